"""Single-op cases: one op of the routing path alone on seeded inputs, timed
with CUDA events; the same command is what a profiler capture of that op runs.

    python -m combine_moe_topk_gate_b200.cases <op> [--workload prefill] [--reps 20]
        [--rows R] [--inter I]

ops: gate, layout, dispatch_<payload> (bf16, fp8, fp8_token, mxfp8, nvfp4,
e5m6), combine, dispatch_backward, combine_backward, swiglu_fp8 (R receive
rows of h = [gate | up], I channels each), quant_fp8_channel (the aligned
receive buffer at align 128).  The first five launches are warm-up; the
timed ones follow (each launch reuses resident inputs, so a capture of launch
6 or later sees the steady state).
"""
from __future__ import annotations

import argparse

import torch

from . import api
from .workloads import DTYPES, WORKLOADS, algorithmic_bytes, make_inputs


def build(op: str, workload: str, rows: int | None, inter: int, device):
    """Inputs for ``op`` and a closure that launches it once; (launch, bytes per launch)."""
    w = WORKLOADS[workload]
    inp = make_inputs(w, 0, with_y=op in ("combine", "combine_backward"))
    logits = inp.logits.to(device)
    idx, wts = api.moe_topk_gate(logits, w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn)
    L = api.moe_get_layout(idx, w.E, w.R)
    x = inp.x.to(device)
    ab = algorithmic_bytes(w)
    if op == "gate":
        return (lambda: api.moe_topk_gate(logits, w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn,
                                          topk_idx=idx, topk_w=wts)), ab["gate"]
    if op == "layout":
        return (lambda: api.moe_get_layout(idx, w.E, w.R, out=L)), ab["layout"]
    if op.startswith("dispatch_") and op[9:] in (*DTYPES, "nvfp4", "e5m6"):
        name = op[9:]
        wd = type(w)(**{**w.__dict__, "dtype": name})
        if name == "nvfp4":
            rx = torch.empty((w.S, w.H // 2), dtype=torch.uint8, device=device)
            bs = torch.empty((w.S, w.H // 16), dtype=torch.uint8, device=device)
            rs = torch.empty((w.S,), dtype=torch.float32, device=device)
            return (lambda: api.moe_dispatch_nvfp4(x, L.token_slot, recv_x=rx, block_scale=bs, row_scale=rs,
                                                   d_status=L.status)), algorithmic_bytes(wd)["dispatch"]
        code = api.MOE_DTYPE_E5M6 if name == "e5m6" else DTYPES[name]
        recv, scale = api.moe_dispatch(x, L.token_slot, code, d_status=L.status)
        return (lambda: api.moe_dispatch(x, L.token_slot, code, recv_x=recv, recv_scale=scale,
                                         d_status=L.status)), algorithmic_bytes(wd)["dispatch"]
    if op == "combine":
        y = inp.y.to(device) if inp.y is not None else \
            torch.randn(w.S, w.H, generator=torch.Generator(device="cpu").manual_seed(4)).to(torch.bfloat16).to(device)
        out = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=device)
        return (lambda: api.moe_combine(y, L.token_slot, wts, out=out, d_status=L.status)), ab["combine"]
    if op in ("dispatch_backward", "combine_backward"):
        g = torch.Generator(device="cpu").manual_seed(1)
        grad_recv = torch.randn(w.S, w.H, generator=g).to(torch.bfloat16).to(device)
        grad_out = torch.randn(w.N, w.H, generator=g).to(torch.bfloat16).to(device)
        if op == "dispatch_backward":
            gx = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=device)
            return (lambda: api.moe_dispatch_backward(grad_recv, L.token_slot, grad_x=gx,
                                                      d_status=L.status)), ab[op]
        gy = torch.empty_like(grad_recv)
        gw = torch.empty((w.N, w.k), dtype=torch.float32, device=device)
        return (lambda: api.moe_combine_backward(grad_out, grad_recv, L.token_slot, wts, grad_y=gy, grad_w=gw,
                                                 d_status=L.status)), ab[op]
    if op == "swiglu_fp8":
        S = rows or w.S
        g = torch.Generator(device="cpu").manual_seed(2)
        h = torch.randn(S, 2 * inter, generator=g).to(torch.bfloat16).to(device)
        out = torch.empty((S, inter), dtype=torch.uint8, device=device)
        sc = torch.empty((S, inter // 128), dtype=torch.float32, device=device)
        return (lambda: api.moe_swiglu_quant(h, api.MOE_DTYPE_FP8_E4M3, out=out, out_scale=sc)), \
            S * (5 * inter + 4 * (inter // 128))
    if op == "quant_fp8_channel":
        La = api.moe_get_layout(idx, w.E, w.R, align=128)
        g = torch.Generator(device="cpu").manual_seed(3)
        recv = torch.randn(La.num_rows, w.H, generator=g).to(torch.bfloat16).to(device)
        out = torch.empty((La.num_rows, w.H), dtype=torch.uint8, device=device)
        sc = torch.empty((w.E, w.H), dtype=torch.float32, device=device)
        ws = torch.zeros(api.moe_quant_fp8_channel_workspace_bytes(w.E, w.H), dtype=torch.uint8, device=device)
        landed = int((La.slot_token >= 0).sum().item())
        return (lambda: api.moe_quant_fp8_channel(recv, La.expert_offset, La.expert_count, out=out, scale=sc,
                                                  workspace=ws, d_status=La.status)), landed * w.H * 3 + 4 * w.E * w.H
    raise SystemExit(f"unknown op {op}")


def main() -> None:
    p = argparse.ArgumentParser()
    p.add_argument("op")
    p.add_argument("--workload", default="prefill", choices=sorted(WORKLOADS))
    p.add_argument("--reps", type=int, default=20)
    p.add_argument("--rows", type=int, default=None)
    p.add_argument("--inter", type=int, default=2048)
    a = p.parse_args()
    device = torch.device("cuda", 0)
    launch, nbytes = build(a.op, a.workload, a.rows, a.inter, device)
    for _ in range(5):
        launch()
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(a.reps):
        launch()
    t1.record()
    t1.synchronize()
    us = t0.elapsed_time(t1) / a.reps * 1e3
    print(f"{a.op} ({a.workload}): {us:.1f} us per launch, {nbytes / us / 1e3:.0f} GB/s of algorithmic traffic "
          f"(back to back, L2 warm between launches)")


if __name__ == "__main__":
    main()
