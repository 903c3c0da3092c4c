"""Runs one workload through the CUDA path (via the C-ABI binding) and through
the CPU oracle on the same seeded inputs, and compares the results.

The oracle only ever sees the seeded CPU inputs and its own intermediate
results; nothing computed on the GPU is fed to it.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from combine_moe_topk_gate_b200.workloads import Inputs, Workload

BF16_REL_TOL = 2.0 ** -7   # combine: at most one bf16 ulp relative per element


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def run_gpu(w: Workload, inp: Inputs, device="cuda:0", topk_idx: torch.Tensor | None = None):
    from combine_moe_topk_gate_b200 import api
    logits = inp.logits.to(device)
    x = inp.x.to(device)
    if topk_idx is None:
        idx, wts = api.moe_topk_gate(logits, w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn)
    else:
        idx = topk_idx.to(device)
        _, wts = api.moe_topk_gate(logits, w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn)
    L = api.moe_get_layout(idx, w.E, w.R)
    recv, scale = api.moe_dispatch(x, L.token_slot, w.dtype_code, d_status=L.status)
    y = recv if w.expert_out == "identity" else inp.y.to(device)
    out = api.moe_combine(y, L.token_slot, wts, d_status=L.status)
    torch.cuda.synchronize()
    res = dict(
        topk_idx=idx.cpu().numpy(), topk_w=wts.cpu().numpy(),
        expert_count=L.expert_count.cpu().numpy(), expert_offset=L.expert_offset.cpu().numpy(),
        rank_count=L.rank_count.cpu().numpy(), rank_offset=L.rank_offset.cpu().numpy(),
        rank_tokens=L.rank_tokens.cpu().numpy(), token_slot=L.token_slot.cpu().numpy(),
        slot_token=L.slot_token.cpu().numpy(), status=int(L.status.item()),
        out=bf16_bits(out),
    )
    if w.dtype != "bf16":
        res["recv"] = recv.cpu().numpy()
        res["scale"] = scale.cpu().numpy()
    else:
        res["recv"] = bf16_bits(recv)
        res["scale"] = None
    return res


def run_oracle(w: Workload, inp: Inputs, topk_idx: np.ndarray | None = None):
    logits = inp.logits.numpy()
    x = bf16_bits(inp.x)
    idx, wts = O.topk_gate(logits, w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn)
    if topk_idx is not None:
        idx = np.ascontiguousarray(topk_idx, np.int32)
    L = O.get_layout(idx, w.E, w.R)
    recv, scale, st_d = O.dispatch(x, L.token_slot, w.dtype_code)
    y = recv if w.expert_out == "identity" else bf16_bits(inp.y)
    out, st_c = O.combine(y, L.token_slot, wts)
    return dict(topk_idx=idx, topk_w=wts, expert_count=L.expert_count, expert_offset=L.expert_offset,
                rank_count=L.rank_count, rank_offset=L.rank_offset, rank_tokens=L.rank_tokens,
                token_slot=L.token_slot, slot_token=L.slot_token, recv=recv, scale=scale, out=out,
                status=max(L.status, st_d, st_c))


def assert_combine_close(got_bits: np.ndarray, ref_bits: np.ndarray):
    g = O.bf16_to_f32(got_bits).astype(np.float64)
    r = O.bf16_to_f32(ref_bits).astype(np.float64)
    err = np.abs(g - r)
    bad = err > BF16_REL_TOL * np.abs(r)
    assert not bad.any(), f"{bad.sum()} combine elements beyond 1 bf16 ulp; first at {np.argwhere(bad)[:3]}"


def compare(gpu: dict, ref: dict, *, exact_combine: bool = True):
    """Bit-exact routing, layout, payload and scales; combine within 1 bf16 ulp
    (and bit-exact when ``exact_combine``, which the shared fp32 definition gives)."""
    assert np.array_equal(gpu["topk_idx"], ref["topk_idx"]), _first_diff(gpu["topk_idx"], ref["topk_idx"])
    assert np.array_equal(f32_bits(gpu["topk_w"]), f32_bits(ref["topk_w"])), \
        _first_diff(gpu["topk_w"], ref["topk_w"])
    for key in ("expert_count", "expert_offset", "rank_count", "rank_offset", "rank_tokens",
                "token_slot", "slot_token"):
        assert np.array_equal(gpu[key], ref[key]), f"{key}: {_first_diff(gpu[key], ref[key])}"
    valid_rows = ref["slot_token"] >= 0
    assert np.array_equal(gpu["recv"][valid_rows], ref["recv"][valid_rows]), "recv payload differs"
    if ref["scale"] is not None:
        g_s = np.ascontiguousarray(gpu["scale"][valid_rows]).view(np.uint8)
        r_s = np.ascontiguousarray(ref["scale"][valid_rows]).view(np.uint8)
        assert np.array_equal(g_s, r_s), "recv scales differ"
    assert_combine_close(gpu["out"], ref["out"])
    if exact_combine:
        assert np.array_equal(gpu["out"], ref["out"]), _first_diff(gpu["out"], ref["out"])
    assert gpu["status"] == ref["status"]


def _first_diff(a, b):
    a, b = np.asarray(a), np.asarray(b)
    if a.shape != b.shape:
        return f"shape {a.shape} vs {b.shape}"
    d = np.argwhere(a != b)
    if len(d) == 0:
        return "equal"
    i = tuple(d[0])
    return f"{len(d)} differences, first at {i}: gpu={a[i]!r} oracle={b[i]!r}"
