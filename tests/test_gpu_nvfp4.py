"""GPU parity of the NVFP4 dispatch (moe_dispatch_nvfp4) against the CPU
oracle, bit for bit (packed e2m1 codes, e4m3 block scales in every layout,
fp32 row scales), and a check that a block-scaled FP4 tensor-core GEMM reads
the tiled block scales as they stand.  Buffers start zeroed on both sides and
are compared whole.
"""
import numpy as np
import pytest
import torch

import oracle as O
from combine_moe_topk_gate_b200.workloads import WORKLOADS, Workload, make_inputs

from _harness import bf16_bits

pytestmark = pytest.mark.gpu

CASES = [
    (WORKLOADS["decode"], 128, 0.05),
    (WORKLOADS["mixtral"], 1, 0.0),
    (Workload("nv_ragged", 333, 384, 24, 3, 6, "softmax", "fp8", "random"), 16, 0.2),
    (Workload("nv_wide", 40, 16384, 16, 2, 4, "softmax", "fp8", "random"), 1, 0.0),
]


def _routed(w, align, frac, seed):
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    inp = make_inputs(w, seed, with_y=False)
    idx, _ = api.moe_topk_gate(inp.logits.to(dev), w.k, w.gate_kind, w.n_groups, w.topk_groups,
                               w.group_topn)
    if frac:
        g = torch.Generator().manual_seed(seed + 3)
        idx = idx.cpu()
        idx[torch.rand(idx.shape, generator=g) < frac] = -1
        idx = idx.to(dev)
    rows = api.moe_aligned_recv_rows(w.N, w.k, w.E, align)
    L = api.moe_get_layout(idx, w.E, w.R, align=align, num_recv_rows=rows)
    return inp, L, rows


@pytest.mark.parametrize("layout", [0, 1, 2])
@pytest.mark.parametrize("case", CASES, ids=[f"{w.name}-a{a}" for w, a, _ in CASES])
def test_nvfp4_parity(case, layout):
    from combine_moe_topk_gate_b200 import api
    w, align, frac = case
    dev = torch.device("cuda", 0)
    inp, L, rows = _routed(w, align, frac, seed=6)
    x = inp.x.clone()
    x[1] = 0.0                                              # an all-zero token
    x[2, :64] = 0.0                                         # all-zero blocks in a live row
    shape, _ = api.scale_shape(rows, w.H, api.MOE_DTYPE_NVFP4, layout)
    rx = torch.zeros((rows, w.H // 2), dtype=torch.uint8, device=dev)
    bs = torch.zeros(shape, dtype=torch.uint8, device=dev)
    rs = torch.zeros((rows,), dtype=torch.float32, device=dev)
    api.moe_dispatch_nvfp4(x.to(dev), L.token_slot, scale_layout=layout, recv_x=rx, block_scale=bs,
                           row_scale=rs, d_status=L.status)
    torch.cuda.synchronize()
    assert int(L.status.item()) == 0
    r_rx, r_bs, r_rs, st = O.dispatch_nvfp4(bf16_bits(x), L.token_slot.cpu().numpy(), layout, recv_rows=rows)
    assert st == 0
    got = rx.cpu().numpy()
    d = np.argwhere(got != r_rx)
    assert len(d) == 0, f"{len(d)} code bytes differ, first at {d[:3].tolist()}: gpu {got[tuple(d[0])]:#x} oracle {r_rx[tuple(d[0])]:#x}"
    assert np.array_equal(bs.cpu().numpy().reshape(-1), r_bs)
    assert np.array_equal(rs.cpu().numpy().view(np.uint32), r_rs.view(np.uint32))


def test_nvfp4_bad_slots_reported():
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    N, H, k = 20, 256, 2
    slots = np.arange(N * k, dtype=np.int32).reshape(N, k)
    slots[3, 1] = N * k + 7
    slots[5, 0] = -1
    x = torch.randn(N, H, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    rx = torch.zeros((N * k, H // 2), dtype=torch.uint8, device=dev)
    api.moe_dispatch_nvfp4(x.to(dev), torch.from_numpy(slots).to(dev), recv_x=rx, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == O.ERR_BAD_INDEX
    r_rx, _, _, rst = O.dispatch_nvfp4(bf16_bits(x), slots)
    assert rst == O.ERR_BAD_INDEX and np.array_equal(rx.cpu().numpy(), r_rx)


def _e2m1_table():
    return torch.tensor([O.e2m1_decode(c) for c in range(16)], dtype=torch.float64)


def test_tiled_nvfp4_scales_feed_block_scaled_fp4_gemm():
    """Per expert of an align-128 layout, the packed e2m1 rows and their tiled
    e4m3 block scales go straight into the block-scaled (1x16) FP4 tensor-core
    GEMM; scaling its rows by the row scales gives the dequantised product."""
    from torch.nn.functional import ScalingType, SwizzleType, scaled_mm

    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    w = Workload("nv_gemm", 512, 1024, 8, 2, 2, "softmax", "fp8", "random")
    inp = make_inputs(w, 3, with_y=False)
    g = torch.Generator().manual_seed(8)
    mag = torch.exp2(torch.randint(-5, 6, (w.N, w.H // 16), generator=g).float()).repeat_interleave(16, 1)
    x = (inp.x.float() * mag).to(torch.bfloat16)
    idx, _ = api.moe_topk_gate(inp.logits.to(dev), w.k, w.gate_kind)
    rows = api.moe_aligned_recv_rows(w.N, w.k, w.E, 128)
    L = api.moe_get_layout(idx, w.E, w.R, align=128, num_recv_rows=rows)
    B = w.H // 16
    shape, _ = api.scale_shape(rows, w.H, api.MOE_DTYPE_NVFP4, api.MOE_SCALE_MMA_TILED)
    rx = torch.zeros((rows, w.H // 2), dtype=torch.uint8, device=dev)
    bs = torch.zeros(shape, dtype=torch.uint8, device=dev)
    rs = torch.zeros((rows,), dtype=torch.float32, device=dev)
    api.moe_dispatch_nvfp4(x.to(dev), L.token_slot, scale_layout=api.MOE_SCALE_MMA_TILED, recv_x=rx,
                           block_scale=bs, row_scale=rs, d_status=L.status)
    # weights: e2m1 codes with unit block scales (e4m3 1.0 = 0x38)
    n_out = 256
    wc = torch.randint(0, 256, (n_out, w.H // 2), generator=g, dtype=torch.uint8)
    w_scale = torch.full((n_out * B,), 0x38, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    assert int(L.status.item()) == 0

    tab = _e2m1_table()
    wdeq = torch.stack([tab[(wc & 0xF).long()], tab[(wc >> 4).long()]], -1).reshape(n_out, w.H)
    r_rx, r_bs, r_rs, _ = O.dispatch_nvfp4(bf16_bits(x), L.token_slot.cpu().numpy(), recv_rows=rows)
    codes = torch.from_numpy(r_rx)
    deq = torch.stack([tab[(codes & 0xF).long()], tab[(codes >> 4).long()]], -1).reshape(rows, w.H)
    e4 = torch.tensor([O.e4m3_decode(c) for c in range(256)], dtype=torch.float64)
    deq = deq * e4[torch.from_numpy(r_bs.reshape(rows, B)).long()].repeat_interleave(16, 1)
    deq = deq * torch.from_numpy(r_rs.astype(np.float64))[:, None]
    off = L.expert_offset.cpu().numpy()
    landed = L.slot_token.cpu().numpy() >= 0
    checked = 0
    for e in range(w.E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        a = rx[lo:hi].view(torch.float4_e2m1fn_x2)
        sa = bs[lo * B: hi * B].view(torch.float8_e4m3fn)
        try:
            out = scaled_mm(a, wc.to(dev).view(torch.float4_e2m1fn_x2).t(), sa, ScalingType.BlockWise1x16,
                            w_scale.view(torch.float8_e4m3fn), ScalingType.BlockWise1x16,
                            swizzle_a=SwizzleType.SWIZZLE_32_4_4, swizzle_b=SwizzleType.SWIZZLE_32_4_4,
                            output_dtype=torch.bfloat16)
        except (RuntimeError, NotImplementedError) as exc:
            pytest.skip(f"1x16 block-scaled FP4 GEMM unavailable: {str(exc).splitlines()[0][:120]}")
        got = out.float().cpu().to(torch.float64) * rs[lo:hi].cpu().to(torch.float64)[:, None]
        ref = deq[lo:hi] @ wdeq.t()
        mag_ref = deq[lo:hi].abs() @ wdeq.abs().t()
        m = torch.from_numpy(landed[lo:hi])
        err = (got - ref).abs()[m]
        tol = (2.0**-8 * ref.abs() + 2.0**-14 * mag_ref)[m]    # bf16 output + fp32 accumulation, K = 1024
        assert (err <= tol).all(), float((err / tol).max())
        checked += int(m.sum())
    assert checked == w.N * w.k
