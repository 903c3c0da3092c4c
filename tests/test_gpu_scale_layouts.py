"""GPU parity of the receive-scale layouts (moe_dispatch_ex) against the CPU
oracle, and a check that a block-scaled tensor-core GEMM reads the tiled
layout as it stands.

The scale buffers start zeroed on both sides and are compared whole, so a
write to a position no landed row owns fails the test.
"""
import numpy as np
import pytest
import torch

import oracle as O
from combine_moe_topk_gate_b200.workloads import WORKLOADS, Workload, make_inputs

from _harness import bf16_bits

pytestmark = pytest.mark.gpu

LAYOUTS = {"mn": 1, "tiled": 2}
CASES = [
    # workload, align, masked fraction
    (WORKLOADS["decode"], 128, 0.05),
    (Workload("sl_ragged", 1500, 384, 96, 6, 8, "softmax_renorm", "fp8", "random"), 32, 0.2),
    (Workload("sl_small", 37, 640, 16, 3, 4, "softmax", "fp8", "random"), 1, 0.0),
    (WORKLOADS["prefill"], 128, 0.0),
    # k <= 4: the FP8 kernels take two 512-channel segments per warp; 1152
    # channels = 3 segments, so the last warp of a token has one segment
    (Workload("sl_k2_odd", 600, 1152, 16, 2, 4, "softmax", "fp8", "random"), 16, 0.1),
    (Workload("sl_k4", 300, 2048, 32, 4, 8, "softmax_renorm", "fp8", "random"), 128, 0.05),
]


def _routed(w, align, frac, seed):
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    inp = make_inputs(w, seed, with_y=False)
    idx, wts = api.moe_topk_gate(inp.logits.to(dev), w.k, w.gate_kind, w.n_groups, w.topk_groups,
                                 w.group_topn)
    if frac:
        g = torch.Generator().manual_seed(seed + 7)
        idx = idx.cpu()
        idx[torch.rand(idx.shape, generator=g) < frac] = -1
        idx = idx.to(dev)
    rows = api.moe_aligned_recv_rows(w.N, w.k, w.E, align)
    L = api.moe_get_layout(idx, w.E, w.R, align=align, num_recv_rows=rows)
    return inp, L, rows


@pytest.mark.parametrize("layout", ["mn", "tiled"])
@pytest.mark.parametrize("dtype", ["fp8", "fp8_token", "mxfp8"])
@pytest.mark.parametrize("case", CASES, ids=[f"{w.name}-a{a}" for w, a, _ in CASES])
def test_scale_layout_parity(case, dtype, layout):
    from combine_moe_topk_gate_b200 import api
    from combine_moe_topk_gate_b200.workloads import DTYPES
    w, align, frac = case
    code, lay = DTYPES[dtype], LAYOUTS[layout]
    if w.H % 128 and layout == "tiled":
        pytest.skip("tiled scales need H % 128 == 0")
    dev = torch.device("cuda", 0)
    inp, L, rows = _routed(w, align, frac, seed=2)
    shape, sdt = api.scale_shape(rows, w.H, code, lay)
    if code != api.MOE_DTYPE_MXFP8_E4M3 and layout == "tiled":
        assert shape is None                                   # no tiled layout for fp32 scales
        with pytest.raises(ValueError):
            api.moe_dispatch(inp.x.to(dev), L.token_slot, code, num_recv_rows=rows, scale_layout=lay)
        return
    recv_scale = torch.zeros(shape, dtype=sdt, device=dev)
    recv_x = torch.zeros((rows, w.H), dtype=torch.uint8, device=dev)
    api.moe_dispatch(inp.x.to(dev), L.token_slot, code, recv_x=recv_x, recv_scale=recv_scale,
                     num_recv_rows=rows, scale_layout=lay, d_status=L.status)
    torch.cuda.synchronize()
    assert int(L.status.item()) == 0
    r_recv, r_scale, st = O.dispatch_scaled(bf16_bits(inp.x), L.token_slot.cpu().numpy(), code, lay,
                                            recv_rows=rows)
    assert st == 0
    assert np.array_equal(recv_x.cpu().numpy(), r_recv)
    got = recv_scale.cpu().numpy().reshape(-1)
    assert got.size == r_scale.size
    assert np.array_equal(np.ascontiguousarray(got).view(np.uint8), r_scale.view(np.uint8))


def _e4m3_to_f64(codes: torch.Tensor) -> torch.Tensor:
    return codes.view(torch.float8_e4m3fn).to(torch.float32).to(torch.float64)


def test_tiled_mxfp8_scales_feed_block_scaled_gemm():
    """Per expert of an align-128 layout, the dispatched e4m3 rows and their
    tiled E8M0 scales go straight into the block-scaled (1x32) tensor-core
    GEMM; the product matches the dequantised rows times the weights."""
    from torch.nn.functional import ScalingType, SwizzleType, scaled_mm

    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    w = Workload("sl_gemm", 512, 1024, 8, 2, 2, "softmax", "mxfp8", "random")
    inp = make_inputs(w, 3, with_y=False)
    # block magnitudes spread over 2^-6..2^6 so a misplaced scale shows
    g = torch.Generator().manual_seed(5)
    mag = torch.exp2(torch.randint(-6, 7, (w.N, w.H // 32), generator=g).float()).repeat_interleave(32, 1)
    x = (inp.x.float() * mag).to(torch.bfloat16)
    idx, _ = api.moe_topk_gate(inp.logits.to(dev), w.k, w.gate_kind)
    rows = api.moe_aligned_recv_rows(w.N, w.k, w.E, 128)
    L = api.moe_get_layout(idx, w.E, w.R, align=128, num_recv_rows=rows)
    B = w.H // 32
    shape, _ = api.scale_shape(rows, w.H, api.MOE_DTYPE_MXFP8_E4M3, api.MOE_SCALE_MMA_TILED)
    sc = torch.zeros(shape, dtype=torch.uint8, device=dev)
    rx = torch.zeros((rows, w.H), dtype=torch.uint8, device=dev)
    api.moe_dispatch(x.to(dev), L.token_slot, api.MOE_DTYPE_MXFP8_E4M3, recv_x=rx, recv_scale=sc,
                     num_recv_rows=rows, scale_layout=api.MOE_SCALE_MMA_TILED, d_status=L.status)
    # weights: e4m3 codes with unit (2^0) scales
    n_out = 256
    wq = (torch.randn(n_out, w.H, generator=g) * 2).to(torch.float8_e4m3fn)
    w_codes = wq.view(torch.uint8).to(dev)
    w_scale = torch.full((n_out * B,), 127, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    assert int(L.status.item()) == 0

    # reference from the oracle's row-major dispatch of the same rows
    r_recv, r_e8, _ = O.dispatch(bf16_bits(x), L.token_slot.cpu().numpy(), O.DT_MXFP8_E4M3, recv_rows=rows)
    deq = _e4m3_to_f64(torch.from_numpy(r_recv)) * torch.exp2(
        torch.from_numpy(r_e8.astype(np.float64) - 127.0)).repeat_interleave(32, 1)
    wdeq = _e4m3_to_f64(wq.view(torch.uint8))
    off = L.expert_offset.cpu().numpy()
    landed = L.slot_token.cpu().numpy() >= 0
    checked = 0
    for e in range(w.E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        a = rx[lo:hi].view(torch.float8_e4m3fn)
        sa = sc[lo * B: hi * B].view(torch.float8_e8m0fnu)
        out = scaled_mm(a, w_codes.view(torch.float8_e4m3fn).t(), sa, ScalingType.BlockWise1x32,
                        w_scale.view(torch.float8_e8m0fnu), ScalingType.BlockWise1x32,
                        swizzle_a=SwizzleType.SWIZZLE_32_4_4, swizzle_b=SwizzleType.SWIZZLE_32_4_4,
                        output_dtype=torch.bfloat16)
        ref = deq[lo:hi] @ wdeq.t()
        mag_ref = deq[lo:hi].abs() @ wdeq.abs().t()
        got = out.float().cpu().to(torch.float64)
        m = torch.from_numpy(landed[lo:hi])
        err = (got - ref).abs()[m]
        tol = (2.0**-8 * ref.abs() + 2.0**-14 * mag_ref)[m]    # bf16 output + fp32 accumulation, K = 1024
        assert (err <= tol).all(), float((err / tol).max())
        checked += int(m.sum())
    assert checked == w.N * w.k


def test_mn_major_fp8_scales_feed_blockwise_gemm():
    """The MN-major fp32 scales of the per-128-block FP8 payload, read as the
    1x128 block-scaled operand of a GEMM (the row count is a multiple of 4 so
    the leading dimension is the row count).  Skipped where the installed
    BLAS has no 1x128 block-scaled FP8 GEMM for this GPU."""
    from torch.nn.functional import ScalingType, scaled_mm

    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    w = Workload("sl_gemm128", 256, 1024, 8, 2, 2, "softmax", "fp8", "random")
    inp = make_inputs(w, 4, with_y=False)
    idx, _ = api.moe_topk_gate(inp.logits.to(dev), w.k, w.gate_kind)
    L = api.moe_get_layout(idx, w.E, w.R)
    S, B = w.N * w.k, w.H // 128
    shape, _ = api.scale_shape(S, w.H, api.MOE_DTYPE_FP8_E4M3, api.MOE_SCALE_MN_MAJOR)
    assert shape == (B, S)
    sc = torch.zeros(shape, dtype=torch.float32, device=dev)
    rx, _ = api.moe_dispatch(inp.x.to(dev), L.token_slot, api.MOE_DTYPE_FP8_E4M3, recv_scale=sc,
                             scale_layout=api.MOE_SCALE_MN_MAJOR, d_status=L.status)
    g = torch.Generator().manual_seed(9)
    n_out = 256
    wq = (torch.randn(n_out, w.H, generator=g) * 2).to(torch.float8_e4m3fn)
    w_scale = torch.ones((n_out // 128, B), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    try:
        out = scaled_mm(rx.view(torch.float8_e4m3fn), wq.to(dev).t(), sc.t(), ScalingType.BlockWise1x128,
                        w_scale, ScalingType.BlockWise128x128, output_dtype=torch.bfloat16)
    except (RuntimeError, NotImplementedError) as exc:   # no 1x128 kernel in this BLAS for sm_100
        pytest.skip(f"1x128 block-scaled GEMM unavailable: {str(exc).splitlines()[0][:120]}")
    r_recv, r_sc, _ = O.dispatch(bf16_bits(inp.x), L.token_slot.cpu().numpy(), O.DT_FP8_E4M3)
    deq = _e4m3_to_f64(torch.from_numpy(r_recv)) * torch.from_numpy(r_sc.astype(np.float64)).repeat_interleave(128, 1)
    wdeq = _e4m3_to_f64(wq.view(torch.uint8))
    ref = deq @ wdeq.t()
    mag_ref = deq.abs() @ wdeq.abs().t()
    err = (out.float().cpu().to(torch.float64) - ref).abs()
    assert (err <= 2.0**-8 * ref.abs() + 2.0**-14 * mag_ref).all()


@pytest.mark.parametrize("layout", [0, 1, 3])
@pytest.mark.parametrize("case", CASES, ids=[f"{w.name}-a{a}" for w, a, _ in CASES])
def test_ue8m0_parity(case, layout):
    """FP8 with power-of-two (UE8M0) 1x128 scales, row-major, MN-major and
    packed MN-major scales, against the oracle over whole zeroed buffers."""
    from combine_moe_topk_gate_b200 import api
    w, align, frac = case
    dev = torch.device("cuda", 0)
    inp, L, rows = _routed(w, align, frac, seed=8)
    g = torch.Generator().manual_seed(3)
    x = (inp.x.float() * torch.exp2(torch.randint(-30, 20, (w.N, w.H // 128), generator=g).float())
         .repeat_interleave(128, 1)).to(torch.bfloat16)
    x[0] = 0.0
    code = api.MOE_DTYPE_FP8_E4M3_UE8M0
    shape, sdt = api.scale_shape(rows, w.H, code, layout)
    sc = torch.zeros(shape, dtype=sdt, device=dev)
    rx = torch.zeros((rows, w.H), dtype=torch.uint8, device=dev)
    api.moe_dispatch(x.to(dev), L.token_slot, code, recv_x=rx, recv_scale=sc, num_recv_rows=rows,
                     scale_layout=layout, d_status=L.status)
    torch.cuda.synchronize()
    assert int(L.status.item()) == 0
    r_recv, r_sc, st = O.dispatch_scaled(bf16_bits(x), L.token_slot.cpu().numpy(), code, layout, recv_rows=rows)
    assert st == 0
    assert np.array_equal(rx.cpu().numpy(), r_recv)
    assert np.array_equal(sc.cpu().numpy().reshape(-1), r_sc.reshape(-1))
