"""GPU parity of the GEMM-aligned layout and of dispatch, combine and both
backward ops on its padded receive buffer, against the CPU oracle.

Every expert's rows start at a multiple of ``align``; rows that no token lands
in (padding, spare rows at the tail) carry slot_token = -1 and are not part of
any op's output, so payloads are compared on the rows a token lands in.
"""
import numpy as np
import pytest
import torch

import oracle as O
from combine_moe_topk_gate_b200.workloads import WORKLOADS, Workload, make_inputs

from _harness import assert_combine_close, bf16_bits

pytestmark = pytest.mark.gpu

LAYOUT_KEYS = ("expert_count", "expert_offset", "rank_count", "rank_offset", "rank_tokens",
               "token_slot", "slot_token")

CASES = [
    # (workload, align, spare rows beyond the minimum, masked fraction)
    (WORKLOADS["tiny"], 8, 0, 0.0),
    (WORKLOADS["tiny"], 128, 5, 0.2),
    (WORKLOADS["decode"], 64, 0, 0.05),
    (WORKLOADS["decode"], 1, 33, 0.0),                     # plain layout in a larger buffer
    (WORKLOADS["mixtral"], 128, 0, 0.0),
    (Workload("al_single", 40, 256, 32, 4, 4, "softmax", "fp8", "random"), 16, 3, 0.1),   # N*k <= 1024
    (Workload("al_k1", 777, 512, 16, 1, 4, "softmax", "bf16", "random"), 4096, 0, 0.0),  # max align
    (Workload("al_ragged", 1500, 384, 96, 6, 8, "softmax_renorm", "fp8", "random"), 32, 7, 0.3),
]
IDS = [f"{w.name}-a{a}-s{s}-m{m}" for w, a, s, m in CASES]


def _mask(idx: torch.Tensor, frac: float, seed: int) -> torch.Tensor:
    if not frac:
        return idx
    g = torch.Generator().manual_seed(seed)
    m = torch.rand(idx.shape, generator=g) < frac
    idx = idx.clone()
    idx[m] = -1
    return idx


def _layout(w, align, spare, frac, seed=0):
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    inp = make_inputs(w, seed, with_y=False)
    idx, wts = api.moe_topk_gate(inp.logits.to(dev), w.k, w.gate_kind, w.n_groups, w.topk_groups,
                                 w.group_topn)
    idx = _mask(idx.cpu(), frac, seed + 1).to(dev)
    rows = api.moe_aligned_recv_rows(w.N, w.k, w.E, align) + spare
    L = api.moe_get_layout(idx, w.E, w.R, align=align, num_recv_rows=rows)
    return inp, idx, wts, L, rows


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_aligned_layout_parity(case):
    w, align, spare, frac = case
    inp, idx, wts, L, rows = _layout(w, align, spare, frac)
    torch.cuda.synchronize()
    ref = O.get_layout_aligned(idx.cpu().numpy(), w.E, w.R, align, rows)
    for key in LAYOUT_KEYS:
        assert np.array_equal(getattr(L, key).cpu().numpy(), getattr(ref, key)), key
    assert int(L.status.item()) == ref.status
    assert L.num_rows == rows
    off = L.expert_offset.cpu().numpy()
    assert (off % align == 0).all()


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "fp8_token", "mxfp8"])
@pytest.mark.parametrize("case", CASES[2:6], ids=IDS[2:6])
def test_aligned_dispatch_combine_parity(case, dtype):
    from combine_moe_topk_gate_b200 import api
    from combine_moe_topk_gate_b200.workloads import DTYPES
    w, align, spare, frac = case
    dev = torch.device("cuda", 0)
    inp, idx, wts, L, rows = _layout(w, align, spare, frac, seed=3)
    code = DTYPES[dtype]
    recv, scale = api.moe_dispatch(inp.x.to(dev), L.token_slot, code, num_recv_rows=rows,
                                   d_status=L.status)
    assert recv.shape[0] == rows
    gen = torch.Generator().manual_seed(17)
    y = torch.randn(rows, w.H, generator=gen).to(torch.bfloat16)
    out = api.moe_combine(y.to(dev), L.token_slot, wts, d_status=L.status)
    torch.cuda.synchronize()
    assert int(L.status.item()) == 0

    slots = L.token_slot.cpu().numpy()
    r_recv, r_scale, st = O.dispatch(bf16_bits(inp.x), slots, code, recv_rows=rows)
    assert st == 0
    valid = L.slot_token.cpu().numpy() >= 0
    got = recv.cpu().numpy() if dtype != "bf16" else bf16_bits(recv)
    assert np.array_equal(got[valid], r_recv[valid])
    if r_scale is not None:
        g_s = np.ascontiguousarray(scale.cpu().numpy()[valid]).view(np.uint8)
        assert np.array_equal(g_s, np.ascontiguousarray(r_scale[valid]).view(np.uint8))
    r_out, st = O.combine(bf16_bits(y), slots, wts.cpu().numpy())
    assert st == 0
    assert_combine_close(bf16_bits(out), r_out)
    assert np.array_equal(bf16_bits(out), r_out)


@pytest.mark.parametrize("case", [CASES[1], CASES[4], CASES[7]], ids=[IDS[1], IDS[4], IDS[7]])
def test_aligned_backward_parity(case):
    from combine_moe_topk_gate_b200 import api
    w, align, spare, frac = case
    dev = torch.device("cuda", 0)
    inp, idx, wts, L, rows = _layout(w, align, spare, frac, seed=9)
    gen = torch.Generator().manual_seed(23)
    grad_recv = torch.randn(rows, w.H, generator=gen).to(torch.bfloat16)
    grad_out = torch.randn(w.N, w.H, generator=gen).to(torch.bfloat16)
    y = torch.randn(rows, w.H, generator=gen).to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    gx = api.moe_dispatch_backward(grad_recv.to(dev), L.token_slot, d_status=st)
    gy, gw = api.moe_combine_backward(grad_out.to(dev), y.to(dev), L.token_slot, wts, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert gy.shape[0] == rows
    slots = L.token_slot.cpu().numpy()
    ref_gx, _ = O.dispatch_backward(bf16_bits(grad_recv), slots)
    assert np.array_equal(bf16_bits(gx), ref_gx)
    ref_gy, ref_gw, mag, _ = O.combine_backward(bf16_bits(grad_out), bf16_bits(y), slots,
                                                wts.cpu().numpy())
    valid = slots[slots >= 0]
    assert np.array_equal(bf16_bits(gy)[valid], ref_gy[valid])
    got_gw = gw.cpu().numpy().astype(np.float64)
    tol = (w.H - 1) * 2.0**-24 * mag + 2.0**-24 * np.abs(ref_gw) + 1e-30
    assert (np.abs(got_gw - ref_gw) <= tol).all()
    assert (got_gw[slots < 0] == 0).all()


def test_aligned_slot_beyond_default_rows_is_accepted():
    """A slot at or beyond N*k is legal in a padded buffer: with the row count
    passed, dispatch and combine use it instead of reporting a bad index."""
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    N, H, k, rows = 8, 256, 2, 64
    slots = (np.arange(N * k, dtype=np.int32) * 3 + 5).reshape(N, k)     # up to 50 > N*k
    gen = torch.Generator().manual_seed(1)
    x = torch.randn(N, H, generator=gen).to(torch.bfloat16)
    w = torch.rand(N, k, generator=gen)
    ts = torch.from_numpy(slots).to(dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    recv, _ = api.moe_dispatch(x.to(dev), ts, api.MOE_DTYPE_BF16, num_recv_rows=rows, d_status=st)
    out = api.moe_combine(recv, ts, w.to(dev), d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    r_recv, _, rst = O.dispatch(bf16_bits(x), slots, O.DT_BF16, recv_rows=rows)
    assert rst == 0
    got = bf16_bits(recv)
    assert np.array_equal(got[slots.ravel()], r_recv[slots.ravel()])
    r_out, _ = O.combine(r_recv, slots, w.numpy())
    assert np.array_equal(bf16_bits(out), r_out)
    # The same slots against the default N*k rows are out of range.
    st.zero_()
    api.moe_dispatch(x.to(dev), ts, api.MOE_DTYPE_BF16, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == O.ERR_BAD_INDEX
