"""GPU parity of the backward ops against the CPU oracle.

dispatch backward (slot-order fp32 sum, bf16 out) and the grad_y rows of
combine backward (bf16 of the fp32 product w * g) are compared bit for bit.
grad_w is an fp32 dot product whose summation order the definition leaves
open; a product of two bf16 values is exact in fp32, so any order is within
(H - 1) * 2^-24 * sum|g * y| of the exact value, and the oracle (exact sum
rounded once to fp32) is within 2^-24 * |value| of it.  That sum of the two
bounds is the tolerance.
"""
import numpy as np
import pytest
import torch

import oracle as O
from combine_moe_topk_gate_b200.workloads import WORKLOADS, Workload, make_inputs

from _harness import bf16_bits

pytestmark = pytest.mark.gpu


def _layout(w, inp, dev, masked_frac=0.0, seed=0):
    from combine_moe_topk_gate_b200 import api
    idx, wts = api.moe_topk_gate(inp.logits.to(dev), w.k, w.gate_kind, w.n_groups, w.topk_groups,
                                 w.group_topn)
    if masked_frac:
        g = torch.Generator().manual_seed(seed)
        m = torch.rand(idx.shape, generator=g) < masked_frac
        idx = idx.cpu()
        idx[m] = -1
        idx = idx.to(dev)
    L = api.moe_get_layout(idx, w.E, w.R)
    return idx, wts, L


CASES = [("prefill", 0.0), ("mixtral", 0.0), ("decode", 0.05), ("tiny", 0.1)]
EXTRA = [Workload("bwd_k32", 64, 264, 64, 32, 4, "softmax_renorm", "bf16", "random"),
         Workload("bwd_k3", 333, 136, 24, 3, 6, "softmax", "bf16", "random"),
         Workload("bwd_k1", 100, 512, 16, 1, 4, "softmax", "bf16", "random"),
         Workload("bwd_k2", 333, 200, 16, 2, 4, "softmax", "bf16", "random"),
         Workload("bwd_k4", 301, 264, 32, 4, 4, "softmax_renorm", "bf16", "random")]


# masked slots reach every compile-time k of the backward consumer (1, 2, 4, 8)
# and the generic one (3, 32)
MASKED_EXTRA = {"bwd_k32": 0.1, "bwd_k3": 0.15, "bwd_k1": 0.2, "bwd_k2": 0.1, "bwd_k4": 0.1}


@pytest.mark.parametrize("w", [WORKLOADS[n] for n, _ in CASES] + EXTRA,
                         ids=[n for n, _ in CASES] + [w.name for w in EXTRA])
def test_backward_parity(w):
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    masked = dict(CASES).get(w.name, MASKED_EXTRA.get(w.name, 0.0))
    inp = make_inputs(w, 5, with_y=False)
    idx, wts, L = _layout(w, inp, dev, masked)
    gen = torch.Generator().manual_seed(11)
    grad_recv = torch.randn(w.S, w.H, generator=gen).to(torch.bfloat16)
    grad_out = torch.randn(w.N, w.H, generator=gen).to(torch.bfloat16)
    y = torch.randn(w.S, w.H, generator=gen).to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    gx = api.moe_dispatch_backward(grad_recv.to(dev), L.token_slot, d_status=st)
    gy, gw = api.moe_combine_backward(grad_out.to(dev), y.to(dev), L.token_slot, wts, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    slots = L.token_slot.cpu().numpy()
    w_np = wts.cpu().numpy()
    ref_gx, _ = O.dispatch_backward(bf16_bits(grad_recv), slots)
    assert np.array_equal(bf16_bits(gx), ref_gx)
    ref_gy, ref_gw, mag, _ = O.combine_backward(bf16_bits(grad_out), bf16_bits(y), slots, w_np)
    valid = slots[slots >= 0]
    assert np.array_equal(bf16_bits(gy)[valid], ref_gy[valid])
    got_gw = gw.cpu().numpy().astype(np.float64)
    tol = (w.H - 1) * 2.0**-24 * mag + 2.0**-24 * np.abs(ref_gw) + 1e-30
    assert (np.abs(got_gw - ref_gw) <= tol).all(), np.max(np.abs(got_gw - ref_gw) / (tol + 1e-300))
    assert (got_gw[slots < 0] == 0).all()


def test_backward_bad_slots_are_reported_and_skipped():
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    N, H, k = 40, 256, 2
    rng = np.random.default_rng(3)
    slots = rng.permutation(N * k).astype(np.int32).reshape(N, k)
    slots[4, 1] = N * k + 3
    slots[7, 0] = -9
    slots[9, 1] = -1
    w = rng.random((N, k)).astype(np.float32)
    gr = torch.from_numpy(rng.normal(size=(N * k, H)).astype(np.float32)).to(torch.bfloat16)
    go = torch.from_numpy(rng.normal(size=(N, H)).astype(np.float32)).to(torch.bfloat16)
    ts = torch.from_numpy(slots).to(dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    gx = api.moe_dispatch_backward(gr.to(dev), ts, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == O.ERR_BAD_INDEX
    ref_gx, rst = O.dispatch_backward(bf16_bits(gr), slots)
    assert rst == O.ERR_BAD_INDEX and np.array_equal(bf16_bits(gx), ref_gx)
    st.zero_()
    gy, gw = api.moe_combine_backward(go.to(dev), gr.to(dev), ts, torch.from_numpy(w).to(dev), d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == O.ERR_BAD_INDEX
    ref_gy, ref_gw, mag, rst = O.combine_backward(bf16_bits(go), bf16_bits(gr), slots, w)
    ok = slots[(slots >= 0) & (slots < N * k)]
    assert np.array_equal(bf16_bits(gy)[ok], ref_gy[ok])
    bad = (slots < 0) | (slots >= N * k)
    assert (gw.cpu().numpy()[bad] == 0).all() and (ref_gw[bad] == 0).all()
