"""GPU parity of the E5M6 dispatch payload (12-bit float, two codes per three
bytes) against the CPU oracle, bit for bit over whole zeroed buffers, with
inputs that reach saturation, the subnormal range and signed zeros."""
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
    (Workload("e5_ragged", 333, 416, 24, 3, 6, "softmax", "bf16", "random"), 8, 0.2),
]


def _spread(x: torch.Tensor, seed: int) -> torch.Tensor:
    """Scale rows by 2^-30 .. 2^20 so that the subnormal and saturating ranges
    of E5M6 are both hit; add exact zeros of both signs."""
    g = torch.Generator().manual_seed(seed)
    e = torch.randint(-30, 21, (x.shape[0], 1), generator=g).float()
    y = x.float() * torch.exp2(e)
    y[:, 0] = 0.0
    y[:, 1] = -0.0
    y[0, :] = 1e38
    return y.to(torch.bfloat16)


@pytest.mark.parametrize("case", CASES, ids=[f"{w.name}-a{a}" for w, a, _ in CASES])
def test_e5m6_parity(case):
    from combine_moe_topk_gate_b200 import api
    w, align, frac = case
    dev = torch.device("cuda", 0)
    inp = make_inputs(w, 4, with_y=False)
    idx, _ = api.moe_topk_gate(inp.logits.to(dev), w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn)
    if frac:
        g = torch.Generator().manual_seed(11)
        idx = idx.cpu()
        idx[torch.rand(idx.shape, generator=g) < frac] = -1
        idx = idx.to(dev)
    rows = api.moe_aligned_recv_rows(w.N, w.k, w.E, align)
    L = api.moe_get_layout(idx, w.E, w.R, align=align, num_recv_rows=rows)
    x = _spread(inp.x, 5)
    rx = torch.zeros((rows, w.H // 2 * 3), dtype=torch.uint8, device=dev)
    api.moe_dispatch(x.to(dev), L.token_slot, api.MOE_DTYPE_E5M6, recv_x=rx, num_recv_rows=rows,
                     d_status=L.status)
    torch.cuda.synchronize()
    assert int(L.status.item()) == 0
    ref, st = O.dispatch_e5m6(bf16_bits(x), L.token_slot.cpu().numpy(), recv_rows=rows)
    assert st == 0
    got = rx.cpu().numpy()
    d = np.argwhere(got != ref)
    assert len(d) == 0, f"{len(d)} bytes differ, first at {d[:3].tolist()}"


def test_e5m6_every_bf16_value():
    """All 65536 bf16 bit patterns except NaNs, dispatched as one token row
    (k = 1), against the oracle's encoder: exhaustive over the input type."""
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = O.bf16_to_f32(bits)
    bits = bits[~np.isnan(f)]
    bits = np.concatenate([bits, np.zeros((-len(bits)) % 32, np.uint16)])
    H = len(bits)
    x = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).reshape(1, H)
    slots = torch.zeros((1, 1), dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    rx, _ = api.moe_dispatch(x.to(dev), slots, api.MOE_DTYPE_E5M6, d_status=st)
    torch.cuda.synchronize()
    ref, rst = O.dispatch_e5m6(bits.reshape(1, H), np.zeros((1, 1), np.int32))
    assert int(st.item()) == 0 and rst == 0
    assert np.array_equal(rx.cpu().numpy(), ref)


def test_e5m6_bad_slots_reported():
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    N, H, k = 12, 64, 2
    slots = np.arange(N * k, dtype=np.int32).reshape(N, k)
    slots[2, 0] = N * k
    x = torch.randn(N, H, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    rx = torch.zeros((N * k, H // 2 * 3), dtype=torch.uint8, device=dev)
    api.moe_dispatch(x.to(dev), torch.from_numpy(slots).to(dev), api.MOE_DTYPE_E5M6, recv_x=rx, d_status=st)
    torch.cuda.synchronize()
    ref, rst = O.dispatch_e5m6(bf16_bits(x), slots)
    assert int(st.item()) == O.ERR_BAD_INDEX == rst
    assert np.array_equal(rx.cpu().numpy(), ref)
