"""GPU parity of the per-(expert, channel) FP8 quantisation of the receive
buffer (moe_quant_fp8_channel) against the CPU oracle, bit for bit, row-major
and transposed.  Padding rows hold +inf: they must be neither read (the
scales would change) nor written (the zeroed output is compared whole)."""
import numpy as np
import pytest
import torch

import oracle as O
from combine_moe_topk_gate_b200.workloads import WORKLOADS, Workload, make_inputs

from _harness import bf16_bits

pytestmark = pytest.mark.gpu

CASES = [
    (WORKLOADS["decode"], 128, 0.0),
    (WORKLOADS["prefill"], 128, 0.0),
    (Workload("ch_ragged", 300, 384, 40, 3, 8, "softmax", "bf16", "random"), 8, 0.25),
    # few experts with thousands of rows each: several CTAs per (expert, slab),
    # combined through a thread-block cluster (2, 4 and 8 CTAs)
    (Workload("ch_q2", 1100, 256, 2, 2, 2, "softmax", "bf16", "random"), 128, 0.1),
    (Workload("ch_q4", 3000, 384, 2, 2, 2, "softmax", "bf16", "random"), 32, 0.3),
    (Workload("ch_q8", 8192, 384, 4, 2, 2, "softmax", "bf16", "random"), 128, 0.2),
    # skewed loads: hot experts next to cold ones
    (Workload("ch_zipf", 4096, 512, 64, 8, 8, "sigmoid_group", "fp8", "random", 8, 4, 2, bias="zipf1.1"), 128, 0.0),
    (Workload("ch_mixtral", 16384, 512, 8, 2, 8, "softmax_renorm", "bf16", "identity", bias="expert0+2"), 128, 0.0),
]


@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("case", CASES, ids=[f"{w.name}-a{a}" for w, a, _ in CASES])
def test_quant_fp8_channel_parity(case, transpose):
    from combine_moe_topk_gate_b200 import api
    w, align, frac = case
    dev = torch.device("cuda", 0)
    inp = make_inputs(w, 2, with_y=False)
    idx, _ = api.moe_topk_gate(inp.logits.to(dev), w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn)
    if frac:
        g = torch.Generator().manual_seed(4)
        idx = idx.cpu()
        idx[torch.rand(idx.shape, generator=g) < frac] = -1
        idx = idx.to(dev)
    rows = api.moe_aligned_recv_rows(w.N, w.k, w.E, align)
    L = api.moe_get_layout(idx, w.E, w.R, align=align, num_recv_rows=rows)
    g = torch.Generator().manual_seed(9)
    recv = torch.randn(rows, w.H, generator=g) * torch.exp2(torch.randint(-12, 12, (1, w.H), generator=g).float())
    recv[:, 3] = 0.0
    recv[:, 7] = torch.randn(rows, generator=g) * 1e-39     # a channel of bf16 subnormals only
    landed = (L.slot_token >= 0).cpu()
    recv[~landed] = float("inf")
    recv = recv.to(torch.bfloat16)
    shape = (w.H, rows) if transpose else (rows, w.H)
    out = torch.zeros(shape, dtype=torch.uint8, device=dev)
    sc = torch.zeros((w.E, w.H), dtype=torch.float32, device=dev)
    api.moe_quant_fp8_channel(recv.to(dev), L.expert_offset, L.expert_count, transpose=transpose, out=out,
                              scale=sc, d_status=L.status)
    torch.cuda.synchronize()
    assert int(L.status.item()) == 0
    r_out, r_sc, st = O.quant_fp8_channel(bf16_bits(recv), L.expert_offset.cpu().numpy(),
                                          L.expert_count.cpu().numpy(), transpose=transpose)
    assert st == 0
    got = out.cpu().numpy()
    d = np.argwhere(got != r_out)
    assert len(d) == 0, f"{len(d)} codes differ, first at {d[:3].tolist()}"
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), r_sc.view(np.uint32))


def test_quant_fp8_channel_reports_bad_ranges():
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    S, H, E = 64, 128, 3
    recv = torch.randn(S, H).to(torch.bfloat16).to(dev)
    off = torch.tensor([0, 20, 40, 64], dtype=torch.int32, device=dev)
    cnt = torch.tensor([20, 30, 10], dtype=torch.int32, device=dev)     # expert 1 runs past expert 2's start: fine
    cnt_bad = torch.tensor([20, 10, 60], dtype=torch.int32, device=dev)  # expert 2 leaves [0, S)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    api.moe_quant_fp8_channel(recv, off, cnt, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    api.moe_quant_fp8_channel(recv, off, cnt_bad, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == O.ERR_BAD_INDEX


@pytest.mark.parametrize("transpose", [False, True])
def test_clustered_split_with_empty_experts(transpose):
    """40 000 rows over 4 experts (8 CTAs per expert and slab), experts 1 and 3
    empty, expert 2 with 37 rows: the empty and short experts' CTAs still meet
    the cluster barriers, and nothing outside the landed rows is touched."""
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    N, H, E = 40000, 256, 4
    idx = torch.zeros((N, 1), dtype=torch.int32)
    idx[:37, 0] = 2
    L = api.moe_get_layout(idx.to(dev), E, 2)
    g = torch.Generator().manual_seed(12)
    recv = (torch.randn(N, H, generator=g) * torch.exp2(torch.randint(-8, 8, (1, H), generator=g).float()))
    recv[5000:5100, 17] = 300.0                                  # a channel maximum deep inside one share
    recv = recv.to(torch.bfloat16)
    shape = (H, N) if transpose else (N, H)
    out = torch.zeros(shape, dtype=torch.uint8, device=dev)
    sc = torch.full((E, H), 5.0, dtype=torch.float32, device=dev)
    api.moe_quant_fp8_channel(recv.to(dev), L.expert_offset, L.expert_count, transpose=transpose, out=out,
                              scale=sc, d_status=L.status)
    torch.cuda.synchronize()
    assert int(L.status.item()) == 0
    off, cnt = L.expert_offset.cpu().numpy(), L.expert_count.cpu().numpy()
    assert list(cnt) == [N - 37, 0, 37, 0]
    r_out, r_sc, st = O.quant_fp8_channel(bf16_bits(recv), off, cnt, transpose=transpose)
    assert st == 0
    assert np.array_equal(out.cpu().numpy(), r_out)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), r_sc.view(np.uint32))
    assert (sc.cpu().numpy()[[1, 3]] == 0).all()
