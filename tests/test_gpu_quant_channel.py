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
    # the largest expert count
    (Workload("ch_e1024", 2048, 256, 1024, 4, 8, "softmax", "bf16", "random"), 32, 0.1),
    # averages of 256 to 1023 rows per expert, where the workspace's task
    # queue runs (ch_zipf above too): skewed top-8, and one hot expert of 4
    (Workload("ch_q_zipf", 8192, 256, 128, 8, 8, "sigmoid_group", "fp8", "random", 8, 4, 2, bias="zipf1.1"), 1, 0.0),
    (Workload("ch_q_hot", 3000, 384, 8, 2, 2, "softmax", "bf16", "random", bias="expert0+2"), 32, 0.2),
]


@pytest.mark.parametrize("workspace", ["new", None], ids=["ws", "nows"])
@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("case", CASES, ids=[f"{w.name}-a{a}" for w, a, _ in CASES])
def test_quant_fp8_channel_parity(case, transpose, workspace):
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
                              scale=sc, workspace=workspace, d_status=L.status)
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


def test_quant_fp8_channel_workspace_left_zero_and_reused():
    """One zeroed workspace serves calls in a row (different shapes, both
    orientations): each call leaves it zero, and the results equal the path
    without scratch."""
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    ws = torch.zeros(api.moe_quant_fp8_channel_workspace_bytes(8, 512), dtype=torch.uint8, device=dev)
    for seed, (S, E) in enumerate([(9000, 2), (3000, 8), (40, 8), (9000, 2)]):
        g = torch.Generator().manual_seed(seed)
        cnt = torch.full((E,), S // E, dtype=torch.int32)
        cnt[0] += S - int(cnt.sum())
        off = torch.cat([torch.zeros(1, dtype=torch.int32), torch.cumsum(cnt, 0).to(torch.int32)])
        recv = torch.randn(S, 512, generator=g).to(torch.bfloat16).to(dev)
        for tr in (False, True):
            o1, s1 = api.moe_quant_fp8_channel(recv, off.to(dev), cnt.to(dev), transpose=tr, workspace=ws)
            o2, s2 = api.moe_quant_fp8_channel(recv, off.to(dev), cnt.to(dev), transpose=tr, workspace=None)
            torch.cuda.synchronize()
            assert int(ws.count_nonzero().item()) == 0
            assert torch.equal(o1, o2) and torch.equal(s1.view(torch.int32), s2.view(torch.int32))


def test_quant_fp8_channel_workspace_on_a_side_stream():
    """The default per-call workspace is zeroed in the order of the stream the
    kernel runs on."""
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    S, E, H = 6500, 16, 256                        # 406 rows per expert: the task queue
    cnt = torch.tensor([5000] + [100] * 15, dtype=torch.int32, device=dev)
    off = torch.cat([torch.zeros(1, dtype=torch.int32, device=dev), torch.cumsum(cnt, 0).to(torch.int32)])
    recv = torch.randn(S, H, device=dev).to(torch.bfloat16)
    ref, rsc = api.moe_quant_fp8_channel(recv, off, cnt, workspace=None)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        o, s = api.moe_quant_fp8_channel(recv, off, cnt, stream=side)
    side.synchronize()
    assert torch.equal(o, ref) and torch.equal(s.view(torch.int32), rsc.view(torch.int32))


def test_quant_fp8_channel_hot_expert_beyond_64_parts():
    """An expert of 20 000 rows next to 31 small ones (722 rows per expert on
    average: the task queue): its parts are capped at 64, so they hold more
    than 256 rows and the last ones are empty; against the oracle, both
    orientations, a zeroed workspace left zero."""
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    E, H = 32, 256
    cnt = np.array([20000] + [100] * (E - 1), dtype=np.int32)
    off = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)
    S = int(off[-1])
    g = torch.Generator().manual_seed(21)
    recv = (torch.randn(S, H, generator=g) * 3.0).to(torch.bfloat16)
    ws = torch.zeros(api.moe_quant_fp8_channel_workspace_bytes(E, H), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    for tr in (False, True):
        o, s = api.moe_quant_fp8_channel(recv.to(dev), torch.from_numpy(off).to(dev), torch.from_numpy(cnt).to(dev),
                                         transpose=tr, workspace=ws, d_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0 and int(ws.count_nonzero().item()) == 0
        r_out, r_sc, rst = O.quant_fp8_channel(bf16_bits(recv), off, cnt, transpose=tr)
        assert rst == 0
        assert np.array_equal(o.cpu().numpy(), r_out)
        assert np.array_equal(s.cpu().numpy().view(np.uint32), r_sc.view(np.uint32))
