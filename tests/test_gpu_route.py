"""Routing in one call (moe_route: gate and layout) through the C ABI, against
the CPU oracle's gate followed by its layout, bit for bit, on the five
workloads and on the shapes that pick each of its paths: the one-launch path
(N*k <= 1024 with E <= 512, lanes or generic gate; the last CTA builds the
layout), the gate and layout launches for larger batches or more experts.  The arrival counter (the workspace's first 256 bytes) must be zero
again after every call, so calls in a row on one workspace agree too."""
import numpy as np
import pytest
import torch

import oracle as O
from combine_moe_topk_gate_b200.workloads import WORKLOADS, Workload, make_inputs

from _harness import f32_bits

pytestmark = pytest.mark.gpu

LAYOUT_KEYS = ("expert_count", "expert_offset", "rank_count", "rank_offset", "rank_tokens",
               "token_slot", "slot_token")


def _route(w, logits, out=None, align=1, num_rows=None):
    from combine_moe_topk_gate_b200 import api
    idx, wts, L = api.moe_route(logits, w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn, w.R,
                                align=align, num_recv_rows=num_rows, out=out)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), wts.cpu().numpy(), L


def _check(w, inp, idx, wts, L, align=1):
    r_idx, r_w = O.topk_gate(inp.logits.numpy(), w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn)
    assert np.array_equal(idx, r_idx)
    assert np.array_equal(f32_bits(wts), f32_bits(r_w))
    RL = O.get_layout(r_idx, w.E, w.R) if align == 1 else \
        O.get_layout_aligned(r_idx, w.E, w.R, align, L.num_rows)
    for key in LAYOUT_KEYS:
        assert np.array_equal(getattr(L, key).cpu().numpy(), getattr(RL, key)), key
    assert int(L.status.item()) == 0
    assert int(L.workspace[:256].count_nonzero().item()) == 0, "arrival counter not left zero"


CASES = [(name, seed) for name in ("tiny", "decode", "prefill", "skewed", "mixtral") for seed in (0, 1, 2)]


@pytest.mark.parametrize("name,seed", CASES, ids=[f"{n}-s{s}" for n, s in CASES])
def test_route_equals_oracle_gate_then_layout(name, seed):
    w = WORKLOADS[name]
    inp = make_inputs(w, seed, with_y=False)
    idx, wts, L = _route(w, inp.logits.cuda())
    _check(w, inp, idx, wts, L)


SHAPES = [
    Workload("small_path_edge", 128, 64, 256, 8, 8, "sigmoid_group", "fp8", "random", 8, 4, 2),      # N*k = 1024
    Workload("large_path_edge", 129, 64, 256, 8, 8, "sigmoid_group", "fp8", "random", 8, 4, 2),      # 1032
    Workload("one_token", 1, 64, 32, 1, 1, "softmax", "bf16", "random"),
    Workload("small_n256", 256, 64, 128, 4, 4, "softmax_renorm", "bf16", "random"),
    Workload("small_n300", 300, 64, 64, 2, 8, "softmax_renorm", "bf16", "random"),
    Workload("e64_group", 700, 64, 64, 6, 8, "sigmoid_group", "fp8", "random", 8, 3, 2),
    Workload("e128_k1", 1000, 64, 128, 1, 4, "softmax_renorm", "bf16", "random"),
    Workload("e33_small", 100, 64, 33, 5, 3, "softmax", "bf16", "random"),                          # generic, one launch
    Workload("e600_small", 40, 64, 600, 6, 6, "sigmoid_group", "fp8", "random", 12, 4, 2),       # generic, two launches
    Workload("e33_large", 900, 64, 33, 5, 3, "softmax", "bf16", "random"),                          # generic + counts
    Workload("max_E_max_k", 64, 64, 1024, 32, 16, "softmax_renorm", "bf16", "random"),
    Workload("max_E_group", 300, 64, 1024, 32, 32, "sigmoid_group", "fp8", "random", 32, 8, 3),
    Workload("many_groups", 90, 64, 256, 8, 4, "sigmoid_group", "fp8", "random", 64, 16, 2),
    Workload("k3_chunks", 2000, 64, 24, 3, 6, "softmax_renorm", "bf16", "identity"),
]


@pytest.mark.parametrize("w", SHAPES, ids=[w.name for w in SHAPES])
def test_route_shapes(w):
    inp = make_inputs(w, 7, with_y=False)
    idx, wts, L = _route(w, inp.logits.cuda())
    _check(w, inp, idx, wts, L)


@pytest.mark.parametrize("name", ["decode", "prefill"])
def test_route_aligned_layout(name):
    from combine_moe_topk_gate_b200 import api
    w = WORKLOADS[name]
    inp = make_inputs(w, 1, with_y=False)
    rows = api.moe_aligned_recv_rows(w.N, w.k, w.E, 128) + 5
    idx, wts, L = _route(w, inp.logits.cuda(), align=128, num_rows=rows)
    _check(w, inp, idx, wts, L, align=128)


@pytest.mark.parametrize("name", ["decode", "prefill"])
def test_route_calls_in_a_row_share_one_workspace(name):
    """Three batches through one workspace (each call must leave it zero for
    the next), and the same batch twice (identical results)."""
    from combine_moe_topk_gate_b200 import api
    w = WORKLOADS[name]
    L = api.Layout.empty(w.N, w.k, w.E, w.R, "cuda", route=True)
    for seed in (3, 4, 3):
        inp = make_inputs(w, seed, with_y=False)
        idx, wts, L = _route(w, inp.logits.cuda(), out=L)
        _check(w, inp, idx, wts, L)


def test_route_empty_batch():
    from combine_moe_topk_gate_b200 import api
    logits = torch.empty((0, 256), dtype=torch.float32, device="cuda")
    idx, wts, L = api.moe_route(logits, 8, api.MOE_GATE_SIGMOID_GROUP, 8, 4, 2, 8)
    torch.cuda.synchronize()
    assert idx.shape == (0, 8) and (L.expert_count.cpu() == 0).all() and (L.rank_offset.cpu() == 0).all()
    assert int(L.workspace[:256].count_nonzero().item()) == 0


def test_route_rejects_a_short_workspace():
    from combine_moe_topk_gate_b200 import api
    w = WORKLOADS["prefill"]
    logits = torch.zeros((w.N, w.E), dtype=torch.float32, device="cuda")
    L = api.Layout.empty(w.N, w.k, w.E, w.R, "cuda")      # moe_get_layout's size: 256 bytes short
    with pytest.raises(ValueError, match="workspace"):
        api.moe_route(logits, w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn, w.R, out=L)


@pytest.mark.parametrize("name", ["decode", "prefill", "mixtral"])
def test_route_with_l2_prefetch_gives_the_same_results(name):
    """The prefetch region (x of the dispatch that follows, more than the
    64 MiB cap on the Mixtral shape) is a hint: results are unchanged, and a
    dispatch right after still matches the oracle."""
    from combine_moe_topk_gate_b200 import api
    w = WORKLOADS[name]
    inp = make_inputs(w, 2, with_y=False)
    x = inp.x.cuda()
    idx, wts, L = api.moe_route(inp.logits.cuda(), w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn, w.R,
                                prefetch=x)
    recv, scale = api.moe_dispatch(x, L.token_slot, w.dtype_code, d_status=L.status)
    torch.cuda.synchronize()
    _check(w, inp, idx.cpu().numpy(), wts.cpu().numpy(), L)
    from _harness import bf16_bits
    r_recv, r_scale, _ = O.dispatch(bf16_bits(inp.x), L.token_slot.cpu().numpy(), w.dtype_code)
    got = recv.cpu().numpy() if w.dtype != "bf16" else bf16_bits(recv)
    assert np.array_equal(got, r_recv)
    if scale is not None:
        assert np.array_equal(scale.cpu().numpy().view(np.uint8), r_scale.view(np.uint8))
