"""The allocation-free layout entry point (moe_get_layout_noalloc).

It exists for callers that cannot allocate device memory -- for example a
serving runtime that has reserved the whole GPU for its own pool, or a
deployment whose memory plan is fixed before the first request -- and so
cannot pass moe_get_layout a workspace.  It must give exactly what
moe_get_layout gives.  Two calls in a row check that the shared scratch array,
which keeps the previous call's contents, does not leak into the next result.
This file is collected last so that a failure here stops a ``-x`` run only
after every other test has run; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _fields(L):
    torch.cuda.synchronize()
    return {k: getattr(L, k).cpu().numpy() for k in ("expert_count", "expert_offset", "rank_count",
                                                     "rank_offset", "rank_tokens", "token_slot",
                                                     "slot_token", "status")}


def _inputs(N, k, E, seed, masked):
    g = torch.Generator().manual_seed(seed)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(N)]).to(torch.int32)
    if masked:
        idx[torch.rand((N, k), generator=g) < 0.05] = -1
    return idx.cuda()


def test_noalloc_layout_equals_workspace_layout_twice_in_a_row():
    from combine_moe_topk_gate_b200 import api
    # two different batches back to back: a DeepSeek-shaped one, then a smaller
    # Mixtral-shaped one with masked slots, so the second call reads scratch the
    # first one left behind
    for (N, k, E, R, seed, masked) in [(4096, 8, 256, 32, 0, False), (3000, 2, 8, 8, 1, True)]:
        idx = _inputs(N, k, E, seed, masked)
        ref = api.moe_get_layout(idx, E, R)
        got = api.Layout.empty(N, k, E, R, idx.device)
        # poison the outputs so a skipped write would show
        for t in (got.expert_count, got.expert_offset, got.rank_count, got.rank_offset,
                  got.rank_tokens, got.token_slot, got.slot_token):
            t.fill_(-12345)
        st = api.lib().moe_get_layout_noalloc(
            ctypes.c_void_p(idx.data_ptr()), N, k, E, R,
            *[ctypes.c_void_p(t.data_ptr()) for t in (got.expert_count, got.expert_offset,
                                                      got.rank_count, got.rank_offset,
                                                      got.rank_tokens, got.token_slot,
                                                      got.slot_token, got.status)],
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == api.MOE_OK
        a, b = _fields(ref), _fields(got)
        for key in a:
            assert np.array_equal(a[key], b[key]), key


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from combine_moe_topk_gate_b200 import api
    N, k, E, R = 1 << 20, 8, 1024, 1024      # needs far more than the fixed scratch
    assert api.moe_layout_workspace_bytes(N, k, E, R) > api.MOE_LAYOUT_NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(256)
    st = api.lib().moe_get_layout_noalloc(p, N, k, E, R, p, p, p, p, p, p, p, None, None)
    assert st == api.MOE_ERR_UNSUPPORTED
