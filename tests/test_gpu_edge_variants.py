"""Edge cases of the quantisation variants and GEMM-facing layouts, each
against the CPU oracle over whole buffers: empty batches, one token, every
slot masked, k = E, the smallest legal widths."""
import numpy as np
import pytest
import torch

import oracle as O

from _harness import bf16_bits

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def _x(N, H, seed=0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(N, H, generator=g) * torch.exp2(torch.randint(-8, 8, (N, 1), generator=g).float())).to(torch.bfloat16)


def _slots(N, k, masked=None, seed=0):
    rng = np.random.default_rng(seed)
    s = rng.permutation(N * k).astype(np.int32).reshape(N, k)
    if masked is not None:
        s[masked] = -1
    return s


@pytest.mark.parametrize("N,H,k", [(1, 64, 1), (1, 7168, 8), (5, 64, 4), (33, 128, 32)])
def test_nvfp4_small_and_wide_k(N, H, k):
    from combine_moe_topk_gate_b200 import api
    x = _x(N, H, N + H)
    s = _slots(N, k)
    rx = torch.zeros((N * k, H // 2), dtype=torch.uint8, device=DEV)
    bs = torch.zeros((N * k, H // 16), dtype=torch.uint8, device=DEV)
    rs = torch.zeros((N * k,), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    api.moe_dispatch_nvfp4(x.to(DEV), torch.from_numpy(s).to(DEV), recv_x=rx, block_scale=bs, row_scale=rs, d_status=st)
    torch.cuda.synchronize()
    r_rx, r_bs, r_rs, rst = O.dispatch_nvfp4(bf16_bits(x), s)
    assert int(st.item()) == rst == 0
    assert np.array_equal(rx.cpu().numpy(), r_rx) and np.array_equal(bs.cpu().numpy().reshape(-1), r_bs)
    assert np.array_equal(rs.cpu().numpy().view(np.uint32), r_rs.view(np.uint32))


@pytest.mark.parametrize("dtype", ["e5m6", "fp8_ue8m0", "mxfp8", "fp8_token"])
def test_all_slots_masked_writes_nothing(dtype):
    from combine_moe_topk_gate_b200 import api
    from combine_moe_topk_gate_b200.workloads import DTYPES
    code = api.MOE_DTYPE_E5M6 if dtype == "e5m6" else DTYPES[dtype]
    N, H, k = 16, 256, 2
    x = _x(N, H)
    s = np.full((N, k), -1, np.int32)
    width = H // 2 * 3 if dtype == "e5m6" else H
    rx = torch.full((N * k, width), 0xAB, dtype=torch.uint8, device=DEV)
    shape, sdt = api.scale_shape(N * k, H, code)
    sc = torch.full(shape, 7, dtype=sdt, device=DEV) if shape else None
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    api.moe_dispatch(x.to(DEV), torch.from_numpy(s).to(DEV), code, recv_x=rx, recv_scale=sc, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert (rx.cpu().numpy() == 0xAB).all()
    if sc is not None:
        assert (sc.cpu().numpy() == 7).all()


@pytest.mark.parametrize("dtype", ["e5m6", "fp8_ue8m0"])
def test_empty_batch(dtype):
    from combine_moe_topk_gate_b200 import api
    from combine_moe_topk_gate_b200.workloads import DTYPES
    code = api.MOE_DTYPE_E5M6 if dtype == "e5m6" else DTYPES[dtype]
    x = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    s = torch.empty((0, 4), dtype=torch.int32, device=DEV)
    rx, sc = api.moe_dispatch(x, s, code)
    torch.cuda.synchronize()
    assert rx.shape[0] == 0
    rx, bs, rs = api.moe_dispatch_nvfp4(x, s)
    assert rx.shape[0] == 0 and rs.shape[0] == 0


def test_quant_channel_empty_experts_and_single_row():
    """Experts with no rows get zero scales; an expert with one row gets
    codes of that row against its own magnitudes."""
    from combine_moe_topk_gate_b200 import api
    S, H, E = 9, 256, 4
    recv = _x(S, H, 3)
    off = np.array([0, 0, 1, 1, 9], np.int32)        # experts 0 and 2 empty, expert 1 one row
    cnt = np.array([0, 1, 0, 8], np.int32)
    out = torch.zeros((S, H), dtype=torch.uint8, device=DEV)
    sc = torch.full((E, H), 3.0, dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    api.moe_quant_fp8_channel(recv.to(DEV), torch.from_numpy(off).to(DEV), torch.from_numpy(cnt).to(DEV),
                              out=out, scale=sc, d_status=st)
    torch.cuda.synchronize()
    r_out, r_sc, rst = O.quant_fp8_channel(bf16_bits(recv), off, cnt)
    assert int(st.item()) == rst == 0
    assert np.array_equal(out.cpu().numpy(), r_out)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), r_sc.view(np.uint32))
    assert (sc.cpu().numpy()[[0, 2]] == 0).all()


def test_swiglu_single_row_every_layout():
    from combine_moe_topk_gate_b200 import api
    I = 128
    h = _x(1, 2 * I, 5)
    for dt, lay in ((api.MOE_DTYPE_FP8_E4M3, 0), (api.MOE_DTYPE_FP8_E4M3, 1), (api.MOE_DTYPE_MXFP8_E4M3, 2),
                    (api.MOE_DTYPE_FP8_E4M3_TOKEN, 1), (api.MOE_DTYPE_BF16, 0)):
        shape, sdt = api.scale_shape(1, I, dt, lay)
        out = torch.zeros((1, I), dtype=torch.bfloat16 if dt == 0 else torch.uint8, device=DEV)
        sc = torch.zeros(shape, dtype=sdt, device=DEV) if shape else None
        api.moe_swiglu_quant(h.to(DEV), dt, scale_layout=lay, out=out, out_scale=sc)
        torch.cuda.synchronize()
        r_out, r_sc, st = O.swiglu_quant(bf16_bits(h), None, dt, lay)
        got = bf16_bits(out) if dt == 0 else out.cpu().numpy()
        assert st == 0 and np.array_equal(got, r_out), (dt, lay)
        if sc is not None:
            assert np.array_equal(np.ascontiguousarray(sc.cpu().numpy().reshape(-1)).view(np.uint8),
                                  r_sc.view(np.uint8)), (dt, lay)


def test_mismatched_layout_handle_is_rejected_before_launch():
    """A caller-supplied layout sized for another batch raises in the binding;
    nothing is launched, so nothing can be written out of bounds."""
    from combine_moe_topk_gate_b200 import api
    idx = torch.zeros((10, 2), dtype=torch.int32, device=DEV)
    with pytest.raises(ValueError, match="out.token_slot"):
        api.moe_get_layout(idx, 4, 2, out=api.Layout.empty(8, 2, 4, 2, DEV))       # 8 tokens, not 10
    with pytest.raises(ValueError, match="out.expert_count"):
        api.moe_get_layout(idx, 4, 2, out=api.Layout.empty(10, 2, 8, 2, DEV))      # 8 experts, not 4
    with pytest.raises(ValueError, match="out.rank_count"):
        api.moe_get_layout_noalloc(idx, 4, 2, out=api.Layout.empty(10, 2, 4, 4, DEV))  # 4 ranks, not 2
    with pytest.raises(ValueError, match="d_status"):
        api.moe_combine(torch.zeros((20, 64), dtype=torch.bfloat16, device=DEV), idx,
                        torch.zeros((10, 2), dtype=torch.float32, device=DEV),
                        d_status=torch.zeros(1, dtype=torch.int32))                   # host status word
    # the no-workspace entry point writes the packed layout's N*k rows: a
    # handle with another row count (or an aligned one) is refused
    with pytest.raises(ValueError, match="N\\*k"):
        api.moe_get_layout_noalloc(idx, 4, 2, out=api.Layout.empty(10, 2, 4, 2, DEV, num_rows=12))
    with pytest.raises(ValueError, match="N\\*k"):
        api.moe_get_layout_noalloc(idx, 4, 2, out=api.Layout.empty(10, 2, 4, 2, DEV, align=8))


def test_shape_mismatches_are_rejected_before_launch():
    """Arrays whose shapes disagree with the batch raise in the binding before
    any kernel could read or write past them."""
    from combine_moe_topk_gate_b200 import api
    x = torch.zeros((10, 128), dtype=torch.bfloat16, device=DEV)
    short = torch.zeros((8, 2), dtype=torch.int32, device=DEV)      # 8 tokens' slots for 10 tokens
    for dt in (api.MOE_DTYPE_BF16, api.MOE_DTYPE_FP8_E4M3):
        with pytest.raises(ValueError, match="token_slot"):
            api.moe_dispatch(x, short, dt)
    with pytest.raises(ValueError, match="token_slot"):
        api.moe_dispatch_nvfp4(x, short)
    with pytest.raises(ValueError, match="token_slot"):
        api.moe_dispatch(x, torch.zeros((12, 2), dtype=torch.int32, device=DEV), 0)
    slots = torch.zeros((10, 2), dtype=torch.int32, device=DEV)
    w = torch.zeros((10, 2), dtype=torch.float32, device=DEV)
    y = torch.zeros((20, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError, match="grad_out"):   # fewer rows than tokens
        api.moe_combine_backward(torch.zeros((9, 128), dtype=torch.bfloat16, device=DEV), y, slots, w)
    with pytest.raises(ValueError, match="grad_out"):   # another width than y
        api.moe_combine_backward(torch.zeros((10, 64), dtype=torch.bfloat16, device=DEV), y, slots, w)
    with pytest.raises(ValueError, match="y must be 2-D"):
        api.moe_combine(torch.zeros(20 * 128, dtype=torch.bfloat16, device=DEV), slots, w)
    with pytest.raises(ValueError, match="grad_recv"):
        api.moe_dispatch_backward(torch.zeros(20 * 128, dtype=torch.bfloat16, device=DEV), slots)


def test_stream_of_another_device_is_rejected():
    from combine_moe_topk_gate_b200 import api

    class _OtherDeviceStream:
        device = torch.device("cuda", torch.cuda.device_count())   # a device that is not the tensors'
        cuda_stream = 0
    logits = torch.zeros((4, 8), dtype=torch.float32, device=DEV)
    with pytest.raises(ValueError, match="stream is on"):
        api.moe_topk_gate(logits, 2, api.MOE_GATE_SOFTMAX, stream=_OtherDeviceStream())
