"""GPU parity of the fused SwiGLU + quantisation (moe_swiglu_quant) against
the CPU oracle, bit for bit: output codes (or bf16), scales in every layout,
and the padding rows of an aligned layout left untouched.  Both sides start
from zeroed buffers and the whole buffers are compared.
"""
import numpy as np
import pytest
import torch

import oracle as O
from combine_moe_topk_gate_b200.workloads import WORKLOADS, make_inputs

from _harness import bf16_bits

pytestmark = pytest.mark.gpu

VARIANTS = [("bf16", 0), ("fp8", 0), ("fp8", 1), ("fp8_token", 0), ("fp8_token", 1),
            ("mxfp8", 0), ("mxfp8", 1), ("mxfp8", 2)]


def _h(rows, I, seed):
    g = torch.Generator().manual_seed(seed)
    h = (torch.randn(rows, 2 * I, generator=g) * 2.0)
    h[:, :7] = 0.0                                   # exact zeros (gate and up)
    h[::17, I + 5] = -0.0
    h[::13, 3] = 30.0                                # silu saturates to the identity
    h[::11, I + 9] = 1e4
    # gate values at and beyond the shortened silu's range (|g| <= 87): the
    # lanes holding them take the full steps; -0 keeps its sign
    h[::7, 10] = -0.0
    h[::19, 11] = -100.0
    h[::23, 12] = 87.5
    h[::29, 13] = -87.0
    h[::31, 14] = 87.0
    h[::37, 15] = -1e4
    return h.to(torch.bfloat16)


def _slot_token(workload, align, seed=1):
    from combine_moe_topk_gate_b200 import api
    w = WORKLOADS[workload]
    dev = torch.device("cuda", 0)
    inp = make_inputs(w, seed, with_y=False)
    idx, _ = api.moe_topk_gate(inp.logits.to(dev), w.k, w.gate_kind, w.n_groups, w.topk_groups,
                               w.group_topn)
    rows = api.moe_aligned_recv_rows(w.N, w.k, w.E, align)
    L = api.moe_get_layout(idx, w.E, w.R, align=align, num_recv_rows=rows)
    return L.slot_token


def _run(h_cpu, slot_token, dtype, layout):
    from combine_moe_topk_gate_b200 import api
    from combine_moe_topk_gate_b200.workloads import DTYPES
    dev = torch.device("cuda", 0)
    code = DTYPES[dtype]
    S, I = h_cpu.shape[0], h_cpu.shape[1] // 2
    if code == 0:
        out = torch.zeros((S, I), dtype=torch.bfloat16, device=dev)
        sc = None
    else:
        out = torch.zeros((S, I), dtype=torch.uint8, device=dev)
        shape, sdt = api.scale_shape(S, I, code, layout)
        sc = torch.zeros(shape, dtype=sdt, device=dev)
    api.moe_swiglu_quant(h_cpu.to(dev), code, slot_token=slot_token, scale_layout=layout, out=out,
                         out_scale=sc)
    torch.cuda.synchronize()
    st_np = slot_token.cpu().numpy() if slot_token is not None else None
    r_out, r_sc, st = O.swiglu_quant(bf16_bits(h_cpu), st_np, code, layout)
    assert st == 0
    got = bf16_bits(out) if code == 0 else out.cpu().numpy()
    d = np.argwhere(got != r_out)
    assert len(d) == 0, f"{len(d)} output differences, first at {d[:3].tolist()}"
    if sc is not None:
        g = np.ascontiguousarray(sc.cpu().numpy().reshape(-1)).view(np.uint8)
        assert np.array_equal(g, r_sc.view(np.uint8))


@pytest.mark.parametrize("dtype,layout", VARIANTS, ids=[f"{d}-sl{l}" for d, l in VARIANTS])
def test_swiglu_parity_decode_aligned(dtype, layout):
    """Receive rows of the decode batch at align 128 (padding rows skipped), I = 2048."""
    st = _slot_token("decode", 128)
    _run(_h(st.numel(), 2048, 3), st, dtype, layout)


@pytest.mark.parametrize("dtype,layout", VARIANTS, ids=[f"{d}-sl{l}" for d, l in VARIANTS])
def test_swiglu_parity_ragged_no_slot_token(dtype, layout):
    """1000 rows (not a multiple of any tile), I = 384, every row processed."""
    _run(_h(1000, 384, 4), None, dtype, layout)


@pytest.mark.parametrize("dtype", ["fp8_token", "bf16", "mxfp8"])
def test_swiglu_parity_wide_rows(dtype):
    """I = 14336: the widest per-row FP8 variant (7 vectors of 8 per thread)."""
    _run(_h(37, 14336, 5), None, dtype, 0)


def test_swiglu_parity_prefill_full_size():
    """The prefill receive buffer at align 128 (65280 rows, 32768 of them
    landed) with I = 2048, per-block FP8, MN-major scales."""
    st = _slot_token("prefill", 128)
    _run(_h(st.numel(), 2048, 6), st, "fp8", 1)


def test_swiglu_empty():
    from combine_moe_topk_gate_b200 import api
    dev = torch.device("cuda", 0)
    out, sc = api.moe_swiglu_quant(torch.empty((0, 512), dtype=torch.bfloat16, device=dev),
                                   api.MOE_DTYPE_FP8_E4M3)
    assert out.shape == (0, 256) and sc.shape == (0, 2)
