"""GPU parity of the per-token FP8 and MXFP8 dispatch payloads against the CPU
oracle: codes and scales bit for bit, on the prefill shape, ragged sizes,
special blocks and bad slots; the rest of the path must be unchanged."""
import numpy as np
import pytest
import torch

import oracle as O
from combine_moe_topk_gate_b200.workloads import WORKLOADS, Workload, make_inputs

from _harness import bf16_bits, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

P = WORKLOADS["prefill"]


def _variant(w, dtype, name=None, **kw):
    return Workload(**{**w.__dict__, "dtype": dtype, "name": name or f"{w.name}-{dtype}", **kw})


CASES = [_variant(P, "fp8_token"), _variant(P, "mxfp8"),
         _variant(WORKLOADS["decode"], "mxfp8"),
         Workload("mx_ragged", 333, 224, 64, 6, 8, "sigmoid_group", "mxfp8", "random", 8, 3, 2),
         Workload("mx_small_h", 77, 96, 16, 3, 4, "softmax", "mxfp8", "random"),
         Workload("tok_ragged", 257, 200, 12, 3, 3, "softmax_renorm", "fp8_token", "random"),
         Workload("tok_max_h", 40, 16384, 32, 4, 4, "softmax", "fp8_token", "random"),
         Workload("tok_min_h", 50, 8, 8, 2, 2, "softmax", "fp8_token", "random"),
         # k <= 4: two 512-channel segments per warp; 1536 = 3 whole segments
         # (16-byte scale stores), 1184 = 2 whole + 160 channels
         Workload("mx_k2", 500, 1536, 16, 2, 4, "softmax", "mxfp8", "random"),
         Workload("mx_k4_ragged", 300, 1184, 16, 4, 4, "softmax_renorm", "mxfp8", "random"),
         Workload("fp8_k2", 500, 1536, 16, 2, 4, "softmax", "fp8", "random"),
         Workload("fp8_k1_ragged", 333, 1152, 8, 1, 2, "softmax", "fp8", "random")]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_variant_parity(w):
    inp = make_inputs(w, 2)
    compare(run_gpu(w, inp), run_oracle(w, inp))


@pytest.mark.parametrize("dtype", [O.DT_FP8_E4M3_TOKEN, O.DT_MXFP8_E4M3])
def test_variant_special_rows_and_bad_slots(dtype):
    from combine_moe_topk_gate_b200 import api
    H = 512
    r = np.random.default_rng(9)
    rows = [np.zeros(H, np.float32)]
    nz = np.zeros(H, np.float32); nz[::3] = -0.0; rows.append(nz)
    rows.append(r.normal(size=H).astype(np.float32) * 1e-37)
    rows.append(r.normal(size=H).astype(np.float32) * 1e-39)
    rows.append(r.normal(size=H).astype(np.float32) * 1e37)
    mx = np.full(H, 3.38e38, np.float32); mx[1::2] *= -1; rows.append(mx)
    rows.append(r.normal(size=H).astype(np.float32) * np.exp2(r.integers(-30, 30, H)).astype(np.float32))
    blk = r.normal(size=H).astype(np.float32); blk[:32] = 0.0; blk[32:64] *= 1e-30; rows.append(blk)
    for special in (np.inf, -np.inf, np.nan):     # the kernels' path with NaN fix-ups
        row = r.normal(size=H).astype(np.float32); row[37] = special; rows.append(row)
    row = r.normal(size=H).astype(np.float32); row[64:96] = np.nan; rows.append(row)
    xf = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    N, k = xf.shape[0], 3
    slots = np.arange(N * k, dtype=np.int32).reshape(N, k)
    slots[1, 2] = N * k + 5          # bad: skipped and reported
    slots[2, 1] = -1                 # masked
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    recv, scale = api.moe_dispatch(xf.cuda(), torch.from_numpy(slots).cuda(), dtype, d_status=st)
    torch.cuda.synchronize()
    ref_recv, ref_scale, ref_st = O.dispatch(bf16_bits(xf), slots, dtype)
    assert int(st.item()) == ref_st == O.ERR_BAD_INDEX
    ok = slots[(slots >= 0) & (slots < N * k)]
    got, ref = recv.cpu().numpy()[ok], ref_recv[ok]
    nan = lambda c: (c & 0x7F) == 0x7F      # NaN codes by class (the sign of inf * 0's NaN)
    assert np.all((got == ref) | (nan(got) & nan(ref)))
    assert np.array_equal(np.ascontiguousarray(scale.cpu().numpy()[ok]).view(np.uint8),
                          np.ascontiguousarray(ref_scale[ok]).view(np.uint8))
