"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element
by element, on the five seeded workloads at their full sizes and on ragged and
degenerate cases.  Routing, layout, FP8 payload and scales must be bit-exact;
combine within one bf16 ulp (and, by the shared fp32 definition, bit-exact)."""
import numpy as np
import pytest
import torch

import oracle as O
from combine_moe_topk_gate_b200.workloads import WORKLOADS, Workload, make_inputs

from _harness import bf16_bits, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

CASES = [(name, seed) for name in ("tiny", "decode", "prefill", "skewed", "mixtral") for seed in (0, 1, 2)]


@pytest.mark.parametrize("name,seed", CASES, ids=[f"{n}-s{s}" for n, s in CASES])
def test_workload_parity(name, seed):
    w = WORKLOADS[name]
    inp = make_inputs(w, seed)
    compare(run_gpu(w, inp), run_oracle(w, inp))


def test_identity_experts_return_x():
    """BF16 dispatch, identity experts, weights summing to 1: combine gives x back."""
    w = WORKLOADS["mixtral"]
    inp = make_inputs(w, 0)
    g = run_gpu(w, inp)
    assert np.array_equal(g["out"], bf16_bits(inp.x))


def test_skewed_load_is_skewed():
    w = WORKLOADS["skewed"]
    inp = make_inputs(w, 0, with_y=False)
    from combine_moe_topk_gate_b200 import api
    idx, _ = api.moe_topk_gate(inp.logits.cuda(), w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn)
    L = api.moe_get_layout(idx, w.E, w.R)
    c = L.expert_count.cpu().numpy()
    assert c.sum() == w.S and c.max() > 4 * c.mean()


RAGGED = [
    Workload("ragged_fp8", 333, 384, 64, 6, 8, "sigmoid_group", "fp8", "random", 8, 3, 2),
    Workload("ragged_bf16", 257, 200, 12, 3, 3, "softmax_renorm", "bf16", "random"),
    Workload("one_token", 1, 128, 4, 1, 1, "softmax", "fp8", "random"),
    Workload("k_equals_E", 50, 64, 8, 8, 4, "softmax", "bf16", "identity"),
    Workload("E33", 100, 136, 33, 5, 3, "softmax", "bf16", "random"),
    Workload("max_E_max_k", 64, 256, 1024, 32, 16, "softmax_renorm", "bf16", "random"),
    Workload("max_E_group", 64, 512, 1024, 32, 32, "sigmoid_group", "fp8", "random", 32, 8, 3),
    Workload("single_group", 200, 256, 64, 8, 8, "sigmoid_group", "fp8", "random", 1, 1, 1),
    Workload("many_groups", 90, 256, 256, 8, 4, "sigmoid_group", "fp8", "random", 64, 16, 2),
    Workload("chunk_edge", 1025, 128, 16, 1, 4, "softmax", "bf16", "random"),
    Workload("k3_chunks", 2000, 128, 24, 3, 6, "softmax_renorm", "bf16", "identity"),
]


@pytest.mark.parametrize("w", RAGGED, ids=[w.name for w in RAGGED])
def test_ragged_and_limits(w):
    inp = make_inputs(w, 3)
    compare(run_gpu(w, inp), run_oracle(w, inp))


def test_empty_batch():
    from combine_moe_topk_gate_b200 import api
    dev = "cuda:0"
    logits = torch.empty((0, 8), dtype=torch.float32, device=dev)
    idx, wts = api.moe_topk_gate(logits, 2, api.MOE_GATE_SOFTMAX)
    L = api.moe_get_layout(idx, 8, 2)
    x = torch.empty((0, 256), dtype=torch.bfloat16, device=dev)
    recv, _ = api.moe_dispatch(x, L.token_slot, api.MOE_DTYPE_BF16)
    out = api.moe_combine(recv, L.token_slot, wts)
    torch.cuda.synchronize()
    assert (L.expert_count.cpu() == 0).all() and (L.expert_offset.cpu() == 0).all()
    assert (L.rank_tokens.cpu() == 0).all() and (L.rank_offset.cpu() == 0).all()
    assert out.shape == (0, 256) and int(L.status.item()) == 0


def test_all_tokens_to_one_expert():
    w = Workload("one_hot", 3000, 256, 32, 2, 4, "softmax", "bf16", "random")
    inp = make_inputs(w, 4)
    inp.logits[:, 7] += 100.0
    g, r = run_gpu(w, inp), run_oracle(w, inp)
    compare(g, r)
    assert r["expert_count"][7] == w.N


def test_masked_and_invalid_ids():
    """-1 entries are masked silently; other out-of-range ids are skipped and set the
    device status word; both sides agree on every output."""
    w = Workload("masked", 500, 256, 16, 4, 4, "softmax", "fp8", "random")
    inp = make_inputs(w, 5)
    rng = np.random.default_rng(0)
    idx = np.stack([rng.choice(16, 4, replace=False) for _ in range(w.N)]).astype(np.int32)
    idx[rng.random(idx.shape) < 0.1] = -1
    g0, r0 = run_gpu(w, inp, topk_idx=torch.from_numpy(idx)), run_oracle(w, inp, topk_idx=idx)
    compare(g0, r0)
    assert g0["status"] == 0
    idx[3, 1] = 16
    idx[77, 0] = -5
    idx[499, 3] = 1 << 30
    g1, r1 = run_gpu(w, inp, topk_idx=torch.from_numpy(idx)), run_oracle(w, inp, topk_idx=idx)
    compare(g1, r1)
    assert g1["status"] == O.ERR_BAD_INDEX


@pytest.mark.parametrize("k", [1, 2, 4, 5, 8])
def test_bulk_combine_every_k_with_masked_slots(k):
    """Sizes past the register kernel (N * k > 4096) so the pipelined kernel
    runs, with its compile-time k (1, 2, 4, 8) or generic (5) consumer; a ragged
    last token group and 10 % masked slots."""
    E = 32
    N = 4096 // k + 37
    w = Workload(f"bulk_k{k}", N, 264, E, k, 4, "softmax", "bf16", "random")
    inp = make_inputs(w, 7)
    rng = np.random.default_rng(k)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(N)]).astype(np.int32)
    idx[rng.random(idx.shape) < 0.1] = -1
    g, r = run_gpu(w, inp, topk_idx=torch.from_numpy(idx)), run_oracle(w, inp, topk_idx=idx)
    compare(g, r)
    assert g["status"] == 0


def test_bad_slots_in_dispatch_and_combine():
    from combine_moe_topk_gate_b200 import api
    N, H, k = 64, 256, 2
    rng = np.random.default_rng(1)
    xf = torch.from_numpy(rng.normal(size=(N, H)).astype(np.float32)).to(torch.bfloat16)
    slots = rng.permutation(N * k).astype(np.int32).reshape(N, k)
    slots[5, 0] = N * k
    slots[9, 1] = -7
    slots[11, 0] = -1
    w_ = rng.random((N, k)).astype(np.float32)
    for dt in (O.DT_BF16, O.DT_FP8_E4M3):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        recv, scale = api.moe_dispatch(xf.cuda(), torch.from_numpy(slots).cuda(), dt, d_status=st)
        torch.cuda.synchronize()
        ref_recv, ref_scale, ref_st = O.dispatch(bf16_bits(xf), slots, dt)
        assert int(st.item()) == ref_st == O.ERR_BAD_INDEX
        ok = slots[(slots >= 0) & (slots < N * k)]
        got = (recv.cpu().numpy() if dt else bf16_bits(recv))[ok]
        assert np.array_equal(got, ref_recv[ok])
        if dt:
            assert np.array_equal(scale.cpu().numpy()[ok], ref_scale[ok])
    y = torch.from_numpy(rng.normal(size=(N * k, H)).astype(np.float32)).to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = api.moe_combine(y.cuda(), torch.from_numpy(slots).cuda(), torch.from_numpy(w_).cuda(), d_status=st)
    torch.cuda.synchronize()
    ref_out, ref_st = O.combine(bf16_bits(y), slots, w_)
    assert int(st.item()) == ref_st == O.ERR_BAD_INDEX
    assert np.array_equal(bf16_bits(out), ref_out)


def _same_codes(got, ref):
    """e4m3 codes equal, NaN codes (0x7f / 0xff) by class: the sign of a NaN
    made by inf * 0 is the host's or the GPU's default, not the definition's."""
    nan = lambda c: (c & 0x7F) == 0x7F
    return bool(np.all((got == ref) | (nan(got) & nan(ref))))


def test_fp8_special_blocks():
    """All-zero, negative-zero, tiny-amax (448/amax overflows fp32), subnormal,
    near-max and mixed-magnitude blocks; blocks holding an infinity or a NaN
    (the kernels' path with NaN fix-ups)."""
    from combine_moe_topk_gate_b200 import api
    H = 128 * 8
    rows = []
    r = np.random.default_rng(2)
    z = np.zeros(H, np.float32)
    rows.append(z.copy())
    nz = z.copy(); nz[::3] = -0.0; rows.append(nz)
    tiny = r.normal(size=H).astype(np.float32) * 1e-37; rows.append(tiny)
    sub = r.normal(size=H).astype(np.float32) * 1e-39; rows.append(sub)
    big = r.normal(size=H).astype(np.float32) * 1e37; rows.append(big)
    mx = np.full(H, 3.38e38, np.float32); mx[1::2] *= -1; rows.append(mx)
    mixed = r.normal(size=H).astype(np.float32) * np.exp2(r.integers(-30, 30, H)).astype(np.float32); rows.append(mixed)
    ties = np.tile(np.array([448, 1, 0.5, 0.25, 3.0 / 64, 13.0 / 1024], np.float32), H // 6 + 1)[:H]; rows.append(ties)
    for special in (np.inf, -np.inf, np.nan):
        row = r.normal(size=H).astype(np.float32)
        row[5] = special                    # one block with it, the others finite
        rows.append(row)
    row = r.normal(size=H).astype(np.float32); row[128:256] = np.nan; rows.append(row)   # an all-NaN block
    xf = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    N, k = xf.shape[0], 3
    slots = np.arange(N * k, dtype=np.int32).reshape(N, k)
    for dt in (O.DT_FP8_E4M3, O.DT_FP8_UE8M0):
        recv, scale = api.moe_dispatch(xf.cuda(), torch.from_numpy(slots).cuda(), dt)
        torch.cuda.synchronize()
        ref_recv, ref_scale, _ = O.dispatch(bf16_bits(xf), slots, dt)
        assert _same_codes(recv.cpu().numpy(), ref_recv)
        assert np.array_equal(np.ascontiguousarray(scale.cpu().numpy()).view(np.uint8).reshape(-1),
                              np.ascontiguousarray(ref_scale).view(np.uint8).reshape(-1))


def test_gate_ties_and_equal_logits():
    w = Workload("ties", 64, 128, 256, 8, 8, "sigmoid_group", "fp8", "random", 8, 4, 2)
    inp = make_inputs(w, 6)
    inp.logits[:16] = 0.5                     # every score equal
    inp.logits[16:32] = torch.round(inp.logits[16:32] * 2) / 2   # many exact ties
    inp.logits[32:40, ::2] = -0.0
    inp.logits[32:40, 1::2] = 0.0
    compare(run_gpu(w, inp), run_oracle(w, inp))
    w2 = Workload("ties_sm", 64, 128, 64, 6, 8, "softmax", "bf16", "random")
    inp2 = make_inputs(w2, 6)
    inp2.logits[:16] = 1.0
    inp2.logits[16:32] = torch.round(inp2.logits[16:32])
    compare(run_gpu(w2, inp2), run_oracle(w2, inp2))


def test_e4m3_encoder_all_fp32_patterns():
    """Every one of the 2^32 fp32 bit patterns through the library's element
    encoder equals the oracle's encoder (NaNs compared by class)."""
    from combine_moe_topk_gate_b200 import api
    chunk = 1 << 28
    dev_in = torch.empty(chunk, dtype=torch.int32, device="cuda")
    dev_out = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    for start in range(0, 1 << 32, chunk):
        bits = np.arange(start, start + chunk, dtype=np.uint64).astype(np.uint32)
        dev_in.copy_(torch.from_numpy(bits.view(np.int32)))
        api.moe_e4m3_encode(dev_in.view(torch.float32), out=dev_out)
        got = dev_out.cpu().numpy()
        ref = O.e4m3_encode_array(bits.view(np.float32))
        assert np.array_equal(got, ref), f"chunk {start:#x}: {np.nonzero(got != ref)[0][:5]}"
