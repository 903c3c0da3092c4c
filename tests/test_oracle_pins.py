"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test ties one oracle routine to a closed form, a library routine
(torch's bf16 / float8 conversions, float64 exp, stable sorts), a brute-force
search on tiny inputs, a hand-worked example under ``tests/golden/``, or an
invariant of the definition.  No expected value here comes from the CUDA path.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _ulp_err(got, ref64):
    ulp = np.spacing(np.abs(ref64).astype(np.float32)).astype(np.float64)
    return np.abs(got.astype(np.float64) - ref64) / ulp


# ----------------------------------------------------------------- exp
def test_dexp_closed_forms():
    assert O.dexp(0.0) == 1.0
    for n in range(-20, 21):
        # e^(n ln2) = 2^n: within one ulp of e^y for the fp32-rounded y = n ln2
        y = np.float32(n * math.log(2))
        ref = 2.0 ** n * math.exp(float(y) - n * math.log(2))
        got = O.dexp(y)
        assert abs(got - ref) <= np.spacing(np.float32(ref))
        assert abs(got - 2.0 ** n) <= 2.0 ** n * 2e-6
    assert abs(O.dexp(1.0) - math.e) <= np.spacing(np.float32(math.e))


def test_dexp_vs_float64_exp_dense():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.uniform(-87, 88, 1_000_000).astype(np.float32),
                        np.linspace(-1, 1, 200_001, dtype=np.float32),
                        np.linspace(-87, -80, 50_001, dtype=np.float32)])
    got = O.dexp_array(x)
    err = _ulp_err(got, np.exp(x.astype(np.float64)))
    assert err.max() <= 1.0, err.max()          # measured 0.90 ulp
    assert err.mean() < 0.3


def test_dexp_saturation_and_monotone():
    assert O.dexp(-100.0) == O.dexp(-87.0)
    assert O.dexp(100.0) == O.dexp(88.0)
    assert O.dexp(float("inf")) == O.dexp(88.0) and O.dexp(float("-inf")) == O.dexp(-87.0)
    # the clamp takes a NaN input to -87 (NaN is outside the contract; the
    # routine is total so that every fp32 pattern has a defined result)
    nans = np.array([0x7F800001, 0x7FC00000, 0x7FFFFFFF, 0xFF800001, 0xFFC00000], dtype=np.uint32).view(np.float32)
    assert (O.dexp_array(nans) == np.float32(O.dexp(-87.0))).all()        # signalling and quiet NaNs alike
    assert (O.sigmoid_array(nans) == np.float32(1.0)).all()
    x = np.sort(np.random.default_rng(2).uniform(-90, 90, 500_000).astype(np.float32))
    assert (np.diff(O.dexp_array(x)) >= 0).all()


def test_sigmoid_vs_float64():
    assert O.sigmoid(0.0) == 0.5
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.normal(0, 3, 500_000), rng.uniform(-80, 80, 200_000)]).astype(np.float32)
    got = O.sigmoid_array(x)
    ref = 1.0 / (1.0 + np.exp(-x.astype(np.float64)))
    assert _ulp_err(got, ref).max() <= 3.0
    # s(x) + s(-x) = 1 to within rounding
    assert np.abs(got + O.sigmoid_array(-x) - 1.0).max() < 2.5e-7


# ----------------------------------------------------------------- bf16
def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(4)
    bits = rng.integers(0, 2**32, 400_000, dtype=np.uint64).astype(np.uint32)
    # force exact ties and near-ties in the low half
    bits[:1000] = (bits[:1000] & 0xFFFF0000) | 0x8000
    bits[1000:2000] = (bits[1000:2000] & 0xFFFF0000) | 0x7FFF
    bits[2000:3000] = (bits[2000:3000] & 0xFFFF0000) | 0x8001
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    lib = O.lib()
    got = np.array([lib.oracle_bf16_from_f32(float(v)) for v in f[:60_000]], np.uint16)
    ref = torch.from_numpy(f[:60_000].copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    # overflow rounds to infinity
    assert O.bf16_from_f32(3.4028235e38) == 0x7F80
    assert O.f32_from_bf16(0x3F80) == 1.0


# ----------------------------------------------------------------- e4m3
def test_e4m3_spec_points():
    g = _gold("e4m3_ocp_points.json")
    for p in g["points"]:
        code = int(p["code"], 16)
        v = O.e4m3_decode(code)
        assert v == p["value"] and math.copysign(1, v) == math.copysign(1, p["value"]), p
        assert O.e4m3_encode(p["value"]) == code, p
    for c in g["nan_codes"]:
        assert math.isnan(O.e4m3_decode(int(c, 16)))


def _torch_e4m3_decode_table():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_matches_torch_table():
    table = _torch_e4m3_decode_table()
    for c in range(256):
        v = O.e4m3_decode(c)
        if math.isnan(table[c]):
            assert math.isnan(v)
        else:
            assert v == table[c], c


def test_e4m3_encode_brute_force_nearest():
    """Nearest code by exhaustive search over the 127 non-negative finite codes,
    ties to the even code (even mantissa), saturation above 448."""
    table = _torch_e4m3_decode_table()[:127]    # codes 0x00..0x7e, increasing
    rng = np.random.default_rng(5)
    mids = (table[:-1] + table[1:]) / 2.0
    xs = np.concatenate([
        table, mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
        np.nextafter(mids.astype(np.float32), np.float32(1e9)),
        rng.uniform(0, 470, 20_000), np.exp2(rng.uniform(-14, 9, 20_000)),
        [448.0, 463.9, 464.0, 464.1, 500.0, 1e30, np.inf, 2.0**-10, 2.0**-10 * 1.0001, 1e-30],
    ]).astype(np.float32)
    for sign in (1.0, -1.0):
        x = (sign * xs).astype(np.float32)
        got = O.e4m3_encode_array(x)
        a = np.abs(x.astype(np.float64))
        d = np.abs(a[:, None] - table[None, :])
        best = d.min(axis=1, keepdims=True)
        cand = d == best
        codes = np.arange(127)
        # tie -> even code
        pick = np.where(cand.sum(1) > 1,
                        np.array([codes[r][(codes[r] % 2) == 0][0] if r.sum() > 1 else -1 for r in cand]),
                        cand.argmax(1))
        pick = np.where(a >= 448.0, 0x7E, pick)
        expect = pick.astype(np.uint8) | (np.uint8(0x80) if sign < 0 else np.uint8(0))
        assert np.array_equal(got, expect), np.nonzero(got != expect)[0][:10]


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(6)
    x = np.concatenate([rng.normal(0, 100, 300_000), rng.uniform(-448, 448, 100_000),
                        np.exp2(rng.uniform(-12, 8.8, 100_000)) * rng.choice([-1, 1], 100_000)])
    x = np.clip(x, -448, 448).astype(np.float32)
    got = O.e4m3_encode_array(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


# ----------------------------------------------------------------- gate
@pytest.mark.parametrize("case", _gold("gate_worked_examples.json")["cases"], ids=lambda c: c["name"])
def test_gate_worked_examples(case):
    logits = np.array(case["logits"], np.float32)
    idx, w = O.topk_gate(logits, case["k"], case["kind"], case["n_groups"],
                         case["topk_groups"], case["group_topn"])
    assert idx.tolist() == case["idx"]
    assert np.abs(w - np.array(case["w"])).max() <= case["tol"]


def test_gate_softmax_vs_torch_float64():
    rng = np.random.default_rng(7)
    for E, k in [(8, 2), (16, 4), (64, 6), (256, 8)]:
        logits = rng.normal(0, 2, (300, E)).astype(np.float32)
        idx, w = O.topk_gate(logits, k, O.GATE_SOFTMAX)
        ref = torch.softmax(torch.from_numpy(logits).double(), dim=1)
        rv, ri = torch.topk(ref, k, dim=1)
        assert np.array_equal(idx, ri.numpy())
        assert np.abs(w - rv.numpy()).max() <= 4 * np.spacing(np.float32(1.0))
        idx2, w2 = O.topk_gate(logits, k, O.GATE_SOFTMAX_RENORM)
        assert np.array_equal(idx2, idx)
        rn = (rv / rv.sum(1, keepdim=True)).numpy()
        assert np.abs(w2 - rn).max() <= 4 * np.spacing(np.float32(1.0))
        assert np.abs(w2.astype(np.float64).sum(1) - 1).max() <= k * 2.0**-23


def test_gate_softmax_closed_form_two_experts():
    rng = np.random.default_rng(8)
    l = rng.normal(0, 3, (2000, 2)).astype(np.float32)
    idx, w = O.topk_gate(l, 1, O.GATE_SOFTMAX)
    d = np.abs(l[:, 0].astype(np.float64) - l[:, 1])
    expect = 1.0 / (1.0 + np.exp(-d))
    assert np.array_equal(idx[:, 0], np.where(l[:, 1] > l[:, 0], 1, 0))
    assert np.abs(w[:, 0] - expect).max() < 4e-7


def _group_limited_brute(s, G, TG, n, k):
    """Exhaustive reference: every subset of TG groups; the kept set is the one
    with the largest sum of group scores (float64), ties to the subset whose
    sorted group ids are lexicographically smallest; experts by stable sort."""
    E = s.shape[0]
    eg = E // G
    gs = []
    for g in range(G):
        v = np.sort(s[g * eg:(g + 1) * eg])[::-1][:n]
        acc = np.float32(v[0])
        for t in v[1:]:
            acc = np.float32(acc + np.float32(t))
        gs.append(float(acc))
    best, best_key = None, None
    for sub in itertools.combinations(range(G), TG):
        key = (sum(gs[g] for g in sub), [-g for g in sub])
        if best is None or key > best_key:
            best, best_key = sub, key
    cand = [e for g in best for e in range(g * eg, (g + 1) * eg)]
    order = sorted(cand, key=lambda e: (-float(s[e]), e))
    return order[:k], best


def test_gate_group_limited_vs_brute_force():
    rng = np.random.default_rng(9)
    for (E, G, TG, n, k) in [(256, 8, 4, 2, 8), (64, 8, 3, 2, 6), (32, 4, 2, 1, 3), (48, 6, 2, 3, 5)]:
        logits = rng.normal(0, 1, (120, E)).astype(np.float32)
        idx, w = O.topk_gate(logits, k, O.GATE_SIGMOID_GROUP, G, TG, n)
        s = O.sigmoid_array(logits)
        for t in range(logits.shape[0]):
            ref, groups = _group_limited_brute(s[t], G, TG, n, k)
            assert idx[t].tolist() == ref, (E, t)
            assert set(int(e) // (E // G) for e in idx[t]) <= set(groups)
            sel = s[t][idx[t]].astype(np.float64)
            assert np.abs(w[t] - sel / sel.sum()).max() <= 4 * 2.0**-24
            assert (w[t] > 0).all()


def test_gate_single_group_equals_plain_sigmoid_topk():
    rng = np.random.default_rng(10)
    logits = rng.normal(0, 1, (200, 64)).astype(np.float32)
    idx, _ = O.topk_gate(logits, 8, O.GATE_SIGMOID_GROUP, 1, 1, 1)
    s = torch.sigmoid(torch.from_numpy(logits).double())
    _, ri = torch.topk(s, 8, dim=1)
    assert np.array_equal(idx, ri.numpy())


def test_gate_ties_go_to_lower_index():
    logits = np.zeros((3, 16), np.float32)
    logits[1, 5] = 1.0
    logits[2] = -0.0
    logits[2, ::2] = 0.0
    idx, _ = O.topk_gate(logits, 4, O.GATE_SOFTMAX)
    assert idx.tolist() == [[0, 1, 2, 3], [5, 0, 1, 2], [0, 1, 2, 3]]
    idx, _ = O.topk_gate(logits, 4, O.GATE_SIGMOID_GROUP, 4, 2, 2)
    assert idx.tolist()[0] == [0, 1, 2, 3]
    # group 1 (holding expert 5) scores s(1)+s(0); groups 0, 2, 3 tie at 2 s(0) and the
    # lower index (group 0) is kept: experts 5, then 0, 1, 2 by the index tie rule
    assert idx.tolist()[1] == [5, 0, 1, 2]


# ----------------------------------------------------------------- layout
def test_layout_worked_example():
    g = _gold("layout_worked_example.json")
    L = O.get_layout(np.array(g["topk_idx"], np.int32), g["E"], g["R"])
    for key in ("expert_count", "expert_offset", "rank_count", "rank_offset", "rank_tokens",
                "token_slot", "slot_token"):
        assert getattr(L, key).tolist() == g[key], key
    assert L.status == O.OK


def _layout_naive(idx, E, R):
    N, k = idx.shape
    flat = idx.reshape(-1)
    counts = np.array([(flat == e).sum() for e in range(E)], np.int64)
    off = np.concatenate([[0], np.cumsum(counts)])
    token_slot = np.full(N * k, -1, np.int64)
    slot_token = np.full(N * k, -1, np.int64)
    for e in range(E):
        pos = np.nonzero(flat == e)[0]          # ascending (token, slot)
        token_slot[pos] = off[e] + np.arange(len(pos))
        slot_token[off[e] + np.arange(len(pos))] = pos // k
    epr = E // R
    rank_of = np.where((flat >= 0) & (flat < E), flat // epr, -1).reshape(N, k)
    rank_tokens = np.array([(rank_of == r).any(1).sum() for r in range(R)])
    rank_count = counts.reshape(R, epr).sum(1)
    return counts, off, token_slot.reshape(N, k), slot_token, rank_count, rank_tokens


@pytest.mark.parametrize("N,k,E,R,mask", [(1, 1, 1, 1, 0.0), (37, 3, 16, 4, 0.0), (200, 8, 256, 32, 0.0),
                                          (333, 2, 8, 8, 0.1), (64, 6, 12, 3, 0.3)])
def test_layout_vs_naive(N, k, E, R, mask):
    rng = np.random.default_rng(N * 7 + k)
    idx = rng.integers(0, E, (N, k)).astype(np.int32)
    idx[rng.random((N, k)) < mask] = -1
    L = O.get_layout(idx, E, R)
    counts, off, ts, st, rc, rt = _layout_naive(idx, E, R)
    assert np.array_equal(L.expert_count, counts)
    assert np.array_equal(L.expert_offset, off)
    assert np.array_equal(L.token_slot, ts)
    assert np.array_equal(L.slot_token, st)
    assert np.array_equal(L.rank_count, rc)
    assert np.array_equal(L.rank_tokens, rt)
    assert np.array_equal(L.rank_offset, off[::E // R])
    # invariants
    valid = idx >= 0
    assert L.expert_count.sum() == valid.sum() == L.expert_offset[E]
    slots = L.token_slot[valid]
    assert len(np.unique(slots)) == len(slots)                 # each (t,j) exactly once
    assert (L.slot_token[slots] == np.nonzero(valid)[0]).all()  # inverse map
    for e in range(E):                                          # ascending tokens per expert
        seg = L.slot_token[L.expert_offset[e]:L.expert_offset[e + 1]]
        assert (np.diff(seg) >= 0).all()
    assert (L.rank_tokens <= np.minimum(N, L.rank_count)).all()
    assert L.status == O.OK


def test_layout_bad_index_is_skipped_and_reported():
    idx = np.array([[0, 5], [-3, 1], [1, -1]], np.int32)
    L = O.get_layout(idx, 4, 2)
    assert L.status == O.ERR_BAD_INDEX
    assert L.token_slot.tolist() == [[0, -1], [-1, 1], [2, -1]]
    assert L.expert_count.tolist() == [1, 2, 0, 0]
    assert L.slot_token.tolist() == [0, 1, 2, -1, -1, -1]


# ----------------------------------------------------------------- dispatch
def _bf16_bits(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_dispatch_bf16_is_row_copy():
    rng = np.random.default_rng(11)
    N, H, E, k = 50, 136, 8, 3
    x = _bf16_bits(rng.normal(size=(N, H)))
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(N)]).astype(np.int32)
    L = O.get_layout(idx, E, 2)
    recv, sc, st = O.dispatch(x, L.token_slot, O.DT_BF16)
    assert st == O.OK and sc is None
    assert np.array_equal(recv[L.token_slot.reshape(-1)], np.repeat(x, k, axis=0))
    assert np.array_equal(recv[L.slot_token >= 0], x[L.slot_token[L.slot_token >= 0]])


def test_dispatch_fp8_worked_example():
    g = _gold("fp8_block_worked_example.json")
    row = np.zeros(128, np.float32)
    for c, v in g["nonzero"].items():
        row[int(c)] = v
    x = _bf16_bits(row[None, :])
    recv, sc, st = O.dispatch(x, np.array([[0]], np.int32), O.DT_FP8_E4M3)
    assert sc[0, 0] == np.float32(g["scale"])
    for c, code in g["codes"].items():
        assert recv[0, int(c)] == int(code, 16), c


def test_dispatch_fp8_properties():
    rng = np.random.default_rng(12)
    N, H, k = 40, 512, 4
    xf = rng.normal(size=(N, H)).astype(np.float32)
    xf[3, 128:256] = 0.0                          # all-zero block
    xf[4, :128] = -0.0
    xf[5, 256:384] *= 1e-3
    x = _bf16_bits(xf)
    ts = np.arange(N * k, dtype=np.int32).reshape(N, k)
    recv, sc, st = O.dispatch(x, ts, O.DT_FP8_E4M3)
    xv = O.bf16_to_f32(x).astype(np.float32)
    blocks = xv.reshape(N, H // 128, 128)
    amax = np.abs(blocks).max(2)
    # scale is the fp32 division amax/448
    expect_scale = (amax.astype(np.float32) / np.float32(448)).astype(np.float32)
    for j in range(k):
        assert np.array_equal(sc[ts[:, j]], expect_scale)
        assert np.array_equal(recv[ts[:, j]], recv[ts[:, 0]])    # same payload in every slot
    q = recv[ts[:, 0]].reshape(N, H // 128, 128)
    # codes match torch's RNE float8 conversion of x * (448/amax) (fp32 product)
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = (np.float32(448) / amax.astype(np.float32)).astype(np.float32)
        prod = (blocks * inv[:, :, None]).astype(np.float32)
    prod = np.where(blocks == 0, blocks, prod)
    ref = torch.from_numpy(np.clip(prod, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)
    # the element at amax maps to +-448
    am = np.abs(blocks).argmax(2)
    top = np.take_along_axis(q, am[:, :, None], 2)[:, :, 0]
    nz = amax > 0
    assert ((top[nz] & 0x7F) == 0x7E).all()
    # round trip within the e4m3 bound: half a mantissa step (2^-4 relative) or half the
    # subnormal step (2^-10 * scale) in the scaled domain
    deq = _torch_e4m3_decode_table()[q] * sc[ts[:, 0]].astype(np.float64)[:, :, None]
    bound = np.maximum(2.0**-4 * np.abs(blocks), 2.0**-10 * sc[ts[:, 0]][:, :, None]) * (1 + 2.0**-20)
    assert (np.abs(deq - blocks) <= bound).all()
    # zero blocks: scale 0, signed-zero codes
    assert sc[ts[3, 0], 1] == 0.0 and (q[3, 1] == 0).all()
    assert (q[4, 0] == 0x80).all()


def test_dispatch_fp8_tiny_amax_block():
    """448/amax overflows fp32 for amax below ~1.3e-36: non-zero elements saturate,
    zeros keep their sign, the scale is still amax/448."""
    xf = np.zeros((1, 128), np.float32)
    xf[0, 0] = 1e-37
    xf[0, 1] = -5e-38
    xf[0, 2] = -0.0
    x = _bf16_bits(xf)
    recv, sc, st = O.dispatch(x, np.array([[0]], np.int32), O.DT_FP8_E4M3)
    amax = O.bf16_to_f32(x)[0, 0]
    assert sc[0, 0] == np.float32(amax) / np.float32(448)
    assert recv[0, 0] == 0x7E and recv[0, 1] == 0xFE and recv[0, 2] == 0x80 and recv[0, 3] == 0


# ----------------------------------------------------------------- combine
def test_combine_identity_experts_return_x():
    rng = np.random.default_rng(13)
    N, H, E, k = 300, 64, 8, 2
    logits = rng.normal(size=(N, E)).astype(np.float32)
    logits[:, 0] += 2.0
    idx, w = O.topk_gate(logits, k, O.GATE_SOFTMAX_RENORM)
    L = O.get_layout(idx, E, 8)
    x = _bf16_bits(rng.normal(size=(N, H)))
    recv, _, _ = O.dispatch(x, L.token_slot, O.DT_BF16)
    out, st = O.combine(recv, L.token_slot, w)
    assert np.array_equal(out, x)


def test_combine_k1_unit_weight_is_gather():
    rng = np.random.default_rng(14)
    N, H = 64, 40
    y = _bf16_bits(rng.normal(size=(N, H)))
    slot = rng.permutation(N).astype(np.int32).reshape(N, 1)
    out, _ = O.combine(y, slot, np.ones((N, 1), np.float32))
    assert np.array_equal(out, y[slot[:, 0]])


def test_combine_vs_float64_within_one_bf16_ulp():
    rng = np.random.default_rng(15)
    N, H, k = 120, 96, 8
    y = _bf16_bits(rng.normal(size=(N * k, H)))
    slot = rng.permutation(N * k).astype(np.int32).reshape(N, k)
    w = rng.random((N, k)).astype(np.float32)
    w /= w.sum(1, keepdims=True)
    out, _ = O.combine(y, slot, w)
    yv = O.bf16_to_f32(y).astype(np.float64)
    ref = np.einsum("tk,tkh->th", w.astype(np.float64), yv[slot])
    got = O.bf16_to_f32(out).astype(np.float64)
    # |got - ref| <= half a bf16 ulp of ref + the fp32 chain error
    tol = np.abs(ref) * 2.0**-8 + k * 2.0**-24 * np.abs(yv[slot]).max(1) + 1e-30
    assert (np.abs(got - ref) <= tol).all()


def test_combine_linear_in_weights_and_masked_slots():
    rng = np.random.default_rng(16)
    N, H, k = 30, 32, 4
    y = _bf16_bits(rng.integers(-8, 8, size=(N * k, H)))      # small integers: exact sums
    slot = rng.permutation(N * k).astype(np.int32).reshape(N, k)
    w = rng.integers(0, 4, (N, k)).astype(np.float32)
    out, _ = O.combine(y, slot, w)
    yv = O.bf16_to_f32(y)
    ref = np.einsum("tk,tkh->th", w, yv[slot])
    assert np.array_equal(O.bf16_to_f32(out), ref.astype(np.float32))
    slot2 = slot.copy()
    slot2[:, 1] = -1
    out2, st = O.combine(y, slot2, w)
    w2 = w.copy()
    w2[:, 1] = 0
    assert np.array_equal(O.bf16_to_f32(out2), np.einsum("tk,tkh->th", w2, yv[slot]).astype(np.float32))
    assert st == O.OK
    slot2[0, 0] = N * k                                   # out of range: skipped, reported
    _, st = O.combine(y, slot2, w)
    assert st == O.ERR_BAD_INDEX


def test_dispatch_combine_adjoint():
    """<combine(y), g> = <y, w * dispatch(g)> (dispatch and combine are each
    other's backward: DeepEP V2 summary, usage patterns)."""
    rng = np.random.default_rng(17)
    N, H, E, k = 80, 48, 16, 4
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(N)]).astype(np.int32)
    w = rng.random((N, k)).astype(np.float32)
    L = O.get_layout(idx, E, 4)
    y = _bf16_bits(rng.normal(size=(N * k, H)))
    g = _bf16_bits(rng.normal(size=(N, H)))
    out, _ = O.combine(y, L.token_slot, w)
    lhs = (O.bf16_to_f32(out).astype(np.float64) * O.bf16_to_f32(g)).sum()
    dg, _, _ = O.dispatch(g, L.token_slot, O.DT_BF16)
    wslot = np.zeros(N * k)
    wslot[L.token_slot.reshape(-1)] = w.reshape(-1)
    rhs = (O.bf16_to_f32(y).astype(np.float64) * O.bf16_to_f32(dg) * wslot[:, None]).sum()
    assert abs(lhs - rhs) <= 2.0**-8 * np.abs(O.bf16_to_f32(out).astype(np.float64) * O.bf16_to_f32(g)).sum()


# ----------------------------------------------------------------- backward
def test_dispatch_backward_is_slot_sum():
    rng = np.random.default_rng(18)
    N, H, k = 60, 40, 4
    slot = rng.permutation(N * k).astype(np.int32).reshape(N, k)
    slot[rng.random((N, k)) < 0.1] = -1
    g = _bf16_bits(rng.integers(-8, 8, size=(N * k, H)))        # small integers: exact sums
    gx, st = O.dispatch_backward(g, slot)
    gv = O.bf16_to_f32(g).astype(np.float64)
    ref = np.zeros((N, H))
    for t in range(N):
        for j in range(k):
            if slot[t, j] >= 0:
                ref[t] += gv[slot[t, j]]
    assert st == O.OK and np.array_equal(O.bf16_to_f32(gx), ref.astype(np.float32))
    # random values: within one bf16 ulp of the float64 sum
    g2 = _bf16_bits(rng.normal(size=(N * k, H)))
    gx2, _ = O.dispatch_backward(g2, slot)
    gv2 = O.bf16_to_f32(g2).astype(np.float64)
    ref2 = np.zeros((N, H))
    for t in range(N):
        for j in range(k):
            if slot[t, j] >= 0:
                ref2[t] += gv2[slot[t, j]]
    got = O.bf16_to_f32(gx2).astype(np.float64)
    assert (np.abs(got - ref2) <= 2.0**-8 * np.abs(ref2) + k * 2.0**-24 * np.abs(gv2).max() + 1e-30).all()


def test_dispatch_backward_adjoint_of_dispatch():
    """<dispatch_backward(G), x> = <G, dispatch(x)> in exact arithmetic."""
    rng = np.random.default_rng(19)
    N, H, E, k = 50, 32, 12, 3
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(N)]).astype(np.int32)
    L = O.get_layout(idx, E, 3)
    x = _bf16_bits(rng.integers(-4, 5, size=(N, H)))
    G = _bf16_bits(rng.integers(-4, 5, size=(N * k, H)))
    dx, _, _ = O.dispatch(x, L.token_slot, O.DT_BF16)
    gx, _ = O.dispatch_backward(G, L.token_slot)
    lhs = (O.bf16_to_f32(gx).astype(np.float64) * O.bf16_to_f32(x)).sum()
    rhs = (O.bf16_to_f32(G).astype(np.float64) * O.bf16_to_f32(dx)).sum()
    assert lhs == rhs


def test_combine_backward_vs_torch_autograd():
    rng = np.random.default_rng(20)
    N, H, k = 24, 64, 4
    S = N * k
    slot = rng.permutation(S).astype(np.int32).reshape(N, k)
    orphan = int(slot[3, 2])           # the row the masked slot would have used
    slot[3, 2] = -1
    w = rng.random((N, k)).astype(np.float32)
    y = _bf16_bits(rng.normal(size=(S, H)))
    g = _bf16_bits(rng.normal(size=(N, H)))
    gy, gw, mag, st = O.combine_backward(g, y, slot, w)
    assert st == O.OK
    yt = torch.from_numpy(O.bf16_to_f32(y).astype(np.float64)).requires_grad_(True)
    wt = torch.from_numpy(w.astype(np.float64)).requires_grad_(True)
    st_ = torch.from_numpy(np.where(slot >= 0, slot, 0).astype(np.int64))
    mask = torch.from_numpy((slot >= 0).astype(np.float64))
    out = (wt[:, :, None] * mask[:, :, None] * yt[st_]).sum(1)
    gt = torch.from_numpy(O.bf16_to_f32(g).astype(np.float64))
    (out * gt).sum().backward()
    # grad_w: the oracle sums in double, so it matches autograd to double rounding
    assert np.allclose(gw, wt.grad.numpy(), rtol=1e-6, atol=1e-12)
    assert gw[3, 2] == 0.0
    # grad_y = bf16(fp32(w * g)) on every valid row; autograd's float64 value is within one rounding
    valid = slot >= 0
    ref_rows = torch.from_numpy((w[:, :, None] * O.bf16_to_f32(g)[:, None, :]).astype(np.float32))
    ref_bits = ref_rows.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(gy[slot[valid]], ref_bits[valid])
    ag = yt.grad.numpy()[slot[valid]]
    assert np.all(np.abs(O.bf16_to_f32(gy[slot[valid]]) - ag) <= 2.0**-8 * np.abs(ag) + 1e-30)
    assert not gy[orphan].any()        # no slot names it: never written
    # magnitude sums bound the dot products
    assert (np.abs(gw) <= mag * (1 + 1e-6) + 1e-30).all()


# ----------------------------------------------------------------- quantisation variants
def test_mxfp8_worked_example():
    g = _gold("mxfp8_block_worked_example.json")
    row = np.zeros(32, np.float32)
    for c, v in g["nonzero"].items():
        row[int(c)] = v
    x = _bf16_bits(row[None, :])
    recv, sc, st = O.dispatch(x, np.array([[0]], np.int32), O.DT_MXFP8_E4M3)
    assert sc.dtype == np.uint8 and sc[0, 0] == g["e8m0"]
    for c, code in g["codes"].items():
        assert recv[0, int(c)] == int(code, 16), c


def test_mxfp8_properties():
    rng = np.random.default_rng(21)
    N, H, k = 30, 256, 3
    xf = (rng.normal(size=(N, H)) * np.exp2(rng.integers(-20, 20, size=(N, 1)))).astype(np.float32)
    xf[2, :32] = 0.0
    xf[3, 32:64] = -0.0
    x = _bf16_bits(xf)
    ts = np.arange(N * k, dtype=np.int32).reshape(N, k)
    recv, sc, st = O.dispatch(x, ts, O.DT_MXFP8_E4M3)
    xv = O.bf16_to_f32(x).astype(np.float32).reshape(N, H // 32, 32)
    amax = np.abs(xv).max(2)
    mant, ex = np.frexp(amax.astype(np.float64))          # amax = mant * 2^ex, mant in [0.5, 1)
    e = np.where(amax > 0, ex - 1 - 8, -127)
    assert np.array_equal(sc[ts[:, 0]], (e + 127).astype(np.uint8))
    for j in range(k):
        assert np.array_equal(recv[ts[:, j]], recv[ts[:, 0]]) and np.array_equal(sc[ts[:, j]], sc[ts[:, 0]])
    scaled = np.ldexp(xv.astype(np.float64), -e[:, :, None]).astype(np.float32)      # exact
    ref = torch.from_numpy(np.clip(scaled, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    q = recv[ts[:, 0]].reshape(N, H // 32, 32)
    assert np.array_equal(q, ref)
    # the largest element of every non-zero block lands in [256, 448] (saturating above)
    top = np.take_along_axis(q, np.abs(xv).argmax(2)[:, :, None], 2)[:, :, 0] & 0x7F
    assert ((top[amax > 0] >= 0x78) & (top[amax > 0] <= 0x7E)).all()
    assert (q[2, 0] == 0).all() and (q[3, 1] == 0x80).all() and sc[ts[2, 0], 0] == 0


def test_fp8_per_token_properties():
    rng = np.random.default_rng(22)
    N, H, k = 20, 384, 2
    xf = rng.normal(size=(N, H)).astype(np.float32) * np.exp2(rng.integers(-10, 10, size=(N, 1))).astype(np.float32)
    xf[5] = 0.0
    x = _bf16_bits(xf)
    ts = np.arange(N * k, dtype=np.int32).reshape(N, k)
    recv, sc, st = O.dispatch(x, ts, O.DT_FP8_E4M3_TOKEN)
    xv = O.bf16_to_f32(x).astype(np.float32)
    amax = np.abs(xv).max(1)
    assert sc.shape == (N * k, 1)
    assert np.array_equal(sc[ts[:, 1], 0], (amax / np.float32(448)).astype(np.float32))
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = (np.float32(448) / amax).astype(np.float32)
        prod = (xv * inv[:, None]).astype(np.float32)
    prod = np.where(xv == 0, xv, prod)
    ref = torch.from_numpy(np.clip(prod, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(recv[ts[:, 0]], ref) and np.array_equal(recv[ts[:, 1]], ref)
    assert sc[ts[5, 0], 0] == 0.0 and (recv[ts[5, 0]] == 0).all()
    # round trip within the e4m3 bound
    deq = _torch_e4m3_decode_table()[recv[ts[:, 0]]] * sc[ts[:, 0]].astype(np.float64)
    bound = np.maximum(2.0**-4 * np.abs(xv), 2.0**-10 * sc[ts[:, 0]]) * (1 + 2.0**-20)
    assert (np.abs(deq - xv) <= bound).all()


# ----------------------------------------------------------------- aligned layout
def test_layout_aligned_worked_example():
    g = _gold("layout_aligned_worked_example.json")
    L = O.get_layout_aligned(np.array(g["topk_idx"], np.int32), g["E"], g["R"], g["align"], g["num_rows"])
    for key in ("expert_count", "expert_offset", "rank_count", "rank_offset", "rank_tokens",
                "token_slot", "slot_token"):
        assert getattr(L, key).tolist() == g[key], key


@pytest.mark.parametrize("N,k,E,R,align,mask", [(200, 8, 256, 32, 128, 0.0), (333, 2, 8, 8, 16, 0.1),
                                                (64, 6, 12, 3, 8, 0.3), (50, 3, 16, 4, 1, 0.0)])
def test_layout_aligned_vs_naive(N, k, E, R, align, mask):
    rng = np.random.default_rng(N + align)
    idx = rng.integers(0, E, (N, k)).astype(np.int32)
    idx[rng.random((N, k)) < mask] = -1
    rows = N * k + E * (align - 1)
    L = O.get_layout_aligned(idx, E, R, align, rows)
    flat = idx.reshape(-1)
    counts = np.array([(flat == e).sum() for e in range(E)])
    padded = -(-counts // align) * align
    off = np.concatenate([[0], np.cumsum(padded)])
    assert np.array_equal(L.expert_count, counts) and np.array_equal(L.expert_offset, off)
    assert (L.expert_offset % align == 0).all()
    ts = np.full(N * k, -1)
    st = np.full(rows, -1)
    for e in range(E):
        pos = np.nonzero(flat == e)[0]
        ts[pos] = off[e] + np.arange(len(pos))
        st[off[e] + np.arange(len(pos))] = pos // k
    assert np.array_equal(L.token_slot.reshape(-1), ts)
    assert np.array_equal(L.slot_token, st)
    epr = E // R
    assert np.array_equal(L.rank_offset, off[::epr])
    assert np.array_equal(L.rank_count, np.diff(off[::epr]))
    if align == 1:   # reduces to the packed layout
        P = O.get_layout(idx, E, R)
        assert np.array_equal(P.token_slot, L.token_slot) and np.array_equal(P.expert_offset, L.expert_offset)


@pytest.mark.parametrize("dtype", [O.DT_BF16, O.DT_FP8_E4M3, O.DT_FP8_E4M3_TOKEN, O.DT_MXFP8_E4M3])
def test_ops_on_padded_buffer_are_relocations_of_packed(dtype):
    """Where a token's rows sit in the receive buffer changes nothing else: every
    op on the padded (aligned) buffer equals the packed op with its rows moved,
    padding rows are never written, and no in-range slot is reported bad."""
    rng = np.random.default_rng(7 + dtype)
    N, k, E, R, H, align = 90, 3, 12, 4, 256, 16
    idx = rng.integers(0, E, (N, k)).astype(np.int32)
    idx[rng.random((N, k)) < 0.15] = -1
    rows = N * k + E * (align - 1) + 5
    P = O.get_layout(idx, E, R)
    A = O.get_layout_aligned(idx, E, R, align, rows)
    assert A.status == 0 and int(A.token_slot.max()) >= N * k       # some rows beyond N*k
    x = rng.normal(size=(N, H)).astype(np.float32)
    x_bits = (torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    valid = P.token_slot >= 0
    sp, sa = P.token_slot[valid], A.token_slot[valid]

    rp, cp, stp = O.dispatch(x_bits, P.token_slot, dtype)
    ra, ca, sta = O.dispatch(x_bits, A.token_slot, dtype, recv_rows=rows)
    assert stp == 0 and sta == 0
    assert np.array_equal(ra[sa], rp[sp])
    unused = A.slot_token < 0
    assert (ra[unused] == 0).all()
    if cp is not None:
        assert np.array_equal(ca[sa], cp[sp]) and (ca[unused] == 0).all()

    w = rng.random((N, k)).astype(np.float32)
    yp = rng.integers(0, 1 << 16, (N * k, H), dtype=np.uint16) & 0xBFFF     # finite bf16 patterns
    ya = np.zeros((rows, H), np.uint16)
    ya[sa] = yp[sp]
    ya[unused] = 0x7FC0                                                       # NaN padding must not leak
    op, s1 = O.combine(yp, P.token_slot, w)
    oa, s2 = O.combine(ya, A.token_slot, w)
    assert s1 == 0 and s2 == 0 and np.array_equal(oa, op)

    gp, s1 = O.dispatch_backward(yp, P.token_slot)
    ga, s2 = O.dispatch_backward(ya, A.token_slot)
    assert s1 == 0 and s2 == 0 and np.array_equal(ga, gp)

    go = x_bits
    gyp, gwp, mp, s1 = O.combine_backward(go, yp, P.token_slot, w)
    gya, gwa, ma, s2 = O.combine_backward(go, ya, A.token_slot, w)
    assert s1 == 0 and s2 == 0
    assert np.array_equal(gya[sa], gyp[sp]) and (gya[unused] == 0).all()
    assert np.array_equal(gwa, gwp) and np.array_equal(ma, mp)


# ----------------------------------------------------------------- scale layouts
def test_scale_layout_worked_offsets():
    g = _gold("scale_layout_offsets.json")
    for c in g["cases"]:
        assert O.scale_elems(c["num_rows"], c["H"], c["dtype"], c["layout"]) == c["elems"], c
        for s, b, off in c["points"]:
            assert O.scale_index(c["layout"], c["num_rows"], c["H"], c["dtype"], s, b) == off, (c, s, b)
    for layout, dtype, H, rows in g["undefined"]:
        assert O.scale_elems(rows, H, dtype, layout) == -1


def _scaled_case(dtype, seed=0, N=70, k=3, E=6, align=32):
    rng = np.random.default_rng(seed)
    H = 512
    idx = rng.integers(0, E, (N, k)).astype(np.int32)
    idx[rng.random((N, k)) < 0.1] = -1
    rows = N * k + E * (align - 1)
    A = O.get_layout_aligned(idx, E, 2, align, rows)
    x = rng.normal(size=(N, H)) * np.exp2(rng.integers(-6, 6, (N, H // 32))).repeat(32, 1)
    x_bits = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return x_bits, A, rows


@pytest.mark.parametrize("dtype", [O.DT_FP8_E4M3, O.DT_FP8_E4M3_TOKEN, O.DT_MXFP8_E4M3])
def test_scale_layout_mn_major_is_padded_transpose(dtype):
    x_bits, A, rows = _scaled_case(dtype)
    r_recv, r_sc, _ = O.dispatch(x_bits, A.token_slot, dtype, recv_rows=rows)
    m_recv, m_sc, st = O.dispatch_scaled(x_bits, A.token_slot, dtype, O.SL_MN_MAJOR, recv_rows=rows)
    assert st == 0 and np.array_equal(m_recv, r_recv)
    B = r_sc.shape[1]
    ld = -(-rows // (16 // r_sc.itemsize)) * (16 // r_sc.itemsize)
    assert m_sc.size == B * ld and (ld * r_sc.itemsize) % 16 == 0
    assert np.array_equal(m_sc.reshape(B, ld)[:, :rows].T, r_sc)      # zeros where nothing lands
    assert (m_sc.reshape(B, ld)[:, rows:] == 0).all()


def test_scale_layout_mma_tiled_is_blocked_reshape():
    """The tiled E8M0 layout, restated as array reshapes: rows s = 128 i + 32 j + r
    and blocks b = 4 m + n go to index (i, m, r, j, n)."""
    x_bits, A, rows = _scaled_case(O.DT_MXFP8_E4M3, seed=4)
    _, r_sc, _ = O.dispatch(x_bits, A.token_slot, O.DT_MXFP8_E4M3, recv_rows=rows)
    t_recv, t_sc, st = O.dispatch_scaled(x_bits, A.token_slot, O.DT_MXFP8_E4M3, O.SL_MMA_TILED,
                                         recv_rows=rows)
    assert st == 0
    B = r_sc.shape[1]
    Sp = -(-rows // 128) * 128
    padded = np.zeros((Sp, B), np.uint8)
    padded[:rows] = r_sc
    want = padded.reshape(Sp // 128, 4, 32, B // 4, 4).transpose(0, 3, 2, 1, 4).reshape(-1)
    assert np.array_equal(t_sc, want)
    # with align = 128 every expert's scales are one contiguous run of whole atoms
    x2, A2, rows2 = _scaled_case(O.DT_MXFP8_E4M3, seed=5, align=128)
    _, t2, _ = O.dispatch_scaled(x2, A2.token_slot, O.DT_MXFP8_E4M3, O.SL_MMA_TILED, recv_rows=rows2)
    _, r2, _ = O.dispatch(x2, A2.token_slot, O.DT_MXFP8_E4M3, recv_rows=rows2)
    for e in range(len(A2.expert_count)):
        lo, hi = A2.expert_offset[e], A2.expert_offset[e + 1]
        seg = t2[lo * B: hi * B].reshape(-1, B // 4, 32, 4, 4).transpose(0, 3, 2, 1, 4).reshape(hi - lo, B)
        assert np.array_equal(seg, r2[lo:hi])


def test_scale_layout_rejects_undefined_pairs():
    x_bits, A, rows = _scaled_case(O.DT_FP8_E4M3)
    for dt, lay in ((O.DT_FP8_E4M3, O.SL_MMA_TILED), (O.DT_BF16, O.SL_MN_MAJOR)):
        with pytest.raises(ValueError):
            O.dispatch_scaled(x_bits, A.token_slot, dt, lay, recv_rows=rows)


# ----------------------------------------------------------------- SwiGLU + quantisation
def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_swiglu_closed_forms():
    g = np.array([0.0, -0.0, 20.0, 37.5, 1e4, -100.0, -1e30, 1.0], np.float32)
    u = np.array([3.0, 3.0, 1.0, -2.0, 0.5, 1.0, 1.0, 1.0], np.float32)
    I = len(g)
    h = np.concatenate([_bf16(g), _bf16(u)])[None, :]
    out, _, st = O.swiglu_quant(h, None, O.DT_BF16)
    got = O.bf16_to_f32(out[0]).astype(np.float64)
    gb, ub = O.bf16_to_f32(h[0, :I]).astype(np.float64), O.bf16_to_f32(h[0, I:]).astype(np.float64)
    assert st == 0
    assert got[0] == 0 and got[1] == 0
    for i in (2, 3, 4):                                  # 1 + e^-g rounds to 1: silu(g) = g exactly
        assert got[i] == O.bf16_to_f32(_bf16(np.float32(gb[i] * ub[i]))[None])[0]
    assert -1e-36 < got[5] < 0                           # -100 / (1 + e^88): tiny, negative
    assert got[6] == -0.0 or got[6] < 0                  # the exponent is clamped, no NaN
    ref = 1.0 / (1.0 + math.exp(-1.0))                   # silu(1) * 1
    assert abs(got[7] - ref) <= 2.0**-8 * ref


def test_swiglu_vs_float64():
    rng = np.random.default_rng(21)
    S, I = 64, 256
    h = _bf16(rng.normal(scale=2.0, size=(S, 2 * I)))
    out, _, st = O.swiglu_quant(h, None, O.DT_BF16)
    hf = O.bf16_to_f32(h).astype(np.float64)
    g, u = hf[:, :I], hf[:, I:]
    ref = g / (1.0 + np.exp(-g)) * u
    got = O.bf16_to_f32(out).astype(np.float64)
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64) * 2.0**16   # one bf16 ulp
    assert st == 0 and (np.abs(got - ref) <= ulp).all()
    assert (np.abs(got - ref) <= 2.0**-8 * np.abs(ref) * (1 + 2.0**-6) + 1e-38).all()


@pytest.mark.parametrize("dtype,layout", [(O.DT_FP8_E4M3, O.SL_ROW_MAJOR), (O.DT_FP8_E4M3, O.SL_MN_MAJOR),
                                          (O.DT_FP8_E4M3_TOKEN, O.SL_ROW_MAJOR), (O.DT_MXFP8_E4M3, O.SL_ROW_MAJOR),
                                          (O.DT_MXFP8_E4M3, O.SL_MMA_TILED), (O.DT_BF16, O.SL_ROW_MAJOR)])
def test_swiglu_quant_equals_dispatch_of_exact_activations(dtype, layout):
    """With gate >= 20 the SiLU is the identity (1 + e^-g rounds to 1) and with
    up = +-1 or +-0 every a = silu(g) * u is an exact bf16 value: the fused op
    must then quantise exactly as dispatch quantises that bf16 row."""
    rng = np.random.default_rng(33 + dtype)
    S, I = 40, 512
    g = np.exp2(rng.integers(5, 21, (S, I))) * rng.uniform(1, 2, (S, I))
    g = O.bf16_to_f32(_bf16(g)).astype(np.float32)
    u = rng.choice(np.array([1.0, -1.0, 0.0, -0.0], np.float32), (S, I), p=[0.45, 0.45, 0.05, 0.05])
    u[3] = 0.0                                           # an all-zero row
    h = np.concatenate([_bf16(g), _bf16(u)], axis=1)
    a = (g * u).astype(np.float32)
    out, sc, st = O.swiglu_quant(h, None, dtype, layout)
    slots = np.arange(S, dtype=np.int32)[:, None]
    r_out, r_sc, rst = O.dispatch_scaled(_bf16(a), slots, dtype, layout)
    assert st == 0 and rst == 0
    assert np.array_equal(out, r_out)
    if sc is not None:
        assert np.array_equal(sc.view(np.uint8), r_sc.view(np.uint8))


def test_swiglu_skips_padding_rows():
    rng = np.random.default_rng(8)
    S, I = 300, 128
    h = _bf16(rng.normal(size=(S, 2 * I)))
    slot_token = rng.integers(-1, 50, S).astype(np.int32)
    full, fsc, _ = O.swiglu_quant(h, None, O.DT_FP8_E4M3)
    part, psc, st = O.swiglu_quant(h, slot_token, O.DT_FP8_E4M3)
    keep = slot_token >= 0
    assert st == 0 and np.array_equal(part[keep], full[keep]) and (part[~keep] == 0).all()
    assert np.array_equal(psc.reshape(S, -1)[keep], fsc.reshape(S, -1)[keep])
    assert (psc.reshape(S, -1)[~keep] == 0).all()
    for dt, lay, I_bad in ((O.DT_FP8_E4M3, O.SL_ROW_MAJOR, 96), (O.DT_BF16, O.SL_MN_MAJOR, 128),
                           (O.DT_FP8_E4M3, O.SL_MMA_TILED, 128)):
        with pytest.raises(ValueError):
            O.swiglu_quant(h[:, :2 * I_bad], None, dt, lay)


# ----------------------------------------------------------------- FP4 E2M1 and NVFP4
def test_e2m1_decode_table():
    g = _gold("nvfp4_worked_example.json")
    for c in range(16):
        v = O.e2m1_decode(c)
        assert v == g["e2m1_values"][c] and math.copysign(1, v) == math.copysign(1, g["e2m1_values"][c])


def test_e2m1_encode_brute_force_nearest_even():
    """Every bf16 value in [-8, 8] and a dense fp32 grid: the code of the nearest
    E2M1 value, ties to the even mantissa bit, saturating beyond 6."""
    mags = np.array([O.e2m1_decode(c) for c in range(8)])
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = O.bf16_to_f32(bits)
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 8)]
    vals = np.concatenate([vals, np.linspace(-7, 7, 20001, dtype=np.float32), mags.astype(np.float32) + 0.25])
    for v in vals:
        a = abs(float(v))
        d = np.abs(mags - a)
        best = np.flatnonzero(d == d.min())
        code = int(best[0]) if len(best) == 1 else int(best[best % 2 == 0][0])
        if a >= 6:
            code = 7
        code |= 8 if math.copysign(1, float(v)) < 0 else 0
        assert O.e2m1_encode(float(v)) == code, (v, O.e2m1_encode(float(v)), code)


def test_nvfp4_worked_example():
    g = _gold("nvfp4_worked_example.json")
    x0 = np.array(g["x_token0"], np.float32)
    x = np.stack([x0, x0 * np.float32(g["token1_factor"])])
    xb = _bf16(x)
    assert np.array_equal(O.bf16_to_f32(xb), x)                 # every value is exact in bf16
    slots = np.array([[1], [0]], np.int32)                      # token 0 -> row 1, token 1 -> row 0
    recv, bs, rs, st = O.dispatch_nvfp4(xb, slots)
    assert st == 0
    assert recv[1].tolist() == g["codes_token0"] and recv[0].tolist() == g["codes_token0"]
    assert bs.reshape(2, -1)[1].tolist() == g["block_scales"] == bs.reshape(2, -1)[0].tolist()
    assert rs.tolist() == [g["row_scales"][1], g["row_scales"][0]]
    x2 = _bf16(np.array(g["x_token2"], np.float32)[None])
    r2, b2, s2, st = O.dispatch_nvfp4(x2, np.array([[0]], np.int32))
    assert st == 0 and r2[0].tolist() == g["codes_token2"] and b2.tolist() == g["block_scales_token2"]
    assert s2.tolist() == [1.0]


def test_nvfp4_round_trip_bound_and_tiled_layout():
    rng = np.random.default_rng(12)
    N, H, k = 50, 512, 2
    x = rng.normal(size=(N, H)) * np.exp2(rng.integers(-8, 8, (N, H // 16))).repeat(16, 1)
    x[3] = 0.0
    xb = _bf16(x)
    xf = O.bf16_to_f32(xb).astype(np.float64)
    slots = rng.permutation(N * k).astype(np.int32).reshape(N, k)
    recv, bs, rs, st = O.dispatch_nvfp4(xb, slots)
    assert st == 0
    lo, hi = recv & 0xF, recv >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(N * k, H)
    dec = np.array([O.e2m1_decode(c) for c in range(16)])[codes]
    sbv = np.array([O.e4m3_decode(c) for c in range(256)])[bs.reshape(N * k, -1)].repeat(16, 1)
    deq = dec * sbv * rs.astype(np.float64)[:, None]
    ref = xf[np.argsort(slots.reshape(-1)) // k]
    amax_b = np.abs(ref).reshape(N * k, -1, 16).max(-1).repeat(16, 1)
    bound = 1.07 * amax_b / 6 + 6.1 * 2.0**-10 * rs.astype(np.float64)[:, None]
    assert (np.abs(deq - ref) <= bound).all()
    # the largest element of each row decodes within 6.25 % (sb rounds by at most half an e4m3 step)
    row_max = np.abs(ref).max(1)
    assert (np.abs(np.abs(deq).max(1) - row_max) <= 0.0625 * row_max + 1e-30).all()
    # tiled block scales are the same bytes in the block-scaled MMA's order
    rows = N * k
    _, bt, _, _ = O.dispatch_nvfp4(xb, slots, O.SL_MMA_TILED)
    B = H // 16
    Sp = -(-rows // 128) * 128
    padded = np.zeros((Sp, B), np.uint8)
    padded[:rows] = bs.reshape(rows, B)
    assert np.array_equal(bt, padded.reshape(Sp // 128, 4, 32, B // 4, 4).transpose(0, 3, 2, 1, 4).reshape(-1))


# ----------------------------------------------------------------- E5M6
def test_e5m6_decode_is_truncated_fp16():
    """E5M6 code c is the FP16 value with bits c << 4 (same exponent field and
    bias, the top 6 of FP16's 10 fraction bits): checked for all 4096 codes
    against numpy's float16."""
    codes = np.arange(4096, dtype=np.uint16)
    want = (codes << 4).astype(np.uint16).view(np.float16).astype(np.float64)
    got = np.array([O.e5m6_decode(int(c)) for c in codes], np.float64)
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()
    assert np.array_equal(np.signbit(got[~np.isnan(got)]), np.signbit(want[~np.isnan(want)]))


def test_e5m6_encode_brute_force_nearest_even():
    codes = np.arange(0x7C0, dtype=np.int64)                     # non-negative finite codes
    vals = (codes.astype(np.uint16) << 4).view(np.float16).astype(np.float64)
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    xs = O.bf16_to_f32(bits)
    xs = np.concatenate([xs[np.isfinite(xs)], np.float32(vals[1:] - np.diff(vals) / 2),   # exact midpoints
                         np.linspace(-70000, 70000, 4001, dtype=np.float32)])
    for x in xs:
        a = abs(float(x))
        if a >= 65024.0:
            code = 0x7BF
        else:
            i = int(np.searchsorted(vals, a))
            cand = [j for j in (i - 1, i) if 0 <= j < len(vals)]
            d = [abs(vals[j] - a) for j in cand]
            best = [cand[n] for n in range(len(cand)) if d[n] == min(d)]
            code = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        code |= 0x800 if math.copysign(1, float(x)) < 0 else 0
        assert O.e5m6_encode(float(x)) == code, (x, hex(O.e5m6_encode(float(x))), hex(code))


def test_dispatch_e5m6_packs_two_codes_in_three_bytes():
    rng = np.random.default_rng(17)
    N, H, k = 30, 96, 3
    x = _bf16(rng.normal(size=(N, H)) * np.exp2(rng.integers(-24, 17, (N, H))))
    slots = rng.permutation(N * k).astype(np.int32).reshape(N, k)
    slots[4, 2] = -1
    recv, st = O.dispatch_e5m6(x, slots)
    assert st == 0 and recv.shape == (N * k, H // 2 * 3)
    w = recv.reshape(N * k, H // 2, 3).astype(np.uint32)
    word = w[..., 0] | (w[..., 1] << 8) | (w[..., 2] << 16)
    codes = np.stack([word & 0xFFF, word >> 12], -1).reshape(N * k, H)
    xf = O.bf16_to_f32(x)
    for t in range(N):
        for j in range(k):
            s = slots[t, j]
            if s < 0:
                continue
            assert [O.e5m6_encode(float(v)) for v in xf[t]] == codes[s].tolist()
    unused = np.setdiff1d(np.arange(N * k), slots.ravel())          # the masked slot's row
    assert len(unused) == 1 and (recv[unused] == 0).all()


# ----------------------------------------------------------------- per-channel FP8
def _channel_case(seed=0, align=16):
    rng = np.random.default_rng(seed)
    N, k, E, H = 120, 3, 10, 96
    idx = rng.integers(0, E, (N, k)).astype(np.int32)
    idx[rng.random((N, k)) < 0.1] = -1
    idx[idx == 7] = -1                                   # an expert with no rows
    rows = N * k + E * (align - 1)
    L = O.get_layout_aligned(idx, E, 2, align, rows)
    x = rng.normal(size=(rows, H)) * np.exp2(rng.integers(-10, 10, (1, H)))   # per-channel magnitudes
    x[:, 5] = 0.0                                        # an all-zero channel
    return _bf16(x), L, rows


def test_fp8_channel_equals_per_token_rule_on_transposed_columns():
    """Channel c of expert e, read as one 'token row' of the expert's landed rows
    (zero-padded to a multiple of 8), quantised by the per-token FP8 dispatch:
    the same codes and the same scale."""
    x, L, rows = _channel_case()
    codes, sc, st = O.quant_fp8_channel(x, L.expert_offset, L.expert_count)
    assert st == 0
    for e in range(len(L.expert_count)):
        r0, n = int(L.expert_offset[e]), int(L.expert_count[e])
        if n == 0:
            assert (sc[e] == 0).all()
            continue
        cols = np.zeros((x.shape[1], -(-n // 8) * 8), np.uint16)
        cols[:, :n] = x[r0:r0 + n].T
        tq, ts, tst = O.dispatch(cols, np.arange(x.shape[1], dtype=np.int32)[:, None], O.DT_FP8_E4M3_TOKEN)
        assert tst == 0
        assert np.array_equal(codes[r0:r0 + n].T, tq[:, :n])
        assert np.array_equal(sc[e].view(np.uint32), ts[:, 0].view(np.uint32))


def test_fp8_channel_transposed_and_padding():
    x, L, rows = _channel_case(3, align=32)
    c0, s0, _ = O.quant_fp8_channel(x, L.expert_offset, L.expert_count)
    c1, s1, st = O.quant_fp8_channel(x, L.expert_offset, L.expert_count, transpose=True)
    assert st == 0 and np.array_equal(c1, c0.T) and np.array_equal(s0, s1)
    landed = L.slot_token >= 0
    assert (c0[~landed] == 0).all()                      # padding rows are not written
    x2 = x.copy()
    x2[~landed] = 0x7F80                                 # +inf in the padding must not matter
    c2, s2, _ = O.quant_fp8_channel(x2, L.expert_offset, L.expert_count)
    assert np.array_equal(c2, c0) and np.array_equal(s2, s0)


# ----------------------------------------------------------------- FP8 with UE8M0 (power-of-two) 1x128 scales
def test_ue8m0_worked_example():
    g = _gold("ue8m0_worked_example.json")
    H = g["H"]
    x = np.zeros((len(g["tokens"]), H), np.float32)
    for t, tok in enumerate(g["tokens"]):
        for c, v in tok["values"].items():
            x[t, int(c)] = v
    xb = _bf16(x)
    assert np.array_equal(O.bf16_to_f32(xb), x)
    recv, sc, st = O.dispatch(xb, np.arange(len(x), dtype=np.int32)[:, None], O.DT_FP8_UE8M0)
    assert st == 0
    for t, tok in enumerate(g["tokens"]):
        want = np.zeros(H, np.uint8)
        for c, code in tok["codes"].items():
            want[int(c)] = code
        assert recv[t].tolist() == want.tolist(), t
        assert sc[t].tolist() == tok["scale_bytes"], t


def test_ue8m0_is_smallest_power_of_two_not_below_quotient():
    rng = np.random.default_rng(31)
    N, H = 64, 1024
    x = rng.normal(size=(N, H)) * np.exp2(rng.integers(-20, 20, (N, H // 128))).repeat(128, 1)
    x[::7, :128] = 0.0
    xb = _bf16(x)
    xf = O.bf16_to_f32(xb)
    recv, sc, st = O.dispatch(xb, np.arange(N, dtype=np.int32)[:, None], O.DT_FP8_UE8M0)
    assert st == 0
    e = sc.astype(np.int64) - 127
    amax = np.abs(xf).reshape(N, -1, 128).max(-1)
    q = (amax / np.float32(448)).astype(np.float32).astype(np.float64)
    live = amax > 0
    assert (np.exp2(e[live] - 1.0) < q[live]).all() and (q[live] <= np.exp2(e[live].astype(np.float64))).all()
    assert (sc[~live] == 0).all()
    scaled = (xf * np.exp2(-e.repeat(128, 1)).astype(np.float32)).astype(np.float32)
    assert np.array_equal(recv, O.e4m3_encode_array(scaled))


def test_ue8m0_block_with_an_infinity():
    """A block whose amax is infinite: ceil(log2(inf / 448)) is +inf, clamped to
    127 like any exponent beyond the byte (scale byte 254); the factor 2^-127
    takes every finite value of the block to a zero of its sign and the
    infinities to +-448; the other blocks of the row are untouched by it."""
    H = 256
    x = np.zeros((1, H), np.float32)
    x[0, :128] = np.linspace(-3.0, 3.0, 128)
    x[0, 5], x[0, 9] = np.inf, -np.inf
    x[0, 128:] = np.linspace(-1.0, 1.0, 128)
    xb = _bf16(x)
    recv, sc, st = O.dispatch(xb, np.zeros((1, 1), np.int32), O.DT_FP8_UE8M0)
    assert st == 0
    assert sc[0, 0] == 254
    codes = recv[0, :128]
    assert codes[5] == 0x7E and codes[9] == 0xFE                     # +-448
    finite = np.ones(128, bool); finite[[5, 9]] = False
    sign = np.signbit(x[0, :128]).astype(np.uint8) << 7
    assert np.array_equal(codes[finite], sign[finite])                # zeros keep their sign
    q = (np.float32(1.0) / np.float32(448)).astype(np.float32)
    e = int(np.ceil(np.log2(np.float64(np.float32(1.0) * q))))        # amax 1.0: the second block as usual
    assert sc[0, 1] == e + 127


def test_pack4_layout_is_word_transpose():
    rng = np.random.default_rng(5)
    N, k, H = 33, 2, 768                                  # 6 blocks: two words, the second half full
    x = _bf16(rng.normal(size=(N, H)) * np.exp2(rng.integers(-9, 9, (N, H // 128))).repeat(128, 1))
    slots = rng.permutation(N * k).astype(np.int32).reshape(N, k)
    _, row, _ = O.dispatch(x, slots, O.DT_FP8_UE8M0)
    _, packed, st = O.dispatch_scaled(x, slots, O.DT_FP8_UE8M0, O.SL_MN_MAJOR_PACK4)
    assert st == 0
    S, B = row.shape
    ld, G = -(-S // 4) * 4, -(-B // 4)
    padded = np.zeros((ld, G * 4), np.uint8)
    padded[:S, :B] = row
    assert np.array_equal(packed, padded.reshape(ld, G, 4).transpose(1, 0, 2).reshape(-1))
