"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of ``oracle/moe_oracle.c`` (a dropped
term, a wrong sign or index, transposed operands, another tie rule), builds it
under a temporary directory and runs the pin suite against it; the suite must
fail.  Everything runs on the CPU; the real oracle is untouched.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTANTS = {
    "exp_drop_7th_taylor_term": ("float p = c7;", "float p = 0.0f;"),
    "exp_drop_ln2_tail": ("r = fmaf(-n, ln2_tail, r);", "r = r + 0.0f;"),
    "sigmoid_wrong_sign": ("float e = oracle_dexp(-x);", "float e = oracle_dexp(x);"),
    "tie_to_higher_index": ("(va == vb && ia < ib)", "(va == vb && ia > ib)"),
    "softmax_renorm_dropped": ("for (int j = 0; j < k; ++j) ow[j] = ow[j] / ps;", "(void)ps;"),
    "group_score_drops_second": ("for (int j = 1; j < group_topn; ++j) sum = sum + gv[gsel[j]];", "(void)0;"),
    "group_candidates_wrong_index": ("cand[(size_t)gsel[j] * eg + i] = 1;", "cand[(size_t)j * eg + i] = 1;"),
    "layout_slot_token_stores_slot_index": ("slot_token[s] = t;", "slot_token[s] = j;", 0),
    "aligned_slot_token_stores_slot_index": ("slot_token[s] = t;", "slot_token[s] = j;", 1),
    "layout_rank_offset_wrong_index": ("rank_count[r] = c;\n        rank_offset[r] = expert_offset[r * epr];",
                                       "rank_count[r] = c;\n        rank_offset[r] = expert_offset[r];"),
    "aligned_rank_offset_wrong_index": ("        rank_offset[r] = expert_offset[r * epr];\n        rank_count[r] = expert_offset[(r + 1) * epr]",
                                        "        rank_offset[r] = expert_offset[r];\n        rank_count[r] = expert_offset[(r + 1) * epr]"),
    "layout_rank_tokens_modulo": ("if (e >= 0 && e < E && e / epr == r) hit = 1;",
                                  "if (e >= 0 && e < E && e % epr == r) hit = 1;", 0),
    "aligned_rank_tokens_modulo": ("if (e >= 0 && e < E && e / epr == r) hit = 1;",
                                   "if (e >= 0 && e < E && e % epr == r) hit = 1;", 1),
    "fp8_scale_transposed": (" sc[b] = amax / 448.0f;", " sc[b] = 448.0f / amax;"),
    "swiglu_fp8_scale_transposed": ("fsc[b] = amax / 448.0f;", "fsc[b] = 448.0f / amax;"),
    "e4m3_ties_away": ("double m = nearbyint(q);                     /* ties to even */",
                       "double m = floor(q + 0.5);", 0),
    "e4m3_subnormal_step": ("double q = a * 512.0;", "double q = a * 256.0;"),
    "bf16_ties_up": ("(lower == 0x8000u && (upper & 1u))", "(lower == 0x8000u)"),
    "combine_weight_index_dropped": ("acc = fmaf(topk_w[(int64_t)t * k + j], v, acc);",
                                     "acc = fmaf(topk_w[(int64_t)t * k], v, acc);"),
    "dispatch_backward_skips_last_slot": ("            for (int j = 0; j < k; ++j) {\n                int32_t s = token_slot[(int64_t)t * k + j];\n                if (s == -1) continue;\n                if (s < -1 || s >= S) { status = ORC_ERR_BAD_INDEX; continue; }\n                acc = acc + ",
                                          "            for (int j = 0; j + 1 < k; ++j) {\n                int32_t s = token_slot[(int64_t)t * k + j];\n                if (s == -1) continue;\n                if (s < -1 || s >= S) { status = ORC_ERR_BAD_INDEX; continue; }\n                acc = acc + "),
    "combine_backward_weight_dropped": ("float prod = topk_w[i] * gc;", "float prod = gc;"),
    "combine_backward_dot_wrong_row": ("double term = (double)gc * (double)oracle_f32_from_bf16(yr[c]);",
                                       "double term = (double)gc * (double)oracle_f32_from_bf16(yr[0]);"),
    "mxfp8_exponent_off_by_one": ("int e = (amax > 0.0f) ? floor_log2_pos(amax) - 8 : -127;",
                                  "int e = (amax > 0.0f) ? floor_log2_pos(amax) - 7 : -127;", 0),
    "swiglu_mxfp8_exponent_off_by_one": ("int e = (amax > 0.0f) ? floor_log2_pos(amax) - 8 : -127;",
                                         "int e = (amax > 0.0f) ? floor_log2_pos(amax) - 7 : -127;", 1),
    "fp8_token_scale_transposed": ("fsc[0] = amax / 448.0f;", "fsc[0] = 448.0f / amax;"),
    "aligned_layout_rounds_down": ("int32_t padded = (expert_count[e] + align - 1) / align * align;",
                                   "int32_t padded = expert_count[e] / align * align;"),
    "dispatch_rows_bound_by_packed_rows": ("    int status = ORC_OK;\n    int64_t S = num_rows;\n    int nb = H / 128;",
                                           "    int status = ORC_OK;\n    int64_t S = (int64_t)N * k;\n    int nb = H / 128;"),
    "mn_major_unpadded_stride": ("if (layout == SL_MN_MAJOR) return (int64_t)b * round_up64(num_rows, 16 / scale_elem_bytes(dtype)) + s;",
                                 "if (layout == SL_MN_MAJOR) return (int64_t)b * num_rows + s;"),
    "mma_tile_row_quarters_swapped": ("return atom * 512 + (s % 32) * 16 + ((s % 128) / 32) * 4 + b % 4;",
                                      "return atom * 512 + ((s % 128) / 32) * 16 + (s % 32) * 4 + b % 4;"),
    "mma_tile_atoms_column_major": ("int64_t atom = (s / 128) * (B / 4) + b / 4;",
                                    "int64_t atom = (b / 4) * ((num_rows + 127) / 128) + s / 128;"),
    "silu_wrong_sign": ("float e = oracle_dexp(-g);", "float e = oracle_dexp(g);"),
    "swiglu_halves_swapped": ("float g = oracle_f32_from_bf16(hr[c]);\n            float u = oracle_f32_from_bf16(hr[I + c]);",
                              "float g = oracle_f32_from_bf16(hr[I + c]);\n            float u = oracle_f32_from_bf16(hr[c]);"),
    "swiglu_padding_not_skipped": ("if (slot_token && slot_token[s] < 0) continue;", "(void)slot_token;"),
    "nvfp4_nibbles_swapped": ("q[c / 2] = (uint8_t)(lo | (hi << 4));", "q[c / 2] = (uint8_t)(hi | (lo << 4));"),
    "nvfp4_ratio_uses_unrounded_block_scale": ("float r = inv / oracle_e4m3_decode(sb[b]);", "float r = inv / sbf;"),
    "nvfp4_block_scale_from_row_amax": ("float sbf = (amax_b / 6.0f) * inv;", "float sbf = (amax_t / 6.0f) * inv;"),
    "nvfp4_row_scale_inverted": ("float g = amax_t / 2688.0f;", "float g = 2688.0f / amax_t;"),
    "e2m1_ties_away": ("if (a < 2.0) return sign | (uint8_t)nearbyint(a * 2.0);", "if (a < 2.0) return sign | (uint8_t)floor(a * 2.0 + 0.5);"),
    "e5m6_ties_away": ("    double m = nearbyint(q);                     /* ties to even */\n    int biased = unb + 15;",
                       "    double m = floor(q + 0.5);\n    int biased = unb + 15;"),
    "e5m6_subnormal_step": ("double m = nearbyint(a * 1048576.0);", "double m = nearbyint(a * 524288.0);"),
    "e5m6_pack_overlaps": ("uint32_t w = c0 | (c1 << 12);", "uint32_t w = c0 | (c1 << 8);"),
    "fp8_channel_amax_over_padded_block": ("int64_t r0 = expert_offset[e], r1 = r0 + expert_count[e];",
                                           "int64_t r0 = expert_offset[e], r1 = expert_offset[e + 1];"),
    "fp8_channel_transpose_index": ("if (transpose) out[(size_t)c * num_rows + s] = q;",
                                    "if (transpose) out[(size_t)c * H + s] = q;"),
    "ue8m0_floor_instead_of_ceil": ("e = (fr == 0.5) ? fe - 1 : fe;", "e = fe - 1;"),
    "ue8m0_ceil_misses_powers_of_two": ("e = (fr == 0.5) ? fe - 1 : fe;", "e = fe;"),
    "ue8m0_infinite_quotient_exponent_zero": ("e = 127;   /* ceil(log2(+inf)) is +inf", "e = 0;   /* ceil(log2(+inf)) is +inf"),
    "pack4_words_row_major": ("return (int64_t)(b / 4) * 4 * round_up64(num_rows, 4) + s * 4 + b % 4;",
                              "return s * 4 * (int64_t)((B + 3) / 4) + (int64_t)(b / 4) * 4 + b % 4;"),
    "combine_no_zero_skip_for_masked": ("if (s == -1) continue;\n                if (s < -1 || s >= S) { status = ORC_ERR_BAD_INDEX; continue; }\n                float v",
                                        "if (s < -1 || s >= S) { status = ORC_ERR_BAD_INDEX; continue; }\n                if (s == -1) s = 0;\n                float v"),
}


def _mutated_source(name: str) -> str:
    src = open(SRC).read()
    old, new, *which = MUTANTS[name]
    if which:   # the anchor occurs in more than one function: mutate occurrence which[0]
        parts = src.split(old)
        assert len(parts) > which[0] + 1, f"mutation anchor occurrence missing: {old!r}"
        return old.join(parts[:which[0] + 1]) + new + old.join(parts[which[0] + 1:])
    assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
    return src.replace(old, new)


def _run_mutant(name: str, work) -> tuple[int, str]:
    """Build the mutated oracle and run the pin suite against it: (return code, tail)."""
    mut = work / f"{name}.c"
    mut.write_text(_mutated_source(name))
    lib = work / f"lib{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                           "-shared", "-w", "-o", str(lib), str(mut), "-lm"])
    env = dict(os.environ, MOE_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    """Every mutant's pin run, several at a time (each is its own process)."""
    from concurrent.futures import ThreadPoolExecutor
    work = tmp_path_factory.mktemp("mutants")
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as pool:
        futs = {n: pool.submit(_run_mutant, n, work) for n in sorted(MUTANTS)}
        return {n: f.result() for n, f in futs.items()}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, mutant_results):
    code, tail = mutant_results[name]
    assert code != 0, f"pins did not catch mutant {name}:\n{tail}"
