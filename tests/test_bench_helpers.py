"""CPU checks of the measurement helpers: the algorithmic byte counts behind
every roofline fraction, written out here term by term for the two shapes
the headline numbers use, and the kernel count per step."""
import importlib.util
import os

import pytest

from combine_moe_topk_gate_b200.workloads import WORKLOADS, Workload, algorithmic_bytes

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_prefill_bytes():
    # N = 4096 tokens, H = 7168, top-8, FP8 dispatch with one fp32 scale per 128 channels
    b = algorithmic_bytes(WORKLOADS["prefill"])
    x_read = 4096 * 7168 * 2
    codes = 4096 * 8 * 7168
    scales = 4096 * 8 * (7168 // 128) * 4
    slots = 4096 * 8 * 4
    assert b["dispatch"] == x_read + codes + scales + slots == 301_072_384
    y_read = 4096 * 8 * 7168 * 2
    out_write = 4096 * 7168 * 2
    meta = 4096 * 8 * (4 + 4)          # slot ids and weights
    assert b["combine"] == y_read + out_write + meta == 528_744_448


def test_mixtral_bytes():
    # N = 16384, H = 4096, top-2, BF16 dispatch
    b = algorithmic_bytes(WORKLOADS["mixtral"])
    assert b["dispatch"] == 16384 * 4096 * 2 + 16384 * 2 * 4096 * 2 + 16384 * 2 * 4 == 402_784_256
    assert b["combine"] == 16384 * 2 * 4096 * 2 + 16384 * 4096 * 2 + 16384 * 2 * 8 == 402_915_328


@pytest.mark.parametrize("dtype,row,scale", [
    ("bf16", lambda H: 2 * H, lambda H: 0),
    ("fp8", lambda H: H, lambda H: 4 * (H // 128)),
    ("fp8_token", lambda H: H, lambda H: 4),
    ("mxfp8", lambda H: H, lambda H: H // 32),
    ("fp8_ue8m0", lambda H: H, lambda H: H // 128),
    ("nvfp4", lambda H: H // 2, lambda H: H // 16 + 4),
    ("e5m6", lambda H: H // 2 * 3, lambda H: 0),
])
def test_dispatch_bytes_per_payload(dtype, row, scale):
    N, H, k = 300, 1024, 3
    w = Workload("b", N, H, 16, k, 4, "softmax", dtype, "random")
    assert algorithmic_bytes(w)["dispatch"] == 2 * N * H + N * k * (row(H) + scale(H)) + 4 * N * k


def test_launches_per_step():
    bench = _bench()
    assert bench.launches_per_step(WORKLOADS["tiny"]) == 3      # E = 8: the generic gate, still one launch
    assert bench.launches_per_step(WORKLOADS["decode"]) == 3    # N*k = 1024: still one launch
    assert bench.launches_per_step(WORKLOADS["prefill"]) == 5   # gate, count, assign


def test_whole_job_rate_is_tokens_over_time():
    bench = _bench()
    assert bench.whole_job_rate(4096, 2, 10, 20.0) == pytest.approx(4096 * 2 * 10 / 0.020)
