"""The gate's exp and sigmoid, and SwiGLU's silu, through the C ABI on every
one of the 2^32 fp32 bit patterns, bit for bit against the oracle's routines.

Every group-limited routing decision compares sums of these sigmoids, and
every softmax weight is a quotient of these exps, so the two routines must
agree with the oracle on the whole input domain, not only on the values a
seeded batch happens to reach ("DeepSeek, DeepEP 오픈소스 공개", Topic Body:
group-limited gating).  SwiGLU's silu takes shortened steps for |g| <= 87
(no clamp, one corrected quotient from an approximate reciprocal in place of
the IEEE division); its gate values are bf16, so the sweep requires equality
on every bf16 pattern and outside [-87, 87], and at most one unit in the last
place on the other fp32 patterns (DeepSeek Tile-Kernels news, "Funktionen der
DeepSeek-Tile-Kernel": SwiGLU).  The oracle side runs on host threads (ctypes releases
the GIL during the C call); the library side generates its inputs from the
bit-pattern counter, so only the outputs cross PCIe.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

CHUNK = 1 << 26


def _oracle(bits: np.ndarray, threads: int):
    x = bits.view(np.float32)
    parts = np.array_split(np.arange(x.size), threads)
    e = np.empty(x.size, dtype=np.float32)
    s = np.empty(x.size, dtype=np.float32)
    g = np.empty(x.size, dtype=np.float32)

    def work(ix):
        a, b = ix[0], ix[-1] + 1
        e[a:b] = O.dexp_array(x[a:b])
        s[a:b] = O.sigmoid_array(x[a:b])
        g[a:b] = O.silu_array(x[a:b])

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, parts))
    return e, s, g


def _silu_bad(start, got, ref):
    """Patterns where the library's silu breaks its contract: bit equality on
    bf16 patterns and on |x| > 87 (NaN results: any NaN, the payload is not
    part of the definition), at most 1 ulp apart on the rest."""
    bits = np.arange(start, start + got.size, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    gi, ri = got.view(np.uint32).astype(np.int64), ref.view(np.uint32).astype(np.int64)
    both_nan = np.isnan(got) & np.isnan(ref)
    exact = ((bits & 0xFFFF) == 0) | ~(np.abs(x) <= 87.0)
    return ~both_nan & np.where(exact, gi != ri, np.abs(gi - ri) > 1)


def test_exp_sigmoid_silu_every_fp32_pattern_bit_exact():
    from combine_moe_topk_gate_b200 import api
    threads = max(1, min(64, os.cpu_count() or 1))
    e_dev = torch.empty(CHUNK, dtype=torch.float32, device="cuda")
    s_dev = torch.empty(CHUNK, dtype=torch.float32, device="cuda")
    g_dev = torch.empty(CHUNK, dtype=torch.float32, device="cuda")
    e_host = torch.empty(CHUNK, dtype=torch.float32).pin_memory()
    s_host = torch.empty(CHUNK, dtype=torch.float32).pin_memory()
    g_host = torch.empty(CHUNK, dtype=torch.float32).pin_memory()
    checked = 0
    with ThreadPoolExecutor(1) as pre:
        nxt = pre.submit(_oracle, np.arange(0, CHUNK, dtype=np.uint32), threads)
        for start in range(0, 1 << 32, CHUNK):
            api.moe_gate_math(start, CHUNK, exp_out=e_dev, sigmoid_out=s_dev, silu_out=g_dev)
            e_host.copy_(e_dev)
            s_host.copy_(s_dev)
            g_host.copy_(g_dev)
            re, rs, rg = nxt.result()
            if start + CHUNK < (1 << 32):
                nxt = pre.submit(_oracle, np.arange(start + CHUNK, start + 2 * CHUNK, dtype=np.uint64)
                                 .astype(np.uint32), threads)
            ge, gs = e_host.numpy().view(np.uint32), s_host.numpy().view(np.uint32)
            be, bs = ge != re.view(np.uint32), gs != rs.view(np.uint32)
            bg = _silu_bad(start, g_host.numpy(), rg)
            assert not be.any(), f"exp differs at pattern {start + int(np.nonzero(be)[0][0]):#010x}"
            assert not bs.any(), f"sigmoid differs at pattern {start + int(np.nonzero(bs)[0][0]):#010x}"
            assert not bg.any(), f"silu differs at pattern {start + int(np.nonzero(bg)[0][0]):#010x}"
            checked += CHUNK
    assert checked == 1 << 32


def test_gate_math_ragged_run_and_wraparound():
    """A run that is not a multiple of the kernel's four patterns per thread,
    starting near the top of the pattern space so that it wraps to 0."""
    from combine_moe_topk_gate_b200 import api
    n, first = 1001, (1 << 32) - 500
    e, s, g = api.moe_gate_math(first, n)
    bits = ((np.arange(n, dtype=np.uint64) + first) % (1 << 32)).astype(np.uint32)
    re, rs, rg = _oracle(bits, 2)
    assert np.array_equal(e.cpu().numpy().view(np.uint32), re.view(np.uint32))
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert not _silu_bad(first, g.cpu().numpy(), rg).any()
    only_sig = torch.full((n,), -1.0, device="cuda")
    api.lib().moe_gate_math(first, n, None, api._ptr(only_sig), None, api._stream(None, only_sig.device))
    torch.cuda.synchronize()
    assert np.array_equal(only_sig.cpu().numpy().view(np.uint32), rs.view(np.uint32))
