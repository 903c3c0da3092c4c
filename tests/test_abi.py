"""CPU checks of the C ABI: the library loads, exports every entry point that
``include/*.h`` declares, answers size queries, and rejects invalid arguments
on the host before anything is launched (no compute call needs a GPU here)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def api():
    from combine_moe_topk_gate_b200 import build
    build.build()
    from combine_moe_topk_gate_b200 import api as A
    return A


def test_every_declared_symbol_is_exported(api):
    names = _declared()
    assert {"moe_topk_gate", "moe_get_layout", "moe_dispatch", "moe_combine"} <= set(names)
    L = api.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_size_queries(api):
    assert api.moe_recv_bytes(4096, 7168, 8, api.MOE_DTYPE_FP8_E4M3) == 4096 * 8 * 7168
    assert api.moe_recv_bytes(16384, 4096, 2, api.MOE_DTYPE_BF16) == 16384 * 2 * 4096 * 2
    assert api.moe_scale_bytes(4096, 7168, 8) == 4096 * 8 * 56 * 4
    assert api.moe_scale_bytes(4096, 7168, 8, api.MOE_DTYPE_FP8_E4M3_TOKEN) == 4096 * 8 * 4
    assert api.moe_scale_bytes(4096, 7168, 8, api.MOE_DTYPE_MXFP8_E4M3) == 4096 * 8 * 224
    assert api.moe_scale_bytes(4096, 7168, 8, api.MOE_DTYPE_BF16) == 0
    ws = api.moe_layout_workspace_bytes(4096, 8, 256, 32)
    assert ws >= 256 and ws % 256 == 0
    assert api.moe_layout_workspace_bytes(0, 8, 256, 32) >= 256
    assert api.moe_layout_workspace_bytes(-1, 8, 256, 32) == 0
    assert api.moe_abi_version() >= 1
    assert api.status_string(api.MOE_ERR_BAD_INDEX)


def _P(v=0x1000):
    return ctypes.c_void_p(v)


def test_gate_rejects_bad_arguments(api):
    L = api.lib()
    ok = dict(N=10, E=8, k=2, kind=0, G=1, TG=1, n=1)

    def call(**kw):
        a = {**ok, **kw}
        return L.moe_topk_gate(_P(), a["N"], a["E"], a["k"], a["kind"], a["G"], a["TG"], a["n"],
                               _P(), _P(), None)
    assert call(k=9) == api.MOE_ERR_INVALID_ARG             # k > E
    assert call(k=0) == api.MOE_ERR_INVALID_ARG
    assert call(N=-1) == api.MOE_ERR_INVALID_ARG
    assert call(kind=7) == api.MOE_ERR_INVALID_ARG
    assert call(E=2048, k=4) == api.MOE_ERR_UNSUPPORTED      # beyond MOE_MAX_EXPERTS
    assert call(E=64, k=33) == api.MOE_ERR_UNSUPPORTED       # beyond MOE_MAX_TOPK
    assert call(kind=2, E=256, G=7, TG=4, n=2, k=8) == api.MOE_ERR_INVALID_ARG   # E % G
    assert call(kind=2, E=256, G=8, TG=9, n=2, k=8) == api.MOE_ERR_INVALID_ARG   # TG > G
    assert call(kind=2, E=256, G=8, TG=4, n=33, k=8) == api.MOE_ERR_INVALID_ARG  # n > E/G
    assert call(kind=2, E=256, G=64, TG=1, n=2, k=8) == api.MOE_ERR_INVALID_ARG  # TG*E/G < k
    assert L.moe_topk_gate(None, 10, 8, 2, 0, 1, 1, 1, _P(), _P(), None) == api.MOE_ERR_INVALID_ARG
    assert L.moe_topk_gate(_P(0x1001), 10, 8, 2, 0, 1, 1, 1, _P(), _P(), None) == api.MOE_ERR_INVALID_ARG
    assert call(N=0) == api.MOE_OK                            # empty: nothing enqueued


def test_layout_rejects_bad_arguments(api):
    L = api.lib()
    ws = api.moe_layout_workspace_bytes(100, 4, 16, 4)

    def call(N=100, k=4, E=16, R=4, wsb=ws, idx=_P(), work=_P()):
        return L.moe_get_layout(idx, N, k, E, R, _P(), _P(), _P(), _P(), _P(), _P(), _P(), work, wsb,
                                None, None)
    assert call(R=3) == api.MOE_ERR_INVALID_ARG       # E % R
    assert call(R=0) == api.MOE_ERR_INVALID_ARG
    assert call(wsb=ws - 1) == api.MOE_ERR_INVALID_ARG
    assert call(idx=None) == api.MOE_ERR_INVALID_ARG
    assert call(work=_P(0x1008)) == api.MOE_ERR_INVALID_ARG   # workspace not 16-byte aligned
    assert call(k=40) == api.MOE_ERR_UNSUPPORTED
    assert call(E=2048, R=4) == api.MOE_ERR_UNSUPPORTED
    assert call(N=1 << 29, k=8, wsb=1 << 40) == api.MOE_ERR_UNSUPPORTED   # N*k >= 2^31


def test_aligned_layout_rejects_bad_arguments(api):
    L = api.lib()
    ws = api.moe_layout_workspace_bytes(100, 4, 16, 4)
    need = api.moe_aligned_recv_rows(100, 4, 16, 64)
    assert need == 100 * 4 + 16 * 63
    assert api.moe_aligned_recv_rows(100, 4, 16, 1) == 400
    assert api.moe_aligned_recv_rows(100, 4, 16, 0) == 0

    def call(align=64, rows=need, slot_token=_P(), N=100, k=4, E=16, R=4):
        return L.moe_get_layout_aligned(_P(), N, k, E, R, align, rows, _P(), _P(), _P(), _P(), _P(),
                                        _P(), slot_token, _P(), ws, None, None)
    assert call(align=0) == api.MOE_ERR_INVALID_ARG
    assert call(align=api.MOE_MAX_ALIGN + 1) == api.MOE_ERR_INVALID_ARG
    assert call(rows=need - 1) == api.MOE_ERR_INVALID_ARG      # buffer cannot hold the padded layout
    assert call(slot_token=None) == api.MOE_ERR_INVALID_ARG
    assert call(N=0, rows=16 * 63 - 1) == api.MOE_ERR_INVALID_ARG  # padding alone needs E*(align-1)
    assert call(N=1 << 26, k=32, E=1024, R=4, align=4096, rows=(1 << 31) - 1) == api.MOE_ERR_UNSUPPORTED


def test_dispatch_combine_reject_bad_arguments(api):
    L = api.lib()
    FP8, BF16 = api.MOE_DTYPE_FP8_E4M3, api.MOE_DTYPE_BF16
    S = 20

    def disp(x, N, H, k, dt, recv, scale, rows=S, ts=_P()):
        return L.moe_dispatch(x, N, H, k, ts, rows, dt, recv, scale, None, None)
    assert disp(_P(), 10, 200, 2, FP8, _P(), _P()) == api.MOE_ERR_INVALID_ARG
    assert disp(_P(), 10, 100, 2, BF16, _P(), None) == api.MOE_ERR_INVALID_ARG
    assert disp(_P(), 10, 256, 2, FP8, _P(), None) == api.MOE_ERR_INVALID_ARG
    assert disp(_P(0x1008), 10, 256, 2, BF16, _P(), None) == api.MOE_ERR_INVALID_ARG
    assert disp(_P(), 10, 256, 2, 9, _P(), None) == api.MOE_ERR_INVALID_ARG
    MX, TOK = api.MOE_DTYPE_MXFP8_E4M3, api.MOE_DTYPE_FP8_E4M3_TOKEN
    assert disp(_P(), 10, 272, 2, MX, _P(), _P()) == api.MOE_ERR_INVALID_ARG  # H % 32
    assert disp(_P(), 10, 256, 2, MX, _P(), _P(0x1008)) == api.MOE_ERR_INVALID_ARG  # scales 16-B
    assert disp(_P(), 10, 20000, 2, TOK, _P(), _P()) == api.MOE_ERR_UNSUPPORTED
    assert disp(_P(), 10, 100, 2, TOK, _P(), _P()) == api.MOE_ERR_INVALID_ARG  # H % 8
    assert disp(_P(), 10, 256, 40, BF16, _P(), None) == api.MOE_ERR_UNSUPPORTED
    assert disp(_P(), 10, 256, 2, BF16, _P(), None, rows=-1) == api.MOE_ERR_INVALID_ARG
    assert disp(None, 0, 256, 2, BF16, None, None, rows=0, ts=None) == api.MOE_OK

    def comb(y, N, H, k, w, out, rows=S, ts=_P()):
        return L.moe_combine(y, N, H, k, ts, rows, w, out, None, None)
    assert comb(_P(), 10, 100, 2, _P(), _P()) == api.MOE_ERR_INVALID_ARG
    assert comb(_P(), 10, 256, 2, _P(), None) == api.MOE_ERR_INVALID_ARG
    assert comb(_P(), 10, 256, 2, _P(), _P(0x1004)) == api.MOE_ERR_INVALID_ARG
    assert comb(_P(), 10, 256, 2, _P(), _P(), rows=-5) == api.MOE_ERR_INVALID_ARG
    assert comb(None, 0, 256, 2, None, None, rows=0, ts=None) == api.MOE_OK
    assert L.moe_dispatch_backward(_P(), 10, 100, 2, _P(), S, _P(), None, None) == api.MOE_ERR_INVALID_ARG
    assert L.moe_dispatch_backward(_P(), 10, 256, 2, _P(), -1, _P(), None, None) == api.MOE_ERR_INVALID_ARG
    assert L.moe_combine_backward(_P(), _P(), 10, 100, 2, _P(), S, _P(), _P(), _P(), None, None) \
        == api.MOE_ERR_INVALID_ARG
    assert L.moe_combine_backward(_P(), _P(), 10, 256, 2, _P(), -1, _P(), _P(), _P(), None, None) \
        == api.MOE_ERR_INVALID_ARG
    assert L.moe_e4m3_encode(None, 0, None, None) == api.MOE_OK
    assert L.moe_e4m3_encode(None, 5, _P(), None) == api.MOE_ERR_INVALID_ARG


def test_scale_layout_sizes_and_validation(api):
    L = api.lib()
    FP8, TOK, MX, BF16 = (api.MOE_DTYPE_FP8_E4M3, api.MOE_DTYPE_FP8_E4M3_TOKEN,
                          api.MOE_DTYPE_MXFP8_E4M3, api.MOE_DTYPE_BF16)
    ROW, MN, TILED = api.MOE_SCALE_ROW_MAJOR, api.MOE_SCALE_MN_MAJOR, api.MOE_SCALE_MMA_TILED
    # payload bytes: every e4m3 payload is one byte per element
    for dt in (FP8, TOK, MX):
        assert api.moe_recv_bytes(10, 256, 2, dt) == 10 * 2 * 256
    assert api.moe_recv_scale_bytes(10, 256, FP8, ROW) == 10 * 2 * 4
    assert api.moe_recv_scale_bytes(10, 256, FP8, MN) == 2 * 12 * 4        # ld = 12 (16 bytes)
    assert api.moe_recv_scale_bytes(10, 256, TOK, MN) == 12 * 4
    assert api.moe_recv_scale_bytes(10, 256, MX, MN) == 8 * 16              # ld = 16 bytes
    assert api.moe_recv_scale_bytes(300, 256, MX, TILED) == 384 * 8         # rows padded to 128
    assert api.moe_recv_scale_bytes(300, 224, MX, TILED) == 0               # 7 blocks: not a multiple of 4
    assert api.moe_recv_scale_bytes(300, 256, FP8, TILED) == 0
    assert api.moe_recv_scale_bytes(300, 256, BF16, MN) == 0
    assert api.scale_shape(10, 256, FP8, MN) == ((2, 12), api.torch.float32)
    assert api.scale_shape(300, 256, MX, TILED) == ((3072,), api.torch.uint8)

    def disp(dt, lay, H=256, scale=_P(), rows=20):
        return L.moe_dispatch_ex(_P(), 10, H, 2, _P(), rows, dt, lay, _P(), scale, None, None)
    assert disp(FP8, TILED) == api.MOE_ERR_INVALID_ARG
    assert disp(TOK, TILED) == api.MOE_ERR_INVALID_ARG
    assert disp(BF16, MN, scale=None) == api.MOE_ERR_INVALID_ARG
    assert disp(MX, TILED, H=224) == api.MOE_ERR_INVALID_ARG
    assert disp(MX, 3) == api.MOE_ERR_INVALID_ARG
    assert disp(FP8, MN, scale=_P(0x1004)) == api.MOE_ERR_INVALID_ARG   # 16-byte alignment
    assert disp(FP8, ROW, H=200) == api.MOE_ERR_INVALID_ARG
    assert L.moe_dispatch_ex(None, 0, 256, 2, None, 0, MX, TILED, None, None, None, None) == api.MOE_OK


def test_swiglu_quant_rejects_bad_arguments(api):
    L = api.lib()
    FP8, TOK, MX, BF16 = (api.MOE_DTYPE_FP8_E4M3, api.MOE_DTYPE_FP8_E4M3_TOKEN,
                          api.MOE_DTYPE_MXFP8_E4M3, api.MOE_DTYPE_BF16)
    ROW, MN, TILED = api.MOE_SCALE_ROW_MAJOR, api.MOE_SCALE_MN_MAJOR, api.MOE_SCALE_MMA_TILED

    def call(dt, I, lay=ROW, rows=10, h=_P(), out=_P(), sc=_P(), st=None):
        return L.moe_swiglu_quant(h, rows, I, st, dt, lay, out, sc, None)
    assert call(FP8, 192) == api.MOE_ERR_INVALID_ARG          # I % 128
    assert call(MX, 48) == api.MOE_ERR_INVALID_ARG            # I % 32
    assert call(MX, 96, TILED) == api.MOE_ERR_INVALID_ARG     # tiled needs I % 128
    assert call(BF16, 24) == api.MOE_ERR_INVALID_ARG          # I % 16
    assert call(BF16, 256, MN) == api.MOE_ERR_INVALID_ARG     # bf16 has no scales
    assert call(TOK, 20000) == api.MOE_ERR_UNSUPPORTED
    assert call(FP8, 256, TILED) == api.MOE_ERR_INVALID_ARG
    assert call(FP8, 256, 7) == api.MOE_ERR_INVALID_ARG
    assert call(FP8, 256, sc=None) == api.MOE_ERR_INVALID_ARG
    assert call(FP8, 256, h=_P(0x1008)) == api.MOE_ERR_INVALID_ARG
    assert call(FP8, 256, MN, sc=_P(0x1004)) == api.MOE_ERR_INVALID_ARG
    assert call(FP8, 256, st=_P(0x1002)) == api.MOE_ERR_INVALID_ARG
    assert call(FP8, 256, rows=-1) == api.MOE_ERR_INVALID_ARG
    assert call(FP8, 256, rows=0, h=None, out=None, sc=None) == api.MOE_OK


def test_nvfp4_sizes_and_validation(api):
    L = api.lib()
    NV = api.MOE_DTYPE_NVFP4
    assert api.moe_recv_bytes(10, 256, 2, NV) == 10 * 2 * 128
    assert api.moe_scale_bytes(10, 256, 2, NV) == 10 * 2 * 16
    assert api.moe_recv_scale_bytes(300, 256, NV, api.MOE_SCALE_MMA_TILED) == 384 * 16
    assert api.moe_recv_scale_bytes(10, 256, NV, api.MOE_SCALE_MN_MAJOR) == 16 * 16
    assert api.scale_shape(10, 256, NV) == ((10, 16), api.torch.uint8)

    def call(H=256, lay=0, bs=_P(), rs=_P(), x=_P(), rows=20):
        return L.moe_dispatch_nvfp4(x, 10, H, 2, _P(), rows, lay, _P(), bs, rs, None, None)
    assert call(H=96) == api.MOE_ERR_INVALID_ARG            # H % 64
    assert call(H=32768) == api.MOE_ERR_UNSUPPORTED
    assert call(lay=5) == api.MOE_ERR_INVALID_ARG
    assert call(rs=None) == api.MOE_ERR_INVALID_ARG
    assert call(bs=_P(0x1004)) == api.MOE_ERR_INVALID_ARG    # 16-byte aligned block scales
    assert call(x=_P(0x1008)) == api.MOE_ERR_INVALID_ARG
    assert call(rows=-1) == api.MOE_ERR_INVALID_ARG
    assert L.moe_dispatch_nvfp4(None, 0, 256, 2, None, 0, 0, None, None, None, None, None) == api.MOE_OK
    # the other entry points do not take NVFP4
    assert L.moe_dispatch_ex(_P(), 10, 256, 2, _P(), 20, NV, 0, _P(), _P(), None, None) == api.MOE_ERR_INVALID_ARG
    assert L.moe_swiglu_quant(_P(), 10, 256, None, NV, 0, _P(), _P(), None) == api.MOE_ERR_INVALID_ARG


def test_e5m6_sizes_and_validation(api):
    L = api.lib()
    E5 = api.MOE_DTYPE_E5M6
    assert api.moe_recv_bytes(10, 256, 2, E5) == 10 * 2 * 384
    assert api.moe_scale_bytes(10, 256, 2, E5) == 0
    assert api.moe_recv_scale_bytes(10, 256, E5, api.MOE_SCALE_MN_MAJOR) == 0
    assert L.moe_dispatch_ex(_P(), 10, 272, 2, _P(), 20, E5, 0, _P(), None, None, None) == api.MOE_ERR_INVALID_ARG
    assert L.moe_dispatch_ex(_P(), 10, 256, 2, _P(), 20, E5, 1, _P(), None, None, None) == api.MOE_ERR_INVALID_ARG
    assert L.moe_dispatch_ex(None, 0, 256, 2, None, 0, E5, 0, None, None, None, None) == api.MOE_OK


def test_quant_fp8_channel_rejects_bad_arguments(api):
    L = api.lib()

    def call(S=64, H=256, E=4, tr=0, recv=_P(), out=_P(), sc=_P(), off=_P(), cnt=_P(), ws=None, wsb=0):
        return L.moe_quant_fp8_channel(recv, S, H, E, off, cnt, tr, out, sc, ws, wsb, None, None)
    need = api.moe_quant_fp8_channel_workspace_bytes(4, 256)
    # header, two counters per (expert, 128-channel slab), one amax per (expert, channel)
    assert need == 4 * (64 + 2 * 4 * 2 + 4 * 256)
    assert api.moe_quant_fp8_channel_workspace_bytes(0, 256) == 0
    # used where the average expert holds 256 to 1023 rows
    assert api.moe_quant_fp8_channel_takes_workspace(78336, 256)          # Zipf-skewed, aligned
    assert not api.moe_quant_fp8_channel_takes_workspace(48640, 256)      # prefill, aligned
    assert not api.moe_quant_fp8_channel_takes_workspace(33280, 8)        # Mixtral shape: clusters
    assert api.moe_quant_fp8_channel_takes_workspace(2048, 8) and not api.moe_quant_fp8_channel_takes_workspace(2047, 8)
    assert not api.moe_quant_fp8_channel_takes_workspace(8192, 8) and api.moe_quant_fp8_channel_takes_workspace(8191, 8)
    assert not api.moe_quant_fp8_channel_takes_workspace(-1, 8) and not api.moe_quant_fp8_channel_takes_workspace(100, 0)
    assert api.moe_quant_fp8_channel_workspace_bytes(4, 192) == 0
    assert call(ws=_P(), wsb=need - 4) == api.MOE_ERR_INVALID_ARG   # short workspace
    assert call(ws=_P(0x1008), wsb=need) == api.MOE_ERR_INVALID_ARG  # not 16-byte aligned
    assert call(H=192) == api.MOE_ERR_INVALID_ARG           # H % 128
    assert call(E=0) == api.MOE_ERR_INVALID_ARG
    assert call(E=2000) == api.MOE_ERR_UNSUPPORTED
    assert call(tr=2) == api.MOE_ERR_INVALID_ARG
    assert call(sc=None) == api.MOE_ERR_INVALID_ARG
    assert call(off=None) == api.MOE_ERR_INVALID_ARG
    assert call(recv=_P(0x1008)) == api.MOE_ERR_INVALID_ARG
    assert call(out=_P(0x1002)) == api.MOE_ERR_INVALID_ARG
    assert call(S=-1) == api.MOE_ERR_INVALID_ARG


def test_ue8m0_and_pack4_sizes_and_validation(api):
    L = api.lib()
    U8, FP8, MX = api.MOE_DTYPE_FP8_E4M3_UE8M0, api.MOE_DTYPE_FP8_E4M3, api.MOE_DTYPE_MXFP8_E4M3
    P4 = api.MOE_SCALE_MN_MAJOR_PACK4
    assert api.moe_recv_bytes(10, 768, 2, U8) == 10 * 2 * 768
    assert api.moe_scale_bytes(10, 768, 2, U8) == 10 * 2 * 6
    assert api.moe_recv_scale_bytes(10, 768, U8, P4) == 2 * 4 * 12          # 6 blocks -> 2 words, rows -> 12
    assert api.moe_recv_scale_bytes(10, 768, U8, api.MOE_SCALE_MN_MAJOR) == 6 * 16
    assert api.moe_recv_scale_bytes(10, 768, U8, api.MOE_SCALE_MMA_TILED) == 0
    assert api.moe_recv_scale_bytes(10, 768, MX, P4) == 0
    assert api.scale_shape(10, 768, U8) == ((10, 6), api.torch.uint8)
    assert api.scale_shape(10, 768, U8, P4) == ((96,), api.torch.uint8)

    def disp(dt, lay, H=768, sc=_P()):
        return L.moe_dispatch_ex(_P(), 10, H, 2, _P(), 20, dt, lay, _P(), sc, None, None)
    assert disp(U8, 0, H=192) == api.MOE_ERR_INVALID_ARG                  # H % 128
    assert disp(U8, api.MOE_SCALE_MMA_TILED) == api.MOE_ERR_INVALID_ARG
    assert disp(FP8, P4) == api.MOE_ERR_INVALID_ARG
    assert disp(U8, 4) == api.MOE_ERR_INVALID_ARG
    assert disp(U8, 0, sc=_P(0x1004)) == api.MOE_ERR_INVALID_ARG           # byte scales: 16-byte aligned


def test_selftest_rejects_bad_arguments(api):
    L = api.lib()
    assert L.moe_selftest_bounded_wait(None, None) == api.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_bounded_wait(_P(0x1002), None) == api.MOE_ERR_INVALID_ARG


def test_scale_buffer_sizes_agree_with_the_oracle(api):
    """For every payload type and scale layout, the three independent size
    rules agree: the library's moe_recv_scale_bytes, the binding's
    scale_shape, and the oracle's scale_elems x element size.  Undefined
    pairs are 0 bytes / None / -1 on the three sides."""
    import math

    import oracle as O
    elem = {api.MOE_DTYPE_FP8_E4M3: 4, api.MOE_DTYPE_FP8_E4M3_TOKEN: 4, api.MOE_DTYPE_MXFP8_E4M3: 1,
            api.MOE_DTYPE_NVFP4: 1, api.MOE_DTYPE_FP8_E4M3_UE8M0: 1}
    layouts = [api.MOE_SCALE_ROW_MAJOR, api.MOE_SCALE_MN_MAJOR, api.MOE_SCALE_MMA_TILED,
               api.MOE_SCALE_MN_MAJOR_PACK4]
    checked = 0
    for dtype, es in elem.items():
        for lay in layouts:
            for rows in (1, 3, 4, 15, 16, 127, 128, 129, 1000, 65280):
                for H in (128, 256, 640, 1024, 7168):
                    nbytes = api.moe_recv_scale_bytes(rows, H, dtype, lay)
                    n_or = O.scale_elems(rows, H, dtype, lay)
                    shape, sdt = api.scale_shape(rows, H, dtype, lay)
                    if n_or < 0:
                        assert nbytes == 0 and shape is None, (dtype, lay, rows, H)
                        continue
                    assert nbytes == n_or * es, (dtype, lay, rows, H, nbytes, n_or)
                    assert shape is not None and math.prod(shape) * (1 if sdt == api.torch.uint8 else 4) == nbytes
                    checked += 1
    assert checked > 300


def test_binding_rejects_mixed_devices_and_bad_status_words(api):
    """The binding's own checks, before anything is called: tensors of one
    call on two devices, and a status word that is not device int32."""
    import torch
    called = []
    with pytest.raises(ValueError, match="one CUDA device"):
        api._launch(lambda *a: called.append(a) or 0, "probe",
                    (torch.empty(1), torch.empty(1, device="meta")), 1, 2)
    assert not called
    with pytest.raises(ValueError, match="CUDA tensor"):
        api._status(torch.zeros(1, dtype=torch.int32))
    assert api._status(None) is None


def test_gate_math_rejects_bad_arguments(api):
    L = api.lib()
    assert L.moe_gate_math(0, 0, None, None, None, None) == api.MOE_OK            # empty run
    assert L.moe_gate_math(0, 16, None, None, None, None) == api.MOE_ERR_INVALID_ARG
    assert L.moe_gate_math(0, 16, 260, None, None, None) == api.MOE_ERR_INVALID_ARG   # not 16-byte aligned
    assert L.moe_gate_math(0, 16, None, 264, None, None) == api.MOE_ERR_INVALID_ARG
    assert L.moe_gate_math(0, 16, None, None, 520, None) == api.MOE_ERR_INVALID_ARG


def test_route_rejects_bad_arguments(api):
    L = api.lib()
    p = 256
    ws = api.moe_route_workspace_bytes(64, 8, 256, 8)
    assert ws == api.moe_layout_workspace_bytes(64, 8, 256, 8) + 256 and ws % 256 == 0
    args = lambda **kw: [kw.get("logits", p), kw.get("N", 64), kw.get("E", 256), kw.get("k", 8),
                         kw.get("kind", api.MOE_GATE_SIGMOID_GROUP), kw.get("G", 8), kw.get("TG", 4),
                         kw.get("topn", 2), kw.get("R", 8), kw.get("align", 1), kw.get("rows", 512),
                         p, p, p, p, p, p, p, p, p, kw.get("ws", p), kw.get("wsb", ws),
                         kw.get("pf", None), kw.get("pfb", 0), None, None]
    assert L.moe_route(*args(k=0)) == api.MOE_ERR_INVALID_ARG
    assert L.moe_route(*args(R=3)) == api.MOE_ERR_INVALID_ARG                 # E % R != 0
    assert L.moe_route(*args(G=3)) == api.MOE_ERR_INVALID_ARG                 # E % G != 0
    assert L.moe_route(*args(rows=511)) == api.MOE_ERR_INVALID_ARG            # fewer rows than N*k
    assert L.moe_route(*args(wsb=ws - 1)) == api.MOE_ERR_INVALID_ARG          # short workspace
    assert L.moe_route(*args(ws=p + 4)) == api.MOE_ERR_INVALID_ARG            # workspace not 16-byte aligned
    assert L.moe_route(*args(E=2048, k=8, G=8)) == api.MOE_ERR_UNSUPPORTED
    assert L.moe_route(*args(align=0)) == api.MOE_ERR_INVALID_ARG
    assert L.moe_route(*args(pf=None, pfb=4096)) == api.MOE_ERR_INVALID_ARG     # prefetch size without a buffer
    assert L.moe_route(*args(pf=p + 8, pfb=4096)) == api.MOE_ERR_INVALID_ARG    # prefetch not 16-byte aligned
