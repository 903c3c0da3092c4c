"""CPU oracle for the MoE top-k gate / layout / dispatch / combine path.

TEST INFRASTRUCTURE ONLY.  The tests, the package's ``smoke()`` check and the
benchmark's CPU-baseline leg are the only callers.  The product library never
imports this package and this package never imports the product: the two share
no code.  The arithmetic lives in ``moe_oracle.c`` (plain single-threaded C,
built with ``-O2 -ffp-contract=off``); this module only marshals numpy arrays.

Arrays: bf16 data is carried as ``numpy.uint16`` bit patterns, FP8 e4m3 as
``numpy.uint8`` codes, indices as ``int32``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

GATE_SOFTMAX = 0
GATE_SOFTMAX_RENORM = 1
GATE_SIGMOID_GROUP = 2
DT_BF16 = 0
DT_FP8_E4M3 = 1
DT_FP8_E4M3_TOKEN = 2
DT_MXFP8_E4M3 = 3
DT_NVFP4 = 4
DT_E5M6 = 5
DT_FP8_UE8M0 = 6
SL_ROW_MAJOR = 0
SL_MN_MAJOR = 1
SL_MMA_TILED = 2
SL_MN_MAJOR_PACK4 = 3
OK = 0
ERR_INVALID_ARG = 1
ERR_BAD_INDEX = 4

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source (gcc, plain C)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    """The oracle library.  ``MOE_ORACLE_LIB`` may name another build of the same
    source (the mutation test loads deliberately broken copies this way)."""
    global _lib
    if _lib is None:
        path = os.environ.get("MOE_ORACLE_LIB") or build()
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t


def _declare(L):
    L.oracle_dexp.argtypes = [ctypes.c_float]
    L.oracle_dexp.restype = ctypes.c_float
    L.oracle_sigmoid.argtypes = [ctypes.c_float]
    L.oracle_sigmoid.restype = ctypes.c_float
    L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    L.oracle_e4m3_encode.restype = ctypes.c_uint8
    L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_decode.restype = ctypes.c_float
    L.oracle_e5m6_encode.argtypes = [ctypes.c_float]
    L.oracle_e5m6_encode.restype = ctypes.c_uint16
    L.oracle_e5m6_decode.argtypes = [ctypes.c_uint16]
    L.oracle_e5m6_decode.restype = ctypes.c_float
    L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
    L.oracle_e2m1_encode.restype = ctypes.c_uint8
    L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
    L.oracle_e2m1_decode.restype = ctypes.c_float
    L.oracle_bf16_from_f32.argtypes = [ctypes.c_float]
    L.oracle_bf16_from_f32.restype = ctypes.c_uint16
    L.oracle_f32_from_bf16.argtypes = [ctypes.c_uint16]
    L.oracle_f32_from_bf16.restype = ctypes.c_float
    for name in ("oracle_e4m3_encode_array", "oracle_dexp_array", "oracle_sigmoid_array",
                 "oracle_silu_array"):
        getattr(L, name).argtypes = [_P, _P, _SZ]
        getattr(L, name).restype = None
    L.oracle_topk_gate.argtypes = [_P, _I, _I, _I, _I, _I, _I, _I, _P, _P]
    L.oracle_topk_gate.restype = _I
    L.oracle_get_layout.argtypes = [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]
    L.oracle_get_layout.restype = _I
    _L64 = ctypes.c_int64
    L.oracle_get_layout_aligned.argtypes = [_P, _I, _I, _I, _I, _I, _L64, _P, _P, _P, _P, _P, _P, _P]
    L.oracle_get_layout_aligned.restype = _I
    L.oracle_dispatch.argtypes = [_P, _I, _I, _I, _P, _I, _P, _P]
    L.oracle_dispatch.restype = _I
    L.oracle_dispatch_rows.argtypes = [_P, _I, _I, _I, _P, _L64, _I, _P, _P]
    L.oracle_dispatch_rows.restype = _I
    L.oracle_scale_elems.argtypes = [_L64, _I, _I, _I]
    L.oracle_scale_elems.restype = _L64
    L.oracle_scale_index.argtypes = [_I, _L64, _I, _I, _L64, _I]
    L.oracle_scale_index.restype = _L64
    L.oracle_dispatch_scaled.argtypes = [_P, _I, _I, _I, _P, _L64, _I, _I, _P, _P]
    L.oracle_dispatch_scaled.restype = _I
    L.oracle_dispatch_e5m6.argtypes = [_P, _I, _I, _I, _P, _L64, _P]
    L.oracle_dispatch_e5m6.restype = _I
    L.oracle_dispatch_nvfp4.argtypes = [_P, _I, _I, _I, _P, _L64, _I, _P, _P, _P]
    L.oracle_dispatch_nvfp4.restype = _I
    L.oracle_quant_fp8_channel.argtypes = [_P, _L64, _I, _I, _P, _P, _I, _P, _P]
    L.oracle_quant_fp8_channel.restype = _I
    L.oracle_swiglu_quant.argtypes = [_P, _L64, _I, _P, _I, _I, _P, _P]
    L.oracle_swiglu_quant.restype = _I
    L.oracle_combine.argtypes = [_P, _L64, _I, _I, _I, _P, _P, _P]
    L.oracle_combine.restype = _I
    L.oracle_dispatch_backward.argtypes = [_P, _L64, _I, _I, _I, _P, _P]
    L.oracle_dispatch_backward.restype = _I
    L.oracle_combine_backward.argtypes = [_P, _P, _L64, _I, _I, _I, _P, _P, _P, _P, _P]
    L.oracle_combine_backward.restype = _I


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- scalars
def dexp(y: float) -> float:
    return lib().oracle_dexp(y)


def sigmoid(x: float) -> float:
    return lib().oracle_sigmoid(x)


def e4m3_encode(f: float) -> int:
    return lib().oracle_e4m3_encode(f)


def e5m6_encode(f: float) -> int:
    return int(lib().oracle_e5m6_encode(f))


def e5m6_decode(c: int) -> float:
    return float(lib().oracle_e5m6_decode(c))


def dispatch_e5m6(x_bf16: np.ndarray, token_slot: np.ndarray, recv_rows: int | None = None):
    """E5M6 dispatch: (recv_x uint8 [S, 3H/2] (two 12-bit codes per 3 bytes), status)."""
    x_bf16 = _c(x_bf16, np.uint16)
    token_slot = _c(token_slot, np.int32)
    N, H = x_bf16.shape
    k = token_slot.shape[1]
    S = N * k if recv_rows is None else recv_rows
    recv = np.zeros((S, H // 2 * 3), np.uint8)
    st = lib().oracle_dispatch_e5m6(_ptr(x_bf16), N, H, k, _ptr(token_slot), S, _ptr(recv))
    if st == ERR_INVALID_ARG:
        raise ValueError("oracle_dispatch_e5m6: invalid argument")
    return recv, st


def e2m1_encode(f: float) -> int:
    return int(lib().oracle_e2m1_encode(f))


def e2m1_decode(c: int) -> float:
    return float(lib().oracle_e2m1_decode(c))


def e4m3_decode(c: int) -> float:
    return lib().oracle_e4m3_decode(c)


def bf16_from_f32(f: float) -> int:
    return lib().oracle_bf16_from_f32(f)


def f32_from_bf16(h: int) -> float:
    return lib().oracle_f32_from_bf16(h)


# ---------------------------------------------------------------- arrays
def e4m3_encode_array(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(x), _ptr(out), x.size)
    return out


def dexp_array(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.float32)
    lib().oracle_dexp_array(_ptr(x), _ptr(out), x.size)
    return out


def sigmoid_array(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.float32)
    lib().oracle_sigmoid_array(_ptr(x), _ptr(out), x.size)
    return out


def silu_array(x: np.ndarray) -> np.ndarray:
    """silu(g) = g / (1 + dexp(-g)) of SwiGLU, fp32, each operation rounded once."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.float32)
    lib().oracle_silu_array(_ptr(x), _ptr(out), x.size)
    return out


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    h = np.asarray(h, np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- steps
def topk_gate(logits: np.ndarray, k: int, kind: int, n_groups: int = 1,
              topk_groups: int = 1, group_topn: int = 1):
    logits = _c(logits, np.float32)
    N, E = logits.shape
    idx = np.empty((N, k), np.int32)
    w = np.empty((N, k), np.float32)
    st = lib().oracle_topk_gate(_ptr(logits), N, E, k, kind, n_groups, topk_groups,
                                group_topn, _ptr(idx), _ptr(w))
    if st != OK:
        raise ValueError(f"oracle_topk_gate status {st}")
    return idx, w


@dataclass
class Layout:
    expert_count: np.ndarray
    expert_offset: np.ndarray
    rank_count: np.ndarray
    rank_offset: np.ndarray
    rank_tokens: np.ndarray
    token_slot: np.ndarray
    slot_token: np.ndarray
    status: int


def get_layout(topk_idx: np.ndarray, E: int, R: int) -> Layout:
    topk_idx = _c(topk_idx, np.int32)
    N, k = topk_idx.shape
    L = Layout(np.empty(E, np.int32), np.empty(E + 1, np.int32), np.empty(R, np.int32),
               np.empty(R + 1, np.int32), np.empty(R, np.int32), np.empty((N, k), np.int32),
               np.empty(N * k, np.int32), OK)
    st = lib().oracle_get_layout(_ptr(topk_idx), N, k, E, R, _ptr(L.expert_count),
                                 _ptr(L.expert_offset), _ptr(L.rank_count), _ptr(L.rank_offset),
                                 _ptr(L.rank_tokens), _ptr(L.token_slot), _ptr(L.slot_token))
    if st == ERR_INVALID_ARG:
        raise ValueError("oracle_get_layout: invalid argument")
    L.status = st
    return L


def get_layout_aligned(topk_idx: np.ndarray, E: int, R: int, align: int, num_rows: int) -> Layout:
    """Layout whose experts start at multiples of ``align`` rows; ``slot_token``
    covers ``num_rows`` rows (-1 where no token lands)."""
    topk_idx = _c(topk_idx, np.int32)
    N, k = topk_idx.shape
    L = Layout(np.empty(E, np.int32), np.empty(E + 1, np.int32), np.empty(R, np.int32),
               np.empty(R + 1, np.int32), np.empty(R, np.int32), np.empty((N, k), np.int32),
               np.empty(num_rows, np.int32), OK)
    st = lib().oracle_get_layout_aligned(_ptr(topk_idx), N, k, E, R, align, num_rows,
                                         _ptr(L.expert_count), _ptr(L.expert_offset),
                                         _ptr(L.rank_count), _ptr(L.rank_offset), _ptr(L.rank_tokens),
                                         _ptr(L.token_slot), _ptr(L.slot_token))
    if st == ERR_INVALID_ARG:
        raise ValueError("oracle_get_layout_aligned: invalid argument")
    L.status = st
    return L


def dispatch(x_bf16: np.ndarray, token_slot: np.ndarray, dtype: int,
             recv_rows: int | None = None):
    """Returns (recv_x, recv_scale or None, status).  Rows no slot names stay 0.
    recv_scale: fp32 [S, H/128] (per block), fp32 [S, 1] (per token) or uint8
    E8M0 bytes [S, H/32] (MXFP8)."""
    x_bf16 = _c(x_bf16, np.uint16)
    token_slot = _c(token_slot, np.int32)
    N, H = x_bf16.shape
    k = token_slot.shape[1]
    S = N * k if recv_rows is None else recv_rows
    if dtype == DT_BF16:
        recv = np.zeros((S, H), np.uint16)
        scale = None
        sp = None
    else:
        recv = np.zeros((S, H), np.uint8)
        if dtype == DT_FP8_E4M3:
            scale = np.zeros((S, H // 128), np.float32)
        elif dtype == DT_FP8_E4M3_TOKEN:
            scale = np.zeros((S, 1), np.float32)
        elif dtype == DT_FP8_UE8M0:                 # UE8M0 bytes, one per 128 channels
            scale = np.zeros((S, H // 128), np.uint8)
        else:                                   # MXFP8: E8M0 bytes, one per 32 channels
            scale = np.zeros((S, H // 32), np.uint8)
        sp = _ptr(scale)
    st = lib().oracle_dispatch_rows(_ptr(x_bf16), N, H, k, _ptr(token_slot), S, dtype, _ptr(recv), sp)
    if st == ERR_INVALID_ARG:
        raise ValueError("oracle_dispatch: invalid argument")
    return recv, scale, st


def scale_elems(num_rows: int, H: int, dtype: int, layout: int) -> int:
    """Elements of the receive-scale buffer in ``layout`` (-1: layout not defined
    for the payload type)."""
    return int(lib().oracle_scale_elems(num_rows, H, dtype, layout))


def scale_index(layout: int, num_rows: int, H: int, dtype: int, s: int, b: int) -> int:
    """Element index of the scale of receive row ``s``, block ``b``."""
    return int(lib().oracle_scale_index(layout, num_rows, H, dtype, s, b))


def dispatch_scaled(x_bf16: np.ndarray, token_slot: np.ndarray, dtype: int, layout: int,
                    recv_rows: int | None = None):
    """dispatch with the receive scales in ``layout``: (recv_x, flat scale
    buffer, status); positions no landed row owns stay 0."""
    if layout == SL_ROW_MAJOR:
        recv, scale, st = dispatch(x_bf16, token_slot, dtype, recv_rows)
        return recv, (scale.reshape(-1) if scale is not None else None), st
    x_bf16 = _c(x_bf16, np.uint16)
    token_slot = _c(token_slot, np.int32)
    N, H = x_bf16.shape
    k = token_slot.shape[1]
    S = N * k if recv_rows is None else recv_rows
    n = scale_elems(S, H, dtype, layout)
    if n < 0:
        raise ValueError("oracle_dispatch_scaled: layout not defined for this payload")
    recv = np.zeros((S, H), np.uint8)
    scale = np.zeros(n, np.uint8 if dtype in (DT_MXFP8_E4M3, DT_FP8_UE8M0) else np.float32)
    st = lib().oracle_dispatch_scaled(_ptr(x_bf16), N, H, k, _ptr(token_slot), S, dtype, layout,
                                      _ptr(recv), _ptr(scale))
    if st == ERR_INVALID_ARG:
        raise ValueError("oracle_dispatch_scaled: invalid argument")
    return recv, scale, st


def dispatch_nvfp4(x_bf16: np.ndarray, token_slot: np.ndarray, layout: int = SL_ROW_MAJOR,
                   recv_rows: int | None = None):
    """NVFP4 dispatch: (recv_x packed e2m1 [S, H/2] uint8, block scales (flat
    uint8, e4m3 codes in ``layout``), row scales fp32 [S], status).  Rows no
    slot names stay 0."""
    x_bf16 = _c(x_bf16, np.uint16)
    token_slot = _c(token_slot, np.int32)
    N, H = x_bf16.shape
    k = token_slot.shape[1]
    S = N * k if recv_rows is None else recv_rows
    n = scale_elems(S, H, DT_NVFP4, layout)
    if n < 0 or H % 64:
        raise ValueError("oracle_dispatch_nvfp4: invalid argument")
    recv = np.zeros((S, H // 2), np.uint8)
    bs = np.zeros(n, np.uint8)
    rs = np.zeros(S, np.float32)
    st = lib().oracle_dispatch_nvfp4(_ptr(x_bf16), N, H, k, _ptr(token_slot), S, layout, _ptr(recv),
                                     _ptr(bs), _ptr(rs))
    if st == ERR_INVALID_ARG:
        raise ValueError("oracle_dispatch_nvfp4: invalid argument")
    return recv, bs, rs, st


def quant_fp8_channel(recv_bf16: np.ndarray, expert_offset: np.ndarray, expert_count: np.ndarray,
                      transpose: bool = False):
    """Per-(expert, channel) FP8 of the receive rows: (codes [S, H] or [H, S],
    scales fp32 [E, H], status); rows outside the experts' landed ranges stay 0."""
    recv_bf16 = _c(recv_bf16, np.uint16)
    expert_offset = _c(expert_offset, np.int32)
    expert_count = _c(expert_count, np.int32)
    S, H = recv_bf16.shape
    E = len(expert_count)
    out = np.zeros((H, S) if transpose else (S, H), np.uint8)
    scale = np.zeros((E, H), np.float32)
    st = lib().oracle_quant_fp8_channel(_ptr(recv_bf16), S, H, E, _ptr(expert_offset), _ptr(expert_count),
                                        int(transpose), _ptr(out), _ptr(scale))
    if st == ERR_INVALID_ARG:
        raise ValueError("oracle_quant_fp8_channel: invalid argument")
    return out, scale, st


def swiglu_quant(h_bf16: np.ndarray, slot_token: np.ndarray | None, dtype: int,
                 layout: int = SL_ROW_MAJOR):
    """a = silu(gate) * up of each row of ``h`` = [gate | up] (bf16 bits [S, 2I]),
    quantised like a dispatched row: (out, flat scale buffer or None, status).
    out is bf16 bits [S, I] (BF16) or e4m3 codes [S, I]; rows whose slot_token
    is -1 are skipped (left 0)."""
    h_bf16 = _c(h_bf16, np.uint16)
    S, I2 = h_bf16.shape
    I = I2 // 2
    st_ptr = None
    if slot_token is not None:
        slot_token = _c(slot_token, np.int32)
        assert slot_token.shape == (S,)
        st_ptr = _ptr(slot_token)
    out = np.zeros((S, I), np.uint16 if dtype == DT_BF16 else np.uint8)
    scale, sp = None, None
    if dtype != DT_BF16:
        n = scale_elems(S, I, dtype, layout)
        if n < 0:
            raise ValueError("oracle_swiglu_quant: layout not defined for this payload")
        scale = np.zeros(n, np.uint8 if dtype == DT_MXFP8_E4M3 else np.float32)
        sp = _ptr(scale)
    st = lib().oracle_swiglu_quant(_ptr(h_bf16), S, I, st_ptr, dtype, layout, _ptr(out), sp)
    if st == ERR_INVALID_ARG:
        raise ValueError("oracle_swiglu_quant: invalid argument")
    return out, scale, st


def combine(y_bf16: np.ndarray, token_slot: np.ndarray, topk_w: np.ndarray):
    """Returns (out bf16 bits [N,H], status)."""
    y_bf16 = _c(y_bf16, np.uint16)
    token_slot = _c(token_slot, np.int32)
    topk_w = _c(topk_w, np.float32)
    N, k = token_slot.shape
    H = y_bf16.shape[1]
    out = np.empty((N, H), np.uint16)
    st = lib().oracle_combine(_ptr(y_bf16), y_bf16.shape[0], N, H, k, _ptr(token_slot), _ptr(topk_w),
                              _ptr(out))
    if st == ERR_INVALID_ARG:
        raise ValueError("oracle_combine: invalid argument")
    return out, st


def dispatch_backward(grad_recv_bf16: np.ndarray, token_slot: np.ndarray):
    """grad_x bf16 bits [N,H] = slot-order fp32 sum of each token's gradient rows; (grad_x, status)."""
    grad_recv_bf16 = _c(grad_recv_bf16, np.uint16)
    token_slot = _c(token_slot, np.int32)
    N, k = token_slot.shape
    H = grad_recv_bf16.shape[1]
    gx = np.empty((N, H), np.uint16)
    st = lib().oracle_dispatch_backward(_ptr(grad_recv_bf16), grad_recv_bf16.shape[0], N, H, k,
                                        _ptr(token_slot), _ptr(gx))
    if st == ERR_INVALID_ARG:
        raise ValueError("oracle_dispatch_backward: invalid argument")
    return gx, st


def combine_backward(grad_out_bf16: np.ndarray, y_bf16: np.ndarray, token_slot: np.ndarray,
                     topk_w: np.ndarray):
    """(grad_y bf16 bits [S,H] (rows no slot names stay 0), grad_w fp32 [N,k],
    sum_c |g*y| float64 [N,k] (for error bounds), status)."""
    grad_out_bf16 = _c(grad_out_bf16, np.uint16)
    y_bf16 = _c(y_bf16, np.uint16)
    token_slot = _c(token_slot, np.int32)
    topk_w = _c(topk_w, np.float32)
    N, k = token_slot.shape
    H = grad_out_bf16.shape[1]
    gy = np.zeros((y_bf16.shape[0], H), np.uint16)
    gw = np.empty((N, k), np.float32)
    mag = np.empty((N, k), np.float64)
    st = lib().oracle_combine_backward(_ptr(grad_out_bf16), _ptr(y_bf16), y_bf16.shape[0], N, H, k,
                                       _ptr(token_slot), _ptr(topk_w), _ptr(gy), _ptr(gw), _ptr(mag))
    if st == ERR_INVALID_ARG:
        raise ValueError("oracle_combine_backward: invalid argument")
    return gy, gw, mag, st

