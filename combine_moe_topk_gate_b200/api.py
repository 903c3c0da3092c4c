"""Thin ctypes binding of ``libmoe.so`` (C ABI in ``include/moe.h``).

The functions carry the C entry points' names.  They only marshal: check that
tensors are CUDA, contiguous and of the right dtype, allocate outputs the
caller did not pass (``torch.empty`` on the input's device), and pass raw
pointers, sizes and the current CUDA stream.  Every step of the routing path
runs in the library's kernels; there is no other implementation behind these
names.  Importing this module fails if the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_LIBRARY may name another build of the same sources (the bounds-checked
# libmoe_bounds_check.so); by default the in-tree libmoe.so is loaded.
LIB_PATH = os.environ.get("MOE_LIBRARY") or os.path.join(_PKG, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_BAD_INDEX, MOE_ERR_TIMEOUT = range(6)
MOE_GATE_SOFTMAX, MOE_GATE_SOFTMAX_RENORM, MOE_GATE_SIGMOID_GROUP = range(3)
(MOE_DTYPE_BF16, MOE_DTYPE_FP8_E4M3, MOE_DTYPE_FP8_E4M3_TOKEN, MOE_DTYPE_MXFP8_E4M3, MOE_DTYPE_NVFP4,
 MOE_DTYPE_E5M6, MOE_DTYPE_FP8_E4M3_UE8M0) = range(7)
MOE_MAX_EXPERTS = 1024
MOE_MAX_ALIGN = 4096
MOE_SCALE_ROW_MAJOR = 0
MOE_SCALE_MN_MAJOR = 1
MOE_SCALE_MMA_TILED = 2
MOE_SCALE_MN_MAJOR_PACK4 = 3
MOE_MAX_TOPK = 32
MOE_FP8_BLOCK = 128


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m combine_moe_topk_gate_b200.build` "
            "(nvcc, sm_100a).  There is no fallback implementation.")
    L = ctypes.CDLL(LIB_PATH)
    P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.moe_topk_gate.argtypes = [P, I, I, I, I, I, I, I, P, P, P]
    L.moe_topk_gate.restype = I
    L.moe_layout_workspace_bytes.argtypes = [I, I, I, I]
    L.moe_layout_workspace_bytes.restype = SZ
    L.moe_get_layout.argtypes = [P, I, I, I, I, P, P, P, P, P, P, P, P, SZ, P, P]
    L.moe_get_layout.restype = I
    L.moe_get_layout_aligned.argtypes = [P, I, I, I, I, I, I, P, P, P, P, P, P, P, P, SZ, P, P]
    L.moe_get_layout_aligned.restype = I
    L.moe_aligned_recv_rows.argtypes = [I, I, I, I]
    L.moe_aligned_recv_rows.restype = SZ
    L.moe_get_layout_noalloc.argtypes = [P, I, I, I, I, P, P, P, P, P, P, P, P, P]
    L.moe_get_layout_noalloc.restype = I
    L.moe_route_workspace_bytes.argtypes = [I, I, I, I]
    L.moe_route_workspace_bytes.restype = SZ
    L.moe_route.argtypes = [P, I, I, I, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, SZ, P, SZ, P, P]
    L.moe_route.restype = I
    L.moe_recv_bytes.argtypes = [I, I, I, I]
    L.moe_recv_bytes.restype = SZ
    L.moe_scale_bytes.argtypes = [I, I, I, I]
    L.moe_scale_bytes.restype = SZ
    L.moe_dispatch.argtypes = [P, I, I, I, P, I, I, P, P, P, P]
    L.moe_dispatch.restype = I
    L.moe_dispatch_ex.argtypes = [P, I, I, I, P, I, I, I, P, P, P, P]
    L.moe_dispatch_ex.restype = I
    L.moe_recv_scale_bytes.argtypes = [I, I, I, I]
    L.moe_recv_scale_bytes.restype = SZ
    L.moe_dispatch_nvfp4.argtypes = [P, I, I, I, P, I, I, P, P, P, P, P]
    L.moe_dispatch_nvfp4.restype = I
    L.moe_selftest_bounded_wait.argtypes = [P, P]
    L.moe_selftest_bounded_wait.restype = I
    L.moe_quant_fp8_channel.argtypes = [P, I, I, I, P, P, I, P, P, P, SZ, P, P]
    L.moe_quant_fp8_channel_workspace_bytes.argtypes = [I, I]
    L.moe_quant_fp8_channel_workspace_bytes.restype = SZ
    L.moe_quant_fp8_channel_takes_workspace.argtypes = [I, I]
    L.moe_quant_fp8_channel_takes_workspace.restype = I
    L.moe_quant_fp8_channel.restype = I
    L.moe_swiglu_quant.argtypes = [P, I, I, P, I, I, P, P, P]
    L.moe_swiglu_quant.restype = I
    L.moe_combine.argtypes = [P, I, I, I, P, I, P, P, P, P]
    L.moe_combine.restype = I
    L.moe_dispatch_backward.argtypes = [P, I, I, I, P, I, P, P, P]
    L.moe_dispatch_backward.restype = I
    L.moe_combine_backward.argtypes = [P, P, I, I, I, P, I, P, P, P, P, P]
    L.moe_combine_backward.restype = I
    L.moe_gate_math.argtypes = [ctypes.c_uint32, SZ, P, P, P, P]
    L.moe_gate_math.restype = I
    L.moe_e4m3_encode.argtypes = [P, SZ, P, P]
    L.moe_e4m3_encode.restype = I
    L.moe_status_string.argtypes = [I]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_abi_version.argtypes = []
    L.moe_abi_version.restype = I
    return L


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def status_string(status: int) -> str:
    return _lib.moe_status_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device) -> ctypes.c_void_p:
    """The stream handle to enqueue on: the device's current stream, or the
    caller's stream, which must belong to the tensors' device (the library
    launches on the current device, and a stream of another device there is
    a CUDA error)."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    else:
        sdev = getattr(stream, "device", None)
        if sdev is not None and device is not None and torch.device(sdev) != torch.device(device):
            raise ValueError(f"stream is on {sdev}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _slots_of(token_slot: torch.Tensor, N: int) -> int:
    """k of a token_slot array that must describe the N tokens of x: int32 [N, k]
    (the kernels read N*k slots)."""
    _need(token_slot, "token_slot", torch.int32)
    if token_slot.dim() != 2 or token_slot.shape[0] != N:
        raise ValueError(f"token_slot must have shape ({N}, k), got {tuple(token_slot.shape)}")
    return int(token_slot.shape[1])


def _status(d_status: torch.Tensor | None) -> torch.Tensor | None:
    """The optional device status word: int32 on the GPU, at least one element."""
    if d_status is not None:
        _need(d_status, "d_status", torch.int32)
        if d_status.numel() < 1:
            raise ValueError("d_status must hold at least one int32")
    return d_status


def _launch(fn, where: str, tensors, *args) -> None:
    """Calls an entry point that launches kernels.  The library launches on
    the calling thread's current CUDA device, so every tensor of the call
    must sit on one device, which is made current for the call."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"{where}: tensors on {sorted(str(d) for d in devs)}; all must be on one CUDA device")
    dev = devs.pop()
    if dev.index == torch.cuda.current_device():
        _check(fn(*args), where)
    else:
        with torch.cuda.device(dev):
            _check(fn(*args), where)


# ---------------------------------------------------------------- gate
def moe_topk_gate(logits: torch.Tensor, k: int, kind: int, n_groups: int = 1,
                  topk_groups: int = 1, group_topn: int = 1, *, topk_idx=None, topk_w=None,
                  stream=None):
    """Top-k router selection and weights; returns ``(topk_idx int32 [N,k], topk_w fp32 [N,k])``."""
    _need(logits, "logits", torch.float32)
    N, E = logits.shape
    if topk_idx is None:
        topk_idx = torch.empty((N, k), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((N, k), dtype=torch.float32, device=logits.device)
    _need(topk_idx, "topk_idx", torch.int32, (N, k))
    _need(topk_w, "topk_w", torch.float32, (N, k))
    _launch(_lib.moe_topk_gate, "moe_topk_gate", (logits, topk_idx, topk_w), _ptr(logits), N, E, k, kind,
            n_groups, topk_groups, group_topn, _ptr(topk_idx), _ptr(topk_w), _stream(stream, logits.device))
    return topk_idx, topk_w


# ---------------------------------------------------------------- layout
@dataclass
class Layout:
    """Routing metadata of one batch (the reusable handle)."""
    expert_count: torch.Tensor   # int32 [E]
    expert_offset: torch.Tensor  # int32 [E+1]
    rank_count: torch.Tensor     # int32 [R]
    rank_offset: torch.Tensor    # int32 [R+1]
    rank_tokens: torch.Tensor    # int32 [R]
    token_slot: torch.Tensor     # int32 [N, k]
    slot_token: torch.Tensor     # int32 [num_rows]
    workspace: torch.Tensor      # uint8 scratch
    status: torch.Tensor         # int32 [1] device status word
    align: int = 1               # expert row alignment of the receive buffer

    @property
    def num_rows(self) -> int:
        """Rows of the receive buffer this layout addresses."""
        return self.slot_token.numel()

    @staticmethod
    def empty(N: int, k: int, E: int, R: int, device, align: int = 1, num_rows: int | None = None,
              workspace: bool = True, route: bool = False) -> "Layout":
        """Uninitialised arrays for an N x k batch over E experts and R ranks;
        ``workspace=False`` gives a 0-byte workspace (for the no-workspace
        entry point); ``route=True`` a zeroed workspace of moe_route's size
        (moe_route keeps its first 256 bytes, an arrival counter, zero)."""
        i32 = dict(dtype=torch.int32, device=device)
        if route:
            ws = moe_route_workspace_bytes(N, k, E, R)
            layout = Layout.empty(N, k, E, R, device, align, num_rows, workspace=False)
            layout.workspace = torch.zeros(ws, dtype=torch.uint8, device=device)
            return layout
        ws = moe_layout_workspace_bytes(N, k, E, R) if workspace else 0
        rows = num_rows if num_rows is not None else moe_aligned_recv_rows(N, k, E, align)
        return Layout(torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(R, **i32),
                      torch.empty(R + 1, **i32), torch.empty(R, **i32), torch.empty((N, k), **i32),
                      torch.empty(rows, **i32), torch.empty(ws, dtype=torch.uint8, device=device),
                      torch.zeros(1, **i32), align)


def _check_layout(out: Layout, N: int, k: int, E: int, R: int, workspace: bool = True) -> None:
    """A caller-supplied layout must have the shapes of the batch it is filled
    for: the kernels write every one of its arrays."""
    for name, shape in (("expert_count", (E,)), ("expert_offset", (E + 1,)), ("rank_count", (R,)),
                        ("rank_offset", (R + 1,)), ("rank_tokens", (R,)), ("token_slot", (N, k))):
        _need(getattr(out, name), f"out.{name}", torch.int32, shape)
    _need(out.slot_token, "out.slot_token", torch.int32, (out.slot_token.numel(),))
    if workspace:
        _need(out.workspace, "out.workspace", torch.uint8, (out.workspace.numel(),))
    _status(out.status)


def moe_route_workspace_bytes(num_tokens: int, k: int, num_experts: int, num_ranks: int) -> int:
    return int(_lib.moe_route_workspace_bytes(num_tokens, k, num_experts, num_ranks))


def moe_layout_workspace_bytes(num_tokens: int, k: int, num_experts: int, num_ranks: int) -> int:
    return int(_lib.moe_layout_workspace_bytes(num_tokens, k, num_experts, num_ranks))


def moe_aligned_recv_rows(num_tokens: int, k: int, num_experts: int, align: int) -> int:
    return int(_lib.moe_aligned_recv_rows(num_tokens, k, num_experts, align))


def moe_get_layout(topk_idx: torch.Tensor, num_experts: int, num_ranks: int, *, align: int = 1,
                   num_recv_rows: int | None = None, out: Layout | None = None, stream=None) -> Layout:
    """Counts, offsets and token<->slot maps; fills (and returns) ``out``.
    ``align > 1`` starts every expert's rows at a multiple of ``align``
    (moe_get_layout_aligned); the receive buffer then has ``out.num_rows`` rows.
    The device status word ``out.status`` is not cleared here: zero it to start
    a fresh error record."""
    _need(topk_idx, "topk_idx", torch.int32)
    N, k = topk_idx.shape
    E, R = num_experts, num_ranks
    if out is None:
        out = Layout.empty(N, k, E, R, topk_idx.device, align, num_recv_rows)
    _check_layout(out, N, k, E, R)
    args = (_ptr(out.expert_count), _ptr(out.expert_offset), _ptr(out.rank_count),
            _ptr(out.rank_offset), _ptr(out.rank_tokens), _ptr(out.token_slot), _ptr(out.slot_token),
            _ptr(out.workspace), out.workspace.numel(), _ptr(out.status),
            _stream(stream, topk_idx.device))
    tensors = (topk_idx, out.expert_count, out.expert_offset, out.rank_count, out.rank_offset,
               out.rank_tokens, out.token_slot, out.slot_token, out.workspace, _status(out.status))
    if align == 1 and out.num_rows == N * k:
        _launch(_lib.moe_get_layout, "moe_get_layout", tensors, _ptr(topk_idx), N, k, E, R, *args)
    else:
        _launch(_lib.moe_get_layout_aligned, "moe_get_layout_aligned", tensors, _ptr(topk_idx), N, k, E, R,
                align, out.num_rows, *args)
    out.align = align
    return out


def moe_route(logits: torch.Tensor, k: int, kind: int, n_groups: int, topk_groups: int, group_topn: int,
              num_ranks: int, *, align: int = 1, num_recv_rows: int | None = None, topk_idx=None, topk_w=None,
              out: Layout | None = None, prefetch: torch.Tensor | None = None, stream=None):
    """Gate and layout in one call (moe_route): returns ``(topk_idx, topk_w,
    layout)`` equal to ``moe_topk_gate`` followed by ``moe_get_layout``.
    ``out.workspace`` must be a moe_route workspace whose first 256 bytes are
    zero (``Layout.empty(..., route=True)``); every call leaves them zero.
    ``prefetch``: a CUDA tensor read next (e.g. x before moe_dispatch), fetched
    into L2 while the routing kernels run (a hint; no result changes)."""
    _need(logits, "logits", torch.float32)
    N, E = logits.shape
    R = num_ranks
    if topk_idx is None:
        topk_idx = torch.empty((N, k), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((N, k), dtype=torch.float32, device=logits.device)
    _need(topk_idx, "topk_idx", torch.int32, (N, k))
    _need(topk_w, "topk_w", torch.float32, (N, k))
    if out is None:
        out = Layout.empty(N, k, E, R, logits.device, align, num_recv_rows, route=True)
    _check_layout(out, N, k, E, R)
    need = moe_route_workspace_bytes(N, k, E, R)
    if out.workspace.numel() < need:
        raise ValueError(f"out.workspace must hold moe_route_workspace_bytes = {need} bytes "
                         f"(Layout.empty(..., route=True)), got {out.workspace.numel()}")
    rows = out.num_rows
    pf_bytes = 0
    if prefetch is not None:
        if not prefetch.is_cuda or not prefetch.is_contiguous():
            raise ValueError("prefetch must be a contiguous CUDA tensor")
        pf_bytes = prefetch.numel() * prefetch.element_size() // 16 * 16
    tensors = (logits, topk_idx, topk_w, out.expert_count, out.expert_offset, out.rank_count, out.rank_offset,
               out.rank_tokens, out.token_slot, out.slot_token, out.workspace, _status(out.status), prefetch)
    _launch(_lib.moe_route, "moe_route", tensors, _ptr(logits), N, E, k, kind, n_groups, topk_groups, group_topn,
            R, align, rows, _ptr(topk_idx), _ptr(topk_w), _ptr(out.expert_count), _ptr(out.expert_offset),
            _ptr(out.rank_count), _ptr(out.rank_offset), _ptr(out.rank_tokens), _ptr(out.token_slot),
            _ptr(out.slot_token), _ptr(out.workspace), out.workspace.numel(),
            _ptr(prefetch) if pf_bytes else None, pf_bytes, _ptr(out.status), _stream(stream, logits.device))
    out.align = align
    return topk_idx, topk_w, out


MOE_LAYOUT_NOALLOC_SCRATCH_BYTES = 1 << 20


def moe_get_layout_noalloc(topk_idx: torch.Tensor, num_experts: int, num_ranks: int, *,
                           out: Layout | None = None, stream=None) -> Layout:
    """``moe_get_layout`` for callers that cannot allocate device scratch: the
    library uses its own fixed array (``MOE_LAYOUT_NOALLOC_SCRATCH_BYTES``)
    instead of ``out.workspace``.  Calls must not overlap on the GPU (they share
    the array); the first call on a device should come before any stream
    capture.  Outputs are still the caller's (allocated here when ``out`` is
    None, like every other binding)."""
    _need(topk_idx, "topk_idx", torch.int32)
    N, k = topk_idx.shape
    E, R = num_experts, num_ranks
    if out is None:
        out = Layout.empty(N, k, E, R, topk_idx.device, workspace=False)
    _check_layout(out, N, k, E, R, workspace=False)
    # the entry point writes the packed layout: exactly N*k receive rows
    if out.slot_token.numel() != N * k:
        raise ValueError(f"out.slot_token must have N*k = {N * k} entries for the packed layout, "
                         f"got {out.slot_token.numel()}")
    tensors = (topk_idx, out.expert_count, out.expert_offset, out.rank_count, out.rank_offset,
               out.rank_tokens, out.token_slot, out.slot_token, _status(out.status))
    _launch(_lib.moe_get_layout_noalloc, "moe_get_layout_noalloc", tensors, _ptr(topk_idx), N, k, E, R,
            _ptr(out.expert_count), _ptr(out.expert_offset), _ptr(out.rank_count), _ptr(out.rank_offset),
            _ptr(out.rank_tokens), _ptr(out.token_slot), _ptr(out.slot_token), _ptr(out.status),
            _stream(stream, topk_idx.device))
    out.align = 1
    return out


# ---------------------------------------------------------------- dispatch / combine
def moe_recv_bytes(num_tokens: int, hidden: int, k: int, dtype: int) -> int:
    return int(_lib.moe_recv_bytes(num_tokens, hidden, k, dtype))


def moe_scale_bytes(num_tokens: int, hidden: int, k: int, dtype: int = MOE_DTYPE_FP8_E4M3) -> int:
    return int(_lib.moe_scale_bytes(num_tokens, hidden, k, dtype))


def moe_recv_scale_bytes(num_recv_rows: int, hidden: int, dtype: int, scale_layout: int) -> int:
    return int(_lib.moe_recv_scale_bytes(num_recv_rows, hidden, dtype, scale_layout))


def scale_shape(S: int, H: int, dtype: int, scale_layout: int = 0):
    """(shape, torch dtype) of recv_scale for a payload type (None for BF16):
    row-major [S, B]; MN-major [B, ld]; MMA-tiled flat bytes."""
    if scale_layout != MOE_SCALE_ROW_MAJOR:
        nbytes = moe_recv_scale_bytes(S, H, dtype, scale_layout)
        if nbytes == 0:
            return None, None
        sdt = torch.uint8 if dtype in (MOE_DTYPE_MXFP8_E4M3, MOE_DTYPE_NVFP4, MOE_DTYPE_FP8_E4M3_UE8M0) \
            else torch.float32
        if scale_layout in (MOE_SCALE_MMA_TILED, MOE_SCALE_MN_MAJOR_PACK4):
            return (nbytes,), sdt
        B = {MOE_DTYPE_FP8_E4M3: H // MOE_FP8_BLOCK, MOE_DTYPE_FP8_E4M3_TOKEN: 1,
             MOE_DTYPE_MXFP8_E4M3: H // 32, MOE_DTYPE_NVFP4: H // 16,
             MOE_DTYPE_FP8_E4M3_UE8M0: H // MOE_FP8_BLOCK}[dtype]
        es = 1 if sdt == torch.uint8 else 4
        return (B, nbytes // es // B), sdt
    if dtype == MOE_DTYPE_FP8_E4M3:
        return (S, H // MOE_FP8_BLOCK), torch.float32
    if dtype == MOE_DTYPE_FP8_E4M3_TOKEN:
        return (S, 1), torch.float32
    if dtype == MOE_DTYPE_MXFP8_E4M3:
        return (S, H // 32), torch.uint8
    if dtype == MOE_DTYPE_NVFP4:
        return (S, H // 16), torch.uint8
    if dtype == MOE_DTYPE_FP8_E4M3_UE8M0:
        return (S, H // MOE_FP8_BLOCK), torch.uint8
    return None, None


def moe_dispatch(x: torch.Tensor, token_slot: torch.Tensor, dtype: int, *, recv_x=None,
                 recv_scale=None, num_recv_rows: int | None = None, scale_layout: int = 0,
                 d_status=None, stream=None):
    """Scatter rows of ``x`` (bf16 [N,H]) to their receive rows.  Returns
    ``(recv_x, recv_scale)``: bf16 [S,H] and None, or uint8 e4m3 codes
    [S,H] with fp32 [S,H/128] (per block), fp32 [S,1] (per token) or
    uint8 E8M0 bytes [S,H/32] (MXFP8), row-major; ``scale_layout`` selects
    the MN-major or MMA-tiled scale layouts (moe_dispatch_ex)."""
    _need(x, "x", torch.bfloat16)
    N, H = x.shape
    k = _slots_of(token_slot, N)
    S = num_recv_rows if num_recv_rows is not None else (recv_x.shape[0] if recv_x is not None else N * k)
    if dtype == MOE_DTYPE_BF16:
        if recv_x is None:
            recv_x = torch.empty((S, H), dtype=torch.bfloat16, device=x.device)
        _need(recv_x, "recv_x", torch.bfloat16, (S, H))
        recv_scale = None
    elif dtype == MOE_DTYPE_E5M6:
        if recv_x is None:
            recv_x = torch.empty((S, H // 2 * 3), dtype=torch.uint8, device=x.device)
        _need(recv_x, "recv_x", torch.uint8, (S, H // 2 * 3))
        recv_scale = None
    else:
        shape, sdt = scale_shape(S, H, dtype, scale_layout)
        if shape is None:
            raise ValueError(f"dispatch dtype {dtype} has no scale layout {scale_layout}")
        if recv_x is None:
            recv_x = torch.empty((S, H), dtype=torch.uint8, device=x.device)
        if recv_scale is None:
            recv_scale = torch.empty(shape, dtype=sdt, device=x.device)
        _need(recv_x, "recv_x", torch.uint8, (S, H))
        _need(recv_scale, "recv_scale", sdt, shape)
    _launch(_lib.moe_dispatch_ex, "moe_dispatch", (x, token_slot, recv_x, recv_scale, _status(d_status)),
            _ptr(x), N, H, k, _ptr(token_slot), S, dtype, scale_layout, _ptr(recv_x), _ptr(recv_scale),
            _ptr(d_status), _stream(stream, x.device))
    return recv_x, recv_scale


def moe_dispatch_nvfp4(x: torch.Tensor, token_slot: torch.Tensor, *, scale_layout: int = 0,
                       recv_x=None, block_scale=None, row_scale=None, num_recv_rows: int | None = None,
                       d_status=None, stream=None):
    """NVFP4 dispatch: returns ``(recv_x uint8 [S, H/2] (two e2m1 codes per
    byte, even channel in the low nibble), block_scale (e4m3 codes, one per
    16 channels, in ``scale_layout``), row_scale fp32 [S])``."""
    _need(x, "x", torch.bfloat16)
    N, H = x.shape
    k = _slots_of(token_slot, N)
    S = num_recv_rows if num_recv_rows is not None else (recv_x.shape[0] if recv_x is not None else N * k)
    shape, _ = scale_shape(S, H, MOE_DTYPE_NVFP4, scale_layout)
    if shape is None:
        raise ValueError(f"NVFP4 has no scale layout {scale_layout} for hidden {H}")
    if recv_x is None:
        recv_x = torch.empty((S, H // 2), dtype=torch.uint8, device=x.device)
    if block_scale is None:
        block_scale = torch.empty(shape, dtype=torch.uint8, device=x.device)
    if row_scale is None:
        row_scale = torch.empty((S,), dtype=torch.float32, device=x.device)
    _need(recv_x, "recv_x", torch.uint8, (S, H // 2))
    _need(block_scale, "block_scale", torch.uint8, shape)
    _need(row_scale, "row_scale", torch.float32, (S,))
    _launch(_lib.moe_dispatch_nvfp4, "moe_dispatch_nvfp4",
            (x, token_slot, recv_x, block_scale, row_scale, _status(d_status)), _ptr(x), N, H, k,
            _ptr(token_slot), S, scale_layout, _ptr(recv_x), _ptr(block_scale), _ptr(row_scale),
            _ptr(d_status), _stream(stream, x.device))
    return recv_x, block_scale, row_scale


def moe_selftest_bounded_wait(d_status: torch.Tensor, stream=None) -> None:
    """Runs the pipelined kernels' bounded wait on an mbarrier nothing completes;
    after about a second MOE_ERR_TIMEOUT is recorded in ``d_status``."""
    _need(d_status, "d_status", torch.int32, (1,))
    _launch(_lib.moe_selftest_bounded_wait, "moe_selftest_bounded_wait", (d_status,), _ptr(d_status),
            _stream(stream, d_status.device))


def moe_quant_fp8_channel_workspace_bytes(num_experts: int, hidden: int) -> int:
    return int(_lib.moe_quant_fp8_channel_workspace_bytes(num_experts, hidden))


def moe_quant_fp8_channel_takes_workspace(num_rows: int, num_experts: int) -> bool:
    return bool(_lib.moe_quant_fp8_channel_takes_workspace(num_rows, num_experts))


def moe_quant_fp8_channel(recv: torch.Tensor, expert_offset: torch.Tensor, expert_count: torch.Tensor, *,
                          transpose: bool = False, out=None, scale=None, workspace="new", d_status=None,
                          stream=None):
    """Per-(expert, channel) FP8 of the receive rows ``recv`` (bf16 [S, H]) over
    each expert's landed rows; returns ``(codes uint8 [S, H] or [H, S], scale
    fp32 [E, H])``.  ``workspace``: a uint8 device tensor of
    ``moe_quant_fp8_channel_workspace_bytes(E, H)`` bytes, zero before its
    first use and left zero by every call (keep one per stream); ``"new"``
    (default) allocates a zeroed one for this call when the call uses one
    (``moe_quant_fp8_channel_takes_workspace``); None takes the path without
    scratch."""
    _need(recv, "recv", torch.bfloat16)
    S, H = recv.shape
    _need(expert_count, "expert_count", torch.int32)
    E = expert_count.numel()
    _need(expert_offset, "expert_offset", torch.int32, (E + 1,))
    shape = (H, S) if transpose else (S, H)
    if out is None:
        out = torch.empty(shape, dtype=torch.uint8, device=recv.device)
    if scale is None:
        scale = torch.empty((E, H), dtype=torch.float32, device=recv.device)
    _need(out, "out", torch.uint8, shape)
    _need(scale, "scale", torch.float32, (E, H))
    ws_bytes = moe_quant_fp8_channel_workspace_bytes(E, H)
    if isinstance(workspace, str):
        if workspace != "new":
            raise ValueError(f"workspace must be a tensor, None or 'new', not {workspace!r}")
        if moe_quant_fp8_channel_takes_workspace(S, E):
            # zeroed in the order of the stream the kernel runs on
            with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream(recv.device)):
                workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=recv.device)
        else:
            workspace = None
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8)
        if workspace.numel() < ws_bytes:
            raise ValueError(f"workspace holds {workspace.numel()} bytes, {ws_bytes} needed")
    _launch(_lib.moe_quant_fp8_channel, "moe_quant_fp8_channel",
            (recv, expert_offset, expert_count, out, scale, workspace, _status(d_status)), _ptr(recv), S, H, E,
            _ptr(expert_offset), _ptr(expert_count), int(transpose), _ptr(out), _ptr(scale), _ptr(workspace),
            workspace.numel() if workspace is not None else 0, _ptr(d_status), _stream(stream, recv.device))
    return out, scale


def moe_swiglu_quant(h: torch.Tensor, dtype: int, *, slot_token=None, scale_layout: int = 0,
                     out=None, out_scale=None, stream=None):
    """a = silu(gate) * up for every row of ``h`` = [gate | up] (bf16 [S, 2I]),
    stored as bf16 [S, I] or quantised like a dispatched row (e4m3 [S, I] plus
    scales in ``scale_layout``).  Rows whose ``slot_token`` (int32 [S]) is
    negative are skipped.  Returns ``(out, out_scale)``."""
    _need(h, "h", torch.bfloat16)
    S, I2 = h.shape
    I = I2 // 2
    if slot_token is not None:
        _need(slot_token, "slot_token", torch.int32, (S,))
    if dtype == MOE_DTYPE_BF16:
        if out is None:
            out = torch.empty((S, I), dtype=torch.bfloat16, device=h.device)
        _need(out, "out", torch.bfloat16, (S, I))
        out_scale = None
    else:
        shape, sdt = scale_shape(S, I, dtype, scale_layout)
        if shape is None:
            raise ValueError(f"swiglu dtype {dtype} has no scale layout {scale_layout}")
        if out is None:
            out = torch.empty((S, I), dtype=torch.uint8, device=h.device)
        if out_scale is None:
            out_scale = torch.empty(shape, dtype=sdt, device=h.device)
        _need(out, "out", torch.uint8, (S, I))
        _need(out_scale, "out_scale", sdt, shape)
    _launch(_lib.moe_swiglu_quant, "moe_swiglu_quant", (h, slot_token, out, out_scale), _ptr(h), S, I,
            _ptr(slot_token), dtype, scale_layout, _ptr(out), _ptr(out_scale), _stream(stream, h.device))
    return out, out_scale


def moe_combine(y: torch.Tensor, token_slot: torch.Tensor, topk_w: torch.Tensor, *, out=None,
                d_status=None, stream=None) -> torch.Tensor:
    """Weighted gather-reduce of expert outputs ``y`` (bf16 [N*k,H]) -> bf16 [N,H]."""
    _need(y, "y", torch.bfloat16)
    if y.dim() != 2:
        raise ValueError(f"y must be 2-D [S, H], got {tuple(y.shape)}")
    _need(token_slot, "token_slot", torch.int32)
    N, k = token_slot.shape
    H = y.shape[1]
    _need(topk_w, "topk_w", torch.float32, (N, k))
    if out is None:
        out = torch.empty((N, H), dtype=torch.bfloat16, device=y.device)
    _need(out, "out", torch.bfloat16, (N, H))
    _launch(_lib.moe_combine, "moe_combine", (y, token_slot, topk_w, out, _status(d_status)), _ptr(y), N, H,
            k, _ptr(token_slot), y.shape[0], _ptr(topk_w), _ptr(out), _ptr(d_status), _stream(stream, y.device))
    return out


def moe_dispatch_backward(grad_recv: torch.Tensor, token_slot: torch.Tensor, *, grad_x=None,
                          d_status=None, stream=None) -> torch.Tensor:
    """Gradient of dispatch: slot-order sum of each token's rows of ``grad_recv``
    (bf16 [N*k,H]) -> bf16 [N,H]."""
    _need(grad_recv, "grad_recv", torch.bfloat16)
    if grad_recv.dim() != 2:
        raise ValueError(f"grad_recv must be 2-D [S, H], got {tuple(grad_recv.shape)}")
    _need(token_slot, "token_slot", torch.int32)
    N, k = token_slot.shape
    H = grad_recv.shape[1]
    if grad_x is None:
        grad_x = torch.empty((N, H), dtype=torch.bfloat16, device=grad_recv.device)
    _need(grad_x, "grad_x", torch.bfloat16, (N, H))
    _launch(_lib.moe_dispatch_backward, "moe_dispatch_backward", (grad_recv, token_slot, grad_x, _status(d_status)),
            _ptr(grad_recv), N, H, k, _ptr(token_slot), grad_recv.shape[0], _ptr(grad_x), _ptr(d_status),
            _stream(stream, grad_recv.device))
    return grad_x


def moe_combine_backward(grad_out: torch.Tensor, y: torch.Tensor, token_slot: torch.Tensor,
                         topk_w: torch.Tensor, *, grad_y=None, grad_w=None, d_status=None,
                         stream=None):
    """Gradients of combine: ``(grad_y bf16 [N*k,H], grad_w fp32 [N,k])``."""
    _need(token_slot, "token_slot", torch.int32)
    N, k = token_slot.shape
    _need(y, "y", torch.bfloat16)
    if y.dim() != 2:
        raise ValueError(f"y must be 2-D [S, H], got {tuple(y.shape)}")
    H = y.shape[1]
    _need(grad_out, "grad_out", torch.bfloat16, (N, H))
    _need(topk_w, "topk_w", torch.float32, (N, k))
    if grad_y is None:
        grad_y = torch.empty(tuple(y.shape), dtype=torch.bfloat16, device=y.device)
    if grad_w is None:
        grad_w = torch.empty((N, k), dtype=torch.float32, device=y.device)
    _need(grad_y, "grad_y", torch.bfloat16, tuple(y.shape))
    _need(grad_w, "grad_w", torch.float32, (N, k))
    _launch(_lib.moe_combine_backward, "moe_combine_backward",
            (grad_out, y, token_slot, topk_w, grad_y, grad_w, _status(d_status)), _ptr(grad_out), _ptr(y), N, H,
            k, _ptr(token_slot), y.shape[0], _ptr(topk_w), _ptr(grad_y), _ptr(grad_w), _ptr(d_status),
            _stream(stream, y.device))
    return grad_y, grad_w


def moe_e4m3_encode(x: torch.Tensor, *, out=None, stream=None) -> torch.Tensor:
    """Element-wise e4m3 codes (uint8) of an fp32 tensor, as dispatch encodes them."""
    _need(x, "x", torch.float32)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _need(out, "out", torch.uint8, x.shape)
    _launch(_lib.moe_e4m3_encode, "moe_e4m3_encode", (x, out), _ptr(x), x.numel(), _ptr(out),
            _stream(stream, x.device))
    return out


def moe_gate_math(first: int, n: int, *, exp_out=None, sigmoid_out=None, silu_out=None, device=None,
                  stream=None):
    """The gate's exp and sigmoid and SwiGLU's silu on the fp32 bit patterns
    first, first+1, ..., first+n-1 (mod 2^32); returns ``(exp_out,
    sigmoid_out, silu_out)``, fp32 [n] each."""
    given = [t for t in (exp_out, sigmoid_out, silu_out) if t is not None]
    dev = given[0].device if given else torch.device("cuda", torch.cuda.current_device())
    if device is not None and torch.device(device) != dev:
        raise ValueError(f"outputs are on {dev}, device is {device}")
    outs = []
    for name, t in (("exp_out", exp_out), ("sigmoid_out", sigmoid_out), ("silu_out", silu_out)):
        if t is None:
            t = torch.empty(n, dtype=torch.float32, device=dev)
        _need(t, name, torch.float32, (n,))
        outs.append(t)
    _launch(_lib.moe_gate_math, "moe_gate_math", tuple(outs), first & 0xFFFFFFFF, n,
            *(_ptr(t) for t in outs), _stream(stream, dev))
    return tuple(outs)


def moe_abi_version() -> int:
    return int(_lib.moe_abi_version())
