"""Single-GPU MoE layout / dispatch / combine for B200 (sm_100a), over the C ABI in include/cgl.h.

Python binding only: this module allocates outputs with torch (device memory),
picks the current CUDA stream, and passes raw pointers to libcgl.so.  Every
step of the computation runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and every call raises if the library is missing or the
tensors are not on a CUDA device.

    lay = get_layout(topk_idx, num_experts=256, num_ranks=64)
    recv_x, recv_scale = dispatch_fp8(x, lay.dst_pos, lay.num_recv_rows)
    out = combine(y, lay.dst_pos, topk_weights)

The operations are the dispatch ("send each token to its gated experts") and
combine ("merge the expert outputs back, accumulating") of the DeepEP pages
(GitHub-issue mirror "Technical Overview of DeepEP"; brainleap "Day2 DeepEP",
"DeepEP是什么" and "All-to-All通信"), with FP8 dispatch and BF16 combine as in
their benchmark settings, run inside one GPU with ranks as expert partitions.
"""

from __future__ import annotations

import ctypes as C
import os
from typing import NamedTuple, Optional

import torch

__all__ = [
    "CglError", "Layout", "RankLayout", "lib", "get_layout", "get_rank_layout", "dispatch_fp8", "dispatch_bf16", "combine",
    "combine_backward", "decode_dispatch_fp8", "layout_workspace_bytes", "layout_kernel_count", "status_bits", "check_status", "new_status",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcgl.so")

OK, EINVAL, EALIGN, ERANGE, ECAPACITY, ETIMEOUT, ECUDA, ENOTIMPL = range(8)
_NAMES = {OK: "CGL_OK", EINVAL: "CGL_EINVAL", EALIGN: "CGL_EALIGN", ERANGE: "CGL_ERANGE",
          ECAPACITY: "CGL_ECAPACITY", ETIMEOUT: "CGL_ETIMEOUT", ECUDA: "CGL_ECUDA",
          ENOTIMPL: "CGL_ENOTIMPL"}


class CglError(RuntimeError):
    """A non-OK status from the library (host-side) or a device error bit."""

    def __init__(self, code: int, where: str, detail: str = ""):
        self.code = code
        super().__init__(f"{where}: {_NAMES.get(code, code)} ({detail or _status_string(code)})")


class Opts(C.Structure):
    _fields_ = [("num_sms", C.c_int32), ("capacity", C.c_int32), ("flags", C.c_uint32), ("scratch", C.c_void_p)]


OPT_UE8M0_SCALES = 1   # cgl_opts.flags: power-of-two (UE8M0) FP8 scales


_lib = None


def lib():
    """The loaded libcgl.so (ctypes), with argument types declared."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libcgl.so is not built ({LIB_PATH}); run "
                               "`python -m combine_get_layout_02_b200.build`")
        L = C.CDLL(LIB_PATH)
        P, I64, I = C.c_void_p, C.c_int64, C.c_int
        OP = C.POINTER(Opts)
        L.cgl_version.argtypes = []
        L.cgl_version.restype = I
        L.cgl_status_string.argtypes = [I]
        L.cgl_status_string.restype = C.c_char_p
        L.cgl_layout_workspace_bytes.argtypes = [I64, I, I, I]
        L.cgl_layout_workspace_bytes.restype = C.c_size_t
        L.cgl_layout_kernel_count.argtypes = [I64, I, I, I]
        L.cgl_layout_kernel_count.restype = I
        L.cgl_get_layout.argtypes = [P, I64, I, I, I, OP, P, P, P, P, P, P, P, P, C.c_size_t, P, P]
        L.cgl_get_layout.restype = I
        L.cgl_get_rank_layout.argtypes = [P, I64, I, I, I, OP, P, P, P, P, P, P, C.c_size_t, P, P]
        L.cgl_get_rank_layout.restype = I
        L.cgl_dispatch_fp8.argtypes = [P, I64, I, I, P, P, P, I64, OP, P, P]
        L.cgl_dispatch_fp8.restype = I
        L.cgl_dispatch_bf16.argtypes = [P, I64, I, I, P, P, I64, OP, P, P]
        L.cgl_dispatch_bf16.restype = I
        L.cgl_combine.argtypes = [P, I64, P, P, I64, I, I, P, OP, P, P]
        L.cgl_combine.restype = I
        L.cgl_decode_dispatch_fp8.argtypes = [P, I64, I, I, I, OP, P, I, P, P, P, P, P, P, P, P, P, P, P]
        L.cgl_decode_dispatch_fp8.restype = I
        L.cgl_layout_dispatch_workspace_bytes.argtypes = [I64, I, I, I]
        L.cgl_layout_dispatch_workspace_bytes.restype = C.c_size_t
        L.cgl_layout_dispatch_kernel_count.argtypes = [I64, I, I, I, I, OP]
        L.cgl_layout_dispatch_kernel_count.restype = I
        L.cgl_layout_dispatch_fp8.argtypes = [P, I64, I, I, I, OP, P, I, P, P, P, P, P, P, P, P, P, P,
                                              C.c_size_t, P, P]
        L.cgl_layout_dispatch_fp8.restype = I
        L.cgl_combine_backward.argtypes = [P, P, I64, P, P, I64, I, I, P, P, OP, P, P]
        L.cgl_combine_backward.restype = I
        _lib = L
    return _lib


def _status_string(code: int) -> str:
    try:
        return lib().cgl_status_string(int(code)).decode()
    except RuntimeError:
        return "status"


def _check(code: int, where: str):
    if code != OK:
        raise CglError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, name: str, dtype=None, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _opts(num_sms: int = 0, capacity: int = 0, pow2_scales: bool = False, scratch: Optional[torch.Tensor] = None):
    sp = None
    if scratch is not None:
        if not scratch.is_cuda or scratch.numel() * scratch.element_size() < 16 or not scratch.is_contiguous():
            raise CglError(EINVAL, "scratch", "a contiguous device tensor of at least 16 bytes")
        sp = scratch.data_ptr()
    return C.byref(Opts(int(num_sms), int(capacity), OPT_UE8M0_SCALES if pow2_scales else 0, sp))


def new_scratch(device=None) -> torch.Tensor:
    """Zeroed 16-byte device scratch (cgl_opts.scratch) for dispatch_fp8 / dispatch_bf16: with it the
    dispatch kernel hands tokens out dynamically; each call leaves it zero.  Calls that may run at the
    same time need their own."""
    return torch.zeros(2, dtype=torch.int64, device=device or "cuda")


def new_status(device=None) -> torch.Tensor:
    """A zeroed device status word (uint32 stored as int32[1])."""
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def status_bits(status: torch.Tensor) -> list:
    """Names of the device error bits set in a status word (reads it: synchronises)."""
    v = int(status.item()) & 0xFFFFFFFF
    return [_NAMES[c] for c in range(1, 8) if v & (1 << c)]


def check_status(status: torch.Tensor, where: str = "device"):
    v = int(status.item()) & 0xFFFFFFFF
    for c in range(1, 8):
        if v & (1 << c):
            raise CglError(c, where, "device-reported")


def layout_workspace_bytes(num_tokens: int, num_topk: int, num_experts: int, num_ranks: int) -> int:
    return int(lib().cgl_layout_workspace_bytes(num_tokens, num_topk, num_experts, num_ranks))


def layout_kernel_count(num_tokens: int, num_topk: int, num_experts: int, num_ranks: int) -> int:
    """Kernels one get_layout call launches for these sizes on the current device (1 or 2)."""
    return int(lib().cgl_layout_kernel_count(num_tokens, num_topk, num_experts, num_ranks))


class Layout(NamedTuple):
    tokens_per_expert: torch.Tensor   # int32 [E]
    tokens_per_rank: torch.Tensor     # int32 [R]
    is_token_in_rank: torch.Tensor    # uint8 [N, R]
    expert_offset: torch.Tensor       # int32 [E + 1]
    max_count: torch.Tensor           # int32 [1]
    dst_pos: torch.Tensor             # int32 [N, k]
    recv_src: torch.Tensor            # int32 [num_recv_rows]
    num_recv_rows: int                # N*k (compact) or E*capacity (padded)
    capacity: int


def get_layout(topk_idx: torch.Tensor, num_experts: int, num_ranks: int, capacity: int = 0, *,
               status: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               out: Optional[Layout] = None, stream=None) -> Layout:
    """Counts, prefix sums and stable receive rows for top-k routing (cgl_get_layout)."""
    idx = _dev(topk_idx, "topk_idx", torch.int32, 2)
    n, k = idx.shape
    E, R = int(num_experts), int(num_ranks)
    dev = idx.device
    rows = E * capacity if capacity > 0 else n * k
    ws_bytes = layout_workspace_bytes(n, k, E, R)
    if ws_bytes == 0:
        raise CglError(EINVAL, "get_layout", "invalid sizes")
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if out is None:
        out = Layout(
            torch.empty(E, dtype=torch.int32, device=dev),
            torch.empty(R, dtype=torch.int32, device=dev),
            torch.empty((n, R), dtype=torch.uint8, device=dev),
            torch.empty(E + 1, dtype=torch.int32, device=dev),
            torch.empty(1, dtype=torch.int32, device=dev),
            torch.empty((n, k), dtype=torch.int32, device=dev),
            torch.empty(rows, dtype=torch.int32, device=dev),
            rows, int(capacity))
    code = lib().cgl_get_layout(
        _ptr(idx), n, k, E, R, _opts(0, capacity), _ptr(out.tokens_per_expert),
        _ptr(out.tokens_per_rank), _ptr(out.is_token_in_rank), _ptr(out.expert_offset),
        _ptr(out.max_count), _ptr(out.dst_pos), _ptr(out.recv_src), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream))
    _check(code, "cgl_get_layout")
    return out


class RankLayout(NamedTuple):
    tokens_per_rank: torch.Tensor     # int32 [R]
    rank_offset: torch.Tensor         # int32 [R + 1]
    max_count: torch.Tensor           # int32 [1]
    rank_dst: torch.Tensor            # int32 [N, k]  (row per first slot on each rank, else -1)
    recv_token: torch.Tensor          # int32 [num_recv_rows]
    num_recv_rows: int                # N*k (compact) or R*capacity (padded)
    capacity: int


def get_rank_layout(topk_idx: torch.Tensor, num_experts: int, num_ranks: int, capacity: int = 0, *,
                    status: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    out: Optional[RankLayout] = None, stream=None) -> RankLayout:
    """One copy per (token, destination rank): the deduplicated layout (cgl_get_rank_layout)."""
    idx = _dev(topk_idx, "topk_idx", torch.int32, 2)
    n, k = idx.shape
    E, R = int(num_experts), int(num_ranks)
    dev = idx.device
    rows = R * capacity if capacity > 0 else n * k
    ws_bytes = layout_workspace_bytes(n, k, R, R)
    if ws_bytes == 0 or E % R:
        raise CglError(EINVAL, "get_rank_layout", "invalid sizes")
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if out is None:
        out = RankLayout(
            torch.empty(R, dtype=torch.int32, device=dev),
            torch.empty(R + 1, dtype=torch.int32, device=dev),
            torch.empty(1, dtype=torch.int32, device=dev),
            torch.empty((n, k), dtype=torch.int32, device=dev),
            torch.empty(rows, dtype=torch.int32, device=dev),
            rows, int(capacity))
    code = lib().cgl_get_rank_layout(
        _ptr(idx), n, k, E, R, _opts(0, capacity), _ptr(out.tokens_per_rank), _ptr(out.rank_offset),
        _ptr(out.max_count), _ptr(out.rank_dst), _ptr(out.recv_token), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream))
    _check(code, "cgl_get_rank_layout")
    return out


def dispatch_fp8(x: torch.Tensor, dst_pos: torch.Tensor, num_recv_rows: int, *,
                 recv_x: Optional[torch.Tensor] = None, recv_scale: Optional[torch.Tensor] = None,
                 status: Optional[torch.Tensor] = None, num_sms: int = 0, pow2_scales: bool = False,
                 scratch: Optional[torch.Tensor] = None, stream=None):
    """FP8 E4M3 dispatch with per-token 1x128 fp32 scales (cgl_dispatch_fp8).

    pow2_scales: power-of-two (UE8M0) scales (CGL_OPT_UE8M0_SCALES).
    scratch: new_scratch() (cgl_opts.scratch): tokens handed out dynamically, same results.
    Returns (recv_x uint8 [rows, H], recv_scale fp32 [rows, H/128]); rows that
    receive no copy are left as they were (uninitialised when allocated here)."""
    x = _dev(x, "x", torch.bfloat16, 2)
    dst = _dev(dst_pos, "dst_pos", torch.int32, 2)
    n, h = x.shape
    k = dst.shape[1]
    if recv_x is None:
        recv_x = torch.empty((num_recv_rows, h), dtype=torch.uint8, device=x.device)
    if recv_scale is None:
        recv_scale = torch.empty((num_recv_rows, h // 128), dtype=torch.float32, device=x.device)
    code = lib().cgl_dispatch_fp8(_ptr(x), n, h, k, _ptr(dst), _ptr(recv_x), _ptr(recv_scale),
                                  int(num_recv_rows), _opts(num_sms, 0, pow2_scales, scratch), _ptr(status),
                                  _stream(stream))
    _check(code, "cgl_dispatch_fp8")
    return recv_x, recv_scale


def dispatch_bf16(x: torch.Tensor, dst_pos: torch.Tensor, num_recv_rows: int, *,
                  recv_x: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                  num_sms: int = 0, scratch: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """BF16 row dispatch (cgl_dispatch_bf16); also the combine-backward re-dispatch of grads.

    scratch: new_scratch() (cgl_opts.scratch): tokens handed out dynamically, same results."""
    x = _dev(x, "x", torch.bfloat16, 2)
    dst = _dev(dst_pos, "dst_pos", torch.int32, 2)
    n, h = x.shape
    k = dst.shape[1]
    if recv_x is None:
        recv_x = torch.empty((num_recv_rows, h), dtype=torch.bfloat16, device=x.device)
    code = lib().cgl_dispatch_bf16(_ptr(x), n, h, k, _ptr(dst), _ptr(recv_x), int(num_recv_rows),
                                   _opts(num_sms, 0, False, scratch), _ptr(status), _stream(stream))
    _check(code, "cgl_dispatch_bf16")
    return recv_x


def combine(y: torch.Tensor, dst_pos: torch.Tensor, topk_weights: torch.Tensor, *,
            out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
            num_sms: int = 0, stream=None) -> torch.Tensor:
    """Top-k weighted BF16 combine with an fp32 fixed-order accumulator (cgl_combine)."""
    y = _dev(y, "y", torch.bfloat16, 2)
    dst = _dev(dst_pos, "dst_pos", torch.int32, 2)
    w = _dev(topk_weights, "topk_weights", torch.float32, 2)
    n, k = dst.shape
    h = y.shape[1]
    if out is None:
        out = torch.empty((n, h), dtype=torch.bfloat16, device=y.device)
    code = lib().cgl_combine(_ptr(y), y.shape[0], _ptr(dst), _ptr(w), n, h, k, _ptr(out),
                             _opts(num_sms), _ptr(status), _stream(stream))
    _check(code, "cgl_combine")
    return out


def combine_backward(grad_out: torch.Tensor, y: torch.Tensor, dst_pos: torch.Tensor,
                     topk_weights: torch.Tensor, *, grad_y: Optional[torch.Tensor] = None,
                     grad_w: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                     num_sms: int = 0, stream=None):
    """Gradient of combine: (grad_y BF16 [rows, H], grad_w fp32 [N, k]) (cgl_combine_backward)."""
    g = _dev(grad_out, "grad_out", torch.bfloat16, 2)
    y = _dev(y, "y", torch.bfloat16, 2)
    dst = _dev(dst_pos, "dst_pos", torch.int32, 2)
    w = _dev(topk_weights, "topk_weights", torch.float32, 2)
    n, k = dst.shape
    h = g.shape[1]
    if grad_y is None:
        grad_y = torch.empty_like(y)
    if grad_w is None:
        grad_w = torch.empty((n, k), dtype=torch.float32, device=g.device)
    code = lib().cgl_combine_backward(_ptr(g), _ptr(y), y.shape[0], _ptr(dst), _ptr(w), n, h, k,
                                      _ptr(grad_y), _ptr(grad_w), _opts(num_sms), _ptr(status),
                                      _stream(stream))
    _check(code, "cgl_combine_backward")
    return grad_y, grad_w


def decode_dispatch_fp8(topk_idx: torch.Tensor, x: torch.Tensor, num_experts: int, num_ranks: int,
                        capacity: int = 0, *, out: Optional[Layout] = None,
                        recv_x: Optional[torch.Tensor] = None, recv_scale: Optional[torch.Tensor] = None,
                        status: Optional[torch.Tensor] = None, num_sms: int = 0, pow2_scales: bool = False,
                        stream=None):
    """Layout + FP8 dispatch of a small (decode) batch in one launch (cgl_decode_dispatch_fp8).

    Returns (Layout, recv_x uint8 [rows, H], recv_scale fp32 [rows, H/128])."""
    idx = _dev(topk_idx, "topk_idx", torch.int32, 2)
    x = _dev(x, "x", torch.bfloat16, 2)
    n, k = idx.shape
    h = x.shape[1]
    E, R = int(num_experts), int(num_ranks)
    dev = idx.device
    rows = E * capacity if capacity > 0 else n * k
    if out is None:
        out = Layout(
            torch.empty(E, dtype=torch.int32, device=dev),
            torch.empty(R, dtype=torch.int32, device=dev),
            torch.empty((n, R), dtype=torch.uint8, device=dev),
            torch.empty(E + 1, dtype=torch.int32, device=dev),
            torch.empty(1, dtype=torch.int32, device=dev),
            torch.empty((n, k), dtype=torch.int32, device=dev),
            torch.empty(rows, dtype=torch.int32, device=dev),
            rows, int(capacity))
    if recv_x is None:
        recv_x = torch.empty((rows, h), dtype=torch.uint8, device=dev)
    if recv_scale is None:
        recv_scale = torch.empty((rows, h // 128), dtype=torch.float32, device=dev)
    code = lib().cgl_decode_dispatch_fp8(
        _ptr(idx), n, k, E, R, _opts(num_sms, capacity, pow2_scales), _ptr(x), h, _ptr(out.tokens_per_expert),
        _ptr(out.tokens_per_rank), _ptr(out.is_token_in_rank), _ptr(out.expert_offset), _ptr(out.max_count),
        _ptr(out.dst_pos), _ptr(out.recv_src), _ptr(recv_x), _ptr(recv_scale), _ptr(status), _stream(stream))
    _check(code, "cgl_decode_dispatch_fp8")
    return out, recv_x, recv_scale


def layout_dispatch_workspace_bytes(num_tokens: int, num_topk: int, num_experts: int, num_ranks: int) -> int:
    return int(lib().cgl_layout_dispatch_workspace_bytes(num_tokens, num_topk, num_experts, num_ranks))


def layout_dispatch_kernel_count(num_tokens: int, num_topk: int, num_experts: int, num_ranks: int,
                                 hidden: int, num_sms: int = 0) -> int:
    return int(lib().cgl_layout_dispatch_kernel_count(num_tokens, num_topk, num_experts, num_ranks, hidden,
                                                      _opts(num_sms, 0)))


def layout_dispatch_fp8(topk_idx: torch.Tensor, x: torch.Tensor, num_experts: int, num_ranks: int,
                        capacity: int = 0, *, out: Optional[Layout] = None,
                        recv_x: Optional[torch.Tensor] = None, recv_scale: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                        num_sms: int = 0, pow2_scales: bool = False, stream=None):
    """Layout + FP8 dispatch of any batch in one call (cgl_layout_dispatch_fp8).

    Returns (Layout, recv_x uint8 [rows, H], recv_scale fp32 [rows, H/128])."""
    idx = _dev(topk_idx, "topk_idx", torch.int32, 2)
    x = _dev(x, "x", torch.bfloat16, 2)
    n, k = idx.shape
    h = x.shape[1]
    E, R = int(num_experts), int(num_ranks)
    dev = idx.device
    rows = E * capacity if capacity > 0 else n * k
    ws_bytes = layout_dispatch_workspace_bytes(n, k, E, R)
    if ws_bytes == 0:
        raise CglError(EINVAL, "layout_dispatch_fp8", "invalid sizes")
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if out is None:
        out = Layout(
            torch.empty(E, dtype=torch.int32, device=dev),
            torch.empty(R, dtype=torch.int32, device=dev),
            torch.empty((n, R), dtype=torch.uint8, device=dev),
            torch.empty(E + 1, dtype=torch.int32, device=dev),
            torch.empty(1, dtype=torch.int32, device=dev),
            torch.empty((n, k), dtype=torch.int32, device=dev),
            torch.empty(rows, dtype=torch.int32, device=dev),
            rows, int(capacity))
    if recv_x is None:
        recv_x = torch.empty((rows, h), dtype=torch.uint8, device=dev)
    if recv_scale is None:
        recv_scale = torch.empty((rows, h // 128), dtype=torch.float32, device=dev)
    code = lib().cgl_layout_dispatch_fp8(
        _ptr(idx), n, k, E, R, _opts(num_sms, capacity, pow2_scales), _ptr(x), h, _ptr(out.tokens_per_expert),
        _ptr(out.tokens_per_rank), _ptr(out.is_token_in_rank), _ptr(out.expert_offset), _ptr(out.max_count),
        _ptr(out.dst_pos), _ptr(out.recv_src), _ptr(recv_x), _ptr(recv_scale), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream))
    _check(code, "cgl_layout_dispatch_fp8")
    return out, recv_x, recv_scale
