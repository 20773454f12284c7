"""CPU oracle for MoE layout / dispatch / combine: numpy front end over liboracle.so.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the bench's
CPU-baseline leg may import this; the product path never does.  It shares no
code with the CUDA library (its own C source, its own loader, its own error
numbering) and imports nothing from the package.

Each function returns freshly allocated numpy arrays; BF16 data are uint16 bit
patterns.  See oracle.c for the arithmetic and the reading of the DeepEP pages
that each step takes.
"""

from __future__ import annotations

import ctypes as C
from typing import NamedTuple

import numpy as np

from . import build as _build

FLAG_RANGE = 1
FLAG_CAPACITY = 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        L.oracle_set_threads.argtypes = [C.c_int]
        L.oracle_set_threads.restype = C.c_int
        L.oracle_bf16_from_f32.argtypes = [C.c_float]
        L.oracle_bf16_from_f32.restype = C.c_uint16
        L.oracle_bf16_to_f32.argtypes = [C.c_uint16]
        L.oracle_bf16_to_f32.restype = C.c_float
        L.oracle_e4m3_encode.argtypes = [C.c_float]
        L.oracle_e4m3_encode.restype = C.c_uint8
        L.oracle_e4m3_decode.argtypes = [C.c_uint8]
        L.oracle_e4m3_decode.restype = C.c_float
        L.oracle_e4m3_encode_array.argtypes = [P, C.c_int64, P]
        L.oracle_e4m3_encode_array.restype = None
        L.oracle_e4m3_decode_array.argtypes = [P, C.c_int64, P]
        L.oracle_e4m3_decode_array.restype = None
        L.oracle_bf16_from_f32_array.argtypes = [P, C.c_int64, P]
        L.oracle_bf16_from_f32_array.restype = None
        L.oracle_get_layout.argtypes = [P, C.c_int64, C.c_int, C.c_int, C.c_int, C.c_int,
                                        P, P, P, P, P, P, P]
        L.oracle_get_layout.restype = C.c_int
        L.oracle_get_rank_layout.argtypes = [P, C.c_int64, C.c_int, C.c_int, C.c_int, C.c_int,
                                             P, P, P, P, P]
        L.oracle_get_rank_layout.restype = C.c_int
        L.oracle_dispatch_fp8.argtypes = [P, C.c_int64, C.c_int, C.c_int, P, P, P]
        L.oracle_dispatch_fp8_pow2.argtypes = [P, C.c_int64, C.c_int, C.c_int, P, P, P]
        L.oracle_dispatch_fp8.restype = None
        L.oracle_dispatch_fp8_pow2.restype = None
        L.oracle_dispatch_bf16.argtypes = [P, C.c_int64, C.c_int, C.c_int, P, P]
        L.oracle_dispatch_bf16.restype = None
        L.oracle_combine_backward.argtypes = [P, P, P, P, C.c_int64, C.c_int, C.c_int, P, P]
        L.oracle_combine_backward.restype = None
        L.oracle_combine.argtypes = [P, P, P, C.c_int64, C.c_int, C.c_int, P]
        L.oracle_combine.restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(C.c_void_p)


def set_threads(n: int = 0) -> int:
    """Set the OpenMP thread count (0 = leave as is); returns the count in effect."""
    return int(lib().oracle_set_threads(int(n)))


def e4m3_encode(values) -> np.ndarray:
    """E4M3 codes (RNE, saturating) of fp32 values."""
    v = np.ascontiguousarray(values, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


def e4m3_decode(codes) -> np.ndarray:
    """fp32 values of E4M3 codes."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().oracle_e4m3_decode_array(_p(c), c.size, _p(out))
    return out


def bf16_from_f32(values) -> np.ndarray:
    """BF16 bit patterns (RNE) of fp32 values."""
    v = np.ascontiguousarray(values, dtype=np.float32)
    out = np.empty(v.shape, np.uint16)
    lib().oracle_bf16_from_f32_array(_p(v), v.size, _p(out))
    return out


class Layout(NamedTuple):
    tokens_per_expert: np.ndarray   # int32 [E]
    tokens_per_rank: np.ndarray     # int32 [R]
    is_token_in_rank: np.ndarray    # uint8 [N, R]
    expert_offset: np.ndarray       # int32 [E + 1]
    max_count: int
    dst_pos: np.ndarray             # int32 [N, k]
    recv_src: np.ndarray            # int32 [N*k] or [E*capacity]
    flags: int


def get_layout(topk_idx: np.ndarray, num_experts: int, num_ranks: int, capacity: int = 0) -> Layout:
    idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    n, k = idx.shape
    E, R = int(num_experts), int(num_ranks)
    if R <= 0 or E % R != 0:
        raise ValueError("num_experts must be a positive multiple of num_ranks")
    tpe = np.zeros(E, np.int32)
    tpr = np.zeros(R, np.int32)
    itr = np.zeros((n, R), np.uint8)
    off = np.zeros(E + 1, np.int32)
    mx = np.zeros(1, np.int32)
    dst = np.zeros((n, k), np.int32)
    rows = E * capacity if capacity > 0 else n * k
    src = np.zeros(rows, np.int32)
    flags = lib().oracle_get_layout(_p(idx), n, k, E, R, int(capacity), _p(tpe), _p(tpr), _p(itr),
                                    _p(off), _p(mx), _p(dst), _p(src))
    return Layout(tpe, tpr, itr, off, int(mx[0]), dst, src, int(flags))


class RankLayout(NamedTuple):
    tokens_per_rank: np.ndarray     # int32 [R]
    rank_offset: np.ndarray         # int32 [R + 1]
    max_count: int
    rank_dst: np.ndarray            # int32 [N, k]
    recv_token: np.ndarray          # int32 [N*k] or [R*capacity]
    flags: int


def get_rank_layout(topk_idx: np.ndarray, num_experts: int, num_ranks: int, capacity: int = 0) -> RankLayout:
    """Per-rank (deduplicated) layout: one row per (token, destination rank)."""
    idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    n, k = idx.shape
    E, R = int(num_experts), int(num_ranks)
    if R <= 0 or E % R != 0:
        raise ValueError("num_experts must be a positive multiple of num_ranks")
    tpr = np.zeros(R, np.int32)
    off = np.zeros(R + 1, np.int32)
    mx = np.zeros(1, np.int32)
    dst = np.zeros((n, k), np.int32)
    rows = R * capacity if capacity > 0 else n * k
    src = np.zeros(rows, np.int32)
    flags = lib().oracle_get_rank_layout(_p(idx), n, k, E, R, int(capacity), _p(tpr), _p(off), _p(mx),
                                         _p(dst), _p(src))
    return RankLayout(tpr, off, int(mx[0]), dst, src, int(flags))


def dispatch_fp8(x: np.ndarray, dst_pos: np.ndarray, num_rows: int, pow2_scales: bool = False):
    """Returns (recv_x uint8 [num_rows, H], recv_scale fp32 [num_rows, H/128]).

    pow2_scales: power-of-two (UE8M0) scales, scale = the smallest 2^e with
    448 * 2^e >= amax_c, inv = 2^-e.  Rows that receive no copy are zero (the
    CUDA path leaves them unwritten)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    dst = np.ascontiguousarray(dst_pos, dtype=np.int32)
    n, h = x.shape
    k = dst.shape[1]
    if h % 128:
        raise ValueError("hidden must be a multiple of 128 for FP8 dispatch")
    rx = np.zeros((num_rows, h), np.uint8)
    rs = np.zeros((num_rows, h // 128), np.float32)
    fn = lib().oracle_dispatch_fp8_pow2 if pow2_scales else lib().oracle_dispatch_fp8
    fn(_p(x), n, h, k, _p(dst), _p(rx), _p(rs))
    return rx, rs


def dispatch_bf16(x: np.ndarray, dst_pos: np.ndarray, num_rows: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.uint16)
    dst = np.ascontiguousarray(dst_pos, dtype=np.int32)
    n, h = x.shape
    k = dst.shape[1]
    out = np.zeros((num_rows, h), np.uint16)
    lib().oracle_dispatch_bf16(_p(x), n, h, k, _p(dst), _p(out))
    return out


def combine(y: np.ndarray, dst_pos: np.ndarray, topk_w: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.uint16)
    dst = np.ascontiguousarray(dst_pos, dtype=np.int32)
    w = np.ascontiguousarray(topk_w, dtype=np.float32)
    n, k = dst.shape
    h = y.shape[1]
    out = np.zeros((n, h), np.uint16)
    lib().oracle_combine(_p(y), _p(dst), _p(w), n, h, k, _p(out))
    return out


def combine_backward(g: np.ndarray, y: np.ndarray, dst_pos: np.ndarray, topk_w: np.ndarray):
    """Returns (grad_y uint16 [rows, H], grad_w fp32 [N, k]); rows with no slot are zero."""
    g = np.ascontiguousarray(g, dtype=np.uint16)
    y = np.ascontiguousarray(y, dtype=np.uint16)
    dst = np.ascontiguousarray(dst_pos, dtype=np.int32)
    w = np.ascontiguousarray(topk_w, dtype=np.float32)
    n, k = dst.shape
    h = g.shape[1]
    gy = np.zeros(y.shape, np.uint16)
    gw = np.zeros((n, k), np.float32)
    lib().oracle_combine_backward(_p(g), _p(y), _p(dst), _p(w), n, h, k, _p(gy), _p(gw))
    return gy, gw
