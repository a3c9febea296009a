"""CPU oracle for the MoE token round trip -- TEST INFRASTRUCTURE ONLY.

A ctypes wrapper over ``moe_oracle.c`` (plain, single-threaded C, built with gcc by
``oracle/build.py``).  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import it; the library under
``combine_moe_layout_07_b200/`` never does, and this package imports nothing from there.

Arrays are numpy; bf16 tensors travel as uint16 bit patterns.  Every function states the
passage it follows in ``moe_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None

OK, ERR_INVALID_ARG, ERR_BAD_EXPERT, ERR_CAPACITY = 0, -1, -2, -3

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_layout.argtypes = [_I64, _I32, _I32, _I32, _I32, _P, _P, _I64, _P, _P, _P, _P, _P, _P, _P, _P]
        L.oracle_layout_by_sort.argtypes = [_I64, _I32, _I32, _I32, _I32, _P, _P, _P, _P]
        L.oracle_dispatch_bf16.argtypes = [_I64, _I32, _I32, _I32, _I32, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _I32]
        L.oracle_dispatch_fp8.argtypes = [_I64, _I32, _I32, _I32, _I32, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I32]
        L.oracle_combine.argtypes = [_I64, _I32, _I32, _I32, _I64, _I64, _P, _P, _P, _P, _P, _P]
        L.oracle_combine_f64.argtypes = [_I64, _I32, _I32, _I32, _I64, _I64, _P, _P, _P, _P, _P, _P]
        L.oracle_combine_f64.restype = None
        L.oracle_e4m3_from_float.argtypes = [ctypes.c_float]
        L.oracle_e4m3_from_float.restype = ctypes.c_uint8
        L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_to_double.restype = ctypes.c_double
        L.oracle_float_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_float_to_bf16.restype = ctypes.c_uint16
        L.oracle_bf16_to_float.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_float.restype = ctypes.c_float
        L.oracle_quantize_block.argtypes = [_P, _I32, _P, _P]
        L.oracle_quantize_block.restype = None
        L.oracle_combine_backward.argtypes = [_I64, _I32, _I32, _I32, _I32, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _I32]
        L.oracle_grad_weights_f64.argtypes = [_I64, _I32, _I32, _I32, _I64, _I64, _P, _P, _P, _P, _P]
        L.oracle_grad_weights_f64.restype = None
        L.oracle_layout_by_rank.argtypes = [_I64, _I32, _I32, _I32, _P, _P, _P]
        L.oracle_dispatch_by_rank.argtypes = [_I64, _I32, _I32, _I32, _I64, _I64, _P, _P, _P, _P, _I32, _P, _P, _P, _P]
        L.oracle_combine_by_rank.argtypes = [_I64, _I32, _I32, _I32, _I64, _I64, _P, _P, _P, _P, _P]
        L.oracle_grouped_gemm_f64.argtypes = [_I32, _I32, _I32, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


@dataclass
class Layout:
    status: int
    cnt: np.ndarray             # int32 [E]
    psum: np.ndarray            # int32 [E]
    rows_per_rank: np.ndarray   # int32 [R]
    tokens_per_rank: np.ndarray # int32 [R]
    token_in_rank: np.ndarray   # uint8 [T, R]
    slot: np.ndarray            # int32 [T, k]
    row_src: np.ndarray         # int32 [R, cap]  (valid below rows_per_rank)
    row_w: np.ndarray           # fp32 [R, cap]
    cap: int


def layout(idx, w, E: int, R: int, A: int, cap: int | None = None) -> Layout:
    """Layout: counts, aligned per-rank inclusive psum, membership and the token->slot handle
    ("From DeepEP to Mega MoE" s2.2/s2.4; "Why MoE gets stuck on communication" s1)."""
    idx = _c(idx, np.int64)
    T, k = idx.shape
    w = _c(w, np.float32)
    if cap is None:
        cap = T * k + E * A  # larger than any rank can need
    cnt = np.zeros(E, np.int32)
    psum = np.zeros(E, np.int32)
    rpr = np.zeros(R, np.int32)
    tpr = np.zeros(R, np.int32)
    tir = np.zeros((T, R), np.uint8)
    slot = np.zeros((T, k), np.int32)
    row_src = np.full((R, max(cap, 0)), -7, np.int32)
    row_w = np.full((R, max(cap, 0)), np.nan, np.float32)
    st = lib().oracle_layout(T, k, E, R, A, _p(idx), _p(w), cap, _p(cnt), _p(psum), _p(rpr), _p(tpr),
                             _p(tir), _p(slot), _p(row_src), _p(row_w))
    return Layout(st, cnt, psum, rpr, tpr, tir, slot, row_src, row_w, cap)


def layout_by_sort(idx, E: int, R: int, A: int):
    """The sort-based second statement of the slot assignment: (status, cnt, psum, slot)."""
    idx = _c(idx, np.int64)
    T, k = idx.shape
    cnt = np.zeros(E, np.int32)
    psum = np.zeros(E, np.int32)
    slot = np.zeros((T, k), np.int32)
    st = lib().oracle_layout_by_sort(T, k, E, R, A, _p(idx), _p(cnt), _p(psum), _p(slot))
    return st, cnt, psum, slot


def dispatch_bf16(lay: Layout, idx, w, x_bits, E: int, R: int, A: int, cap: int,
                  zero_padding: bool, fill: int = 0xA5A5, want_w: bool = True):
    """BF16 dispatch: (status, recv_x uint16 [R, cap, H], recv_w fp32 [R, cap] or None).
    Rows the method leaves unwritten keep ``fill``."""
    idx = _c(idx, np.int64)
    x_bits = _c(x_bits, np.uint16)
    w = _c(w, np.float32)
    T, k = idx.shape
    H = x_bits.shape[1]
    recv = np.full((R, cap, H), fill, np.uint16)
    rw = np.full((R, cap), np.nan, np.float32) if want_w else None
    st = lib().oracle_dispatch_bf16(T, k, E, R, A, H, cap, _p(idx), _p(w), _p(lay.cnt), _p(lay.psum),
                                    _p(lay.slot), _p(x_bits), _p(recv), _p(rw), int(zero_padding))
    return st, recv, rw


def dispatch_fp8(lay: Layout, idx, w, x_bits, E: int, R: int, A: int, cap: int,
                 zero_padding: bool, fill: int = 0xA5, want_w: bool = True):
    """FP8 dispatch: (status, codes uint8 [R, cap, H], scales fp32 [R, cap, H/128], recv_w)."""
    idx = _c(idx, np.int64)
    x_bits = _c(x_bits, np.uint16)
    w = _c(w, np.float32)
    T, k = idx.shape
    H = x_bits.shape[1]
    codes = np.full((R, cap, H), fill, np.uint8)
    scales = np.full((R, cap, H // 128), np.nan, np.float32)
    rw = np.full((R, cap), np.nan, np.float32) if want_w else None
    st = lib().oracle_dispatch_fp8(T, k, E, R, A, H, cap, _p(idx), _p(w), _p(lay.cnt), _p(lay.psum),
                                   _p(lay.slot), _p(x_bits), _p(codes), _p(scales), _p(rw),
                                   int(zero_padding))
    return st, codes, scales, rw


def combine(idx, slot, y_bits, E: int, R: int, w=None, bias_bits=None):
    """Combine: (status, out uint16 [T, H]) -- fp32, ascending j, bias last, one bf16 rounding
    ("From DeepEP to Mega MoE" s2.3/s2.5; "Why MoE gets stuck on communication" s1)."""
    idx = _c(idx, np.int64)
    slot = _c(slot, np.int32)
    y_bits = _c(y_bits, np.uint16)
    w = _c(w, np.float32)
    bias_bits = _c(bias_bits, np.uint16)
    T, k = idx.shape
    _, cap, H = y_bits.shape
    out = np.zeros((T, H), np.uint16)
    st = lib().oracle_combine(T, k, E, R, H, cap, _p(idx), _p(slot), _p(y_bits), _p(w), _p(bias_bits), _p(out))
    return st, out


def combine_f64(idx, slot, y_bits, E: int, R: int, w=None, bias_bits=None) -> np.ndarray:
    """The same sums in binary64, before any rounding to bf16."""
    idx = _c(idx, np.int64)
    slot = _c(slot, np.int32)
    y_bits = _c(y_bits, np.uint16)
    w = _c(w, np.float32)
    bias_bits = _c(bias_bits, np.uint16)
    T, k = idx.shape
    _, cap, H = y_bits.shape
    out = np.zeros((T, H), np.float64)
    lib().oracle_combine_f64(T, k, E, R, H, cap, _p(idx), _p(slot), _p(y_bits), _p(w), _p(bias_bits), _p(out))
    return out


def e4m3_from_float(v: float) -> int:
    return int(lib().oracle_e4m3_from_float(float(v)))


def e4m3_to_double(c: int) -> float:
    return float(lib().oracle_e4m3_to_double(int(c)))


def quantize_block(x_bits) -> tuple[np.ndarray, float]:
    x_bits = _c(x_bits, np.uint16)
    codes = np.zeros(x_bits.size, np.uint8)
    s = np.zeros(1, np.float32)
    lib().oracle_quantize_block(_p(x_bits), x_bits.size, _p(codes), _p(s))
    return codes, float(s[0])


def float_to_bf16(v: float) -> int:
    return int(lib().oracle_float_to_bf16(float(v)))


def bf16_to_float(b: int) -> float:
    return float(lib().oracle_bf16_to_float(int(b)))


def combine_backward(lay: Layout, idx, grad_out_bits, E: int, R: int, A: int, cap: int, w=None,
                     zero_padding: bool = True, fill: int = 0xA5A5):
    """Backward of combine: (status, grad_y uint16 [R, cap, H]) -- grad_out scattered to every
    routed row, scaled by the pair weight (one fp32 multiply, bf16 rounding) when w is given."""
    idx = _c(idx, np.int64)
    g = _c(grad_out_bits, np.uint16)
    w = _c(w, np.float32)
    T, k = idx.shape
    H = g.shape[1]
    gy = np.full((R, cap, H), fill, np.uint16)
    st = lib().oracle_combine_backward(T, k, E, R, A, H, cap, _p(idx), _p(lay.cnt), _p(lay.psum), _p(lay.slot),
                                       _p(g), _p(w), _p(gy), int(zero_padding))
    return st, gy


def grad_weights_f64(idx, slot, grad_out_bits, y_bits, E: int, R: int) -> np.ndarray:
    """grad_w[t, j] = <grad_out[t], y[row(t, j)]> in binary64 (0 for masked pairs)."""
    idx = _c(idx, np.int64)
    slot = _c(slot, np.int32)
    g = _c(grad_out_bits, np.uint16)
    y = _c(y_bits, np.uint16)
    T, k = idx.shape
    _, cap, H = y.shape
    gw = np.zeros((T, k), np.float64)
    lib().oracle_grad_weights_f64(T, k, E, R, H, cap, _p(idx), _p(slot), _p(g), _p(y), _p(gw))
    return gw


def layout_by_rank(idx, E: int, R: int):
    """(status, token_row int32 [T, R], rows_per_rank int32 [R]) of the non-expanded layout."""
    idx = _c(idx, np.int64)
    T, k = idx.shape
    tr = np.zeros((T, R), np.int32)
    rows = np.zeros(R, np.int32)
    st = lib().oracle_layout_by_rank(T, k, E, R, _p(idx), _p(tr), _p(rows))
    return st, tr, rows


def dispatch_by_rank(idx, w, token_row, x_bits, E: int, R: int, cap: int, fp8: bool, fill: int = 0xA5):
    """By-rank dispatch: (status, recv [R, cap, H] (uint8 codes or uint16 bf16), scales or None,
    recv_topk_idx int32 [R, cap, k], recv_topk_w fp32 [R, cap, k]); untouched entries keep fill /
    -7 / NaN."""
    idx = _c(idx, np.int64)
    w = _c(w, np.float32)
    tr = _c(token_row, np.int32)
    x_bits = _c(x_bits, np.uint16)
    T, k = idx.shape
    H = x_bits.shape[1]
    if fp8:
        recv = np.full((R, cap, H), fill, np.uint8)
        scales = np.full((R, cap, H // 128), np.nan, np.float32)
    else:
        recv = np.full((R, cap, H), fill | (fill << 8), np.uint16)
        scales = None
    ti = np.full((R, cap, k), -7, np.int32)
    tw = np.full((R, cap, k), np.nan, np.float32)
    st = lib().oracle_dispatch_by_rank(T, k, E, R, H, cap, _p(idx), _p(w), _p(tr), _p(x_bits), int(fp8), _p(recv),
                                       _p(scales), _p(ti), _p(tw))
    return st, recv, scales, ti, tw


def combine_by_rank(idx, token_row, y_bits, E: int, R: int, bias_bits=None):
    """By-rank combine: (status, out uint16 [T, H])."""
    idx = _c(idx, np.int64)
    tr = _c(token_row, np.int32)
    y_bits = _c(y_bits, np.uint16)
    bias_bits = _c(bias_bits, np.uint16)
    T, k = idx.shape
    _, cap, H = y_bits.shape
    out = np.zeros((T, H), np.uint16)
    st = lib().oracle_combine_by_rank(T, k, E, R, H, cap, _p(idx), _p(tr), _p(y_bits), _p(bias_bits), _p(out))
    return st, out


def grouped_gemm_f64(lay: Layout, codes, scales, w_codes, w_scales, E: int, R: int, A: int):
    """Expert GEMM over the dispatch layout, binary64 ("From DeepEP to Mega MoE" s3.2 Linear1 and
    s4.5 GEMM L1 on the expert buffer): (status, out float64 [R, cap, N]); rows outside every
    expert range stay NaN."""
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    w_codes = _c(w_codes, np.uint8)
    w_scales = _c(w_scales, np.float32)
    _, cap, H = codes.shape
    N = w_codes.shape[1]
    out = np.full((R, cap, N), np.nan, np.float64)
    st = lib().oracle_grouped_gemm_f64(E, R, A, cap, H, N, _p(lay.cnt), _p(lay.psum), _p(codes), _p(scales),
                                       _p(w_codes), _p(w_scales), _p(out))
    return st, out

