"""Python binding of the single-B200 MoE round-trip library (``include/moe.h``).

Argument marshalling only: every function below passes torch tensors' device pointers and the
current CUDA stream to the C ABI of ``libmoe_b200.so`` and raises ``MoeError`` on a non-OK status.
All layout, dispatch and combine work runs in the library's CUDA kernels; there is no CPU path.
If the library cannot be loaded (or built with nvcc), importing the entry points raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

from . import build as _build

MOE_NOT_READY = 1
MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_BAD_EXPERT = -2
MOE_ERR_CAPACITY = -3
MOE_ERR_CUDA = -4
MOE_ERR_OOM = -5
MOE_ERR_UNSUPPORTED = -6
MOE_ERR_SCRATCH_LIMIT = -7
MOE_ERR_TIMEOUT = -8
MOE_DTYPE_BF16 = 0
MOE_DTYPE_FP8_E4M3 = 1
MOE_LAYOUT_BY_RANK = 1
MOE_DEFER_EPILOGUE = 2

_lib: Optional[ctypes.CDLL] = None


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class MoeParams(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int64),
        ("num_logical_ranks", ctypes.c_int32),
        ("num_experts", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("hidden", ctypes.c_int32),
        ("expert_alignment", ctypes.c_int32),
        ("num_sms", ctypes.c_int32),
        ("do_cpu_sync", ctypes.c_int32),
        ("flags", ctypes.c_int32),
        ("recv_capacity_rows", ctypes.c_int64),
    ]


def params(num_tokens: int, num_logical_ranks: int, num_experts: int, topk: int, hidden: int,
           expert_alignment: int, recv_capacity_rows: int = 0, num_sms: int = 0,
           do_cpu_sync: bool = True, by_rank: bool = False, defer_epilogue: bool = False) -> MoeParams:
    flags = (MOE_LAYOUT_BY_RANK if by_rank else 0) | (MOE_DEFER_EPILOGUE if defer_epilogue else 0)
    return MoeParams(num_tokens, num_logical_ranks, num_experts, topk, hidden, expert_alignment,
                     num_sms, int(do_cpu_sync), flags, recv_capacity_rows)


_P, _I64, _I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int


def lib() -> ctypes.CDLL:
    """Load (building first if the sources are newer) the in-tree CUDA library."""
    global _lib
    if _lib is None:
        path = _build.build(debug=os.environ.get("MOE_B200_DEBUG") == "1")
        L = ctypes.CDLL(path)
        PP = ctypes.POINTER(MoeParams)
        L.moe_recv_capacity_hint.argtypes = [PP, _I64]
        L.moe_recv_capacity_hint.restype = _I64
        L.moe_layout.argtypes = [PP, _P, _P, _P, ctypes.POINTER(_P), _P]
        L.moe_dispatch.argtypes = [_P, _P, _I32, _P, _P, _P, _I64, _I32, _I32, _I32, _P]
        L.moe_layout_dispatch.argtypes = [PP, _P, _P, _P, _I32, _P, _P, _P, _I32, _P, ctypes.POINTER(_P)]
        L.moe_combine.argtypes = [_P, _P, _P, _P, _P, _I64, _I32, _P]
        L.moe_handle_status.argtypes = [_P, _P]
        L.moe_combine_backward.argtypes = [_P, _P, _P, _P, _I64, _I32, _P, _P, _I32, _P]
        L.moe_dispatch_by_rank.argtypes = [_P, _P, _P, _I32, _P, _P, _P, _P, _I64, _I32, _P]
        L.moe_combine_by_rank.argtypes = [_P, _P, _P, _P, _I64, _I32, _P]
        for name in ("counts", "psum", "rows_per_rank", "tokens_per_rank", "token_in_rank", "slots",
                     "row_src", "row_weights", "token_rows"):
            f = getattr(L, f"moe_handle_{name}")
            f.argtypes = [_P]
            f.restype = _P
        L.moe_handle_row_capacity.argtypes = [_P]
        L.moe_handle_row_capacity.restype = _I64
        L.moe_handle_free.argtypes = [_P]
        L.moe_handle_wait.argtypes = [_P, _P]
        L.moe_expert_gemm_fp8.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I32, _P]
        L.moe_event_record.argtypes = [_P, ctypes.POINTER(_P)]
        for name in ("wait",):
            getattr(L, f"moe_event_{name}").argtypes = [_P, _P]
        for name in ("synchronize", "query", "free"):
            getattr(L, f"moe_event_{name}").argtypes = [_P]
        L.moe_status_string.argtypes = [_I32]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_kernel_launch_count.argtypes = []
        L.moe_kernel_launch_count.restype = _I64
        _lib = L
    return _lib


def library_path() -> str:
    return _build.DEBUG_LIB if os.environ.get("MOE_B200_DEBUG") == "1" else _build.LIB


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(rc: int, where: str) -> None:
    if rc != MOE_OK:
        raise MoeError(rc, where)


class _DeviceView:
    """A device array owned by the handle, exposed through the CUDA array interface."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (ptr, False), "version": 3, "strides": None}


class Handle:
    """Owns a ``moe_handle_t*``; free with ``moe_handle_free`` (or let it be collected)."""

    def __init__(self, ptr: int, p: MoeParams, host_rows: Optional[np.ndarray]):
        self.ptr = ptr
        self.params = p
        self.host_rows_per_rank = host_rows

    def _view(self, fn: str, shape, typestr: str) -> torch.Tensor:
        addr = getattr(lib(), f"moe_handle_{fn}")(self.ptr)
        if not addr or 0 in shape:
            dt = {"<i4": torch.int32, "<f4": torch.float32, "|u1": torch.uint8}[typestr]
            return torch.zeros(shape, dtype=dt, device="cuda")
        return torch.as_tensor(_DeviceView(addr, shape, typestr), device="cuda")

    # copies of the handle's device arrays (clones: valid after the handle is freed)
    def counts(self):
        return self._view("counts", (self.params.num_experts,), "<i4").clone()

    def psum(self):
        return self._view("psum", (self.params.num_experts,), "<i4").clone()

    def rows_per_rank(self):
        return self._view("rows_per_rank", (self.params.num_logical_ranks,), "<i4").clone()

    def tokens_per_rank(self):
        return self._view("tokens_per_rank", (self.params.num_logical_ranks,), "<i4").clone()

    def token_in_rank(self):
        return self._view("token_in_rank", (self.params.num_tokens, self.params.num_logical_ranks), "|u1").clone()

    def slots(self):
        return self._view("slots", (self.params.num_tokens, self.params.topk), "<i4").clone()

    def token_rows(self):
        return self._view("token_rows", (self.params.num_tokens, self.params.num_logical_ranks), "<i4").clone()

    def row_capacity(self) -> int:
        return int(lib().moe_handle_row_capacity(self.ptr))

    def row_src(self):
        return self._view("row_src", (self.params.num_logical_ranks, self.row_capacity()), "<i4").clone()

    def row_weights(self):
        return self._view("row_weights", (self.params.num_logical_ranks, self.row_capacity()), "<f4").clone()

    def __del__(self):
        # stream-ordered free on the layout stream (see moe_handle_free)
        if getattr(self, "ptr", None) and _lib is not None:
            _lib.moe_handle_free(self.ptr)
            self.ptr = None


def moe_recv_capacity_hint(p: MoeParams, max_tokens_per_rank: int) -> int:
    v = lib().moe_recv_capacity_hint(ctypes.byref(p), max_tokens_per_rank)
    if v < 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_recv_capacity_hint")
    return int(v)


def moe_layout(p: MoeParams, topk_idx: torch.Tensor, topk_weights: Optional[torch.Tensor] = None,
               stream=None) -> Handle:
    """Layout of one dispatch; with ``do_cpu_sync`` the host row counts are on the handle (with
    ``defer_epilogue`` only after ``moe_handle_wait``)."""
    h = ctypes.c_void_p()
    deferred = bool(p.flags & MOE_DEFER_EPILOGUE)
    rows = np.zeros(p.num_logical_ranks, np.int32) if p.do_cpu_sync and not deferred else None
    rc = lib().moe_layout(ctypes.byref(p), _ptr(topk_idx), _ptr(topk_weights), _stream(stream),
                          ctypes.byref(h), None if rows is None else rows.ctypes.data_as(_P))
    _check(rc, "moe_layout")
    return Handle(h.value, p, rows)


def moe_dispatch(handle: Handle, x: torch.Tensor, out_dtype: int, recv_x: torch.Tensor,
                 recv_scales: Optional[torch.Tensor] = None, recv_weights: Optional[torch.Tensor] = None,
                 cap: Optional[int] = None, do_expand: bool = True, do_zero_padding: bool = True,
                 num_sms: int = 0, stream=None) -> None:
    cap = recv_x.shape[1] if cap is None else cap
    rc = lib().moe_dispatch(handle.ptr, _ptr(x), out_dtype, _ptr(recv_x), _ptr(recv_scales), _ptr(recv_weights),
                            cap, int(do_expand), int(do_zero_padding), num_sms, _stream(stream))
    _check(rc, "moe_dispatch")


def moe_layout_dispatch(p: MoeParams, topk_idx: torch.Tensor, topk_weights: Optional[torch.Tensor], x: torch.Tensor,
                        out_dtype: int, recv_x: torch.Tensor, recv_scales: Optional[torch.Tensor] = None,
                        recv_weights: Optional[torch.Tensor] = None, do_zero_padding: bool = True,
                        stream=None) -> Handle:
    """Layout and expanded dispatch in one call (no host sync): the same results as moe_layout
    followed by moe_dispatch with cap = p.recv_capacity_rows and num_sms = p.num_sms."""
    h = ctypes.c_void_p()
    rc = lib().moe_layout_dispatch(ctypes.byref(p), _ptr(topk_idx), _ptr(topk_weights), _ptr(x), out_dtype,
                                   _ptr(recv_x), _ptr(recv_scales), _ptr(recv_weights), int(do_zero_padding),
                                   _stream(stream), ctypes.byref(h))
    _check(rc, "moe_layout_dispatch")
    return Handle(h.value, p, None)


def moe_combine(handle: Handle, y: torch.Tensor, out: torch.Tensor, topk_weights: Optional[torch.Tensor] = None,
                bias: Optional[torch.Tensor] = None, cap: Optional[int] = None, num_sms: int = 0,
                stream=None) -> None:
    cap = y.shape[1] if cap is None else cap
    rc = lib().moe_combine(handle.ptr, _ptr(y), _ptr(topk_weights), _ptr(bias), _ptr(out), cap, num_sms,
                           _stream(stream))
    _check(rc, "moe_combine")


def moe_dispatch_by_rank(handle: Handle, x: torch.Tensor, out_dtype: int, recv_x: torch.Tensor,
                         recv_scales: Optional[torch.Tensor] = None, topk_idx: Optional[torch.Tensor] = None,
                         recv_topk_idx: Optional[torch.Tensor] = None,
                         recv_topk_weights: Optional[torch.Tensor] = None, cap: Optional[int] = None,
                         num_sms: int = 0, stream=None) -> None:
    """Non-expanded dispatch: one row per (token, rank) with the token's per-rank top-k views."""
    cap = recv_x.shape[1] if cap is None else cap
    rc = lib().moe_dispatch_by_rank(handle.ptr, _ptr(x), _ptr(topk_idx), out_dtype, _ptr(recv_x), _ptr(recv_scales),
                                    _ptr(recv_topk_idx), _ptr(recv_topk_weights), cap, num_sms, _stream(stream))
    _check(rc, "moe_dispatch_by_rank")


def moe_combine_by_rank(handle: Handle, y: torch.Tensor, out: torch.Tensor, bias: Optional[torch.Tensor] = None,
                        cap: Optional[int] = None, num_sms: int = 0, stream=None) -> None:
    """Non-expanded combine: sum of the token's per-rank partial sums (+ bias)."""
    cap = y.shape[1] if cap is None else cap
    rc = lib().moe_combine_by_rank(handle.ptr, _ptr(y), _ptr(bias), _ptr(out), cap, num_sms, _stream(stream))
    _check(rc, "moe_combine_by_rank")


def moe_combine_backward(handle: Handle, grad_out: torch.Tensor, grad_y: torch.Tensor,
                         topk_weights: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                         grad_weights: Optional[torch.Tensor] = None, cap: Optional[int] = None,
                         do_zero_padding: bool = True, num_sms: int = 0, stream=None) -> None:
    """Backward of moe_combine: grad_y (and grad_weights when given, which needs y)."""
    cap = grad_y.shape[1] if cap is None else cap
    rc = lib().moe_combine_backward(handle.ptr, _ptr(grad_out), _ptr(topk_weights), _ptr(grad_y), cap,
                                    int(do_zero_padding), _ptr(y), _ptr(grad_weights), num_sms, _stream(stream))
    _check(rc, "moe_combine_backward")


def moe_handle_status(handle: Handle, stream=None) -> int:
    return int(lib().moe_handle_status(handle.ptr, _stream(stream)))


def moe_handle_free(handle: Handle) -> None:
    if handle.ptr:
        rc = lib().moe_handle_free(handle.ptr)
        handle.ptr = None
        _check(rc, "moe_handle_free")


def moe_kernel_launch_count() -> int:
    return int(lib().moe_kernel_launch_count())


def moe_layout_static_scratch(p: MoeParams, topk_idx: torch.Tensor, topk_weights: Optional[torch.Tensor],
                              counts: torch.Tensor, psum: torch.Tensor, rows_per_rank: torch.Tensor,
                              tokens_per_rank: torch.Tensor, token_in_rank: torch.Tensor, slots: torch.Tensor,
                              row_src: torch.Tensor, row_weights: torch.Tensor,
                              device_status: Optional[torch.Tensor] = None, stream=None) -> Optional[np.ndarray]:
    """The layout into caller-owned buffers, with no allocation by the library (see the C header).
    Returns the host row counts when ``p.do_cpu_sync`` is set."""
    L = lib()
    f = L.moe_layout_static_scratch
    f.argtypes = [ctypes.POINTER(MoeParams)] + [_P] * 13
    rows = np.zeros(p.num_logical_ranks, np.int32) if p.do_cpu_sync else None
    rc = f(ctypes.byref(p), _ptr(topk_idx), _ptr(topk_weights), _ptr(counts), _ptr(psum), _ptr(rows_per_rank),
           _ptr(tokens_per_rank), _ptr(token_in_rank), _ptr(slots), _ptr(row_src), _ptr(row_weights),
           _ptr(device_status), None if rows is None else rows.ctypes.data_as(_P), _stream(stream))
    _check(rc, "moe_layout_static_scratch")
    return rows


def moe_handle_wait(handle: Handle) -> np.ndarray:
    """The deferred epilogue of a ``defer_epilogue`` layout: blocks until the counts are on the
    host, raises ``MoeError`` on a bad expert id or a capacity overflow, and returns (and keeps on
    the handle) the rows each logical rank receives."""
    rows = np.zeros(handle.params.num_logical_ranks, np.int32)
    _check(lib().moe_handle_wait(handle.ptr, rows.ctypes.data_as(_P)), "moe_handle_wait")
    handle.host_rows_per_rank = rows
    return rows


class Event:
    """A point recorded on a stream (``moe_event_record``); freed when collected."""

    def __init__(self, stream=None):
        e = ctypes.c_void_p()
        _check(lib().moe_event_record(_stream(stream), ctypes.byref(e)), "moe_event_record")
        self.ptr = e.value

    def wait(self, stream=None) -> None:
        """Work enqueued on ``stream`` after this call waits for the event (returns at once)."""
        _check(lib().moe_event_wait(self.ptr, _stream(stream)), "moe_event_wait")

    def synchronize(self) -> None:
        _check(lib().moe_event_synchronize(self.ptr), "moe_event_synchronize")

    def query(self) -> bool:
        rc = lib().moe_event_query(self.ptr)
        if rc == MOE_NOT_READY:
            return False
        _check(rc, "moe_event_query")
        return True

    def __del__(self):
        if getattr(self, "ptr", None) and _lib is not None:
            _lib.moe_event_free(self.ptr)
            self.ptr = None


def moe_event_record(stream=None) -> Event:
    return Event(stream)


def moe_expert_gemm_fp8(handle: Handle, recv_x: torch.Tensor, recv_scales: torch.Tensor, w: torch.Tensor,
                        w_scales: torch.Tensor, out: torch.Tensor, cap: Optional[int] = None, num_sms: int = 0,
                        stream=None) -> None:
    """The first expert GEMM on an FP8 dispatch's output: out [R, cap, N] (bf16) from recv_x
    [R, cap, H] (E4M3 codes as uint8), recv_scales, w [E, N, H] (E4M3 codes) and w_scales
    [E, N/128, H/128]."""
    cap = recv_x.shape[1] if cap is None else cap
    rc = lib().moe_expert_gemm_fp8(handle.ptr, _ptr(recv_x), _ptr(recv_scales), _ptr(w), _ptr(w_scales), _ptr(out),
                                   w.shape[1], cap, num_sms, _stream(stream))
    _check(rc, "moe_expert_gemm_fp8")

