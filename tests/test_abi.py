"""The C ABI library loads, exports every entry point include/moe.h declares, and rejects bad
arguments on the host before touching a GPU (no CUDA device needed for any of these)."""
import ctypes
import os
import re

import pytest

import combine_moe_layout_07_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_round_trip():
    names = declared_functions()
    for required in ("moe_layout", "moe_dispatch", "moe_combine", "moe_handle_free", "moe_handle_status",
                     "moe_recv_capacity_hint"):
        assert required in names


def test_library_exports_every_declared_symbol():
    L = moe.lib()
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_capacity_hint_formula():
    # decode shape: 8 ranks, 256 experts, top-8, A=128, 256 tokens per rank
    p = moe.params(1024, 8, 256, 8, 7168, 128, recv_capacity_rows=1, do_cpu_sync=False)
    assert moe.moe_recv_capacity_hint(p, 256) == 8 * 256 * 8 + 32 * 127
    # top-k larger than the experts of one rank: a token reaches at most E_loc of them
    p = moe.params(64, 4, 8, 6, 256, 4, recv_capacity_rows=1)
    assert moe.moe_recv_capacity_hint(p, 10) == 4 * 10 * 2 + 2 * 3


@pytest.mark.parametrize("field,value,code", [
    ("num_experts", 7, moe.MOE_ERR_INVALID_ARG),        # E % R != 0
    ("num_logical_ranks", 0, moe.MOE_ERR_INVALID_ARG),
    ("topk", 0, moe.MOE_ERR_INVALID_ARG),
    ("topk", 33, moe.MOE_ERR_UNSUPPORTED),
    ("num_experts", 8192, moe.MOE_ERR_UNSUPPORTED),
    ("hidden", 100, moe.MOE_ERR_INVALID_ARG),           # not a multiple of 8
    ("expert_alignment", 0, moe.MOE_ERR_INVALID_ARG),
    ("num_tokens", -1, moe.MOE_ERR_INVALID_ARG),
    ("flags", 4, moe.MOE_ERR_INVALID_ARG),               # only MOE_LAYOUT_BY_RANK | MOE_DEFER_EPILOGUE
    ("do_cpu_sync", 2, moe.MOE_ERR_INVALID_ARG),
    ("num_tokens", 1 << 40, moe.MOE_ERR_UNSUPPORTED),   # row indices would overflow int32
])
def test_layout_rejects_bad_params_before_any_launch(field, value, code):
    p = moe.params(64, 2, 8, 2, 256, 16, recv_capacity_rows=0, do_cpu_sync=True)
    setattr(p, field, value)
    h = ctypes.c_void_p(123)
    rc = moe.lib().moe_layout(ctypes.byref(p), ctypes.c_void_p(0x1000), None, None, ctypes.byref(h), None)
    assert rc == code
    assert h.value is None          # *out_handle cleared


def test_layout_without_host_sync_needs_capacity():
    p = moe.params(64, 2, 8, 2, 256, 16, recv_capacity_rows=0, do_cpu_sync=False)
    h = ctypes.c_void_p()
    assert moe.lib().moe_layout(ctypes.byref(p), ctypes.c_void_p(0x1000), None, None, ctypes.byref(h),
                                None) == moe.MOE_ERR_INVALID_ARG


def test_null_and_misaligned_arguments():
    L = moe.lib()
    p = moe.params(64, 2, 8, 2, 256, 16)
    assert L.moe_layout(ctypes.byref(p), ctypes.c_void_p(0x1000), None, None, None, None) == moe.MOE_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert L.moe_layout(ctypes.byref(p), None, None, None, ctypes.byref(h), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_layout(ctypes.byref(p), ctypes.c_void_p(0x1004), None, None, ctypes.byref(h), None) \
        == moe.MOE_ERR_INVALID_ARG        # int64 topk_idx must be 8-byte aligned
    assert L.moe_dispatch(None, None, 0, None, None, None, 1, 1, 1, 0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_combine(None, None, None, None, None, 1, 0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_handle_status(None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_handle_free(None) == moe.MOE_OK


def test_status_strings():
    for code in range(-8, 1):
        assert moe.status_string(code) and moe.status_string(code) != "unknown status"


def test_deferred_epilogue_needs_a_host_sync():
    p = moe.params(64, 2, 8, 2, 256, 16, recv_capacity_rows=64, do_cpu_sync=False, defer_epilogue=True)
    h = ctypes.c_void_p(123)
    rc = moe.lib().moe_layout(ctypes.byref(p), ctypes.c_void_p(0x1000), None, None, ctypes.byref(h), None)
    assert rc == moe.MOE_ERR_INVALID_ARG and h.value is None


def test_wait_and_event_calls_reject_null_on_the_host():
    L = moe.lib()
    assert L.moe_handle_wait(None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_event_wait(None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_event_synchronize(None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_event_query(None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_event_record(None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_event_free(None) == moe.MOE_OK
    assert moe.status_string(moe.MOE_NOT_READY) == "not complete yet"


def test_layout_dispatch_rejects_bad_arguments_on_the_host():
    L = moe.lib()
    h = ctypes.c_void_p(123)
    ok = moe.params(64, 2, 8, 2, 256, 16, recv_capacity_rows=64, do_cpu_sync=False)

    def call(p, x=0x1000, dtype=moe.MOE_DTYPE_BF16, recv=0x2000, scales=None, zp=1, out=ctypes.byref(h)):
        return L.moe_layout_dispatch(ctypes.byref(p), ctypes.c_void_p(0x3000), None, ctypes.c_void_p(x), dtype,
                                     ctypes.c_void_p(recv), scales, None, zp, None, out)

    assert call(moe.params(64, 2, 8, 2, 256, 16, recv_capacity_rows=64, do_cpu_sync=True)) == moe.MOE_ERR_INVALID_ARG
    assert h.value is None                                   # *out_handle cleared
    assert call(moe.params(64, 2, 8, 2, 256, 16, recv_capacity_rows=64, do_cpu_sync=False,
                           by_rank=True)) == moe.MOE_ERR_INVALID_ARG
    assert call(moe.params(64, 2, 8, 2, 256, 16, recv_capacity_rows=0, do_cpu_sync=False)) == moe.MOE_ERR_INVALID_ARG
    assert call(ok, dtype=7) == moe.MOE_ERR_INVALID_ARG
    assert call(ok, x=0x1008) == moe.MOE_ERR_INVALID_ARG      # rows must be 16-byte aligned
    assert call(ok, zp=2) == moe.MOE_ERR_INVALID_ARG
    assert call(ok, dtype=moe.MOE_DTYPE_FP8_E4M3) == moe.MOE_ERR_INVALID_ARG   # FP8 needs scales
    assert call(ok, out=None) == moe.MOE_ERR_INVALID_ARG
