"""moe_layout_static_scratch: the allocation-free layout entry point, for callers that cannot
call cudaMalloc (their device memory belongs to another allocator, or their serving loop forbids
allocation calls).  Called through the C ABI; its outputs must equal those of moe_layout (the
layout is integer work, so equal means bit-exact), on two calls in a row with different problems
so that the second call runs on scratch the first one left behind.  This file is collected last
so that a run stopping at the first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import combine_moe_layout_07_b200 as moe
import workloads as W

pytestmark = pytest.mark.gpu


def _c_entry():
    f = moe.lib().moe_layout_static_scratch
    f.argtypes = [ctypes.POINTER(moe.MoeParams)] + [ctypes.c_void_p] * 13
    f.restype = ctypes.c_int
    return f


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _static_layout(wl, idx, w, cap, cpu_sync, with_status):
    T, k, E, R = wl.tokens, wl.topk, wl.experts, wl.ranks
    dev = "cuda"
    out = {
        "counts": torch.full((E,), -9, dtype=torch.int32, device=dev),
        "psum": torch.full((E,), -9, dtype=torch.int32, device=dev),
        "rows_per_rank": torch.full((R,), -9, dtype=torch.int32, device=dev),
        "tokens_per_rank": torch.full((R,), -9, dtype=torch.int32, device=dev),
        "token_in_rank": torch.full((T, R), 7, dtype=torch.uint8, device=dev),
        "slots": torch.full((T, k), -9, dtype=torch.int32, device=dev),
        "row_src": torch.full((R, cap), -9, dtype=torch.int32, device=dev),
        "row_weights": torch.full((R, cap), float("nan"), device=dev),
    }
    status = torch.full((1,), 12345, dtype=torch.int32, device=dev) if with_status else None
    host_rows = np.zeros(R, np.int32)
    p = moe.params(T, R, E, k, wl.hidden, wl.alignment, recv_capacity_rows=cap, do_cpu_sync=cpu_sync)
    stream = torch.cuda.current_stream()
    rc = _c_entry()(ctypes.byref(p), _p(idx), _p(w), _p(out["counts"]), _p(out["psum"]), _p(out["rows_per_rank"]),
                    _p(out["tokens_per_rank"]), _p(out["token_in_rank"]), _p(out["slots"]), _p(out["row_src"]),
                    _p(out["row_weights"]), _p(status), host_rows.ctypes.data_as(ctypes.c_void_p),
                    ctypes.c_void_p(stream.cuda_stream))
    torch.cuda.synchronize()
    return rc, out, status, host_rows


def _reference_layout(wl, idx, w, cap):
    p = moe.params(wl.tokens, wl.ranks, wl.experts, wl.topk, wl.hidden, wl.alignment, recv_capacity_rows=cap,
                   do_cpu_sync=True)
    h = moe.moe_layout(p, idx, w)
    ref = {"counts": h.counts(), "psum": h.psum(), "rows_per_rank": h.rows_per_rank(),
           "tokens_per_rank": h.tokens_per_rank(), "token_in_rank": h.token_in_rank(), "slots": h.slots(),
           "row_src": h.row_src(), "row_weights": h.row_weights()}
    moe.moe_handle_free(h)
    torch.cuda.synchronize()
    return ref


def _assert_same(out, ref):
    for key in ("counts", "psum", "rows_per_rank", "tokens_per_rank", "token_in_rank", "slots"):
        assert torch.equal(out[key], ref[key]), key
    rows = ref["rows_per_rank"].cpu()
    for r in range(rows.numel()):
        n = int(rows[r])
        assert torch.equal(out["row_src"][r, :n], ref["row_src"][r, :n]), ("row_src", r)
        assert torch.equal(out["row_weights"][r, :n].view(torch.int32), ref["row_weights"][r, :n].view(torch.int32))


def test_static_scratch_layout_matches_moe_layout_on_two_calls_in_a_row():
    cases = [
        # DeepSeek-V3 shape at 2048 tokens per rank, host-synced, status left in the scratch array
        (W.WORKLOADS["deepseek"].with_(tokens_per_rank=2048), 0.0, True, False),
        # a different problem next (fewer experts and chunks, masked entries, no host sync): it
        # reads scratch regions the first call wrote with other values
        (W.WORKLOADS["tiny"].with_(tokens_per_rank=700, experts=64, ranks=4, topk=6), 0.2, False, True),
    ]
    for wl, mask, cpu_sync, with_status in cases:
        idx, w = W.gen_routing(wl)
        if mask:
            idx = W.mask_entries(wl, idx, mask)
        idx, w = idx.cuda(), w.cuda()
        ref = _reference_layout(wl, idx, w, cap=0)  # rows sized from the counts first
        cap = int(ref["rows_per_rank"].max())
        ref = _reference_layout(wl, idx, w, cap=cap)
        rc, out, status, host_rows = _static_layout(wl, idx, w, cap, cpu_sync, with_status)
        assert rc == moe.MOE_OK, moe.status_string(rc)
        _assert_same(out, ref)
        if cpu_sync:
            assert (host_rows == ref["rows_per_rank"].cpu().numpy()).all()
        if with_status:
            assert int(status.item()) == 0


def test_static_scratch_reports_errors_and_limit():
    wl = W.WORKLOADS["tiny"]
    idx, w = W.gen_routing(wl)
    bad = idx.clone()
    bad[3, 0] = wl.experts
    rc, _, _, _ = _static_layout(wl, bad.cuda(), w.cuda(), cap=256, cpu_sync=True, with_status=False)
    assert rc == moe.MOE_ERR_BAD_EXPERT
    rc, _, status, _ = _static_layout(wl, bad.cuda(), w.cuda(), cap=256, cpu_sync=False, with_status=True)
    assert rc == moe.MOE_OK and int(status.item()) & 1
    rc, _, _, _ = _static_layout(wl, idx.cuda(), w.cuda(), cap=4, cpu_sync=True, with_status=False)
    assert rc == moe.MOE_ERR_CAPACITY
    # a problem larger than the static scratch is refused before any GPU work
    big = moe.params(1 << 20, 8, 256, 8, 7168, 128, recv_capacity_rows=1 << 20, do_cpu_sync=True)
    rc = _c_entry()(ctypes.byref(big), *([ctypes.c_void_p(256)] * 10), None, None, None)
    assert rc == moe.MOE_ERR_SCRATCH_LIMIT
    # and the entry point still agrees with moe_layout afterwards
    cap = 200
    ref = _reference_layout(wl, idx.cuda(), w.cuda(), cap)
    rc, out, _, _ = _static_layout(wl, idx.cuda(), w.cuda(), cap, cpu_sync=True, with_status=False)
    assert rc == moe.MOE_OK
    _assert_same(out, ref)
