"""moe_layout_static_scratch: the allocation-free layout entry point, for callers that cannot
call cudaMalloc (their device memory belongs to another allocator, or their serving loop forbids
allocation calls).  Its outputs must equal the oracle's and those of moe_layout (the layout is
integer work, so equal means bit-exact), on two calls in a row with different problems so that
the second call runs on scratch the first one left behind; one call goes through the Python
binding, the others through the C ABI directly.  Repeated calls must leave the device's free
memory and torch's reserved memory unchanged.  This file is collected last so that a run
stopping at the first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import combine_moe_layout_07_b200 as moe
import oracle
import workloads as W

pytestmark = pytest.mark.gpu

KEYS = ("counts", "psum", "rows_per_rank", "tokens_per_rank", "token_in_rank", "slots", "row_src", "row_weights")


def _c_entry():
    f = moe.lib().moe_layout_static_scratch
    f.argtypes = [ctypes.POINTER(moe.MoeParams)] + [ctypes.c_void_p] * 13
    f.restype = ctypes.c_int
    return f


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _buffers(wl, cap):
    T, k, E, R = wl.tokens, wl.topk, wl.experts, wl.ranks
    dev = "cuda"
    return {
        "counts": torch.full((E,), -9, dtype=torch.int32, device=dev),
        "psum": torch.full((E,), -9, dtype=torch.int32, device=dev),
        "rows_per_rank": torch.full((R,), -9, dtype=torch.int32, device=dev),
        "tokens_per_rank": torch.full((R,), -9, dtype=torch.int32, device=dev),
        "token_in_rank": torch.full((T, R), 7, dtype=torch.uint8, device=dev),
        "slots": torch.full((T, k), -9, dtype=torch.int32, device=dev),
        "row_src": torch.full((R, cap), -9, dtype=torch.int32, device=dev),
        "row_weights": torch.full((R, cap), float("nan"), device=dev),
    }


def _static_layout(wl, idx, w, cap, cpu_sync, with_status, out=None, via_binding=False):
    T, k, E, R = wl.tokens, wl.topk, wl.experts, wl.ranks
    out = _buffers(wl, cap) if out is None else out
    status = torch.full((1,), 12345, dtype=torch.int32, device="cuda") if with_status else None
    p = moe.params(T, R, E, k, wl.hidden, wl.alignment, recv_capacity_rows=cap, do_cpu_sync=cpu_sync)
    stream = torch.cuda.current_stream()
    if via_binding:
        rows = moe.moe_layout_static_scratch(p, idx, w, *(out[key] for key in KEYS), device_status=status,
                                             stream=stream)
        host_rows, rc = (rows if rows is not None else np.zeros(R, np.int32)), moe.MOE_OK
    else:
        host_rows = np.zeros(R, np.int32)
        rc = _c_entry()(ctypes.byref(p), _p(idx), _p(w), *(_p(out[key]) for key in KEYS), _p(status),
                        host_rows.ctypes.data_as(ctypes.c_void_p), ctypes.c_void_p(stream.cuda_stream))
    torch.cuda.synchronize()
    return rc, out, status, host_rows


def _moe_layout(wl, idx, w, cap):
    p = moe.params(wl.tokens, wl.ranks, wl.experts, wl.topk, wl.hidden, wl.alignment, recv_capacity_rows=cap,
                   do_cpu_sync=True)
    h = moe.moe_layout(p, idx, w)
    ref = {"counts": h.counts(), "psum": h.psum(), "rows_per_rank": h.rows_per_rank(),
           "tokens_per_rank": h.tokens_per_rank(), "token_in_rank": h.token_in_rank(), "slots": h.slots(),
           "row_src": h.row_src(), "row_weights": h.row_weights()}
    torch.cuda.synchronize()
    ref = {key: val.clone() for key, val in ref.items()}
    moe.moe_handle_free(h)
    return ref


def _assert_same_as_moe_layout(out, ref):
    for key in ("counts", "psum", "rows_per_rank", "tokens_per_rank", "token_in_rank", "slots"):
        assert torch.equal(out[key], ref[key]), key
    rows = ref["rows_per_rank"].cpu()
    for r in range(rows.numel()):
        n = int(rows[r])
        assert torch.equal(out["row_src"][r, :n], ref["row_src"][r, :n]), ("row_src", r)
        assert torch.equal(out["row_weights"][r, :n].view(torch.int32), ref["row_weights"][r, :n].view(torch.int32))


def _assert_same_as_oracle(out, lay: oracle.Layout):
    assert (out["counts"].cpu().numpy() == lay.cnt).all()
    assert (out["psum"].cpu().numpy() == lay.psum).all()
    assert (out["rows_per_rank"].cpu().numpy() == lay.rows_per_rank).all()
    assert (out["tokens_per_rank"].cpu().numpy() == lay.tokens_per_rank).all()
    assert (out["token_in_rank"].cpu().numpy() == lay.token_in_rank).all()
    assert (out["slots"].cpu().numpy() == lay.slot).all()
    src, rw = out["row_src"].cpu().numpy(), out["row_weights"].cpu().numpy()
    for r in range(lay.rows_per_rank.size):
        n = int(lay.rows_per_rank[r])
        assert (src[r, :n] == lay.row_src[r, :n]).all(), ("row_src", r)
        assert (rw[r, :n].view(np.uint32) == lay.row_w[r, :n].view(np.uint32)).all(), ("row_weights", r)


def _routing(wl, mask):
    idx, w = W.gen_routing(wl)
    if mask:
        idx = W.mask_entries(wl, idx, mask)
    return idx, w


def test_static_scratch_layout_matches_the_oracle_and_moe_layout_on_two_calls_in_a_row():
    cases = [
        # DeepSeek-V3 shape at 2048 tokens per rank (the multi-CTA kernels), host-synced, no status
        (W.WORKLOADS["deepseek"].with_(tokens_per_rank=2048), 0.0, True, False, False),
        # a different problem next (fewer experts and chunks, masked entries, no host sync, the
        # one-CTA kernel) through the Python binding: it reads scratch the first call wrote
        (W.WORKLOADS["tiny"].with_(tokens_per_rank=700, experts=64, ranks=4, topk=6), 0.2, False, True, True),
        # and the multi-CTA kernels again without the host wait, after the one-CTA call
        (W.WORKLOADS["tiny"].with_(tokens_per_rank=1500, experts=32, ranks=4, topk=4), 0.1, False, True, False),
    ]
    for wl, mask, cpu_sync, with_status, via_binding in cases:
        idx_c, w_c = _routing(wl, mask)
        lay = oracle.layout(idx_c.numpy(), w_c.numpy(), wl.experts, wl.ranks, wl.alignment)
        assert lay.status == oracle.OK
        cap = int(lay.rows_per_rank.max())
        lay = oracle.layout(idx_c.numpy(), w_c.numpy(), wl.experts, wl.ranks, wl.alignment, cap=cap)
        idx, w = idx_c.cuda(), w_c.cuda()
        rc, out, status, host_rows = _static_layout(wl, idx, w, cap, cpu_sync, with_status, via_binding=via_binding)
        assert rc == moe.MOE_OK, moe.status_string(rc)
        _assert_same_as_oracle(out, lay)
        _assert_same_as_moe_layout(out, _moe_layout(wl, idx, w, cap))
        if cpu_sync:
            assert (host_rows == lay.rows_per_rank).all()
        if with_status:
            assert int(status.item()) == 0


def test_static_scratch_allocates_no_device_memory():
    """After a first call (which looks up the scratch address and loads the kernels), further
    calls on both kernel paths change neither the device's free memory nor torch's reserved
    memory."""
    cases = [(W.WORKLOADS["deepseek"].with_(tokens_per_rank=512), True),               # multi-CTA
             (W.WORKLOADS["tiny"].with_(tokens_per_rank=100, experts=16, topk=4), False)]  # one CTA
    prepared = []
    for wl, cpu_sync in cases:
        idx, w = (t.cuda() for t in _routing(wl, 0.0))
        cap = wl.tokens * wl.topk
        out = _buffers(wl, cap)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc, _, _, _ = _static_layout(wl, idx, w, cap, cpu_sync, True, out=out)
        assert rc == moe.MOE_OK
        prepared.append((wl, idx, w, cap, cpu_sync, out, status))
    torch.cuda.synchronize()
    free0, reserved0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()
    p_list = [moe.params(wl.tokens, wl.ranks, wl.experts, wl.topk, wl.hidden, wl.alignment, recv_capacity_rows=cap,
                         do_cpu_sync=cpu_sync) for wl, _, _, cap, cpu_sync, _, _ in prepared]
    rows = np.zeros(64, np.int32)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(3):
        for p, (wl, idx, w, cap, cpu_sync, out, status) in zip(p_list, prepared):
            rc = _c_entry()(ctypes.byref(p), _p(idx), _p(w), *(_p(out[key]) for key in KEYS), _p(status),
                            rows.ctypes.data_as(ctypes.c_void_p), stream)
            assert rc == moe.MOE_OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_reserved() == reserved0


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
    # without the host wait the flags have nowhere else to go: a status word is required
    rc, _, _, _ = _static_layout(wl, idx.cuda(), w.cuda(), cap=256, cpu_sync=False, with_status=False)
    assert rc == moe.MOE_ERR_INVALID_ARG
    # a problem larger than the static scratch is refused before any GPU work
    big = moe.params(1 << 20, 8, 256, 8, 7168, 128, recv_capacity_rows=1 << 20, do_cpu_sync=True)
    rc = _c_entry()(ctypes.byref(big), *([ctypes.c_void_p(256)] * 10), None, None, None)
    assert rc == moe.MOE_ERR_SCRATCH_LIMIT
    # and the entry point still agrees with the oracle afterwards
    cap = 200
    lay = oracle.layout(idx.numpy(), w.numpy(), wl.experts, wl.ranks, wl.alignment, cap=cap)
    rc, out, _, _ = _static_layout(wl, idx.cuda(), w.cuda(), cap, cpu_sync=True, with_status=False)
    assert rc == moe.MOE_OK
    _assert_same_as_oracle(out, lay)


def test_static_scratch_capacity_overflow_without_host_wait():
    """The multi-CTA kernels with do_cpu_sync = 0 and too small a capacity: the overflow bit
    reaches device_status, and nothing is written past the caller's row maps."""
    wl = W.WORKLOADS["deepseek"].with_(tokens_per_rank=512)   # 4096 tokens, 32768 pairs
    idx, w = (t.cuda() for t in _routing(wl, 0.0))
    cap, guard, R = 100, 4096, wl.ranks
    out = _buffers(wl, cap)
    src_flat = torch.full((R * cap + guard,), -9, dtype=torch.int32, device="cuda")
    rw_flat = torch.full((R * cap + guard,), -3.0, device="cuda")
    out["row_src"] = src_flat[:R * cap].view(R, cap)
    out["row_weights"] = rw_flat[:R * cap].view(R, cap)
    rc, _, status, _ = _static_layout(wl, idx, w, cap, cpu_sync=False, with_status=True, out=out)
    assert rc == moe.MOE_OK
    assert int(status.item()) & 2
    assert (src_flat[-guard:] == -9).all()
    assert (rw_flat[-guard:] == -3.0).all()
