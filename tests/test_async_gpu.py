"""The asynchronous surface on the GPU, against the oracle.

- A deferred count epilogue: moe_layout with do_cpu_sync and MOE_DEFER_EPILOGUE returns at once,
  dispatch and combine are issued before the host waits, and moe_handle_wait delivers the counts
  (or the device-detected conditions).
- Events that run the round trip on a communication stream, ordered after a compute stream and
  awaited by it ("Why MoE gets stuck on communication", sections 1 and 2: issue, independent
  work, wait).
Every result is compared bit-exactly with the oracle on the same seeded inputs.
"""
import numpy as np
import pytest
import torch

import combine_moe_layout_07_b200 as moe
import oracle
import workloads as W
from gpu_helpers import bits, compare_layout, inputs

pytestmark = pytest.mark.gpu


def _wl():
    return W.WORKLOADS["tiny"].with_(hidden=512, fp8=True, tokens_per_rank=300, experts=16, topk=4)


def _params(wl, cap, **kw):
    return moe.params(wl.tokens, wl.ranks, wl.experts, wl.topk, wl.hidden, wl.alignment,
                      recv_capacity_rows=cap, **kw)


def _check_round_trip(wl, h, idx, w, x, recv, sc, y, out, cap):
    E, R, A = wl.experts, wl.ranks, wl.alignment
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A, cap=cap)
    compare_layout(h, lay, wl)
    st, r_codes, r_scales, _ = oracle.dispatch_fp8(lay, idx.numpy(), w.numpy(), bits(x), E, R, A, cap, True)
    assert st == oracle.OK
    st, ref = oracle.combine(idx.numpy(), lay.slot, bits(y), E, R)
    assert st == oracle.OK
    torch.cuda.synchronize()
    assert (recv.cpu().numpy() == r_codes).all()
    assert (sc.cpu().numpy().view(np.uint32) == r_scales.view(np.uint32)).all()
    assert (bits(out) == ref).all()
    assert moe.moe_handle_status(h) == moe.MOE_OK


@pytest.mark.parametrize("give_cap", [True, False])
def test_deferred_epilogue_issues_the_round_trip_before_the_host_wait(give_cap):
    wl = _wl()
    idx, w, x = inputs(wl, 0.1)
    rows_ref = oracle.layout(idx.numpy(), w.numpy(), wl.experts, wl.ranks, wl.alignment).rows_per_rank
    cap = int(rows_ref.max()) + 1
    h = moe.moe_layout(_params(wl, cap if give_cap else 0, do_cpu_sync=True, defer_epilogue=True),
                       idx.cuda(), w.cuda())
    assert h.host_rows_per_rank is None            # nothing on the host yet
    if not give_cap:                                # sizing the buffers needs the counts first
        cap = int(moe.moe_handle_wait(h).max())
    recv = torch.full((wl.ranks, cap, wl.hidden), 0xA5, dtype=torch.uint8, device="cuda")
    sc = torch.full((wl.ranks, cap, wl.hidden // 128), float("nan"), device="cuda")
    moe.moe_dispatch(h, x.cuda(), moe.MOE_DTYPE_FP8_E4M3, recv, sc, cap=cap)
    y = W.gen_y(wl, cap)
    out = torch.empty(wl.tokens, wl.hidden, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(h, y.cuda(), out, cap=cap)
    rows = moe.moe_handle_wait(h)                   # the deferred epilogue
    assert (rows == rows_ref).all()
    assert (moe.moe_handle_wait(h) == rows).all()   # kept on the handle
    assert (h.host_rows_per_rank == rows_ref).all()
    _check_round_trip(wl, h, idx, w, x, recv, sc, y, out, cap)
    moe.moe_handle_free(h)


@pytest.mark.parametrize("kind", ["capacity", "bad_expert"])
def test_deferred_epilogue_reports_device_conditions_at_the_wait(kind):
    wl = _wl()
    idx, w, _ = inputs(wl, 0.1)
    cap = 0
    if kind == "capacity":
        cap = int(oracle.layout(idx.numpy(), w.numpy(), wl.experts, wl.ranks, wl.alignment).rows_per_rank.max()) - 1
        expected = moe.MOE_ERR_CAPACITY
    else:
        idx[7, 1] = wl.experts
        expected = moe.MOE_ERR_BAD_EXPERT
    h = moe.moe_layout(_params(wl, cap, do_cpu_sync=True, defer_epilogue=True), idx.cuda(), w.cuda())
    for _ in range(2):                              # the result is kept
        with pytest.raises(moe.MoeError) as e:
            moe.moe_handle_wait(h)
        assert e.value.status == expected
    moe.moe_handle_free(h)


def test_wait_on_a_handle_without_host_counts():
    wl = _wl()
    idx, w, _ = inputs(wl)
    h = moe.moe_layout(_params(wl, 4096, do_cpu_sync=False), idx.cuda(), w.cuda())
    with pytest.raises(moe.MoeError) as e:
        moe.moe_handle_wait(h)
    assert e.value.status == moe.MOE_ERR_INVALID_ARG
    moe.moe_handle_free(h)
    h = moe.moe_layout(_params(wl, 0, do_cpu_sync=True), idx.cuda(), w.cuda())
    assert (moe.moe_handle_wait(h) == h.host_rows_per_rank).all()   # not deferred: already there
    moe.moe_handle_free(h)


def test_events_order_a_communication_stream_against_the_compute_stream():
    wl = _wl()
    idx, w, x = inputs(wl, 0.1)
    rows_ref = oracle.layout(idx.numpy(), w.numpy(), wl.experts, wl.ranks, wl.alignment).rows_per_rank
    cap = int(rows_ref.max())
    compute, comm = torch.cuda.Stream(), torch.cuda.Stream()
    x_host, y_host = x.pin_memory(), W.gen_y(wl, cap).pin_memory()
    idx_d, w_d = idx.cuda(), w.cuda()
    torch.cuda.synchronize()
    with torch.cuda.stream(compute):
        a = torch.randn(2048, 2048, device="cuda")
        for _ in range(8):                          # compute work the copy of x must wait for
            a = (a @ a) * 1e-3
        x_d = torch.empty_like(x, device="cuda")
        x_d.copy_(x_host, non_blocking=True)
    produced = moe.moe_event_record(compute)
    produced.wait(comm)                             # the communication stream starts after it
    h = moe.moe_layout(_params(wl, cap, do_cpu_sync=False), idx_d, w_d, stream=comm)
    recv = torch.full((wl.ranks, cap, wl.hidden), 0xA5, dtype=torch.uint8, device="cuda")
    sc = torch.full((wl.ranks, cap, wl.hidden // 128), float("nan"), device="cuda")
    torch.cuda.current_stream().synchronize()       # recv / sc filled before comm writes them
    moe.moe_dispatch(h, x_d, moe.MOE_DTYPE_FP8_E4M3, recv, sc, cap=cap, stream=comm)
    dispatched = moe.moe_event_record(comm)
    with torch.cuda.stream(compute):                # independent work (the shared expert's place)
        b = (a @ a) * 1e-3
        y_d = torch.empty(y_host.shape, dtype=y_host.dtype, device="cuda")
        y_d.copy_(y_host, non_blocking=True)
    dispatched.wait(compute)
    out = torch.empty(wl.tokens, wl.hidden, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(h, y_d, out, cap=cap, stream=compute)
    done = moe.moe_event_record(compute)
    assert done.query() in (True, False)
    done.synchronize()
    assert done.query()
    assert torch.isfinite(b).all()
    _check_round_trip(wl, h, idx, w, x, recv, sc, W.gen_y(wl, cap), out, cap)
    moe.moe_handle_free(h)
