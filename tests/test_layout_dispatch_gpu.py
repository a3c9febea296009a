"""moe_layout_dispatch (layout and expanded dispatch in one call, without host sync) against the
oracle, every byte: the handle's layout, every row of the receive buffers (routed, padding and
untouched rows), FP8 scales and receive weights, then a combine through the returned handle.
Batches of at most 8 tokens per SM run as one cooperative kernel (one launch, counted by the
library); larger ones run the layout's launches and then the dispatch kernel."""
import numpy as np
import pytest
import torch

import combine_moe_layout_07_b200 as moe
import oracle
import workloads as W
from gpu_helpers import assert_bf16_close, bits, compare_layout, inputs

pytestmark = pytest.mark.gpu

FILL8, FILL16 = 0xA5, 0xA5A5


def _placed(t: torch.Tensor, offset_elems: int) -> torch.Tensor:
    """A copy of t on the GPU starting offset_elems elements into a fresh allocation (an int64
    table 8 but not 16 bytes aligned, fp32 scales 4 but not 16 bytes aligned, ...)."""
    flat = torch.empty(t.numel() + offset_elems, dtype=t.dtype, device="cuda")
    v = flat[offset_elems:].view(t.shape)
    v.copy_(t.cuda() if not t.is_cuda else t)
    return v


def _round_trip(wl, mask=0.0, zero_padding=True, num_sms=0, cap=None, want_w=True, launches=None, bias=False,
                idx_offset=0, scales_offset=0):
    idx, w, x = inputs(wl, mask)
    E, R, A, H = wl.experts, wl.ranks, wl.alignment, wl.hidden
    idx_n, w_n = idx.numpy(), w.numpy()
    lay = oracle.layout(idx_n, w_n, E, R, A)
    assert lay.status == oracle.OK
    cap = int(lay.rows_per_rank.max()) + 3 if cap is None else cap
    lay = oracle.layout(idx_n, w_n, E, R, A, cap=cap)
    p = moe.params(wl.tokens, R, E, wl.topk, H, A, recv_capacity_rows=cap, num_sms=num_sms, do_cpu_sync=False)
    rw = torch.full((R, cap), float("nan"), device="cuda") if want_w else None
    if wl.fp8:
        recv = torch.full((R, cap, H), FILL8, dtype=torch.uint8, device="cuda")
        scales = _placed(torch.full((R, cap, H // 128), float("nan")), scales_offset)
    else:
        recv = torch.full((R, cap, H), FILL16 - 65536, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        scales = None
    n0 = moe.moe_kernel_launch_count()
    h = moe.moe_layout_dispatch(p, _placed(idx, idx_offset), w.cuda(), x.cuda(),
                                moe.MOE_DTYPE_FP8_E4M3 if wl.fp8 else moe.MOE_DTYPE_BF16, recv, scales, rw,
                                do_zero_padding=zero_padding)
    if launches is not None:
        assert moe.moe_kernel_launch_count() - n0 == launches
    torch.cuda.synchronize()
    assert moe.moe_handle_status(h) == moe.MOE_OK
    compare_layout(h, lay, wl)
    if wl.fp8:
        st, rc, rs, rww = oracle.dispatch_fp8(lay, idx_n, w_n, bits(x), E, R, A, cap, zero_padding, fill=FILL8,
                                              want_w=want_w)
        assert st == oracle.OK
        for r in range(R):
            bad = recv[r].cpu().numpy() != rc[r]
            assert not bad.any(), f"rank {r}: {bad.sum()} code bytes differ, first at {np.argwhere(bad)[0]}"
        assert (scales.cpu().numpy().view(np.uint32) == rs.view(np.uint32)).all()
    else:
        st, rc, rww = oracle.dispatch_bf16(lay, idx_n, w_n, bits(x), E, R, A, cap, zero_padding, fill=FILL16,
                                           want_w=want_w)
        assert st == oracle.OK
        assert (bits(recv) == rc).all()
    if want_w:
        assert (rw.cpu().numpy().view(np.uint32) == rww.view(np.uint32)).all()
    # the returned handle serves the combine like one from moe_layout
    y = W.gen_y(wl, cap)
    b = W.gen_bias(wl) if bias else None
    out = torch.empty(wl.tokens, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(h, y.cuda(), out, bias=None if b is None else b.cuda())
    st, ref = oracle.combine(idx_n, lay.slot, bits(y), E, R, bias_bits=None if b is None else bits(b))
    got = bits(out)
    assert_bf16_close(got, ref)
    assert (got == ref).all()
    assert moe.moe_handle_status(h) == moe.MOE_OK
    moe.moe_handle_free(h)


def test_decode_workload_one_launch():
    """The decode workload (1024 tokens, top-8 of 256, FP8, receive capacity for 256 tokens per
    rank): one cooperative launch, every byte."""
    wl = W.WORKLOADS["decode"]
    p = moe.params(wl.tokens, wl.ranks, wl.experts, wl.topk, wl.hidden, wl.alignment, recv_capacity_rows=1,
                   do_cpu_sync=False)
    cap = moe.moe_recv_capacity_hint(p, wl.max_tokens_per_rank)
    _round_trip(wl, zero_padding=False, cap=cap, launches=1, bias=True)


@pytest.mark.parametrize("zero_padding", [True, False])
def test_decode_shape_with_padding_and_masking(zero_padding):
    wl = W.WORKLOADS["decode"].with_(tokens_per_rank=100)
    _round_trip(wl, mask=0.1, zero_padding=zero_padding, launches=1)


@pytest.mark.parametrize("kw", [
    dict(),                                                       # tiny: 64 tokens, fewer than the CTAs
    dict(hidden=512, fp8=True, tokens_per_rank=300, experts=16, topk=4),    # 600 tokens
    dict(hidden=136, tokens_per_rank=37, ranks=4, experts=16, topk=3),     # ragged rows, odd T
    dict(hidden=7168, fp8=True, tokens_per_rank=1, ranks=1, experts=4, topk=1),   # one token
    dict(hidden=256, tokens_per_rank=64, ranks=8, experts=2048, topk=8, alignment=1),   # E = 2048
    dict(hidden=1024, fp8=True, tokens_per_rank=16, ranks=4, experts=64, topk=32),      # k = 32
    dict(hidden=384, fp8=True, tokens_per_rank=50, ranks=2, experts=8, topk=3),         # 3 scales a row
    dict(hidden=256, fp8=True, tokens_per_rank=2, ranks=128, experts=256, topk=4),      # R > 64
])
@pytest.mark.parametrize("zero_padding", [True, False])
def test_small_batches_one_launch(kw, zero_padding):
    wl = W.WORKLOADS["tiny"].with_(**kw)
    _round_trip(wl, mask=0.1, zero_padding=zero_padding, launches=1)


@pytest.mark.parametrize("kw", [
    dict(hidden=512, fp8=True, tokens_per_rank=150, experts=32, topk=8),             # 16-byte id pairs
    dict(hidden=384, fp8=True, tokens_per_rank=25, ranks=1, experts=12, topk=3),     # T * k = 75: one id left
])
@pytest.mark.parametrize("idx_offset,scales_offset", [(1, 0), (0, 1), (1, 1)])
def test_unaligned_routing_table_and_scales(kw, idx_offset, scales_offset):
    """A routing table 8 but not 16 bytes aligned takes the batch-wide count one id at a time; FP8
    scales not 16 bytes aligned are written 4 bytes at a time by the storer.  Same bytes."""
    wl = W.WORKLOADS["tiny"].with_(**kw)
    _round_trip(wl, mask=0.1, zero_padding=True, launches=1, idx_offset=idx_offset, scales_offset=scales_offset)


def _random_case(seed: int):
    rng = np.random.default_rng(3000 + seed)
    R = int(rng.choice([1, 2, 4, 8, 16]))
    E = R * int(rng.integers(1, 33))
    k = int(rng.integers(1, min(E, 12) + 1))
    fp8 = bool(rng.integers(0, 2))
    H = 128 * int(rng.integers(1, 9)) if fp8 else 8 * int(rng.integers(1, 129))
    tpr = int(rng.integers(1, 1100 // R + 1))
    kw = dict(tokens_per_rank=tpr, ranks=R, experts=E, topk=k, hidden=H, fp8=fp8,
              alignment=int(rng.choice([1, 4, 16, 128])), seed=seed)
    opts = dict(mask=float(rng.choice([0.0, 0.05, 0.3])), zero_padding=bool(rng.integers(0, 2)),
                want_w=bool(rng.integers(0, 2)), idx_offset=int(rng.integers(0, 2)),
                scales_offset=int(rng.integers(0, 2)) if fp8 else 0)
    return kw, opts


@pytest.mark.parametrize("seed", range(16))
def test_random_shapes_one_launch(seed):
    """Seeded random shapes of at most 8 tokens per SM (one launch), every byte against the oracle."""
    kw, opts = _random_case(seed)
    wl = W.WORKLOADS["tiny"].with_(**kw)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    _round_trip(wl, launches=1 if wl.tokens <= 8 * sms else 2, **opts)


def test_sm_cap():
    """num_sms = 24: 192 tokens are 8 per CTA (one launch); 200 tokens are more (two kernels)."""
    wl = W.WORKLOADS["tiny"].with_(hidden=512, fp8=True, tokens_per_rank=96, experts=16, topk=4)
    _round_trip(wl, num_sms=24, launches=1)
    wl = wl.with_(tokens_per_rank=100)
    _round_trip(wl, num_sms=24, launches=2)


def test_large_batches_take_the_separate_kernels():
    """16 tokens per SM: the layout's launches, then the dispatch kernel; the same bytes."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    wl = W.WORKLOADS["decode"].with_(tokens_per_rank=2 * sms)
    _round_trip(wl, zero_padding=True, launches=2)


def test_bad_expert_and_capacity_are_reported_by_the_status():
    wl = W.WORKLOADS["tiny"].with_(hidden=256, fp8=True, tokens_per_rank=100, experts=16, topk=4)
    idx, w, x = inputs(wl)
    E, R, H = wl.experts, wl.ranks, wl.hidden
    bad = idx.clone()
    bad[5, 1] = E + 3
    cap = 512
    p = moe.params(wl.tokens, R, E, wl.topk, H, wl.alignment, recv_capacity_rows=cap, do_cpu_sync=False)
    recv = torch.zeros(R, cap, H, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(R, cap, H // 128, device="cuda")
    h = moe.moe_layout_dispatch(p, bad.cuda(), w.cuda(), x.cuda(), moe.MOE_DTYPE_FP8_E4M3, recv, sc)
    assert moe.moe_handle_status(h) == moe.MOE_ERR_BAD_EXPERT
    moe.moe_handle_free(h)
    # too small a capacity: flagged, and nothing lands past the receive buffers
    cap, guard = 40, 1 << 14
    p = moe.params(wl.tokens, R, E, wl.topk, H, wl.alignment, recv_capacity_rows=cap, do_cpu_sync=False)
    flat = torch.full((R * cap * H + guard,), FILL8, dtype=torch.uint8, device="cuda")
    sflat = torch.full((R * cap * (H // 128) + guard,), -3.0, device="cuda")
    wflat = torch.full((R * cap + guard,), -3.0, device="cuda")
    h = moe.moe_layout_dispatch(p, idx.cuda(), w.cuda(), x.cuda(), moe.MOE_DTYPE_FP8_E4M3,
                                flat[:-guard].view(R, cap, H), sflat[:-guard].view(R, cap, H // 128),
                                wflat[:-guard].view(R, cap))
    assert moe.moe_handle_status(h) == moe.MOE_ERR_CAPACITY
    assert (flat[-guard:] == FILL8).all() and (sflat[-guard:] == -3.0).all() and (wflat[-guard:] == -3.0).all()
    moe.moe_handle_free(h)


def test_decode_step_in_a_cuda_graph():
    """moe_layout_dispatch + combine + free captured once, replayed with new routing and inputs
    copied into the captured buffers: every byte against the oracle after each replay."""
    wl = W.WORKLOADS["decode"].with_(tokens_per_rank=64)
    E, R, A, H, k, T = wl.experts, wl.ranks, wl.alignment, wl.hidden, wl.topk, wl.tokens
    p = moe.params(T, R, E, k, H, A, recv_capacity_rows=1, do_cpu_sync=False)
    cap = moe.moe_recv_capacity_hint(p, 128)
    p = moe.params(T, R, E, k, H, A, recv_capacity_rows=cap, do_cpu_sync=False)
    idx_d = torch.zeros(T, k, dtype=torch.int64, device="cuda")
    w_d = torch.zeros(T, k, device="cuda")
    x_d = torch.zeros(T, H, dtype=torch.bfloat16, device="cuda")
    y_d = torch.zeros(R, cap, H, dtype=torch.bfloat16, device="cuda")
    recv = torch.zeros(R, cap, H, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(R, cap, H // 128, device="cuda")
    out = torch.zeros(T, H, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.Stream()

    def step():
        h = moe.moe_layout_dispatch(p, idx_d, w_d, x_d, moe.MOE_DTYPE_FP8_E4M3, recv, sc, None,
                                    do_zero_padding=False, stream=stream)
        moe.moe_combine(h, y_d, out, stream=stream)
        moe.moe_handle_free(h)

    with torch.cuda.stream(stream):
        step()  # warm-up outside the capture (first-use set-up of the library)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    for seed in (3, 4):
        swl = wl.with_(seed=seed)
        idx, w = W.gen_routing(swl)
        x, y = W.gen_x(swl), W.gen_y(swl, cap)
        idx_d.copy_(idx)
        w_d.copy_(w)
        x_d.copy_(x)
        y_d.copy_(y)
        recv.fill_(FILL8)
        g.replay()
        torch.cuda.synchronize()
        lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A, cap=cap)
        st, rc, rs, _ = oracle.dispatch_fp8(lay, idx.numpy(), w.numpy(), bits(x), E, R, A, cap, False, fill=FILL8,
                                            want_w=False)
        assert (recv.cpu().numpy() == rc).all()
        valid = lay.row_src >= 0                                  # scales of routed rows
        got_s = sc.cpu().numpy()
        assert (got_s[valid].view(np.uint32) == rs[valid].view(np.uint32)).all()
        st, ref = oracle.combine(idx.numpy(), lay.slot, bits(y), E, R)
        assert (bits(out) == ref).all()
    del g
