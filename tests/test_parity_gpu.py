"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs.

Bit-exact for counts, psum, rows, membership, slots, row maps, dispatched BF16 rows, FP8 codes
and scales, receive weights; combine within one bf16 ulp (|d| <= 2^-7 |ref| + 1e-6), expected
bit-exact given the fixed accumulation order.  Small cases compare every byte of every buffer
(including rows the method must leave untouched); so do the full-size workloads, against the
oracle run over the whole batch.
"""
import numpy as np
import pytest
import torch

import combine_moe_layout_07_b200 as moe
import oracle
import workloads as W
from gpu_helpers import assert_bf16_close, bits, compare_layout, gpu_layout, inputs

pytestmark = pytest.mark.gpu

FILL16 = 0xA5A5
FILL8 = 0xA5


def _full_bf16(shape, pattern=FILL16):
    return torch.full(shape, pattern - 65536 if pattern >= 32768 else pattern, dtype=torch.int16,
                      device="cuda").view(torch.bfloat16)


def _roundtrip_small(wl, idx, w, x, cap_extra=3, zero_padding=True, weighted=False, with_bias=False,
                     num_sms=0, cpu_sync=True):
    """Full-buffer comparison of layout, dispatch (BF16 or FP8) and combine."""
    E, R, A = wl.experts, wl.ranks, wl.alignment
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A)
    assert lay.status == oracle.OK
    cap = int(lay.rows_per_rank.max()) + cap_extra
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A, cap=cap)
    h = gpu_layout(wl, idx, w, cap=cap, cpu_sync=cpu_sync, num_sms=num_sms)
    compare_layout(h, lay, wl)
    xd = x.cuda()
    rw = torch.full((R, cap), float("nan"), device="cuda")
    if wl.fp8:
        recv = torch.full((R, cap, wl.hidden), FILL8, dtype=torch.uint8, device="cuda")
        scales = torch.full((R, cap, wl.hidden // 128), float("nan"), device="cuda")
        moe.moe_dispatch(h, xd, moe.MOE_DTYPE_FP8_E4M3, recv, scales, rw, cap=cap,
                         do_zero_padding=zero_padding, num_sms=num_sms)
        st, rc, rs, rww = oracle.dispatch_fp8(lay, idx.numpy(), w.numpy(), bits(x), E, R, A, cap, zero_padding,
                                              fill=FILL8)
        torch.cuda.synchronize()
        assert st == oracle.OK
        assert (recv.cpu().numpy() == rc).all()
        assert (scales.cpu().numpy().view(np.uint32) == rs.view(np.uint32)).all()
    else:
        recv = _full_bf16((R, cap, wl.hidden))
        moe.moe_dispatch(h, xd, moe.MOE_DTYPE_BF16, recv, None, rw, cap=cap, do_zero_padding=zero_padding,
                         num_sms=num_sms)
        st, rc, rww = oracle.dispatch_bf16(lay, idx.numpy(), w.numpy(), bits(x), E, R, A, cap, zero_padding,
                                           fill=FILL16)
        torch.cuda.synchronize()
        assert st == oracle.OK
        assert (bits(recv) == rc).all()
    assert (rw.cpu().numpy().view(np.uint32) == rww.view(np.uint32)).all()
    assert moe.moe_handle_status(h) == moe.MOE_OK

    y = W.gen_y(wl, cap)
    bias = W.gen_bias(wl) if with_bias else None
    out = torch.empty(wl.tokens, wl.hidden, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(h, y.cuda(), out, topk_weights=w.cuda() if weighted else None,
                    bias=None if bias is None else bias.cuda(), num_sms=num_sms)
    st, ref = oracle.combine(idx.numpy(), lay.slot, bits(y), E, R, w=w.numpy() if weighted else None,
                             bias_bits=None if bias is None else bits(bias))
    got = bits(out)
    assert_bf16_close(got, ref)
    assert (got == ref).all(), f"{(got != ref).sum()} elements differ in the last bit"
    assert moe.moe_handle_status(h) == moe.MOE_OK
    moe.moe_handle_free(h)
    return lay


# ----------------------------------------------------------------------------- small, every byte

@pytest.mark.parametrize("zero_padding", [True, False])
@pytest.mark.parametrize("mask", [0.0, 0.25])
@pytest.mark.parametrize("weighted,with_bias", [(False, False), (True, False), (True, True), (False, True)])
def test_tiny_bf16_roundtrip(zero_padding, mask, weighted, with_bias):
    wl = W.WORKLOADS["tiny"]
    idx, w, x = inputs(wl, mask)
    _roundtrip_small(wl, idx, w, x, zero_padding=zero_padding, weighted=weighted, with_bias=with_bias)


@pytest.mark.parametrize("hidden", [128, 640, 1024, 2048, 7168])
@pytest.mark.parametrize("zero_padding", [True, False])
def test_small_fp8_roundtrip(hidden, zero_padding):
    wl = W.WORKLOADS["tiny"].with_(hidden=hidden, fp8=True, tokens_per_rank=300, experts=16, topk=4)
    idx, w, x = inputs(wl, 0.1)
    _roundtrip_small(wl, idx, w, x, zero_padding=zero_padding, weighted=True, with_bias=True)


@pytest.mark.parametrize("kw", [
    dict(alignment=1),                                   # plain inclusive scan
    dict(alignment=7, experts=12, ranks=3, topk=3),      # odd alignment, 3 ranks
    dict(tokens_per_rank=513, ranks=2),                  # ragged chunk tail (1026 tokens)
    dict(tokens_per_rank=1, ranks=1, experts=4, topk=1), # one token
    dict(topk=1, experts=2, ranks=2),
    dict(topk=32, experts=64, ranks=4, tokens_per_rank=40),   # widest top-k
    dict(experts=1, ranks=1, topk=1),                    # one expert
    dict(experts=16, ranks=16, topk=3),                  # one expert per rank
    dict(hidden=8),                                      # one 16-byte vector per row
    dict(hidden=136),                                    # ragged vector tail in the warp loop
    dict(experts=512, ranks=8, topk=8, tokens_per_rank=700, alignment=128),
    dict(hidden=7168, tokens_per_rank=300, experts=32, ranks=4, topk=8),   # several column chunks
    dict(tokens_per_rank=1024, ranks=1, experts=8, topk=8),   # 8192 pairs, 32 chunks (fused layout)
    dict(tokens_per_rank=1025, ranks=1, experts=8, topk=8),   # a one-token last chunk
    dict(experts=128, ranks=128, topk=4, tokens_per_rank=2),  # more than 64 ranks (membership)
    dict(experts=128, ranks=128, topk=4, tokens_per_rank=70), # ... 8960 tokens: 70 chunks of 128 (fused)
    dict(hidden=4104, tokens_per_rank=200, experts=16, ranks=2, topk=3),   # ragged last chunk
])
def test_shapes_and_edges(kw):
    wl = W.WORKLOADS["tiny"].with_(**kw)
    idx, w, x = inputs(wl, 0.1)
    _roundtrip_small(wl, idx, w, x, weighted=True, with_bias=True)


@pytest.mark.parametrize("extra", [0, 1])
def test_fused_and_three_kernel_layouts_at_the_boundary(extra):
    """The handle's layout runs as one cooperative kernel while some chunk of 32..256 tokens gives
    at most one chunk per SM, else as count -> scan -> assign: both sides of that boundary (256
    tokens per SM), every byte."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    wl = W.WORKLOADS["tiny"].with_(tokens_per_rank=128 * sms + extra, ranks=2, experts=16, topk=4, hidden=64)
    assert -(-wl.tokens // 256) == sms + extra
    idx, w, x = inputs(wl, 0.1)
    _roundtrip_small(wl, idx, w, x, weighted=True, with_bias=True)
    _roundtrip_small(wl, idx, w, x, cpu_sync=False)


def test_fused_layout_respects_the_sm_budget():
    """With num_sms = 24 a 32-chunk batch may not take the one-launch layout (it needs a CTA per
    chunk resident at once); the results are the same either way."""
    wl = W.WORKLOADS["tiny"].with_(tokens_per_rank=512, ranks=2, experts=16, topk=4, hidden=64)
    idx, w, x = inputs(wl, 0.1)
    _roundtrip_small(wl, idx, w, x, weighted=True, num_sms=24)
    _roundtrip_small(wl, idx, w, x, weighted=True, num_sms=32)


@pytest.mark.parametrize("num_sms,kw", [
    (24, dict(tokens_per_rank=512, ranks=16, experts=128, topk=8)),   # skewed shape: 24 chunks of 352 tokens
    (16, dict(tokens_per_rank=512, ranks=16, experts=128, topk=8)),   # 512-token chunks: 4096 pairs, the limit
    (16, dict(tokens_per_rank=512, ranks=16, experts=144, topk=9)),   # 4608 pairs per chunk: three kernels
    (3, dict(tokens_per_rank=300, ranks=3, experts=12, topk=3, alignment=5)),   # chunks of 320, 320, 260 tokens
    (16, dict(tokens_per_rank=576, ranks=8, experts=2048, topk=8, alignment=2)),  # E > 1024: 256 threads, 16 rounds
])
def test_wide_chunk_layout_under_an_sm_cap(num_sms, kw):
    """Under a num_sms cap the one-launch layout takes one chunk per SM of the budget, wider than
    256 tokens, while the chunk's pairs fit its warps' registers: 32 warps of 4 rounds of 32 pairs
    for E <= 1024, else 8 warps of 16 rounds; beyond that, the three kernels.  Each case with and
    without host sync, every byte."""
    wl = W.WORKLOADS["tiny"].with_(hidden=64, **kw)
    idx, w, x = inputs(wl, 0.05)
    _roundtrip_small(wl, idx, w, x, weighted=True, with_bias=True, num_sms=num_sms)
    _roundtrip_small(wl, idx, w, x, cpu_sync=False, num_sms=num_sms)


@pytest.mark.parametrize("kw", [
    dict(tokens_per_rank=64, ranks=8, experts=2048, topk=8, alignment=1, hidden=64),   # E at the fused limit
    dict(tokens_per_rank=64, ranks=8, experts=4096, topk=8, alignment=1, hidden=64),   # beyond it: three kernels
    dict(tokens_per_rank=256, ranks=8, experts=1024, topk=4, alignment=2, hidden=64),  # C * E = 65536: fused
    dict(tokens_per_rank=260, ranks=8, experts=1024, topk=4, alignment=2, hidden=64),  # C * E = 66560: three kernels
])
def test_fused_layout_expert_limits(kw):
    """The one-launch layout also stops at E = 2048 and at C * E = 65536 chunk counts (the last
    CTA sums C - 1 of each expert's); both sides of each limit, every byte."""
    wl = W.WORKLOADS["tiny"].with_(**kw)
    idx, w, x = inputs(wl, 0.1)
    _roundtrip_small(wl, idx, w, x, weighted=True)


def test_duplicate_experts_in_one_token():
    wl = W.WORKLOADS["tiny"].with_(topk=4)
    idx, w, x = inputs(wl)
    idx[:, 1] = idx[:, 0]            # every token sends two rows to the same expert
    idx[::3, 3] = idx[::3, 0]
    _roundtrip_small(wl, idx, w, x, weighted=True)


def test_all_masked_and_empty_rows():
    wl = W.WORKLOADS["tiny"]
    idx, w, x = inputs(wl)
    idx[5] = -1                       # a token routed nowhere: combine gives bias (or 0)
    idx[:, :][idx == 3] = -1          # expert 3 receives nothing
    _roundtrip_small(wl, idx, w, x, weighted=True, with_bias=True)


def test_no_host_sync_path():
    wl = W.WORKLOADS["tiny"].with_(fp8=True, hidden=512)
    idx, w, x = inputs(wl, 0.1)
    _roundtrip_small(wl, idx, w, x, cpu_sync=False)


@pytest.mark.parametrize("num_sms", [1, 3, 24])
def test_num_sms_cap_same_bytes(num_sms):
    wl = W.WORKLOADS["tiny"].with_(fp8=True, hidden=1024, tokens_per_rank=700)
    idx, w, x = inputs(wl)
    _roundtrip_small(wl, idx, w, x, num_sms=num_sms, weighted=True)


def test_zero_tokens():
    wl = W.WORKLOADS["tiny"].with_(tokens_per_rank=0)
    p = moe.params(0, wl.ranks, wl.experts, wl.topk, wl.hidden, wl.alignment, recv_capacity_rows=4)
    h = moe.moe_layout(p, torch.zeros(0, wl.topk, dtype=torch.int64, device="cuda"), None)
    assert (h.counts() == 0).all() and (h.rows_per_rank() == 0).all()
    recv = torch.zeros(wl.ranks, 4, wl.hidden, dtype=torch.bfloat16, device="cuda")
    moe.moe_dispatch(h, torch.zeros(0, wl.hidden, dtype=torch.bfloat16, device="cuda"), moe.MOE_DTYPE_BF16, recv)
    out = torch.zeros(0, wl.hidden, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(h, recv, out)
    assert moe.moe_handle_status(h) == moe.MOE_OK
    moe.moe_handle_free(h)


def test_row_capacity_from_counts():
    wl = W.WORKLOADS["tiny"]
    idx, w, x = inputs(wl)
    h = gpu_layout(wl, idx, w, cap=0, cpu_sync=True)
    lay = oracle.layout(idx.numpy(), w.numpy(), wl.experts, wl.ranks, wl.alignment)
    e_loc = wl.experts_per_rank          # without a capacity the row maps take the worst case
    assert h.row_capacity() == wl.tokens * min(wl.topk, e_loc) + e_loc * (wl.alignment - 1)
    assert h.row_capacity() >= int(lay.rows_per_rank.max())
    assert (h.host_rows_per_rank == lay.rows_per_rank).all()
    compare_layout(h, oracle.layout(idx.numpy(), w.numpy(), wl.experts, wl.ranks, wl.alignment,
                                    cap=h.row_capacity()), wl)


# ----------------------------------------------------------------------------- FP8 conversion sweep

def test_fp8_codes_over_all_bf16_values():
    """Every finite bf16 pattern, shuffled into 1x128 blocks (8 permutations, so each value meets
    many block maxima and hence many 448/amax factors), quantised by the dispatch kernel and by
    the oracle: codes and scales bit-exact."""
    pats = np.arange(65536, dtype=np.uint32)
    finite = pats[((pats >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    rng = np.random.default_rng(7)
    H = 1024
    rows = []
    for _ in range(8):
        perm = rng.permutation(finite)
        n = (perm.size // H) * H
        rows.append(perm[:n].reshape(-1, H))
    xb = np.concatenate(rows)
    # blocks that sit in every magnitude band: scale whole rows by powers of two
    T = xb.shape[0]
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16)
    idx = torch.zeros(T, 1, dtype=torch.int64)
    w = torch.ones(T, 1)
    wl = W.WORKLOADS["tiny"].with_(tokens_per_rank=T, ranks=1, experts=1, topk=1, alignment=1, hidden=H,
                                   fp8=True)
    _roundtrip_small(wl, idx, w, x, cap_extra=0)


# ----------------------------------------------------------------------------- errors

def test_bad_expert_detected():
    wl = W.WORKLOADS["tiny"]
    idx, w, x = inputs(wl)
    idx[7, 1] = wl.experts           # out of range
    with pytest.raises(moe.MoeError) as e:
        gpu_layout(wl, idx, w, cpu_sync=True)
    assert e.value.status == moe.MOE_ERR_BAD_EXPERT
    h = gpu_layout(wl, idx, w, cap=256, cpu_sync=False)
    assert moe.moe_handle_status(h) == moe.MOE_ERR_BAD_EXPERT
    idx[7, 1] = -5
    h = gpu_layout(wl, idx, w, cap=256, cpu_sync=False)
    assert moe.moe_handle_status(h) == moe.MOE_ERR_BAD_EXPERT


def test_capacity_overflow_detected_without_out_of_range_writes():
    wl = W.WORKLOADS["tiny"]
    idx, w, x = inputs(wl)
    lay = oracle.layout(idx.numpy(), w.numpy(), wl.experts, wl.ranks, wl.alignment)
    need = int(lay.rows_per_rank.max())
    with pytest.raises(moe.MoeError) as e:
        gpu_layout(wl, idx, w, cap=need - 1, cpu_sync=True)
    assert e.value.status == moe.MOE_ERR_CAPACITY
    # host-synced handle, dispatch into a buffer that is too small: rejected before launch
    h = gpu_layout(wl, idx, w, cap=need, cpu_sync=True)
    small = torch.zeros(wl.ranks, need - 1, wl.hidden, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.moe_dispatch(h, x.cuda(), moe.MOE_DTYPE_BF16, small)
    assert e.value.status == moe.MOE_ERR_CAPACITY
    # device-side detection: the kernels skip rows >= cap and set the status word
    cap = need - 20
    h = gpu_layout(wl, idx, w, cap=cap, cpu_sync=False)
    assert moe.moe_handle_status(h) == moe.MOE_ERR_CAPACITY
    guard = 4096
    flat = _full_bf16((wl.ranks * cap * wl.hidden + guard,))
    recv = flat[:-guard].view(wl.ranks, cap, wl.hidden)
    rw_flat = torch.full((wl.ranks * cap + guard,), -3.0, device="cuda")
    moe.moe_dispatch(h, x.cuda(), moe.MOE_DTYPE_BF16, recv, None, rw_flat[:-guard].view(wl.ranks, cap), cap=cap)
    out_flat = _full_bf16((wl.tokens * wl.hidden + guard,))
    moe.moe_combine(h, recv, out_flat[:-guard].view(wl.tokens, wl.hidden), cap=cap)
    torch.cuda.synchronize()
    assert (bits(flat[-guard:]) == FILL16).all()
    assert (rw_flat[-guard:] == -3.0).all()
    assert (bits(out_flat[-guard:]) == FILL16).all()
    assert moe.moe_handle_status(h) == moe.MOE_ERR_CAPACITY


def test_bad_dispatch_arguments():
    wl = W.WORKLOADS["tiny"]
    idx, w, x = inputs(wl)
    h = gpu_layout(wl, idx, w, cap=256)
    recv = torch.zeros(wl.ranks, 256, wl.hidden, dtype=torch.bfloat16, device="cuda")
    rc = moe.lib().moe_dispatch(h.ptr, x.cuda().data_ptr(), 0, recv.data_ptr(), None, None, 256, 2, 1, 0, None)
    assert rc == moe.MOE_ERR_INVALID_ARG          # do_expand is 0 or 1
    with pytest.raises(moe.MoeError) as e:        # FP8 needs H % 128 == 0 and scales
        moe.moe_dispatch(h, x.cuda(), moe.MOE_DTYPE_FP8_E4M3, recv.view(torch.uint8), None)
    assert e.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError) as e:        # misaligned row pointer
        moe.lib()
        rc = moe.lib().moe_dispatch(h.ptr, x.cuda().data_ptr() + 2, 0, recv.data_ptr(), None, None, 256, 1, 1, 0,
                                    None)
        moe._check(rc, "moe_dispatch")
    assert e.value.status == moe.MOE_ERR_INVALID_ARG


def test_determinism_three_runs():
    wl = W.WORKLOADS["tiny"].with_(fp8=True, hidden=2048, tokens_per_rank=1000, experts=64, ranks=4, topk=6)
    idx, w, x = inputs(wl)
    outs = []
    cap = int(oracle.layout(idx.numpy(), w.numpy(), wl.experts, wl.ranks, wl.alignment).rows_per_rank.max())
    for _ in range(3):
        h = gpu_layout(wl, idx, w, cap=cap)
        recv = torch.zeros(wl.ranks, cap, wl.hidden, dtype=torch.uint8, device="cuda")
        sc = torch.zeros(wl.ranks, cap, wl.hidden // 128, device="cuda")
        moe.moe_dispatch(h, x.cuda(), moe.MOE_DTYPE_FP8_E4M3, recv, sc)
        outs.append((h.slots().cpu(), recv.cpu(), sc.cpu()))
    for o in outs[1:]:
        assert all(torch.equal(a, b) for a, b in zip(o, outs[0]))


# ----------------------------------------------------------------------------- full-size workloads

def _full_roundtrip(wl: W.Workload):
    """Every byte at full size, against the oracle run over the whole batch: the layout; every row
    of every receive buffer (routed rows, padding rows, and the rows past each rank's count, which
    must keep their fill); every FP8 scale; every combined token.  Buffers are compared one
    logical rank at a time so that the host holds one oracle buffer and one rank of the GPU's."""
    idx, w, x = inputs(wl)
    E, R, A, H = wl.experts, wl.ranks, wl.alignment, wl.hidden
    idx_n, w_n = idx.numpy(), w.numpy()
    lay0 = oracle.layout(idx_n, w_n, E, R, A)
    assert lay0.status == oracle.OK
    if wl.max_tokens_per_rank:
        p = moe.params(wl.tokens, R, E, wl.topk, H, A, recv_capacity_rows=1, do_cpu_sync=False)
        cap = moe.moe_recv_capacity_hint(p, wl.max_tokens_per_rank)
    else:
        cap = int(lay0.rows_per_rank.max())
    del lay0
    lay = oracle.layout(idx_n, w_n, E, R, A, cap=cap)
    h = gpu_layout(wl, idx, w, cap=0 if wl.cpu_sync else cap, num_sms=wl.num_sms)
    compare_layout(h, lay, wl)

    xd = x.cuda()
    if wl.fp8:
        recv = torch.full((R, cap, H), FILL8, dtype=torch.uint8, device="cuda")
        scales = torch.full((R, cap, H // 128), float("nan"), device="cuda")
        moe.moe_dispatch(h, xd, moe.MOE_DTYPE_FP8_E4M3, recv, scales, cap=cap, do_zero_padding=wl.zero_padding,
                         num_sms=wl.num_sms)
        st, rc, rs, _ = oracle.dispatch_fp8(lay, idx_n, w_n, bits(x), E, R, A, cap, wl.zero_padding, fill=FILL8,
                                            want_w=False)
        assert st == oracle.OK
        torch.cuda.synchronize()
        for r in range(R):
            bad = recv[r].cpu().numpy() != rc[r]
            assert not bad.any(), f"rank {r}: {bad.sum()} code bytes differ, first at (row, col) {np.argwhere(bad)[0]}"
        bad = scales.cpu().numpy().view(np.uint32) != rs.view(np.uint32)
        assert not bad.any(), f"{bad.sum()} scales differ, first at {np.argwhere(bad)[0]}"
        del recv, scales, rc, rs
    else:
        recv = _full_bf16((R, cap, H))
        moe.moe_dispatch(h, xd, moe.MOE_DTYPE_BF16, recv, cap=cap, do_zero_padding=wl.zero_padding,
                         num_sms=wl.num_sms)
        st, rc, _ = oracle.dispatch_bf16(lay, idx_n, w_n, bits(x), E, R, A, cap, wl.zero_padding, fill=FILL16,
                                         want_w=False)
        assert st == oracle.OK
        torch.cuda.synchronize()
        for r in range(R):
            bad = bits(recv[r]) != rc[r]
            assert not bad.any(), f"rank {r}: {bad.sum()} elements differ, first at (row, col) {np.argwhere(bad)[0]}"
        del recv, rc
    assert moe.moe_handle_status(h) == moe.MOE_OK

    # combine: y drawn on the GPU, brought to the host whole for the oracle
    y = W.gen_y_device(wl, cap)
    bias = W.gen_bias(wl) if wl.bias else None
    weighted = wl.weighted_combine
    out = torch.empty(wl.tokens, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(h, y, out, topk_weights=w.cuda() if weighted else None,
                    bias=None if bias is None else bias.cuda(), num_sms=wl.num_sms)
    yb = bits(y)
    del y
    st, ref = oracle.combine(idx_n, lay.slot, yb, E, R, w=w_n if weighted else None,
                             bias_bits=None if bias is None else bits(bias))
    assert st == oracle.OK
    got = bits(out)
    assert_bf16_close(got, ref)
    assert (got == ref).all(), f"{(got != ref).sum()} elements differ in the last bit"
    assert moe.moe_handle_status(h) == moe.MOE_OK
    moe.moe_handle_free(h)


@pytest.mark.parametrize("name", ["deepseek", "decode", "large", "skewed"])
def test_workload_full_size(name):
    _full_roundtrip(W.WORKLOADS[name])


def test_deepseek_weighted_with_bias():
    _full_roundtrip(W.WORKLOADS["deepseek"].with_(weighted_combine=True, bias=True))


@pytest.mark.parametrize("kw", [
    dict(hidden=7168, topk=8, experts=64, ranks=8, tokens_per_rank=64),    # DeepSeek row shape
    dict(hidden=7168, topk=8, experts=64, ranks=8, tokens_per_rank=64, fp8=True),
    dict(hidden=4096, topk=8, experts=128, ranks=16, tokens_per_rank=32),  # skewed row shape
])
def test_multi_chunk_rows_plain_combine(kw):
    """Row shapes whose combine stages hold several column chunks, unweighted and without bias
    (the stage-ring geometry of the full-size workloads)."""
    wl = W.WORKLOADS["tiny"].with_(**kw)
    idx, w, x = inputs(wl)
    _roundtrip_small(wl, idx, w, x)
