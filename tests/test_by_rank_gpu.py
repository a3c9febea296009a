"""The non-expanded (by-rank) round trip on the GPU against the oracle: token rows per rank,
dispatch (BF16 copies or FP8 codes + scales, per-row top-k ids and weights) and combine of
per-rank partial sums, all bit-exact; every byte of every buffer on small cases."""
import numpy as np
import pytest
import torch

import combine_moe_layout_07_b200 as moe
import oracle
import workloads as W
from gpu_helpers import bits, gpu_layout, inputs

pytestmark = pytest.mark.gpu


def _round_trip(wl, mask=0.1, with_bias=True, via_moe_dispatch=False, num_sms=0):
    idx, w, x = inputs(wl, mask)
    E, R = wl.experts, wl.ranks
    st, tr, rows = oracle.layout_by_rank(idx.numpy(), E, R)
    assert st == oracle.OK
    cap = int(rows.max()) + 2
    h = gpu_layout(wl, idx, w, cap=0, by_rank=True, num_sms=num_sms)
    torch.cuda.synchronize()
    assert (h.token_rows().cpu().numpy() == tr).all()
    assert (h.tokens_per_rank().cpu().numpy() == rows).all()
    k, H = wl.topk, wl.hidden
    if wl.fp8:
        recv = torch.full((R, cap, H), 0xA5, dtype=torch.uint8, device="cuda")
        sc = torch.full((R, cap, H // 128), float("nan"), device="cuda")
    else:
        recv = torch.full((R, cap, H), -23131, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        sc = None
    ti = torch.full((R, cap, k), -7, dtype=torch.int32, device="cuda")
    tw = torch.full((R, cap, k), float("nan"), device="cuda")
    dt = moe.MOE_DTYPE_FP8_E4M3 if wl.fp8 else moe.MOE_DTYPE_BF16
    if via_moe_dispatch:
        moe.moe_dispatch(h, x.cuda(), dt, recv, sc, tw, cap=cap, do_expand=False)
    else:
        moe.moe_dispatch_by_rank(h, x.cuda(), dt, recv, sc, topk_idx=idx.cuda(), recv_topk_idx=ti,
                                 recv_topk_weights=tw, cap=cap)
    st, r_recv, r_sc, r_ti, r_tw = oracle.dispatch_by_rank(idx.numpy(), w.numpy(), tr, bits(x), E, R, cap, wl.fp8)
    torch.cuda.synchronize()
    if wl.fp8:
        assert (recv.cpu().numpy() == r_recv).all()
        assert (sc.cpu().numpy().view(np.uint32) == r_sc.view(np.uint32)).all()
    else:
        assert (bits(recv) == r_recv).all()
    if not via_moe_dispatch:
        assert (ti.cpu().numpy() == r_ti).all()
    assert (tw.cpu().numpy().view(np.uint32) == r_tw.view(np.uint32)).all()
    # combine of per-rank partial sums
    y = W.gen_y(wl, cap)
    bias = W.gen_bias(wl) if with_bias else None
    out = torch.empty(wl.tokens, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine_by_rank(h, y.cuda(), out, bias=None if bias is None else bias.cuda(), cap=cap)
    st, ref = oracle.combine_by_rank(idx.numpy(), tr, bits(y), E, R, bias_bits=None if bias is None else bits(bias))
    torch.cuda.synchronize()
    assert (bits(out) == ref).all()
    assert moe.moe_handle_status(h) == moe.MOE_OK
    moe.moe_handle_free(h)


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("kw", [
    dict(tokens_per_rank=100, ranks=4, experts=16, topk=4),          # fused layout (13 chunks of 32)
    dict(tokens_per_rank=5000, ranks=8, experts=64, topk=4),         # three-kernel layout (157 chunks of 256)
    dict(tokens_per_rank=600, ranks=8, experts=64, topk=6),          # fused layout (75 chunks of 64)
    dict(tokens_per_rank=40, ranks=64, experts=128, topk=8),         # 64 ranks
    dict(tokens_per_rank=200, ranks=2, experts=8, topk=2, alignment=1),
])
def test_by_rank_round_trip(fp8, kw):
    wl = W.WORKLOADS["tiny"].with_(hidden=512, fp8=fp8, **kw)
    _round_trip(wl)


def test_by_rank_wide_chunks_under_an_sm_cap():
    """num_sms = 24 over 8192 tokens: the one-launch layout's chunks of 352 tokens hold several
    groups of token rows each."""
    wl = W.WORKLOADS["tiny"].with_(hidden=256, tokens_per_rank=512, ranks=16, experts=128, topk=8)
    _round_trip(wl, num_sms=24)


@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("kw", [
    dict(hidden=7168, fp8=True, tokens_per_rank=64, ranks=8, experts=64, topk=8),   # rows of 1..8 ranks
    dict(hidden=1000, tokens_per_rank=50, ranks=4, experts=16, topk=2),              # H not a chunk multiple
])
def test_by_rank_combine_items_sized_by_rows(kw, with_bias):
    """The by-rank combine takes as many column chunks per item as the token's rows leave room for
    (one rank: the whole row at once; no rows and no bias: nothing loaded).  90 % of the routing
    entries masked gives every row count from none to all ranks; every byte against the oracle."""
    wl = W.WORKLOADS["tiny"].with_(**kw)
    _round_trip(wl, mask=0.9, with_bias=with_bias)
    _round_trip(wl.with_(seed=5), mask=0.3, with_bias=with_bias)


def test_moe_dispatch_without_expansion():
    wl = W.WORKLOADS["tiny"].with_(hidden=256, tokens_per_rank=64, ranks=4, experts=16, topk=4)
    _round_trip(wl, via_moe_dispatch=True, with_bias=False)


def test_by_rank_needs_the_layout_flag():
    wl = W.WORKLOADS["tiny"]
    idx, w, x = inputs(wl)
    h = gpu_layout(wl, idx, w, cap=0)
    assert h.token_rows().abs().sum() == 0          # not built (the accessor returns NULL)
    recv = torch.zeros(wl.ranks, 64, wl.hidden, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.moe_dispatch_by_rank(h, x.cuda(), moe.MOE_DTYPE_BF16, recv)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED


def test_by_rank_needs_at_most_64_ranks():
    wl = W.WORKLOADS["tiny"].with_(tokens_per_rank=2, ranks=128, experts=128, topk=4)
    idx, w, x = inputs(wl)
    h = gpu_layout(wl, idx, w, cap=0, by_rank=True)
    recv = torch.zeros(wl.ranks, 8, wl.hidden, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.moe_dispatch_by_rank(h, x.cuda(), moe.MOE_DTYPE_BF16, recv)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED


def test_by_rank_full_size():
    """DeepSeek-V3 prefill without expansion: token rows, every byte of the FP8 rows and scales, the
    per-row top-k ids and weights (one logical rank at a time), and every combined token, against
    the oracle over the whole batch."""
    wl = W.WORKLOADS["deepseek"]
    idx, w, x = inputs(wl)
    E, R, k, H = wl.experts, wl.ranks, wl.topk, wl.hidden
    idx_n, w_n = idx.numpy(), w.numpy()
    st, tr, rows = oracle.layout_by_rank(idx_n, E, R)
    assert st == oracle.OK
    cap = int(rows.max())
    h = gpu_layout(wl, idx, w, cap=0, by_rank=True)
    torch.cuda.synchronize()
    assert (h.token_rows().cpu().numpy() == tr).all()
    assert (h.tokens_per_rank().cpu().numpy() == rows).all()
    recv = torch.full((R, cap, H), 0xA5, dtype=torch.uint8, device="cuda")
    sc = torch.full((R, cap, H // 128), float("nan"), device="cuda")
    ti = torch.full((R, cap, k), -7, dtype=torch.int32, device="cuda")
    tw = torch.full((R, cap, k), float("nan"), device="cuda")
    moe.moe_dispatch_by_rank(h, x.cuda(), moe.MOE_DTYPE_FP8_E4M3, recv, sc, topk_idx=idx.cuda(), recv_topk_idx=ti,
                             recv_topk_weights=tw, cap=cap)
    st, r_recv, r_sc, r_ti, r_tw = oracle.dispatch_by_rank(idx_n, w_n, tr, bits(x), E, R, cap, True)
    assert st == oracle.OK
    torch.cuda.synchronize()
    for r in range(R):
        bad = recv[r].cpu().numpy() != r_recv[r]
        assert not bad.any(), f"rank {r}: {bad.sum()} code bytes differ, first at (row, col) {np.argwhere(bad)[0]}"
    assert (sc.cpu().numpy().view(np.uint32) == r_sc.view(np.uint32)).all()
    assert (ti.cpu().numpy() == r_ti).all()
    assert (tw.cpu().numpy().view(np.uint32) == r_tw.view(np.uint32)).all()
    del recv, sc, ti, tw, r_recv, r_sc, r_ti, r_tw
    # combine of per-rank partial sums, with the shared-expert bias
    y = W.gen_y_device(wl, cap)
    bias = W.gen_bias(wl)
    out = torch.empty(wl.tokens, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine_by_rank(h, y, out, bias=bias.cuda(), cap=cap)
    yb = bits(y)
    del y
    st, ref = oracle.combine_by_rank(idx_n, tr, yb, E, R, bias_bits=bits(bias))
    assert st == oracle.OK
    got = bits(out)
    assert (got == ref).all(), f"{(got != ref).sum()} elements differ"
    assert moe.moe_handle_status(h) == moe.MOE_OK
    moe.moe_handle_free(h)
