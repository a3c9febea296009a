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


def _round_trip(wl, mask=0.1, with_bias=True, via_moe_dispatch=False):
    idx, w, x = inputs(wl, mask)
    E, R = wl.experts, wl.ranks
    st, tr, rows = oracle.layout_by_rank(idx.numpy(), E, R)
    assert st == oracle.OK
    cap = int(rows.max()) + 2
    h = gpu_layout(wl, idx, w, cap=0, by_rank=True)
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


def test_by_rank_full_size_sampled():
    wl = W.WORKLOADS["deepseek"]
    idx, w, x = inputs(wl)
    E, R, k, H = wl.experts, wl.ranks, wl.topk, wl.hidden
    st, tr, rows = oracle.layout_by_rank(idx.numpy(), E, R)
    cap = int(rows.max())
    h = gpu_layout(wl, idx, w, cap=0, by_rank=True)
    torch.cuda.synchronize()
    assert (h.token_rows().cpu().numpy() == tr).all()
    recv = torch.full((R, cap, H), 0xA5, dtype=torch.uint8, device="cuda")
    sc = torch.full((R, cap, H // 128), float("nan"), device="cuda")
    ti = torch.full((R, cap, k), -7, dtype=torch.int32, device="cuda")
    moe.moe_dispatch_by_rank(h, x.cuda(), moe.MOE_DTYPE_FP8_E4M3, recv, sc, topk_idx=idx.cuda(), recv_topk_idx=ti,
                             cap=cap)
    torch.cuda.synchronize()
    rng = np.random.default_rng(6)
    ts = np.unique(rng.integers(0, wl.tokens, 48))
    xb = bits(x)
    e_loc = wl.experts_per_rank
    for t in ts:
        blocks = [oracle.quantize_block(xb[t, b:b + 128]) for b in range(0, H, 128)]
        codes = np.concatenate([c for c, _ in blocks])
        scal = np.array([s for _, s in blocks], np.float32)
        for r in range(R):
            if tr[t, r] < 0:
                continue
            assert (recv[r, tr[t, r]].cpu().numpy() == codes).all()
            assert (sc[r, tr[t, r]].cpu().numpy().view(np.uint32) == scal.view(np.uint32)).all()
            got = ti[r, tr[t, r]].cpu().numpy()
            exp = [int(e) - r * e_loc if e >= 0 and e // e_loc == r else -1 for e in idx[t].tolist()]
            assert got.tolist() == exp
    assert moe.moe_handle_status(h) == moe.MOE_OK
