"""Cached dispatch (one handle, several dispatches) and the backward of combine on the GPU, against
the oracle: grad_y bit-exact (it is one fp32 multiply and one bf16 rounding per element, or a
copy); grad_w within the error bound of its fp32 summation order against the binary64 value:
|d| <= (8 * ceil(H / 256) + 6) * 2^-24 * sum_h |g_h * y_h| (per-lane FMA chains of
8 * ceil(H / 256) terms, then a 5-level tree)."""
import math

import numpy as np
import pytest
import torch

import combine_moe_layout_07_b200 as moe
import oracle
import workloads as W
from gpu_helpers import bits, compare_layout, gpu_layout, inputs

pytestmark = pytest.mark.gpu


def _f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def _grad_w_bound(H, g_rows, y_rows):
    return (8 * math.ceil(H / 256) + 6) * 2.0 ** -24 * np.abs(g_rows * y_rows).sum(axis=-1) + 1e-30


@pytest.mark.parametrize("fp8", [True, False])
def test_cached_dispatch_reuses_one_handle(fp8):
    wl = W.WORKLOADS["tiny"].with_(hidden=512, fp8=fp8, tokens_per_rank=200, experts=16, topk=4)
    idx, w, x1 = inputs(wl, 0.1)
    x2 = W.gen_x(wl.with_(seed=5))
    E, R, A = wl.experts, wl.ranks, wl.alignment
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A)
    cap = int(lay.rows_per_rank.max())
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A, cap=cap)
    h = gpu_layout(wl, idx, w, cap=cap)
    compare_layout(h, lay, wl)
    for x in (x1, x2, x1):          # the same handle, three dispatches
        if fp8:
            recv = torch.full((R, cap, wl.hidden), 0xA5, dtype=torch.uint8, device="cuda")
            sc = torch.full((R, cap, wl.hidden // 128), float("nan"), device="cuda")
            moe.moe_dispatch(h, x.cuda(), moe.MOE_DTYPE_FP8_E4M3, recv, sc, cap=cap)
            st, rc, rs, _ = oracle.dispatch_fp8(lay, idx.numpy(), w.numpy(), bits(x), E, R, A, cap, True)
            torch.cuda.synchronize()
            assert (recv.cpu().numpy() == rc).all()
            assert (sc.cpu().numpy().view(np.uint32) == rs.view(np.uint32)).all()
        else:
            recv = torch.full((R, cap, wl.hidden), -23131, dtype=torch.int16, device="cuda").view(torch.bfloat16)
            moe.moe_dispatch(h, x.cuda(), moe.MOE_DTYPE_BF16, recv, cap=cap)
            st, rc, _ = oracle.dispatch_bf16(lay, idx.numpy(), w.numpy(), bits(x), E, R, A, cap, True)
            torch.cuda.synchronize()
            assert (bits(recv) == rc).all()
    assert moe.moe_handle_status(h) == moe.MOE_OK


@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("zero_padding", [True, False])
@pytest.mark.parametrize("hidden", [256, 7168])
def test_combine_backward_small(weighted, zero_padding, hidden):
    wl = W.WORKLOADS["tiny"].with_(hidden=hidden, tokens_per_rank=96, experts=16, topk=4)
    idx, w, _ = inputs(wl, 0.15)
    E, R, A = wl.experts, wl.ranks, wl.alignment
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A)
    cap = int(lay.rows_per_rank.max()) + 2
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A, cap=cap)
    y = W.gen_y(wl, cap)
    g = W.gen_bias(wl.with_(seed=9))       # grad_out
    h = gpu_layout(wl, idx, w, cap=cap)
    gy = torch.full((R, cap, hidden), -23131, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    gw = torch.full((wl.tokens, wl.topk), float("nan"), device="cuda")
    moe.moe_combine_backward(h, g.cuda(), gy, topk_weights=w.cuda() if weighted else None, y=y.cuda(),
                             grad_weights=gw, cap=cap, do_zero_padding=zero_padding)
    st, ref = oracle.combine_backward(lay, idx.numpy(), bits(g), E, R, A, cap, w=w.numpy() if weighted else None,
                                      zero_padding=zero_padding)
    torch.cuda.synchronize()
    assert st == oracle.OK
    assert (bits(gy) == ref).all()
    ref_w = oracle.grad_weights_f64(idx.numpy(), lay.slot, bits(g), bits(y), E, R)
    got_w = gw.cpu().numpy().astype(np.float64)
    e_loc = E // R
    for t in range(wl.tokens):
        for j in range(wl.topk):
            if idx[t, j] < 0:
                assert got_w[t, j] == 0.0
                continue
            yrow = _f32(bits(y)[idx[t, j] // e_loc, lay.slot[t, j]])
            tol = _grad_w_bound(hidden, _f32(bits(g)[t]), yrow)
            assert abs(got_w[t, j] - ref_w[t, j]) <= tol, (t, j)
    assert moe.moe_handle_status(h) == moe.MOE_OK


def test_combine_backward_full_size():
    """DeepSeek-V3 prefill, weighted: every element of grad_y (one logical rank at a time) bit-exact
    against the oracle's backward over the whole batch, and every grad_w within its bound."""
    wl = W.WORKLOADS["deepseek"]
    idx, w, _ = inputs(wl)
    E, R, A, k, H = wl.experts, wl.ranks, wl.alignment, wl.topk, wl.hidden
    idx_n, w_n = idx.numpy(), w.numpy()
    cap = int(oracle.layout(idx_n, w_n, E, R, A).rows_per_rank.max())
    lay = oracle.layout(idx_n, w_n, E, R, A, cap=cap)
    h = gpu_layout(wl, idx, w, cap=0)
    compare_layout(h, lay, wl)
    y = W.gen_y_device(wl, cap)
    g = W.gen_bias(wl)
    gy = torch.full((R, cap, H), -23131, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    gw = torch.full((wl.tokens, k), float("nan"), device="cuda")
    moe.moe_combine_backward(h, g.cuda(), gy, topk_weights=w.cuda(), y=y, grad_weights=gw, cap=cap)
    gb = bits(g)
    st, ref = oracle.combine_backward(lay, idx_n, gb, E, R, A, cap, w=w_n, zero_padding=True)
    assert st == oracle.OK
    torch.cuda.synchronize()
    assert moe.moe_handle_status(h) == moe.MOE_OK
    for r in range(R):
        bad = bits(gy[r]) != ref[r]
        assert not bad.any(), f"rank {r}: {bad.sum()} elements differ, first at (row, col) {np.argwhere(bad)[0]}"
    del gy, ref
    yb = bits(y)
    del y
    ref_w = oracle.grad_weights_f64(idx_n, lay.slot, gb, yb, E, R)
    got_w = gw.cpu().numpy().astype(np.float64)
    e_loc = wl.experts_per_rank
    gf = bf16_f32(gb)
    for t0 in range(0, wl.tokens, 1024):           # the bound needs sum |g * y| of every pair
        t1 = min(wl.tokens, t0 + 1024)
        rows = yb[idx_n[t0:t1] // e_loc, lay.slot[t0:t1]]            # [n, k, H]
        # a bf16 x bf16 product is exact in binary32; the sum is taken in binary64
        mag = np.abs(gf[t0:t1, None, :] * bf16_f32(rows)).sum(axis=-1, dtype=np.float64)
        tol = (8 * math.ceil(H / 256) + 6) * 2.0 ** -24 * mag + 1e-30
        bad = np.abs(got_w[t0:t1] - ref_w[t0:t1]) > tol
        assert not bad.any(), f"grad_w outside the bound at {np.argwhere(bad)[0] + [t0, 0]}"
