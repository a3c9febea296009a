"""The first expert GEMM (tcgen05, E4M3 x E4M3 per 128-wide K-block, fp32 promotion) on the FP8
dispatch layout, against the binary64 oracle.

Tolerance, from a stated model of the arithmetic.  With M = sum_b |sx * sw| * sum_h |qx * qw|
(the magnitude the sums run over) and KB = H / 128 K-blocks:
  * Products of two E4M3 values are exact.  Each MMA step (K = 32) adds its 32 products to the
    fp32 accumulator in a fixed-point window aligned to the largest magnitude among them and the
    accumulator: an addend loses only the bits more than 25 binary places below that exponent
    (an E4M3 product 2^26 times smaller than the largest one is dropped, 2^25 times smaller is
    kept exactly, measured on the B200 through this GEMM with crafted operands, the accumulator
    carried from an earlier step included).  Per step the error is below 33 addends x 2^-25 x
    the largest magnitude, plus 2^-23 for the fp32 result; over the 4 steps of a K-block below
    4 (33 + 4) 2^-25 = 148 * 2^-25 of sum_h |qx * qw|.
  * The promotion acc = fma(partial, fp32(sx * sw), acc) adds 2^-24 relative for the scale
    product and 2^-24 of the running sum per K-block: (KB + 1) * 2^-24 * M.
  * The final bf16 rounding (8 significant bits) is at most 2^-8 of the result.
So |got - ref| <= 2^-8 |ref| + (1 + 2^-8) (148 * 2^-25 + (KB + 1) * 2^-24) M.  A lost K-block or a
wrong scale gives errors near M / 50 and fails by far.  The identity case below has one nonzero
product per output, so no accumulation error at all: it must match bit for bit.  Rows outside
the expert ranges must keep their fill pattern.
"""
import numpy as np
import pytest
import torch

import combine_moe_layout_07_b200 as moe
import oracle
import workloads as W
from gpu_helpers import bits, gpu_layout, inputs

pytestmark = pytest.mark.gpu

FILL = -23131  # 0xA5A5 as int16


def _e4m3_table():
    return np.array([oracle.e4m3_to_double(c) for c in range(256)], np.float64)


def _weights(E, N, H, seed):
    """Synthetic E4M3 weights (no NaN codes) and 128 x 128 block scales."""
    g = torch.Generator().manual_seed(seed)
    qw = torch.randint(0, 256, (E, N, H), generator=g, dtype=torch.uint8)
    qw[(qw & 0x7F) == 0x7F] = 0x38
    sw = (torch.rand((E, N // 128, H // 128), generator=g) * 1.5 + 0.25) / 64
    return qw, sw


def _dispatch_fp8(wl, h, x, cap):
    recv = torch.zeros((wl.ranks, cap, wl.hidden), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((wl.ranks, cap, wl.hidden // 128), device="cuda")
    moe.moe_dispatch(h, x.cuda(), moe.MOE_DTYPE_FP8_E4M3, recv, sc, cap=cap, do_zero_padding=True)
    return recv, sc


def _magnitude(codes, scales, qw, sw, e_of_rows):
    """M = sum_b |sx * sw| * sum_h |qx * qw| for rows [n_rows, N] whose experts are e_of_rows."""
    t = _e4m3_table()
    ax = np.abs(t[codes]) * np.repeat(np.abs(scales.astype(np.float64)), 128, axis=-1)      # [rows, H]
    M = np.zeros((codes.shape[0], qw.shape[1]), np.float64)
    for e in np.unique(e_of_rows):
        sel = e_of_rows == e
        aw = np.abs(t[qw[e]]) * np.repeat(np.repeat(sw[e].astype(np.float64), 128, axis=0), 128, axis=1)
        M[sel] = ax[sel] @ aw.T
    return M


def m_factor(H):
    """The factor of M in the bound: (1 + 2^-8) (148 * 2^-25 + (KB + 1) * 2^-24), KB = H / 128."""
    return (1 + 2.0 ** -8) * (148 * 2.0 ** -25 + (H // 128 + 1) * 2.0 ** -24)


def _bound(ref, codes, scales, qw, sw, e_of_rows):
    """2^-8 |ref| + m_factor(H) M."""
    return 2.0 ** -8 * np.abs(ref) + m_factor(codes.shape[-1]) * _magnitude(codes, scales, qw, sw, e_of_rows)


def _rows_expert(lay, E, R, A):
    """Expert of every row of every rank's ranges ([R, cap], -1 outside), from cnt and psum."""
    e_loc = E // R
    out = np.full((R, lay.row_src.shape[1]), -1, np.int64)
    for e in range(E):
        end = int(lay.psum[e]); beg = end - -(-int(lay.cnt[e]) // A) * A
        out[e // e_loc, beg:end] = e
    return out


@pytest.mark.parametrize("kw,N", [
    (dict(hidden=256, tokens_per_rank=100, ranks=2, experts=8, topk=2), 128),
    (dict(hidden=512, tokens_per_rank=300, ranks=2, experts=8, topk=4), 256),
    (dict(hidden=384, tokens_per_rank=64, ranks=4, experts=16, topk=3), 384),
    (dict(hidden=1024, tokens_per_rank=700, ranks=1, experts=4, topk=2), 128),   # several row tiles per expert
])
def test_expert_gemm_small_every_row(kw, N):
    wl = W.WORKLOADS["tiny"].with_(fp8=True, alignment=128, **kw)
    idx, w, x = inputs(wl, 0.1)
    E, R, A, H = wl.experts, wl.ranks, wl.alignment, wl.hidden
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A)
    cap = int(lay.rows_per_rank.max()) + 3
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A, cap=cap)
    h = gpu_layout(wl, idx, w, cap=cap)
    recv, sc = _dispatch_fp8(wl, h, x, cap)
    qw, sw = _weights(E, N, H, seed=11)
    out = torch.full((R, cap, N), FILL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    moe.moe_expert_gemm_fp8(h, recv, sc, qw.cuda(), sw.cuda(), out, cap=cap)
    codes, scales = recv.cpu().numpy(), sc.cpu().numpy()
    st, ref = oracle.grouped_gemm_f64(lay, codes, scales, qw.numpy(), sw.numpy(), E, R, A)
    assert st == 0
    got = bits(out)
    gotf = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ex = _rows_expert(lay, E, R, A)
    worst = rel_m = 0.0
    for r in range(R):
        n = int(lay.rows_per_rank[r])
        M = _magnitude(codes[r, :n], scales[r, :n], qw.numpy(), sw.numpy(), ex[r, :n])
        tol = 2.0 ** -8 * np.abs(ref[r, :n]) + m_factor(H) * M
        err = np.abs(gotf[r, :n] - ref[r, :n])
        if (M > 0).any():
            rel_m = max(rel_m, float((err[M > 0] / M[M > 0]).max()))
        assert (err <= tol).all(), f"rank {r}: {(err > tol).sum()} outside the bound"
        pos = tol > 0
        if pos.any():
            worst = max(worst, float((err[pos] / tol[pos]).max()))
        assert (got[r, n:] == np.uint16(0xA5A5)).all()          # rows beyond the ranges untouched
    assert moe.moe_handle_status(h) == moe.MOE_OK
    print(f"largest error / bound = {worst:.3f}; largest error / M = 2^{np.log2(max(rel_m, 1e-300)):.2f}")


def test_expert_gemm_identity_weights_bit_exact():
    """W_e = I (E4M3 1.0 on the diagonal, scales 1): out[row, n] = bf16(fp32(sx[row, n/128] *
    deq(qx[row, n]))) exactly -- tiles, swizzle, expert selection and scales with nothing summed."""
    wl = W.WORKLOADS["tiny"].with_(fp8=True, alignment=128, hidden=512, tokens_per_rank=150, ranks=2, experts=8,
                                   topk=3)
    idx, w, x = inputs(wl, 0.1)
    E, R, A, H = wl.experts, wl.ranks, wl.alignment, wl.hidden
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A)
    cap = int(lay.rows_per_rank.max())
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A, cap=cap)
    h = gpu_layout(wl, idx, w, cap=cap)
    recv, sc = _dispatch_fp8(wl, h, x, cap)
    qw = torch.zeros((E, H, H), dtype=torch.uint8)
    qw[:, torch.arange(H), torch.arange(H)] = 0x38
    sw = torch.ones((E, H // 128, H // 128))
    out = torch.full((R, cap, H), FILL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    moe.moe_expert_gemm_fp8(h, recv, sc, qw.cuda(), sw.cuda(), out, cap=cap)
    st, ref = oracle.grouped_gemm_f64(lay, recv.cpu().numpy(), sc.cpu().numpy(), qw.numpy(), sw.numpy(), E, R, A)
    assert st == 0
    got = bits(out)
    for r in range(R):
        n = int(lay.rows_per_rank[r])
        f32 = ref[r, :n].astype(np.float32)                       # one rounding to fp32 (exact product)
        want = np.vectorize(oracle.float_to_bf16, otypes=[np.uint16])(f32)
        assert (got[r, :n] == want).all(), f"rank {r}: {(got[r, :n] != want).sum()} differ"


def test_expert_gemm_full_size_sampled():
    """DeepSeek-V3 prefill layout (32768 tokens, 256 experts, H = 7168) with N = 256: rows sampled
    on every rank, recomputed by the oracle per expert."""
    wl = W.WORKLOADS["deepseek"]
    idx, w, x = inputs(wl)
    E, R, A, H, N = wl.experts, wl.ranks, wl.alignment, wl.hidden, 256
    h = gpu_layout(wl, idx, w, cap=0)
    cap = int(h.host_rows_per_rank.max())
    recv, sc = _dispatch_fp8(wl, h, x, cap)
    qw, sw = _weights(E, N, H, seed=12)
    out = torch.full((R, cap, N), FILL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    moe.moe_expert_gemm_fp8(h, recv, sc, qw.cuda(), sw.cuda(), out, cap=cap)
    torch.cuda.synchronize()
    assert moe.moe_handle_status(h) == moe.MOE_OK
    cnt, psum = h.counts().cpu().numpy(), h.psum().cpu().numpy()
    e_loc = E // R
    rng = np.random.default_rng(8)
    for e in rng.choice(E, 12, replace=False):
        r = e // e_loc
        end = int(psum[e]); beg = end - -(-int(cnt[e]) // A) * A
        rows = np.unique(rng.integers(beg, end, 6))
        codes = recv[r, rows].cpu().numpy()[None]
        scales = sc[r, rows].cpu().numpy()[None]
        n = len(rows)
        sub = oracle.Layout(status=0, cnt=np.array([n], np.int32), psum=np.array([n], np.int32),
                            rows_per_rank=np.array([n], np.int32), tokens_per_rank=None, token_in_rank=None,
                            slot=None, row_src=np.zeros((1, n), np.int32), row_w=None, cap=n)
        st, ref = oracle.grouped_gemm_f64(sub, codes, scales, qw.numpy()[e:e + 1], sw.numpy()[e:e + 1], 1, 1, 1)
        assert st == 0
        got = bits(out[r, rows])
        gotf = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        tol = _bound(ref[0], codes[0], scales[0], qw.numpy()[e:e + 1], sw.numpy()[e:e + 1], np.zeros(n, np.int64))
        assert (np.abs(gotf - ref[0]) <= tol).all(), e


def test_expert_gemm_rejects_unsupported_shapes():
    wl = W.WORKLOADS["tiny"].with_(fp8=True, hidden=256, alignment=16)
    idx, w, _ = inputs(wl)
    h = gpu_layout(wl, idx, w, cap=0)
    cap = int(h.host_rows_per_rank.max())
    recv = torch.zeros((wl.ranks, cap, wl.hidden), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((wl.ranks, cap, 2), device="cuda")
    qw, sw = _weights(wl.experts, 128, wl.hidden, 1)
    out = torch.zeros((wl.ranks, cap, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as e:     # expert_alignment 16: tiles would straddle experts
        moe.moe_expert_gemm_fp8(h, recv, sc, qw.cuda(), sw.cuda(), out, cap=cap)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED
    wl = wl.with_(alignment=128)
    h = gpu_layout(wl, idx, w, cap=0)
    cap = int(h.host_rows_per_rank.max())
    recv = torch.zeros((wl.ranks, cap, wl.hidden), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((wl.ranks, cap, 2), device="cuda")
    out = torch.zeros((wl.ranks, cap, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as e:     # fewer rows than the counts need
        moe.moe_expert_gemm_fp8(h, recv, sc, qw.cuda(), sw.cuda(), out, cap=cap - 1)
    assert e.value.status == moe.MOE_ERR_CAPACITY
    qw2, sw2 = _weights(wl.experts, 192, wl.hidden, 1)
    with pytest.raises(moe.MoeError) as e:     # N = 192 is not a multiple of 128
        moe.moe_expert_gemm_fp8(h, recv, sc, qw2.cuda(), sw2.cuda(), out, cap=cap)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED


def test_expert_gemm_capacity_overflow_writes_nothing_beyond_cap():
    """Without host counts, a capacity overflow is flagged by the layout; the GEMM computes only
    the row tiles that fit in cap and writes nothing past the buffer."""
    wl = W.WORKLOADS["tiny"].with_(fp8=True, hidden=256, alignment=128, tokens_per_rank=200, experts=8, topk=4)
    idx, w, x = inputs(wl)
    E, R, H, N = wl.experts, wl.ranks, wl.hidden, 128
    rows = oracle.layout(idx.numpy(), w.numpy(), E, R, wl.alignment).rows_per_rank
    cap = int(rows.max()) - 100                 # not a multiple of 128 either
    h = gpu_layout(wl, idx, w, cap=cap, cpu_sync=False)
    recv = torch.zeros((R, cap, H), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((R, cap, H // 128), device="cuda")
    moe.moe_dispatch(h, x.cuda(), moe.MOE_DTYPE_FP8_E4M3, recv, sc, cap=cap)
    qw, sw = _weights(E, N, H, 2)
    buf = torch.full((R * cap * N + 4096,), FILL, dtype=torch.int16, device="cuda")
    out = buf[:R * cap * N].view(R, cap, N).view(torch.bfloat16)
    moe.moe_expert_gemm_fp8(h, recv, sc, qw.cuda(), sw.cuda(), out, cap=cap)
    assert moe.moe_handle_status(h) == moe.MOE_ERR_CAPACITY
    assert (buf[R * cap * N:].cpu() == FILL).all()
