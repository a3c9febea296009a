"""A seeded sweep of random problem shapes, every byte against the oracle.

Each case draws the token count, logical ranks, experts per rank, top-k, expert alignment,
hidden size, dtype, masking and host-sync mode, then runs layout -> dispatch -> combine through
the C ABI and compares everything bit-exactly (the full-buffer comparison of the parity suite).
Small batches take the fused one-launch layout, larger ones the three kernels, so the sweep
crosses that boundary too.  When the shape allows it (expert_alignment and H multiples of 128,
FP8), the expert GEMM runs on the dispatch output and is checked against the binary64 oracle."""
import numpy as np
import pytest
import torch

import combine_moe_layout_07_b200 as moe
import oracle
import workloads as W
from gpu_helpers import bits, gpu_layout
from test_expert_gemm_gpu import m_factor
from test_parity_gpu import _roundtrip_small

pytestmark = pytest.mark.gpu


def _case(seed: int):
    rng = np.random.default_rng(1000 + seed)
    R = int(rng.choice([1, 2, 3, 4, 8, 16]))
    e_loc = int(rng.integers(1, 33))
    E = R * e_loc
    k = int(rng.integers(1, min(E, 9) + 1))
    A = int(rng.choice([1, 2, 7, 16, 128]))
    fp8 = bool(rng.integers(0, 2))
    H = int(rng.choice([128, 256, 384, 640])) if fp8 else int(8 * rng.integers(1, 90))
    tpr = int(rng.integers(1, 6000 // R + 2))
    mask = float(rng.choice([0.0, 0.05, 0.3]))
    cpu_sync = bool(rng.integers(0, 2))
    wl = W.WORKLOADS["tiny"].with_(tokens_per_rank=tpr, ranks=R, experts=E, topk=k, alignment=A, hidden=H,
                                   fp8=fp8, seed=seed)
    return wl, mask, cpu_sync


@pytest.mark.parametrize("seed", range(24))
def test_random_shape_round_trip(seed):
    wl, mask, cpu_sync = _case(seed)
    idx, w = W.gen_routing(wl)
    if mask:
        idx = W.mask_entries(wl, idx, mask)
    x = W.gen_x(wl)
    _roundtrip_small(wl, idx, w, x, weighted=bool(seed % 2), with_bias=bool(seed % 3 == 0), cpu_sync=cpu_sync)


@pytest.mark.parametrize("seed", range(8))
def test_random_shape_expert_gemm(seed):
    # sizes kept small: the binary64 oracle decodes every product (a few seconds per case here)
    rng = np.random.default_rng(2000 + seed)
    R = int(rng.choice([1, 2, 4]))
    E = R * int(rng.integers(1, 5))
    k = int(rng.integers(1, min(E, 6) + 1))
    H = int(rng.choice([128, 256]))
    N = int(rng.choice([128, 256, 384]))
    wl = W.WORKLOADS["tiny"].with_(tokens_per_rank=int(rng.integers(1, 65)), ranks=R, experts=E, topk=k,
                                   alignment=128, hidden=H, fp8=True, seed=100 + seed)
    idx, w = W.gen_routing(wl)
    idx = W.mask_entries(wl, idx, 0.1)
    x = W.gen_x(wl)
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, 128)
    cap = int(lay.rows_per_rank.max()) + 1
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, 128, cap=cap)
    h = gpu_layout(wl, idx, w, cap=cap)
    recv = torch.zeros((R, cap, H), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((R, cap, H // 128), device="cuda")
    moe.moe_dispatch(h, x.cuda(), moe.MOE_DTYPE_FP8_E4M3, recv, sc, cap=cap)
    g = torch.Generator().manual_seed(seed)
    qw = torch.randint(0, 256, (E, N, H), generator=g, dtype=torch.uint8)
    qw[(qw & 0x7F) == 0x7F] = 0x38
    sw = torch.rand((E, N // 128, H // 128), generator=g) / 32 + 1 / 256
    out = torch.full((R, cap, N), -23131, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    moe.moe_expert_gemm_fp8(h, recv, sc, qw.cuda(), sw.cuda(), out, cap=cap)
    codes, scales = recv.cpu().numpy(), sc.cpu().numpy()
    st, ref = oracle.grouped_gemm_f64(lay, codes, scales, qw.numpy(), sw.numpy(), E, R, 128)
    assert st == 0
    got = bits(out)
    gotf = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    table = np.array([oracle.e4m3_to_double(c) for c in range(256)], np.float64)
    e_loc = E // R
    for r in range(R):
        n = int(lay.rows_per_rank[r])
        assert (got[r, n:] == np.uint16(0xA5A5)).all()
        ax = np.abs(table[codes[r, :n]]) * np.repeat(scales[r, :n].astype(np.float64), 128, axis=1)
        for e in range(r * e_loc, (r + 1) * e_loc):          # the bound of the expert GEMM tests
            end = int(lay.psum[e]); beg = end - -(-int(lay.cnt[e]) // 128) * 128
            if end == beg:
                continue
            aw = np.abs(table[qw[e].numpy()]) * np.repeat(np.repeat(sw[e].numpy().astype(np.float64), 128, 0), 128, 1)
            M = ax[beg:end] @ aw.T
            tol = 2.0 ** -8 * np.abs(ref[r, beg:end]) + m_factor(wl.hidden) * M
            assert (np.abs(gotf[r, beg:end] - ref[r, beg:end]) <= tol).all(), (r, e)
    assert moe.moe_handle_status(h) == moe.MOE_OK
