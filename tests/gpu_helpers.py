"""Shared helpers for the GPU parity tests: run the round trip through the C ABI binding and
run the oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import combine_moe_layout_07_b200 as moe
import oracle
import workloads as W


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_from_bits(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def assert_bf16_close(got_bits: np.ndarray, ref_bits: np.ndarray):
    """The combine tolerance: |got - ref| <= 2^-7 |ref| + 1e-6 (one bf16 ulp)."""
    g = bf16_from_bits(got_bits).astype(np.float64)
    r = bf16_from_bits(ref_bits).astype(np.float64)
    bad = np.abs(g - r) > 2.0 ** -7 * np.abs(r) + 1e-6
    assert not bad.any(), f"{bad.sum()} elements outside 1 bf16 ulp; first at {np.argwhere(bad)[:3]}"


def inputs(wl: W.Workload, mask: float = 0.0):
    idx, w = W.gen_routing(wl)
    if mask:
        idx = W.mask_entries(wl, idx, mask)
    x = W.gen_x(wl)
    return idx, w, x


def gpu_layout(wl: W.Workload, idx: torch.Tensor, w: torch.Tensor | None, cap: int = 0,
               cpu_sync: bool | None = None, num_sms: int = 0, by_rank: bool = False):
    cpu_sync = wl.cpu_sync if cpu_sync is None else cpu_sync
    p = moe.params(wl.tokens, wl.ranks, wl.experts, wl.topk, wl.hidden, wl.alignment,
                   recv_capacity_rows=cap, num_sms=num_sms, do_cpu_sync=cpu_sync, by_rank=by_rank)
    return moe.moe_layout(p, idx.cuda(), None if w is None else w.cuda())


def compare_layout(h: moe.Handle, lay: oracle.Layout, wl: W.Workload):
    """Bit-exact: counts, psum, rows, tokens, membership, slots, row maps (rows in use)."""
    torch.cuda.synchronize()
    assert (h.counts().cpu().numpy() == lay.cnt).all()
    assert (h.psum().cpu().numpy() == lay.psum).all()
    assert (h.rows_per_rank().cpu().numpy() == lay.rows_per_rank).all()
    assert (h.tokens_per_rank().cpu().numpy() == lay.tokens_per_rank).all()
    assert (h.token_in_rank().cpu().numpy() == lay.token_in_rank).all()
    assert (h.slots().cpu().numpy() == lay.slot).all()
    src, rw = h.row_src().cpu().numpy(), h.row_weights().cpu().numpy()
    for r in range(wl.ranks):
        n = int(lay.rows_per_rank[r])
        assert (src[r, :n] == lay.row_src[r, :n]).all(), r
        assert (rw[r, :n].view(np.uint32) == lay.row_w[r, :n].view(np.uint32)).all(), r
