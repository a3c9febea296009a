"""The no-host-sync round trip (layout -> dispatch -> combine -> handle release) captured in a
CUDA graph and replayed with new inputs in the same buffers: every replay must match the oracle
exactly as the eager path does.  ("Why MoE gets stuck on communication", section 4, lists graph
capture as unsupported on the pages' Ascend port; here the do_cpu_sync=0 path is capturable.)"""
import numpy as np
import pytest
import torch

import combine_moe_layout_07_b200 as moe
import oracle
import workloads as W
from gpu_helpers import bits

pytestmark = pytest.mark.gpu


def _oracle_round_trip(wl, idx, w, x, y, bias, cap):
    E, R, A = wl.experts, wl.ranks, wl.alignment
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A, cap=cap)
    st, codes, scales, _ = oracle.dispatch_fp8(lay, idx.numpy(), w.numpy(), bits(x), E, R, A, cap, False, fill=0)
    st2, out = oracle.combine(idx.numpy(), lay.slot, bits(y), E, R, bias_bits=bits(bias))
    assert st == st2 == oracle.OK
    return lay, codes, scales, out


def test_decode_round_trip_in_a_cuda_graph():
    wl = W.WORKLOADS["decode"].with_(tokens_per_rank=32, hidden=1024, experts=64)
    p = moe.params(wl.tokens, wl.ranks, wl.experts, wl.topk, wl.hidden, wl.alignment, recv_capacity_rows=1,
                   do_cpu_sync=False)
    cap = moe.moe_recv_capacity_hint(p, 64)
    p.recv_capacity_rows = cap
    dev = "cuda"
    idx_s = torch.zeros(wl.tokens, wl.topk, dtype=torch.int64, device=dev)
    w_s = torch.zeros(wl.tokens, wl.topk, device=dev)
    x_s = torch.zeros(wl.tokens, wl.hidden, dtype=torch.bfloat16, device=dev)
    y_s = torch.zeros(wl.ranks, cap, wl.hidden, dtype=torch.bfloat16, device=dev)
    b_s = torch.zeros(wl.tokens, wl.hidden, dtype=torch.bfloat16, device=dev)
    out_s = torch.zeros(wl.tokens, wl.hidden, dtype=torch.bfloat16, device=dev)
    recv = torch.zeros(wl.ranks, cap, wl.hidden, dtype=torch.uint8, device=dev)
    scales = torch.zeros(wl.ranks, cap, wl.hidden // 128, device=dev)

    def round_trip():
        h = moe.moe_layout(p, idx_s, w_s)
        moe.moe_dispatch(h, x_s, moe.MOE_DTYPE_FP8_E4M3, recv, scales, cap=cap, do_zero_padding=False)
        moe.moe_combine(h, y_s, out_s, bias=b_s, cap=cap)
        moe.moe_handle_free(h)

    def load(seed):
        wls = wl.with_(seed=seed)
        idx, w = W.gen_routing(wls)
        x, y, bias = W.gen_x(wls), W.gen_y(wls, cap), W.gen_bias(wls)
        idx_s.copy_(idx)
        w_s.copy_(w)
        x_s.copy_(x)
        y_s.copy_(y)
        b_s.copy_(bias)
        return idx, w, x, y, bias

    load(0)
    round_trip()  # eager warm-up (one-time attributes, memory pool)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        round_trip()
    for seed in (1, 2):
        idx, w, x, y, bias = load(seed)
        recv.zero_()
        scales.zero_()
        g.replay()
        torch.cuda.synchronize()
        lay, codes, sc, ref = _oracle_round_trip(wl, idx, w, x, y, bias, cap)
        assert (bits(out_s) == ref).all()
        for r in range(wl.ranks):
            n = int(lay.rows_per_rank[r])
            valid = lay.row_src[r, :n] >= 0
            assert (recv[r, :n].cpu().numpy()[valid] == codes[r, :n][valid]).all()
            assert (scales[r, :n].cpu().numpy()[valid].view(np.uint32) == sc[r, :n][valid].view(np.uint32)).all()
