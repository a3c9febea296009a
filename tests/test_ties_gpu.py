"""Hand-worked rounding ties on the GPU, through the C ABI: inputs where only the documented
sequence of fp32 operations gives the stated bf16 / E4M3 result (ascending j, bias last, one
fused multiply-add per weighted row, first-appearance rank order, one fp32 multiply in the
backward, one IEEE division for the FP8 inverse).  Random inputs almost never land on such a tie,
so these cases pin the kernels' arithmetic where random parity cannot.  Each result is also
compared with the oracle's."""
import numpy as np
import pytest
import torch

import combine_moe_layout_07_b200 as moe
import oracle
from gpu_helpers import bits

pytestmark = pytest.mark.gpu

ONE, P2M8, P2M24 = 0x3F80, 0x3B80, 0x3380   # bf16 patterns of 1.0, 2^-8, 2^-24
CAP = 8


def _bf16_rows(shape, fill=0):
    return torch.full(shape, fill, dtype=torch.int16)


def _combine_one_token(rows, weights=None, bias=None, H=64):
    """One token routed to experts 0..k-1 of one rank, expert j's row holding the pattern rows[j];
    returns the GPU output bits [H] after checking them against the oracle."""
    k = len(rows)
    idx = torch.arange(k, dtype=torch.int64)[None, :]
    w = torch.tensor([weights if weights is not None else [1.0] * k], dtype=torch.float32)
    p = moe.params(1, 1, k, k, H, 1, recv_capacity_rows=CAP, do_cpu_sync=True)
    h = moe.moe_layout(p, idx.cuda(), w.cuda())
    slots = h.slots().cpu().numpy()
    y = _bf16_rows((1, CAP, H))
    for j, v in enumerate(rows):
        y[0, int(slots[0, j]), :] = v
    y = y.view(torch.bfloat16)
    b = None if bias is None else _bf16_rows((1, H), bias).view(torch.bfloat16)
    out = torch.empty(1, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(h, y.cuda(), out, topk_weights=w.cuda() if weights is not None else None,
                    bias=None if b is None else b.cuda(), cap=CAP)
    torch.cuda.synchronize()
    got = bits(out)[0]
    st, ref = oracle.combine(idx.numpy(), slots, bits(y), k, 1, w=w.numpy() if weights is not None else None,
                             bias_bits=None if b is None else bits(b))
    assert st == oracle.OK and (got == ref[0]).all()
    assert moe.moe_handle_status(h) == moe.MOE_OK
    moe.moe_handle_free(h)
    return got


def test_combine_adds_the_rows_in_ascending_j():
    # 1 + 2^-8, then two half-ulp additions that round back to even: the bf16 tie, to even
    assert (_combine_one_token([ONE, P2M8, P2M24, P2M24]) == ONE).all()
    # the same values with the small ones first: exact 1 + 2^-8 + 2^-23, above the tie
    assert (_combine_one_token([P2M24, P2M24, P2M8, ONE]) == 0x3F81).all()


def test_combine_adds_the_bias_last():
    assert (_combine_one_token([P2M24, P2M24, P2M8], bias=ONE) == 0x3F81).all()


def test_weighted_combine_uses_one_fused_multiply_add():
    # w * y = 2^-8 + 2^-24 + 2^-32 exactly; only fma(w, y, 1) lands above the bf16 tie
    w1 = 11184982 * 2.0 ** -24
    assert (_combine_one_token([ONE, 0x3BC0], weights=[1.0, w1]) == 0x3F81).all()


def test_combine_by_rank_adds_ranks_in_first_appearance_order():
    T, R, H = 4, 4, 64
    idx = torch.tensor([[3, 2, 1, 0]] * T, dtype=torch.int64)
    w = torch.ones(T, 4)
    p = moe.params(T, R, 4, 4, H, 1, recv_capacity_rows=0, do_cpu_sync=True, by_rank=True)
    h = moe.moe_layout(p, idx.cuda(), w.cuda())
    tr = h.token_rows().cpu().numpy()
    y = _bf16_rows((R, CAP, H))
    for r, v in zip((3, 2, 1, 0), (ONE, P2M8, P2M24, P2M24)):
        for t in range(T):
            y[r, int(tr[t, r]), :] = v
    y = y.view(torch.bfloat16)
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine_by_rank(h, y.cuda(), out, cap=CAP)
    torch.cuda.synchronize()
    got = bits(out)
    st, ref = oracle.combine_by_rank(idx.numpy(), tr, bits(y), 4, R)
    assert st == oracle.OK and (got == ref).all()
    assert (got == ONE).all()
    assert moe.moe_handle_status(h) == moe.MOE_OK
    moe.moe_handle_free(h)


def test_fp8_inverse_is_one_ieee_division():
    # 9 * 2^-13 * fl(448 / 504) is exactly 2^-10, the E4M3 tie between 0 and 2^-9: code 0
    x = torch.tensor([[504.0, 9 * 2.0 ** -13] + [0.0] * 126]).to(torch.bfloat16)
    p = moe.params(1, 1, 1, 1, 128, 1, recv_capacity_rows=CAP, do_cpu_sync=True)
    idx = torch.zeros((1, 1), dtype=torch.int64)
    h = moe.moe_layout(p, idx.cuda(), torch.ones(1, 1).cuda())
    recv = torch.full((1, CAP, 128), 0xA5, dtype=torch.uint8, device="cuda")
    sc = torch.full((1, CAP, 1), float("nan"), device="cuda")
    moe.moe_dispatch(h, x.cuda(), moe.MOE_DTYPE_FP8_E4M3, recv, sc, cap=CAP)
    torch.cuda.synchronize()
    codes, scale = recv[0, 0].cpu().numpy(), float(sc[0, 0, 0].item())
    assert codes[0] == 0x7E and codes[1] == 0x00 and (codes[2:] == 0).all()
    assert scale == 1.125
    ref_codes, ref_scale = oracle.quantize_block(bits(x)[0])
    assert (codes == ref_codes).all() and scale == ref_scale
    assert moe.moe_handle_status(h) == moe.MOE_OK
    moe.moe_handle_free(h)


def test_backward_rounds_w_times_g_once_in_fp32():
    # w * g = 1 + 2^-8 + 2^-24 exactly: fp32 rounds it to the bf16 tie 1 + 2^-8, then to even
    H = 256
    w = torch.tensor([[11228502 * 2.0 ** -24]], dtype=torch.float32)
    p = moe.params(1, 1, 1, 1, H, 1, recv_capacity_rows=CAP, do_cpu_sync=True)
    h = moe.moe_layout(p, torch.zeros((1, 1), dtype=torch.int64).cuda(), w.cuda())
    g = _bf16_rows((1, H), 0x3FC0).view(torch.bfloat16)          # 1.5
    gy = torch.full((1, CAP, H), -23131, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    moe.moe_combine_backward(h, g.cuda(), gy, topk_weights=w.cuda(), cap=CAP)
    torch.cuda.synchronize()
    assert (bits(gy)[0, 0] == ONE).all()
    assert moe.moe_handle_status(h) == moe.MOE_OK
    moe.moe_handle_free(h)
