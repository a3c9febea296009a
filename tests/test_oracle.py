"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test checks the oracle against what the pages or the mathematics fix: the worked padding
example, closed forms, invariants that determine the answer uniquely, brute-force enumeration on
tiny inputs, a second (sort-based) statement of the slot assignment, the OCP E4M3 definition
(hand table, nearest-value search, torch's own conversion), and round-trip / exactness bounds.
"""
import itertools
import json
import math
import os
import struct

import numpy as np
import pytest
import torch

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def align_up(n, a):
    return -(-n // a) * a


def check_layout_invariants(idx, E, R, A, lay):
    """Independent checker: these properties determine slot/psum/rows uniquely."""
    idx = np.asarray(idx)
    T, k = idx.shape
    e_loc = E // R
    valid = [(t, j, int(idx[t, j])) for t in range(T) for j in range(k) if idx[t, j] >= 0]
    cnt = np.zeros(E, np.int64)
    for _, _, e in valid:
        cnt[e] += 1
    assert (lay.cnt == cnt).all()
    assert lay.cnt.sum() == T * k - int((idx == -1).sum())
    for r in range(R):
        start = 0
        for e in range(r * e_loc, (r + 1) * e_loc):
            seg = [(t, j) for (t, j, ee) in valid if ee == e]     # ascending (t, j)
            got = [int(lay.slot[t, j]) for (t, j) in seg]
            assert got == list(range(start, start + len(seg))), (e, got, start)
            for (t, j) in seg:
                assert lay.row_src[r, lay.slot[t, j]] == t
            for row in range(start + len(seg), start + align_up(len(seg), A)):
                assert lay.row_src[r, row] == -1
                assert lay.row_w[r, row] == 0.0
            start += align_up(len(seg), A)
            assert lay.psum[e] == start
        assert lay.rows_per_rank[r] == start
    for t in range(T):
        for j in range(k):
            if idx[t, j] < 0:
                assert lay.slot[t, j] == -1
    members = [set(int(e) // e_loc for e in idx[t] if e >= 0) for t in range(T)]
    for r in range(R):
        assert lay.tokens_per_rank[r] == sum(r in m for m in members)
        assert all(lay.token_in_rank[t, r] == (r in members[t]) for t in range(T))


# ----------------------------------------------------------------------------- layout

def test_padding_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "padding_worked_example.json")))
    A, counts = g["alignment"], g["counts"]
    idx = np.concatenate([np.full(c, e) for e, c in enumerate(counts)]).reshape(-1, 1)
    lay = oracle.layout(idx, None, E=len(counts), R=1, A=A)
    assert lay.status == oracle.OK
    assert list(lay.cnt) == counts
    assert list(lay.psum) == [128, 256, 384]
    assert lay.rows_per_rank[0] == g["slots_total"]
    assert lay.cnt.sum() == g["valid_rows"]
    assert lay.rows_per_rank[0] / lay.cnt.sum() == g["A_pad"]


def test_alignment_one_is_plain_inclusive_scan():
    wl = W.WORKLOADS["tiny"].with_(alignment=1)
    idx, w = W.gen_routing(wl)
    lay = oracle.layout(idx.numpy(), w.numpy(), wl.experts, wl.ranks, 1)
    cnt = np.bincount(idx.numpy().ravel(), minlength=wl.experts)
    e_loc = wl.experts_per_rank
    expect = np.concatenate([np.cumsum(cnt[r * e_loc:(r + 1) * e_loc]) for r in range(wl.ranks)])
    assert (lay.psum == expect).all()


@pytest.mark.parametrize("name", ["tiny", "skewed"])
@pytest.mark.parametrize("mask", [0.0, 0.2])
def test_layout_invariants_workloads(name, mask):
    wl = W.WORKLOADS[name]
    if name == "skewed":
        wl = wl.with_(tokens_per_rank=8)   # 128 tokens keeps the pure-Python checker quick
    idx, w = W.gen_routing(wl)
    if mask:
        idx = W.mask_entries(wl, idx, mask)
    lay = oracle.layout(idx.numpy(), w.numpy(), wl.experts, wl.ranks, wl.alignment)
    assert lay.status == oracle.OK
    check_layout_invariants(idx.numpy(), wl.experts, wl.ranks, wl.alignment, lay)
    # weights travel bit-exactly into row_w
    for t in range(wl.tokens):
        for j in range(wl.topk):
            e = int(idx[t, j])
            if e >= 0:
                assert lay.row_w[e // wl.experts_per_rank, lay.slot[t, j]] == w[t, j].item()


@pytest.mark.parametrize("E,R,A,k", [(8, 2, 16, 2), (256, 8, 128, 8), (12, 3, 5, 4), (5, 1, 1, 3),
                                     (64, 64, 7, 2)])
def test_layout_equals_sort_formulation(E, R, A, k):
    rng = np.random.default_rng(E * 1000 + A)
    T = 300
    idx = rng.integers(-1, E, size=(T, k)).astype(np.int64)
    lay = oracle.layout(idx, None, E, R, A)
    st, cnt, psum, slot = oracle.layout_by_sort(idx, E, R, A)
    assert lay.status == st == oracle.OK
    assert (lay.cnt == cnt).all() and (lay.psum == psum).all() and (lay.slot == slot).all()


def test_layout_brute_force_tiny():
    """Every routing of T tokens over E experts (with masked entries) for tiny sizes."""
    n = 0
    for E, R, k, T in [(2, 1, 1, 4), (2, 2, 2, 2), (4, 2, 2, 2), (4, 1, 2, 2), (3, 3, 1, 3)]:
        choices = list(range(-1, E))
        for A in (1, 2, 3):
            for flat in itertools.product(choices, repeat=T * k):
                idx = np.array(flat, np.int64).reshape(T, k)
                lay = oracle.layout(idx, None, E, R, A)
                st, cnt, psum, slot = oracle.layout_by_sort(idx, E, R, A)
                assert lay.status == st == oracle.OK
                assert (lay.slot == slot).all() and (lay.psum == psum).all()
                check_layout_invariants(idx, E, R, A, lay)
                n += 1
    assert n > 1000


def test_layout_without_weights_gives_zero_row_weights():
    """topk_weights may be NULL: every row weight then reads 0, routed rows and padding alike."""
    wl = W.WORKLOADS["tiny"]
    idx, _ = W.gen_routing(wl)
    lay = oracle.layout(idx.numpy(), None, wl.experts, wl.ranks, wl.alignment)
    for r in range(wl.ranks):
        assert (lay.row_w[r, :int(lay.rows_per_rank[r])] == 0.0).all()


def test_layout_errors():
    idx = np.array([[0, 1], [2, 7]], np.int64)
    assert oracle.layout(idx, None, 8, 2, 4).status == oracle.OK
    assert oracle.layout(np.array([[0, 8]]), None, 8, 2, 4).status == oracle.ERR_BAD_EXPERT
    assert oracle.layout(np.array([[0, -2]]), None, 8, 2, 4).status == oracle.ERR_BAD_EXPERT
    # rank 0 needs 4 rows (A=4) but capacity 3
    assert oracle.layout(np.array([[0, 1]]), None, 8, 2, 4, cap=3).status == oracle.ERR_CAPACITY
    assert oracle.layout(np.array([[0, 1]]), None, 8, 2, 4, cap=8).status == oracle.OK


# ----------------------------------------------------------------------------- E4M3

def _golden_e4m3():
    rows = []
    for line in open(os.path.join(GOLDEN, "e4m3_edges.txt")):
        line = line.split("#")[0].strip()
        if line:
            v, c = line.split()[:2]
            rows.append((float(v), int(c, 16)))
    return rows


def test_e4m3_hand_table():
    for v, c in _golden_e4m3():
        assert oracle.e4m3_from_float(v) == c, (v, hex(c), hex(oracle.e4m3_from_float(v)))


def test_e4m3_decode_definition():
    assert oracle.e4m3_to_double(0x7E) == 448.0
    assert oracle.e4m3_to_double(0x01) == 2.0 ** -9
    assert oracle.e4m3_to_double(0x08) == 2.0 ** -6
    assert math.isnan(oracle.e4m3_to_double(0x7F)) and math.isnan(oracle.e4m3_to_double(0xFF))
    finite = [c for c in range(256) if c & 0x7F != 0x7F]
    vals = [oracle.e4m3_to_double(c) for c in finite]
    pos = sorted(v for v in vals if v > 0)
    assert len(pos) == 126 and len(set(pos)) == 126     # 126 distinct positive finite values


def test_e4m3_matches_nearest_value_search():
    """Encoder == argmin |v - value(code)| over all finite codes, ties to the even code,
    magnitudes above 448 saturated: a brute-force statement of round-to-nearest-even."""
    codes = [c for c in range(128) if c != 0x7F]
    table = np.array([oracle.e4m3_to_double(c) for c in codes])
    rng = np.random.default_rng(1)
    samples = np.concatenate([
        rng.standard_normal(3000) * 50, rng.standard_normal(2000) * 0.01,
        rng.uniform(-500, 500, 2000), np.array(table),                      # exact codes
        (table[:-1] + table[1:]) / 2,                                        # exact ties
    ]).astype(np.float32)
    for v in samples:
        a = abs(float(v))
        if a >= 448.0:
            c = 0x7E
        else:
            d = np.abs(table - a)
            best = np.flatnonzero(d == d.min())
            c = codes[best[0]] if len(best) == 1 else [codes[i] for i in best if codes[i] % 2 == 0][0]
        if math.copysign(1.0, float(v)) < 0:
            c |= 0x80
        assert oracle.e4m3_from_float(float(v)) == c, (float(v), hex(c))


def test_e4m3_matches_torch_conversion_in_range():
    """torch's float8_e4m3fn cast (round-to-nearest-even, no saturation) agrees wherever
    saturation does not enter."""
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(20000) * 30, rng.standard_normal(5000) * 1e-3]).astype(np.float32)
    v = v[np.abs(v) <= 448.0]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_from_float(float(a)) for a in v], np.uint8)
    assert (ref == got).all()


# ----------------------------------------------------------------------------- FP8 quantisation

def test_quantize_block_roundtrip_bound_and_max_code():
    wl = W.WORKLOADS["tiny"].with_(hidden=1024)
    x = W.gen_x(wl)[:16]
    xb = bits(x)
    for row in xb:
        for b in range(0, row.size, 128):
            blk = row[b:b + 128]
            codes, s = oracle.quantize_block(blk)
            xf = np.array([oracle.bf16_to_float(u) for u in blk], np.float64)
            q = np.array([oracle.e4m3_to_double(c) for c in codes])
            amax = np.abs(xf).max()
            assert s == np.float32(np.float32(max(amax, 1e-4)) / np.float32(448.0))
            err = np.abs(xf - q * s)
            normal = np.abs(xf) / s >= 2.0 ** -6
            assert (err[normal] <= 2.0 ** -4 * np.abs(xf[normal]) * (1 + 1e-6)).all()
            assert (err[~normal] <= s * 2.0 ** -10 * (1 + 1e-6)).all()
            i = int(np.argmax(np.abs(xf)))
            assert codes[i] & 0x7F == 0x7E            # the block's largest element codes to 448


def test_quantize_block_inv_is_one_ieee_division():
    """Block [504, 9 * 2^-13, 0, ...]: a = 504, inv = fl(448 / 504) = fl(8 / 9), and
    9 * 2^-13 * fl(8 / 9) rounds to exactly 2^-10, half the smallest E4M3 subnormal: a tie, to
    even, code 0x00.  inv taken as 448 * fl(1 / 504) is one ulp larger and would give code 0x01.
    The amax element codes to 448 (0x7E) and the scale is 504 / 448 = 1.125 exactly."""
    xb = bits(torch.tensor([504.0, 9 * 2.0 ** -13] + [0.0] * 126).to(torch.bfloat16))
    codes, scale = oracle.quantize_block(xb)
    assert codes[0] == 0x7E and codes[1] == 0x00 and (codes[2:] == 0).all()
    assert scale == 1.125


def test_quantize_block_zero_and_floor():
    codes, s = oracle.quantize_block(np.zeros(128, np.uint16))
    assert (codes == 0).all() and s == np.float32(1e-4) / np.float32(448.0)
    neg0 = np.full(128, 0x8000, np.uint16)
    codes, _ = oracle.quantize_block(neg0)
    assert (codes == 0x80).all()


# ----------------------------------------------------------------------------- dispatch

def _tiny(mask=0.0, **kw):
    wl = W.WORKLOADS["tiny"].with_(**kw)
    idx, w = W.gen_routing(wl)
    if mask:
        idx = W.mask_entries(wl, idx, mask)
    x = W.gen_x(wl)
    return wl, idx.numpy(), w.numpy(), x


@pytest.mark.parametrize("zero_padding", [True, False])
@pytest.mark.parametrize("mask", [0.0, 0.25])
def test_dispatch_bf16_is_a_gather(zero_padding, mask):
    wl, idx, w, x = _tiny(mask)
    E, R, A = wl.experts, wl.ranks, wl.alignment
    lay = oracle.layout(idx, w, E, R, A)
    cap = int(lay.rows_per_rank.max()) + 3
    st, recv, rw = oracle.dispatch_bf16(lay, idx, w, bits(x), E, R, A, cap, zero_padding)
    assert st == oracle.OK
    xb = bits(x)
    e_loc = E // R
    for t in range(wl.tokens):
        for j in range(wl.topk):
            if idx[t, j] >= 0:
                r = idx[t, j] // e_loc
                assert (recv[r, lay.slot[t, j]] == xb[t]).all()
                assert rw[r, lay.slot[t, j]] == w[t, j]
    for r in range(R):
        pad = lay.row_src[r, :lay.rows_per_rank[r]] == -1
        rows = recv[r, :lay.rows_per_rank[r]][pad]
        assert (rows == (0 if zero_padding else 0xA5A5)).all()
        assert (rw[r, :lay.rows_per_rank[r]][pad] == 0).all()
        assert (recv[r, lay.rows_per_rank[r]:] == 0xA5A5).all()      # beyond the rows: untouched


def test_dispatch_fp8_rows_match_block_quantiser():
    wl, idx, w, x = _tiny(0.1, hidden=512)
    E, R, A = wl.experts, wl.ranks, wl.alignment
    lay = oracle.layout(idx, w, E, R, A)
    cap = int(lay.rows_per_rank.max())
    st, codes, scales, rw = oracle.dispatch_fp8(lay, idx, w, bits(x), E, R, A, cap, True)
    assert st == oracle.OK
    xb = bits(x)
    e_loc = E // R
    for t in range(wl.tokens):
        ref = [oracle.quantize_block(xb[t, b:b + 128]) for b in range(0, 512, 128)]
        for j in range(wl.topk):
            if idx[t, j] >= 0:
                r, s = idx[t, j] // e_loc, lay.slot[t, j]
                assert (codes[r, s] == np.concatenate([c for c, _ in ref])).all()
                assert (scales[r, s] == np.array([v for _, v in ref], np.float32)).all()
    for r in range(R):
        pad = lay.row_src[r, :lay.rows_per_rank[r]] == -1
        assert (codes[r, :lay.rows_per_rank[r]][pad] == 0).all()
        assert (scales[r, :lay.rows_per_rank[r]][pad] == 0).all()


# ----------------------------------------------------------------------------- combine

def _roundtrip(wl, idx, w, x):
    E, R, A = wl.experts, wl.ranks, wl.alignment
    lay = oracle.layout(idx, w, E, R, A)
    cap = int(lay.rows_per_rank.max())
    _, recv, _ = oracle.dispatch_bf16(lay, idx, w, bits(x), E, R, A, cap, True)
    return lay, recv


def test_combine_identity_expert_unit_weights_reproduces_x():
    wl, idx, w, x = _tiny()
    lay, recv = _roundtrip(wl, idx, w, x)
    st, out = oracle.combine(idx, lay.slot, recv, wl.experts, wl.ranks, w=w)
    assert st == oracle.OK
    xf = x.float().numpy()
    of = out.astype(np.uint32) << 16
    of = of.view(np.float32)
    assert (np.abs(of - xf) <= 2.0 ** -7 * np.abs(xf) + 1e-6).all()


def test_combine_single_expert_unit_weight_exact():
    wl, idx, w, x = _tiny(topk=1)
    lay, recv = _roundtrip(wl, idx, w, x)
    st, out = oracle.combine(idx, lay.slot, recv, wl.experts, wl.ranks, w=np.ones_like(w))
    assert (out == bits(x)).all()
    st, out = oracle.combine(idx, lay.slot, recv, wl.experts, wl.ranks)
    assert (out == bits(x)).all()


def test_combine_bias_only_exact():
    wl, idx, w, x = _tiny(mask=0.3)
    lay, recv = _roundtrip(wl, idx, w, x)
    bias = W.gen_bias(wl)
    st, out = oracle.combine(idx, lay.slot, np.zeros_like(recv), wl.experts, wl.ranks, w=w, bias_bits=bits(bias))
    assert (out == bits(bias)).all()


def test_combine_unweighted_sum_of_copies():
    """With an identity expert and no weights, each token gets k_valid * x: exact in fp32 and,
    for k_valid a power of two, exact in bf16 too."""
    wl, idx, w, x = _tiny()
    lay, recv = _roundtrip(wl, idx, w, x)
    st, out = oracle.combine(idx, lay.slot, recv, wl.experts, wl.ranks)
    assert (out == bits((x.float() * 2).to(torch.bfloat16))).all()   # tiny has k = 2


@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("with_bias", [False, True])
def test_combine_fp32_within_tolerance_of_f64(weighted, with_bias):
    wl, idx, w, x = _tiny(mask=0.1, topk=4)
    lay = oracle.layout(idx, w, wl.experts, wl.ranks, wl.alignment)
    cap = int(lay.rows_per_rank.max())
    y = W.gen_y(wl, cap)
    bias = bits(W.gen_bias(wl)) if with_bias else None
    ww = w if weighted else None
    st, out = oracle.combine(idx, lay.slot, bits(y), wl.experts, wl.ranks, w=ww, bias_bits=bias)
    ref = oracle.combine_f64(idx, lay.slot, bits(y), wl.experts, wl.ranks, w=ww, bias_bits=bias)
    got = (out.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert (np.abs(got - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-6).all()
    # the f64 statement against a numpy gather-and-sum of the same rows
    e_loc = wl.experts // wl.ranks
    yf = y.float().numpy().astype(np.float64)
    for t in range(0, wl.tokens, 7):
        acc = np.zeros(wl.hidden)
        for j in range(wl.topk):
            if idx[t, j] >= 0:
                acc += (float(w[t, j]) if weighted else 1.0) * yf[idx[t, j] // e_loc, lay.slot[t, j]]
        if with_bias:
            acc += W.gen_bias(wl)[t].float().numpy()
        assert np.allclose(acc, ref[t], rtol=0, atol=1e-12)


# bf16 bit patterns of the hand-worked order cases below
_ONE, _2M8, _2M24 = 0x3F80, 0x3B80, 0x3380       # 1.0, 2^-8, 2^-24


def _one_token(rows, bias=None, weighted=False, H=8):
    """One token whose k = len(rows) pairs hit experts 0..k-1 of one rank, slot j holding rows[j]."""
    k = len(rows)
    idx = np.arange(k, dtype=np.int64)[None, :]
    slot = np.arange(k, dtype=np.int32)[None, :]
    y = np.repeat(np.array(rows, np.uint16)[None, :, None], H, axis=2)
    w = np.ones((1, k), np.float32) if weighted else None
    b = None if bias is None else np.full((1, H), bias, np.uint16)
    st, out = oracle.combine(idx, slot, y, k, 1, w=w, bias_bits=b)
    assert st == oracle.OK
    return out[0]


@pytest.mark.parametrize("weighted", [False, True])
def test_combine_adds_the_rows_in_ascending_j(weighted):
    """Rows 1, 2^-8, 2^-24, 2^-24 in that j order.  In fp32: 1 + 2^-8 is exact; each + 2^-24 is
    half an ulp (2^-23) from an even value and rounds back to 1 + 2^-8; that is a bf16 tie,
    which rounds to even: 1.0.  Summed in descending j the two 2^-24 first make 2^-23, the total
    1 + 2^-8 + 2^-23 is exact and lies above the tie: bf16 1 + 2^-7 (0x3F81).  Unit weights
    (fma(1, y, acc)) change nothing."""
    assert (_one_token([_ONE, _2M8, _2M24, _2M24], weighted=weighted) == _ONE).all()
    assert (_one_token([_2M24, _2M24, _2M8, _ONE], weighted=weighted) == 0x3F81).all()


def test_combine_weighted_rows_use_one_fused_multiply_add():
    """Rows 1.0 (w = 1) and y = 1.5 * 2^-8 with w = 11184982 * 2^-24: w * y is exactly
    2^-8 + 2^-24 + 2^-32.  With fma(w, y, acc) the fp32 sum 1 + 2^-8 + 2^-24 + 2^-32 lies above
    the tie at 2^-24 and rounds to 1 + 2^-8 + 2^-23, above the bf16 tie: 0x3F81.  Rounding the
    product first gives 2^-8 + 2^-24 (a tie, to even), then the sum 1 + 2^-8 + 2^-24 rounds to
    even, 1 + 2^-8, the bf16 tie, and the result would be 1.0."""
    idx = np.arange(2, dtype=np.int64)[None, :]
    slot = np.arange(2, dtype=np.int32)[None, :]
    y = np.array([[[_ONE] * 8, [0x3BC0] * 8]], np.uint16)      # 1.0, 1.5 * 2^-8
    w = np.array([[1.0, 11184982 * 2.0 ** -24]], np.float32)
    assert float(w[0, 1]) == 11184982 * 2.0 ** -24               # exactly representable
    st, out = oracle.combine(idx, slot, y, 2, 1, w=w)
    assert st == oracle.OK and (out == 0x3F81).all()


def test_combine_by_rank_adds_ranks_in_first_appearance_order():
    """One token whose experts sit on ranks 3, 2, 1, 0 in j order, each rank's partial row being
    1, 2^-8, 2^-24, 2^-24: in that order the sum rounds to bf16 1.0 (the ascending-j case above);
    in ascending rank order it would be 1 + 2^-7."""
    idx = np.array([[3, 2, 1, 0]], np.int64)
    token_row = np.zeros((1, 4), np.int32)
    y = np.zeros((4, 1, 8), np.uint16)
    for r, v in zip((3, 2, 1, 0), (_ONE, _2M8, _2M24, _2M24)):
        y[r, 0, :] = v
    st, out = oracle.combine_by_rank(idx, token_row, y, 4, 4)
    assert st == oracle.OK and (out == _ONE).all()


def test_combine_by_rank_adds_the_bias_last():
    """By rank, partial rows 2^-24, 2^-24, 2^-8 (ranks 0, 1, 2 in j order) and bias 1.0 give
    1 + 2^-8 + 2^-23 exactly, above the bf16 tie: 0x3F81; the bias first would give 1.0."""
    idx = np.array([[0, 1, 2]], np.int64)
    y = np.zeros((3, 1, 8), np.uint16)
    for r, v in enumerate((_2M24, _2M24, _2M8)):
        y[r, 0, :] = v
    st, out = oracle.combine_by_rank(idx, np.zeros((1, 3), np.int32), y, 3, 3,
                                     bias_bits=np.full((1, 8), _ONE, np.uint16))
    assert st == oracle.OK and (out == 0x3F81).all()


def test_combine_adds_the_bias_last():
    """Rows 2^-24, 2^-24, 2^-8 and bias 1.0: the rows sum exactly to 2^-8 + 2^-23, then the bias
    gives 1 + 2^-8 + 2^-23 exactly, above the bf16 tie: 0x3F81.  Had the bias come first, 1 +
    2^-24 would round back to 1 twice and the result would be the tie 1 + 2^-8, rounded to 1.0."""
    assert (_one_token([_2M24, _2M24, _2M8], bias=_ONE) == 0x3F81).all()
    assert (_one_token([_ONE, _2M24, _2M24, _2M8]) == _ONE).all()   # the same values, bias-first order


def test_bf16_rounding_definition():
    for v in [1.0, -2.5, 3.0e38, 1e-40, 0.1, 1.00390625, 1.01171875]:
        assert oracle.float_to_bf16(v) == bits(torch.tensor([v], dtype=torch.float32).to(torch.bfloat16))[0]
    assert oracle.float_to_bf16(float("nan")) == 0x7FC0
    # any NaN, whatever its sign or payload, becomes the one canonical pattern
    payload_nan = struct.unpack("<f", struct.pack("<I", 0x7FC12345))[0]
    assert oracle.float_to_bf16(payload_nan) == 0x7FC0
    assert oracle.float_to_bf16(-float("nan")) == 0x7FC0
    # ties: 1 + 2^-8 is halfway between 1 and 1 + 2^-7 -> even (1.0)
    assert oracle.float_to_bf16(1.00390625) == 0x3F80


# ----------------------------------------------------------------------------- backward of combine

def _bwd_case(mask=0.1, topk=4):
    wl, idx, w, x = _tiny(mask, topk=topk)
    E, R, A = wl.experts, wl.ranks, wl.alignment
    lay = oracle.layout(idx, w, E, R, A)
    cap = int(lay.rows_per_rank.max())
    y = W.gen_y(wl, cap)
    g = W.gen_bias(wl)          # any bf16 [T, H] tensor serves as grad_out
    return wl, idx, w, lay, cap, bits(y), bits(g)


def test_combine_backward_unweighted_is_the_bf16_dispatch_of_grad_out():
    wl, idx, w, lay, cap, y, g = _bwd_case()
    E, R, A = wl.experts, wl.ranks, wl.alignment
    st, gy = oracle.combine_backward(lay, idx, g, E, R, A, cap, w=None)
    st2, ref, _ = oracle.dispatch_bf16(lay, idx, w, g, E, R, A, cap, True)
    assert st == st2 == oracle.OK
    assert (gy == ref).all()


def test_combine_backward_rounds_w_times_g_once_in_fp32():
    """w = 11228502 * 2^-24 and g = 1.5: w * g is exactly 1 + 2^-8 + 2^-24, half an fp32 ulp
    above 1 + 2^-8, so the fp32 product rounds to even, 1 + 2^-8, a bf16 tie that rounds to
    even: 1.0 (0x3F80).  Rounding the exact product straight to bf16 would give 0x3F81."""
    w = np.array([[11228502 * 2.0 ** -24]], np.float32)
    assert float(w[0, 0]) == 11228502 * 2.0 ** -24
    idx = np.array([[0]], np.int64)
    lay = oracle.layout(idx, w, 1, 1, 1)
    st, gy = oracle.combine_backward(lay, idx, np.full((1, 8), 0x3FC0, np.uint16), 1, 1, 1, 1, w=w)
    assert st == oracle.OK and (gy[0, 0] == 0x3F80).all()


def test_combine_backward_is_the_adjoint_of_combine():
    """<g, C(y)> == <C^T(g), y> in binary64, up to the bf16 rounding of grad_y (weighted case)."""
    wl, idx, w, lay, cap, y, g = _bwd_case()
    E, R = wl.experts, wl.ranks
    out64 = oracle.combine_f64(idx, lay.slot, y, E, R, w=w)
    lhs = float(((g.astype(np.uint32) << 16).view(np.float32).astype(np.float64) * out64).sum())
    st, gy = oracle.combine_backward(lay, idx, g, E, R, wl.alignment, cap, w=w, fill=0)
    gyf = (gy.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    yf = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    rhs = float((gyf * yf).sum())
    scale = float(np.abs(gyf * yf).sum())
    assert abs(lhs - rhs) <= 2.0 ** -8 * scale
    # and exactly: each grad_y row is the bf16 rounding of w * g for its (t, j)
    e_loc = E // R
    gf = (g.astype(np.uint32) << 16).view(np.float32)
    for t in range(wl.tokens):
        for j in range(wl.topk):
            if idx[t, j] >= 0:
                row = gy[idx[t, j] // e_loc, lay.slot[t, j]]
                expect = bits(torch.from_numpy((np.float32(w[t, j]) * gf[t]).astype(np.float32)).to(torch.bfloat16))
                assert (row == expect).all()


def test_grad_weights_is_the_derivative_of_combine():
    """Central finite difference of L(w) = <g, combine_f64(y; w)> reproduces grad_w (L is
    linear in each weight, so the difference quotient is exact up to binary64 rounding)."""
    wl, idx, w, lay, cap, y, g = _bwd_case()
    E, R = wl.experts, wl.ranks
    gw = oracle.grad_weights_f64(idx, lay.slot, g, y, E, R)
    gf = (g.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    rng = np.random.default_rng(3)
    for _ in range(12):
        t, j = int(rng.integers(wl.tokens)), int(rng.integers(wl.topk))
        h = 0.25
        wp, wm = w.copy(), w.copy()
        wp[t, j] += h
        wm[t, j] -= h
        lp = float((gf * oracle.combine_f64(idx, lay.slot, y, E, R, w=wp)).sum())
        lm = float((gf * oracle.combine_f64(idx, lay.slot, y, E, R, w=wm)).sum())
        fd = (lp - lm) / (float(wp[t, j]) - float(wm[t, j]))  # the weights are fp32: use the real step
        assert abs(fd - gw[t, j]) <= 1e-9 * max(1.0, abs(gw[t, j])), (t, j, fd, gw[t, j])
        if idx[t, j] < 0:
            assert gw[t, j] == 0.0


# ----------------------------------------------------------------------------- non-expanded (by rank)

def test_layout_by_rank_invariants():
    wl, idx, w, x = _tiny(0.2, topk=4, experts=16, ranks=4)
    st, tr, rows = oracle.layout_by_rank(idx, wl.experts, wl.ranks)
    assert st == oracle.OK
    e_loc = wl.experts // wl.ranks
    lay = oracle.layout(idx, w, wl.experts, wl.ranks, wl.alignment)
    assert (rows == lay.tokens_per_rank).all()          # one row per member token
    for r in range(wl.ranks):
        members = [t for t in range(wl.tokens) if any(e >= 0 and e // e_loc == r for e in idx[t])]
        assert [int(tr[t, r]) for t in members] == list(range(len(members)))   # ascending tokens
        assert all(tr[t, r] == -1 for t in range(wl.tokens) if t not in members)


def test_by_rank_round_trip_equals_the_expanded_one():
    """Two-level reduction: with per-(token, rank) partial sums built from an expanded expert
    output, the by-rank combine equals the expanded combine in binary64 (then within one bf16
    rounding of each other)."""
    wl, idx, w, x = _tiny(0.15, topk=4, experts=16, ranks=4)
    E, R, A = wl.experts, wl.ranks, wl.alignment
    lay = oracle.layout(idx, w, E, R, A)
    cap = int(lay.rows_per_rank.max())
    y = bits(W.gen_y(wl, cap))
    e_loc = E // R
    st, tr, rows = oracle.layout_by_rank(idx, E, R)
    yf = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    part = np.zeros((R, int(rows.max()), wl.hidden))
    for t in range(wl.tokens):
        for j in range(wl.topk):
            e = idx[t, j]
            if e >= 0:
                part[e // e_loc, tr[t, e // e_loc]] += w[t, j] * yf[e // e_loc, lay.slot[t, j]]
    part_bits = bits(torch.from_numpy(part.astype(np.float32)).to(torch.bfloat16))
    st, out_rank = oracle.combine_by_rank(idx, tr, part_bits, E, R)
    ref = oracle.combine_f64(idx, lay.slot, y, E, R, w=w)
    got = (out_rank.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # each partial sum was rounded to bf16 once, the final sum once more
    assert (np.abs(got - ref) <= 2.0 ** -7 * (np.abs(ref) + np.abs(part).max(axis=(0, 1)).max()) + 1e-6).all()


def test_by_rank_dispatch_copies_and_topk_views():
    wl, idx, w, x = _tiny(0.1, topk=4, experts=16, ranks=4, hidden=256)
    E, R = wl.experts, wl.ranks
    st, tr, rows = oracle.layout_by_rank(idx, E, R)
    cap = int(rows.max())
    st, recv, _, ti, tw = oracle.dispatch_by_rank(idx, w, tr, bits(x), E, R, cap, fp8=False)
    e_loc = E // R
    xb = bits(x)
    for t in range(wl.tokens):
        for r in range(R):
            if tr[t, r] >= 0:
                assert (recv[r, tr[t, r]] == xb[t]).all()
                for j in range(wl.topk):
                    e = idx[t, j]
                    on = e >= 0 and e // e_loc == r
                    assert ti[r, tr[t, r], j] == (e - r * e_loc if on else -1)
                    assert tw[r, tr[t, r], j] == (w[t, j] if on else 0.0)
    # identity expert: the by-rank combine of the received copies gives (#member ranks) * x
    st, out = oracle.combine_by_rank(idx, tr, recv, E, R)
    members = np.array([[tr[t, r] >= 0 for r in range(R)] for t in range(wl.tokens)]).sum(1)
    expect = bits((x.float() * torch.from_numpy(members).float()[:, None]).to(torch.bfloat16))
    assert (out == expect).all()
    # FP8: each member row holds the token's 1x128 block codes and scales, at its own row
    st, codes, scales, _, _ = oracle.dispatch_by_rank(idx, w, tr, xb, E, R, cap, fp8=True)
    assert st == oracle.OK
    for t in range(wl.tokens):
        blocks = [oracle.quantize_block(xb[t, b:b + 128]) for b in range(0, wl.hidden, 128)]
        want_c = np.concatenate([c for c, _ in blocks])
        want_s = np.array([sc for _, sc in blocks], np.float32)
        for r in range(R):
            if tr[t, r] >= 0:
                assert (codes[r, tr[t, r]] == want_c).all()
                assert (scales[r, tr[t, r]].view(np.uint32) == want_s.view(np.uint32)).all()


# ----------------------------------------------------------------------------- expert GEMM
def _gemm_case(H=256, N=256, mask=0.1):
    wl = W.WORKLOADS["tiny"].with_(hidden=H, fp8=True, tokens_per_rank=40, experts=4, topk=2, alignment=128)
    idx, w = W.gen_routing(wl)
    idx = W.mask_entries(wl, idx, mask)
    x = W.gen_x(wl)
    E, R, A = wl.experts, wl.ranks, wl.alignment
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A)
    cap = int(lay.rows_per_rank.max()) + 5
    lay = oracle.layout(idx.numpy(), w.numpy(), E, R, A, cap=cap)
    st, codes, scales, _ = oracle.dispatch_fp8(lay, idx.numpy(), w.numpy(), bits(x), E, R, A, cap, True, fill=0)
    assert st == oracle.OK
    return wl, idx.numpy(), lay, codes, scales


def _e4m3_table():
    return np.array([oracle.e4m3_to_double(c) for c in range(256)], np.float64)


def test_grouped_gemm_identity_weights_return_the_dequantised_rows():
    """W_e = I (code 0x38 = 1.0 on the diagonal, scale 1): every row of every expert comes back
    as its dequantised dispatch row, exactly (one nonzero product per output)."""
    wl, _, lay, codes, scales = _gemm_case()
    E, R, A, H = wl.experts, wl.ranks, wl.alignment, wl.hidden
    qw = np.zeros((E, H, H), np.uint8)
    qw[:, np.arange(H), np.arange(H)] = 0x38
    sw = np.ones((E, H // 128, H // 128), np.float32)
    st, out = oracle.grouped_gemm_f64(lay, codes, scales, qw, sw, E, R, A)
    assert st == 0
    deq = _e4m3_table()[codes] * np.repeat(scales.astype(np.float64), 128, axis=2)
    for r in range(R):
        n = int(lay.rows_per_rank[r])
        assert (out[r, :n] == deq[r, :n]).all()
        assert np.isnan(out[r, n:]).all()          # rows beyond the rank's rows untouched


def test_grouped_gemm_selects_each_rows_expert_and_block_scales():
    """All-ones weights with scale (e + 1) * (c + 1) * 2^b for column block c and K-block b:
    out[row, n] = (e + 1) * (n // 128 + 1) * sum_b 2^b * sx[row, b] * sum_{h in b} deq(x[row, h])
    for the row's expert e, read from the routing (row slot[t, j] of expert idx[t, j]); padding
    rows, zero-filled, give 0."""
    wl, idx, lay, codes, scales = _gemm_case(H=384, N=256)
    E, R, A, H, N = wl.experts, wl.ranks, wl.alignment, wl.hidden, 256
    KB = H // 128
    qw = np.full((E, N, H), 0x38, np.uint8)
    sw = np.empty((E, N // 128, KB), np.float32)
    for e in range(E):
        for c in range(N // 128):
            for b in range(KB):
                sw[e, c, b] = (e + 1) * (c + 1) * 2.0 ** b
    st, out = oracle.grouped_gemm_f64(lay, codes, scales, qw, sw, E, R, A)
    assert st == 0
    table = _e4m3_table()
    e_loc = E // R
    seen = np.zeros((R, codes.shape[1]), bool)
    T, k = idx.shape
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            if e < 0:
                continue
            r, row = e // e_loc, int(lay.slot[t, j])
            blocks = table[codes[r, row]].reshape(KB, 128).sum(axis=1)
            base = (e + 1) * sum(2.0 ** b * float(scales[r, row, b]) * blocks[b] for b in range(KB))
            ref = base * (np.arange(N) // 128 + 1)
            assert np.allclose(out[r, row], ref, rtol=1e-12, atol=0), (t, j)
            seen[r, row] = True
    for r in range(R):
        n = int(lay.rows_per_rank[r])
        assert (out[r, :n][~seen[r, :n]] == 0).all()   # padding rows


def test_grouped_gemm_random_weights_match_a_dense_blockwise_product():
    """Random E4M3 weights and block scales against the same sum written as dense float64 matrix
    products, one per 128-wide K-block: out[rows of e] = sum_b (sx[:, b] outer sw[e, n / 128, b])
    * (deq(x[:, b]) @ deq(w[e, :, b])^T).  Square H = N, so a transposed weight operand stays in
    bounds and fails here by value."""
    wl, _, lay, codes, scales = _gemm_case(H=256, N=256)
    E, R, A, H, N = wl.experts, wl.ranks, wl.alignment, wl.hidden, 256
    KB = H // 128
    rng = np.random.default_rng(17)
    qw = rng.integers(0, 256, (E, N, H), dtype=np.uint8)
    qw[(qw & 0x7F) == 0x7F] = 0x38                     # no NaN codes
    sw = rng.uniform(0.25, 4.0, (E, N // 128, KB)).astype(np.float32)
    st, out = oracle.grouped_gemm_f64(lay, codes, scales, qw, sw, E, R, A)
    assert st == 0
    table = _e4m3_table()
    e_loc = E // R
    checked = 0
    for e in range(E):
        r = e // e_loc
        end = int(lay.psum[e]); beg = end - align_up(int(lay.cnt[e]), A)
        if end == beg:
            continue
        X = table[codes[r, beg:end]]                   # [m, H]
        Wd = table[qw[e]]                              # [N, H]
        sx = scales[r, beg:end].astype(np.float64)     # [m, KB]
        swn = np.repeat(sw[e].astype(np.float64), 128, axis=0)   # [N, KB]
        ref = np.zeros((end - beg, N))
        mag = np.zeros((end - beg, N))
        for b in range(KB):
            cols = slice(128 * b, 128 * b + 128)
            f = np.outer(sx[:, b], swn[:, b])
            ref += f * (X[:, cols] @ Wd[:, cols].T)
            mag += np.abs(f) * (np.abs(X[:, cols]) @ np.abs(Wd[:, cols]).T)
        assert (np.abs(out[r, beg:end] - ref) <= 1e-12 * mag + 1e-300).all(), e
        checked += end - beg
    assert checked > 0


def test_grouped_gemm_is_linear_in_the_weight_scales():
    wl, _, lay, codes, scales = _gemm_case(H=256, N=128)
    E, R, A, H = wl.experts, wl.ranks, wl.alignment, wl.hidden
    rng = np.random.default_rng(3)
    qw = rng.integers(0, 256, (E, 128, H), dtype=np.uint8)
    qw[(qw & 0x7F) == 0x7F] = 0                        # no NaN codes
    sw = rng.uniform(0.5, 2.0, (E, 1, H // 128)).astype(np.float32)
    st, a = oracle.grouped_gemm_f64(lay, codes, scales, qw, sw, E, R, A)
    st2, b = oracle.grouped_gemm_f64(lay, codes, scales, qw, (sw * 2).astype(np.float32), E, R, A)
    assert st == st2 == 0
    ok = ~np.isnan(a)
    assert (b[ok] == 2 * a[ok]).all()                  # a power-of-two scale is exact
    # swapping two experts' weights swaps nothing else: experts keep their own rows
    qw2, sw2 = qw.copy(), sw.copy()
    qw2[[0, 1]], sw2[[0, 1]] = qw[[1, 0]], sw[[1, 0]]
    st3, c = oracle.grouped_gemm_f64(lay, codes, scales, qw2, sw2, E, R, A)
    assert st3 == 0
    e_loc = E // R
    for e in range(2, E):                              # rows of experts 2.. are unchanged
        r = e // e_loc
        end = int(lay.psum[e]); beg = end - align_up(int(lay.cnt[e]), A)
        assert (c[r, beg:end] == a[r, beg:end]).all()


def test_grouped_gemm_rejects_unaligned_shapes():
    wl, _, lay, codes, scales = _gemm_case()
    E, R, A = wl.experts, wl.ranks, wl.alignment
    st, _ = oracle.grouped_gemm_f64(lay, codes, scales, np.zeros((E, 100, 256), np.uint8),
                                    np.ones((E, 1, 2), np.float32), E, R, A)
    assert st == -1
