"""Host-side logic of the benchmark (no GPU): the algorithmic byte model, the sizing of the
reference arm's sample, and the clock summary read from nvidia-smi samples."""
import datetime

import numpy as np

import bench
import oracle
import workloads as W


def test_byte_model_matches_an_independent_estimate_for_deepseek_v3():
    """The bytes a DeepSeek-V3 prefill step must move, from the model and the oracle's own counts,
    against an estimate made row by row: dispatch = x 469.8 MB + codes 1879.0 MB + scales
    58.7 MB + about 120 MB of zeroed padding + ids 2.1 MB; combine = rows 3758.1 MB + out
    469.8 MB + ids 2.1 MB."""
    wl = W.WORKLOADS["deepseek"]
    idx, w = W.gen_routing(wl)
    lay = oracle.layout(idx.numpy(), w.numpy(), wl.experts, wl.ranks, wl.alignment)
    assert lay.status == oracle.OK
    valid = int(lay.cnt.sum())
    pad = int(lay.rows_per_rank.sum()) - valid
    assert valid == wl.tokens * wl.topk  # no masked entries in this workload
    assert 0 <= pad < wl.experts * wl.alignment
    b = bench.algorithmic_bytes(wl, valid, pad)
    assert abs(b["dispatch"] - (469.8 + 1879.0 + 58.7 + 120 + 2.1) * 1e6) < 0.01 * 2.53e9
    assert abs(b["combine"] - (3758.1 + 469.8 + 2.1) * 1e6) < 1e6
    # a padding row costs what a routed row costs, and only with zero padding
    no_pad = bench.algorithmic_bytes(wl.with_(zero_padding=False), valid, pad)
    assert b["dispatch"] - no_pad["dispatch"] == pad * (wl.hidden + 4 * wl.hidden // 128)
    assert no_pad["combine"] == b["combine"]


def test_byte_model_counts_bias_and_weights_once():
    wl = W.WORKLOADS["decode"]
    T, H, k = wl.tokens, wl.hidden, wl.topk
    plain = bench.algorithmic_bytes(wl.with_(bias=False), T * k, 0)
    biased = bench.algorithmic_bytes(wl, T * k, 0)
    weighted = bench.algorithmic_bytes(wl, T * k, 0, weighted=True)
    assert biased["combine"] - plain["combine"] == T * H * 2
    assert weighted["combine"] - biased["combine"] == T * k * 4


def test_reference_sample_shrinks_with_the_run_length():
    wl = W.WORKLOADS["deepseek"]
    assert bench.reference_tokens(wl, 2, 3) == 4096
    long_run = bench.reference_tokens(wl, 200, 10)
    assert 16 * wl.ranks <= long_run < 4096 and long_run % wl.ranks == 0
    assert bench.reference_tokens(wl, 100000, 10) == 16 * wl.ranks


def _sample_line(ts: float, mhz: float, reasons=("Not Active",) * 4) -> str:
    stamp = datetime.datetime.fromtimestamp(ts).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return ", ".join([stamp, f"{mhz:.0f}", "1965", "700.0", "0x0", *reasons])


def test_clock_summary_keeps_the_timed_window_and_its_reasons():
    c = bench.ClockSampler(0)
    t0 = 1_700_000_000.0
    c.t0, c.t1 = t0 + 1.0, t0 + 2.0
    lines = [_sample_line(t0 + 0.2, 1200, ("Not Active", "Not Active", "Active", "Not Active"))]  # before
    lines += [_sample_line(t0 + 1.0 + 0.1 * i, 1900 + i) for i in range(11)]                     # inside
    lines += [_sample_line(t0 + 1.5, 1950, ("Not Active", "Not Active", "Not Active", "Active"))]
    lines += [_sample_line(t0 + 3.0, 800)]                                                         # after
    c.out = "\n".join(lines) + "\nnot a sample line\n"
    s = c.summary()
    assert s["samples"] == 12
    assert s["sm_max_mhz"] == 1965.0
    assert s["sm_mhz"] == float(np.median([1900 + i for i in range(11)] + [1950]))
    assert s["reasons"] == ["sw_power_cap"]  # the thermal slowdown lies outside the window


def test_clock_summary_without_samples():
    c = bench.ClockSampler(0)
    c.out = ""
    s = c.summary()
    assert s["samples"] == 0 and s["reasons"] == ["unavailable"]


def test_clock_summary_falls_back_to_the_nearest_samples():
    c = bench.ClockSampler(0)
    t0 = 1_700_000_000.0
    lines = [_sample_line(t0 + 0.1 * i, 1000 + i) for i in range(10)]          # a gap after t0 + 0.9
    lines += [_sample_line(t0 + 5.0, 1900), _sample_line(t0 + 5.1, 1901, ("Active",) + ("Not Active",) * 3)]
    c.out = "\n".join(lines)
    s = c.summary(t0 + 2.0, t0 + 2.1)                   # nothing inside: t0 + 0.9 and t0 + 0.8 are nearest
    assert s["samples"] == 2 and s["window"].startswith("nearest")
    assert s["sm_mhz"] == float(np.median([1009, 1008]))
    assert s["reasons"] == []
    s = c.summary(t0 + 4.0, t0 + 4.1)                   # t0 + 5.0 and t0 + 5.1, one with hw_slowdown
    assert s["sm_mhz"] == float(np.median([1900, 1901])) and s["reasons"] == ["hw_slowdown"]


def test_by_rank_and_backward_byte_models():
    """The widened paths' byte models at the DeepSeek-V3 shape, from a count of the (token, rank)
    rows made here from the routing: by rank, one FP8 row (7168 codes + 56 scales) with 8 ids and
    8 weights per (token, rank); backward, one bf16 grad row per routed or padding row."""
    wl = W.WORKLOADS["deepseek"]
    idx, w = W.gen_routing(wl)
    ranks = idx.numpy() // (wl.experts // wl.ranks)
    token_rank_rows = sum(len(set(r.tolist())) for r in ranks)      # distinct ranks per token
    st, tr, rows = oracle.layout_by_rank(idx.numpy(), wl.experts, wl.ranks)
    assert st == oracle.OK and int(rows.sum()) == token_rank_rows
    assert token_rank_rows <= 4 * wl.tokens                          # group-limited: at most 4 groups
    T, H = wl.tokens, wl.hidden
    b = bench.by_rank_bytes(wl, token_rank_rows)
    assert b["dispatch_by_rank"] == (T * H * 2 + token_rank_rows * (7168 + 224 + 64)
                                     + T * 8 * 12 + T * 8 * 4)
    assert b["combine_by_rank"] == token_rank_rows * H * 2 + T * H * 2 + T * 8 * 4
    lay = oracle.layout(idx.numpy(), w.numpy(), wl.experts, wl.ranks, wl.alignment)
    valid = int(lay.cnt.sum())
    pad = int(lay.rows_per_rank.sum()) - valid
    bw = bench.backward_bytes(wl, valid, pad)
    assert bw["dispatch_cached"] == bench.algorithmic_bytes(wl, valid, pad)["dispatch"]
    assert bw["combine_backward"] == T * H * 2 + (valid + pad) * H * 2 + T * 8 * 8
    assert bench.backward_bytes(wl.with_(zero_padding=False), valid, pad)["combine_backward"] == \
        T * H * 2 + valid * H * 2 + T * 8 * 8
