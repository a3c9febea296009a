"""The oracle's pins have teeth: each test plants one plausible mistake in a copy of the oracle
(on the CPU), rebuilds it, and requires the pin suite (tests/test_oracle.py) to fail against it."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

# (name, exact text in moe_oracle.c, replacement)
MUTATIONS = [
    ("psum exclusive instead of inclusive", "            run += align_up(cnt[e], A);\n            psum[e] = (int32_t)run;",
     "            psum[e] = (int32_t)run;\n            run += align_up(cnt[e], A);"),
    ("alignment dropped", "            run += align_up(cnt[e], A);", "            run += cnt[e];"),
    ("slot order reversed inside a segment", "            int32_t row = seg_start + fill[e]++;",
     "            int32_t row = seg_start + (cnt[e] - 1 - fill[e]++);"),
    ("row_src holds the pair index", "                row_src[(int64_t)r * cap + row] = (int32_t)t;",
     "                row_src[(int64_t)r * cap + row] = (int32_t)(t * k + j);"),
    ("masked entries counted", "            if (e == -1) continue;\n            if (e < -1 || e >= E)",
     "            if (e == -1) { cnt[0] += 1; continue; }\n            if (e < -1 || e >= E)"),
    ("E4M3 rounds half away from zero", "    double m = nearbyint(ldexp(a, 3 - e));", "    double m = round(ldexp(a, 3 - e));"),
    ("E4M3 truncates", "    double m = nearbyint(ldexp(a, 3 - e));", "    double m = floor(ldexp(a, 3 - e));"),
    ("E4M3 saturation threshold off", "    if (a >= 448.0) return (uint8_t)(sign | 0x7E);",
     "    if (a >= 480.0) return (uint8_t)(sign | 0x7F);"),
    ("FP8 scale inverted", "    float inv = 448.0f / a;", "    float inv = a / 448.0f;"),
    ("combine ignores the weights", "                acc = w ? fmaf(w[t * k + j], v, acc) : acc + v;",
     "                acc = acc + v;"),
    ("combine drops the bias", "            if (bias) acc = acc + oracle_bf16_to_float(bias[t * H + h]);\n            out[t * H + h] = oracle_float_to_bf16(acc);\n        }\n    return status;\n}\n\n/* The same sum",
     "            out[t * H + h] = oracle_float_to_bf16(acc);\n        }\n    return status;\n}\n\n/* The same sum"),
    ("bf16 NaN keeps its sign and payload", "return 0x7FC0;", "return (uint16_t)(u >> 16);"),
    ("bf16 rounding truncates", "    if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1;", "    (void)lo;"),
    ("expert GEMM uses the next expert's weights", "const uint8_t* wr = qw + ((int64_t)e * N + n) * H;",
     "const uint8_t* wr = qw + ((int64_t)((e + 1) % E) * N + n) * H;"),
    ("expert GEMM reads the first weight-scale block", "const float* ws = sw + ((int64_t)e * NB + n / 128) * KB;",
     "const float* ws = sw + ((int64_t)e * NB) * KB;"),
    ("expert GEMM drops the row scale", "acc += (double)xs[b] * (double)ws[b] * dot;",
     "acc += (double)ws[b] * dot;"),
    ("combine sums in descending j",
     "            float acc = 0.0f;\n            for (int j = 0; j < k; ++j) {\n                int32_t row = slot[t * k + j];\n"
     "                if (row < 0) continue;\n                if (row >= cap) { status = ORC_ERR_CAPACITY; continue; }",
     "            float acc = 0.0f;\n            for (int j = k - 1; j >= 0; --j) {\n                int32_t row = slot[t * k + j];\n"
     "                if (row < 0) continue;\n                if (row >= cap) { status = ORC_ERR_CAPACITY; continue; }"),
    ("combine adds the bias first",
     '            float acc = 0.0f;\n            for (int j = 0; j < k; ++j) {\n                int32_t row = slot[t * k + j];\n                if (row < 0) continue;\n                if (row >= cap) { status = ORC_ERR_CAPACITY; continue; }\n                int r = (int)(idx[t * k + j] / E_loc);\n                float v = oracle_bf16_to_float(y[((int64_t)r * cap + row) * H + h]);\n                acc = w ? fmaf(w[t * k + j], v, acc) : acc + v;\n            }\n            if (bias) acc = acc + oracle_bf16_to_float(bias[t * H + h]);',
     '            float acc = bias ? oracle_bf16_to_float(bias[t * H + h]) : 0.0f;\n            for (int j = 0; j < k; ++j) {\n                int32_t row = slot[t * k + j];\n                if (row < 0) continue;\n                if (row >= cap) { status = ORC_ERR_CAPACITY; continue; }\n                int r = (int)(idx[t * k + j] / E_loc);\n                float v = oracle_bf16_to_float(y[((int64_t)r * cap + row) * H + h]);\n                acc = w ? fmaf(w[t * k + j], v, acc) : acc + v;\n            }'),
    ("FP8 inv by a reciprocal multiply", "float inv = 448.0f / a;", "float inv = 448.0f * (1.0f / a);"),
    ("weighted combine rounds the product first", "acc = w ? fmaf(w[t * k + j], v, acc) : acc + v;",
     "acc = w ? w[t * k + j] * v + acc : acc + v;"),
    ("by-rank combine in ascending rank order",
     "            for (int j = 0; j < k; ++j) {\n                int64_t e = idx[t * k + j];\n                if (e < 0 || e >= E) continue;\n"
     "                int r = (int)(e / E_loc);\n                if (seen[r]) continue;\n                seen[r] = 1;",
     "            for (int r = 0; r < R; ++r) {\n                int hit = 0;\n"
     "                for (int j = 0; j < k; ++j) { int64_t e = idx[t * k + j]; if (e >= 0 && e < E && e / E_loc == r) hit = 1; }\n"
     "                if (!hit) continue;\n                if (seen[r]) continue;\n                seen[r] = 1;"),
    ("by-rank combine adds the bias first",
     '            float acc = 0.0f;\n            for (int j = 0; j < k; ++j) {\n                int64_t e = idx[t * k + j];\n                if (e < 0 || e >= E) continue;\n                int r = (int)(e / E_loc);\n                if (seen[r]) continue;\n                seen[r] = 1;\n                int32_t row = token_row[t * R + r];\n                if (row >= cap) { status = ORC_ERR_CAPACITY; continue; }\n                acc = acc + oracle_bf16_to_float(y[((int64_t)r * cap + row) * H + h]);\n            }\n            if (bias) acc = acc + oracle_bf16_to_float(bias[t * H + h]);',
     '            float acc = bias ? oracle_bf16_to_float(bias[t * H + h]) : 0.0f;\n            for (int j = 0; j < k; ++j) {\n                int64_t e = idx[t * k + j];\n                if (e < 0 || e >= E) continue;\n                int r = (int)(e / E_loc);\n                if (seen[r]) continue;\n                seen[r] = 1;\n                int32_t row = token_row[t * R + r];\n                if (row >= cap) { status = ORC_ERR_CAPACITY; continue; }\n                acc = acc + oracle_bf16_to_float(y[((int64_t)r * cap + row) * H + h]);\n            }'),
    ("row weights without topk_weights read 1", "row_w[(int64_t)r * cap + row] = w ? w[t * k + j] : 0.0f;",
     "row_w[(int64_t)r * cap + row] = w ? w[t * k + j] : 1.0f;"),
    ("by-rank FP8 scales written at the row index", "                memcpy(recv_scales + g * nb, scales, sizeof(float) * (size_t)nb);",
     "                memcpy(recv_scales + g, scales, sizeof(float) * (size_t)nb);"),
    ("expert GEMM reads the weights transposed",
     "dot += oracle_e4m3_to_double(x[h]) * oracle_e4m3_to_double(wr[h]);",
     "dot += oracle_e4m3_to_double(x[h]) * oracle_e4m3_to_double(qw[((int64_t)e * H + h) * N + n]);"),
    ("expert GEMM drops the last K-block", "for (int64_t b = 0; b < KB; ++b) {\n                    double dot",
     "for (int64_t b = 0; b + 1 < KB; ++b) {\n                    double dot"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(name, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not found exactly once: {name}"
    mutated = tmp_path / "moe_oracle_mutated.c"
    mutated.write_text(src.replace(old, new))
    sys.path.insert(0, ROOT)
    from oracle import build as oracle_build
    lib = oracle_build.build_from(str(mutated), str(tmp_path / "libmutated.so"))
    env = dict(os.environ, MOE_ORACLE_LIB=lib)
    # A planted mistake can make the oracle write past its buffers (e.g. padding rows beyond the
    # smaller row count), which may crash or hang the pin run: either way the pins did not pass.
    try:
        r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle.py"), "-x", "-q",
                            "-p", "no:cacheprovider", "-k", "not brute_force"], cwd=ROOT, env=env,
                           capture_output=True, text=True, timeout=120)
    except subprocess.TimeoutExpired:
        return
    assert r.returncode != 0, f"no pin caught the planted mistake '{name}'"
