/*
 * moe_oracle.c -- CPU oracle for the MoE token round trip (layout, dispatch, combine).
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, single-threaded statement of what the
 * round trip computes, written so that a reader can check it against the source pages by eye.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may load it.  It shares
 * no code, header, table or helper with the CUDA library; the product path never calls it.
 *
 * Sources (page title, then section):
 *   [P1] "From DeepEP to Mega MoE: three-way verification of the MoE runtime's evolution"
 *        (backyes.github.io), section 2.2 "Dispatch Kernel", 2.3 "Combine Kernel",
 *        2.4 "Dispatch Copy Epilogue", 2.5 "Combine Reduce Epilogue".
 *   [P2] "DeepEP expert-parallel communication" (blog.hotdry.top), "Performance benchmark"
 *        and "Key techniques" (FP8 dispatch, num_sms).
 *   [P3] "Why MoE gets stuck on communication -- one expert-parallel round trip, end to end"
 *        (locsic.com), section 1 (round-trip timeline, dispatch flags, handle) and
 *        section 3 "Padding" (the 1/1/126 worked example).
 *   [P4] "deepep-expert-parallel-dispatch-combine" (phantomic12.github.io), "Arithmetic
 *        intensity" (do_cpu_sync=False exposes psum_num_recv_tokens_per_expert).
 *   [P5] "Chapter 2: repository map and module responsibilities" (bowenzhou.top),
 *        section 2.1, the layout.cu row (rank count, expert count, membership).
 *   [P1] again for the expert GEMM: section 3.2 (Linear1, the first expert GEMM, fed by the
 *        dispatched tokens and their scale factors) and section 4.5 (the separated dataflow:
 *        dispatch -> expert buffer in HBM -> GEMM L1).
 *
 * Conventions shared with the library's C ABI (argument meaning only, no code):
 *   T tokens, k top-k, E experts, R logical ranks, E_loc = E/R, A = expert_alignment.
 *   Expert e lives on logical rank e / E_loc (contiguous blocks).
 *   topk_idx[t*k + j] == -1 is a masked entry; any other value outside [0, E) is an error.
 *   bf16 values travel as their 16-bit patterns (uint16_t).
 *
 * Readings of the pages that the code below takes (listed again in the design notes):
 *   - psum_num_recv_tokens_per_expert is an INCLUSIVE sum of counts rounded up to A,
 *     restarting at each logical rank (each receiving rank's buffer begins at row 0).
 *   - inside one expert's segment rows are ordered by ascending (token, j); the pages place
 *     rows with an atomic counter, whose order is not defined.
 *   - FP8 block quantisation recipe: amax over 1x128, a = max(amax, 1e-4), inv = 448/a,
 *     scale = a/448, code = E4M3(x*inv) round-to-nearest-even with saturation to +-448.
 *   - combine accumulates in fp32 in ascending j (fma when weights are given), adds the
 *     bias last and rounds once to bf16.
 *
 * Compile with -ffp-contract=off: every float operation below is one IEEE operation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_INVALID_ARG -1
#define ORC_ERR_BAD_EXPERT -2
#define ORC_ERR_CAPACITY -3

static int64_t align_up(int64_t n, int64_t a) { return ((n + a - 1) / a) * a; }

/* ---------------------------------------------------------------------------------------
 * bf16 <-> fp32 (IEEE binary32 with the low 16 mantissa bits dropped).
 * ------------------------------------------------------------------------------------- */
float oracle_bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a binary32 value to the nearest bf16, ties to even.  NaN becomes the canonical
 * quiet NaN 0x7FC0.  Implemented from the definition: split the value at the 16th bit and
 * compare the discarded half against one half-ulp, in exact integer arithmetic. */
uint16_t oracle_float_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0) return 0x7FC0;
    uint32_t hi = u >> 16;
    uint32_t lo = u & 0xFFFFu;
    if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1; /* carries into the exponent */
    return (uint16_t)hi;
}

/* ---------------------------------------------------------------------------------------
 * OCP FP8 E4M3 ("E4M3FN"): 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities;
 * S.1111.111 is NaN; largest finite 0x7E = 448; smallest normal 2^-6; smallest subnormal 2^-9.
 * ------------------------------------------------------------------------------------- */
double oracle_e4m3_to_double(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);              /* subnormal: m * 2^-9 */
    else v = ldexp(1.0 + m / 8.0, e - 7);               /* normal */
    return s ? -v : v;
}

/* Encode a binary32 value as E4M3 with round-to-nearest-even and saturation to the
 * largest finite magnitude (448).  The sign is kept, also for zero.  NaN -> 0x7F|sign. */
uint8_t oracle_e4m3_from_float(float f) {
    uint8_t sign = signbit(f) ? 0x80 : 0x00;
    if (isnan(f)) return (uint8_t)(sign | 0x7F);
    double a = fabs((double)f);                          /* exact */
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);       /* saturate (also +-inf) */
    if (a < ldexp(1.0, -6)) {                            /* subnormal range, quantum 2^-9 */
        double m = nearbyint(ldexp(a, 9));               /* ties to even: default mode */
        /* m == 8 is the smallest normal 2^-6, whose code is 0x08 == m as well */
        return (uint8_t)(sign | (uint8_t)m);
    }
    int e2;
    frexp(a, &e2);                                       /* a = f * 2^e2, f in [0.5, 1) */
    int e = e2 - 1;                                      /* a in [2^e, 2^(e+1)), e in [-6, 8] */
    double m = nearbyint(ldexp(a, 3 - e));               /* significand in eighths, [8, 16] */
    if (m == 16.0) { m = 8.0; e += 1; }
    if (e > 8 || (e == 8 && m > 14.0)) return (uint8_t)(sign | 0x7E);
    return (uint8_t)(sign | (uint8_t)((e + 7) << 3) | (uint8_t)((int)m - 8));
}

/* ---------------------------------------------------------------------------------------
 * Layout  [P1 s2.2 notify warps: per-expert counts, then do_psum(..., warp_inclusive_sum)]
 *         [P3 s1: expert_alignment matches the grouped GEMM's token alignment]
 *         [P5 s2.1: layout.cu turns top-k into rank counts, expert counts, membership]
 *         [P1 s2.4: each routed row is placed at a position inside its expert's range]
 *
 * Outputs
 *   cnt[E]              rows routed to expert e (masked entries not counted)
 *   psum[E]             inclusive sum over the experts of e's rank, up to and including e,
 *                       of align_up(cnt, A)
 *   rows_per_rank[R]    psum of the rank's last expert
 *   tokens_per_rank[R]  tokens with at least one expert on rank r
 *   token_in_rank[T*R]  membership flag (nullable)
 *   slot[T*k]           row of (t, j) inside its rank's receive buffer, -1 when masked
 *   row_src[R*cap]      source token of every row below rows_per_rank[r], -1 for padding
 *   row_w[R*cap]        topk_weights of that pair (0 for padding; 0 for all if w == NULL)
 * Returns ORC_ERR_BAD_EXPERT for an id outside [-1, E), ORC_ERR_CAPACITY when some rank
 * needs more than cap rows (rows at or beyond cap are then not written).
 * ------------------------------------------------------------------------------------- */
int oracle_layout(int64_t T, int k, int E, int R, int A, const int64_t* idx, const float* w,
                  int64_t cap, int32_t* cnt, int32_t* psum, int32_t* rows_per_rank,
                  int32_t* tokens_per_rank, uint8_t* token_in_rank, int32_t* slot,
                  int32_t* row_src, float* row_w) {
    if (T < 0 || k < 1 || E < 1 || R < 1 || A < 1 || E % R != 0 || cap < 0) return ORC_ERR_INVALID_ARG;
    const int E_loc = E / R;
    int status = ORC_OK;

    /* 1. per-expert counts */
    for (int e = 0; e < E; ++e) cnt[e] = 0;
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int64_t e = idx[t * k + j];
            if (e == -1) continue;
            if (e < -1 || e >= E) { status = ORC_ERR_BAD_EXPERT; continue; }
            cnt[e] += 1;
        }

    /* 2. aligned inclusive prefix sum, restarting at every rank */
    for (int r = 0; r < R; ++r) {
        int64_t run = 0;
        for (int e = r * E_loc; e < (r + 1) * E_loc; ++e) {
            run += align_up(cnt[e], A);
            psum[e] = (int32_t)run;
        }
        rows_per_rank[r] = psum[(r + 1) * E_loc - 1];
        if (rows_per_rank[r] > cap && status == ORC_OK) status = ORC_ERR_CAPACITY;
    }

    /* 3. token -> rank membership */
    for (int r = 0; r < R; ++r) tokens_per_rank[r] = 0;
    for (int64_t t = 0; t < T; ++t)
        for (int r = 0; r < R; ++r) {
            int in = 0;
            for (int j = 0; j < k; ++j) {
                int64_t e = idx[t * k + j];
                if (e >= 0 && e < E && e / E_loc == r) in = 1;
            }
            if (token_in_rank) token_in_rank[t * R + r] = (uint8_t)in;
            tokens_per_rank[r] += in;
        }

    /* 4. slots: walk pairs in (t, j) order, each expert filling its segment from the start */
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int64_t e = idx[t * k + j];
            if (e < 0 || e >= E) { slot[t * k + j] = -1; continue; }
            int32_t seg_start = psum[e] - (int32_t)align_up(cnt[e], A);
            int32_t row = seg_start + fill[e]++;
            slot[t * k + j] = row;
            int r = (int)(e / E_loc);
            if (row < cap) {
                row_src[(int64_t)r * cap + row] = (int32_t)t;
                row_w[(int64_t)r * cap + row] = w ? w[t * k + j] : 0.0f;
            }
        }
    free(fill);

    /* 5. padding rows of every segment: [psum - pad, psum) */
    for (int e = 0; e < E; ++e) {
        int r = e / E_loc;
        int32_t pad = (int32_t)align_up(cnt[e], A) - cnt[e];
        for (int32_t row = psum[e] - pad; row < psum[e]; ++row)
            if (row < cap) {
                row_src[(int64_t)r * cap + row] = -1;
                row_w[(int64_t)r * cap + row] = 0.0f;
            }
    }
    return status;
}

/* ---------------------------------------------------------------------------------------
 * A second, deliberately different statement of the slot assignment, used only to check
 * oracle_layout: list every valid (expert, token, j) triple, sort them, and give each one the
 * index it has inside its expert's group, offset by the aligned sizes of the rank's earlier
 * experts.  Writes cnt, psum and slot.
 * ------------------------------------------------------------------------------------- */
typedef struct { int64_t e, t; int j; } orc_triple;

static int orc_triple_cmp(const void* pa, const void* pb) {
    const orc_triple* a = (const orc_triple*)pa;
    const orc_triple* b = (const orc_triple*)pb;
    if (a->e != b->e) return a->e < b->e ? -1 : 1;
    if (a->t != b->t) return a->t < b->t ? -1 : 1;
    return (a->j > b->j) - (a->j < b->j);
}

int oracle_layout_by_sort(int64_t T, int k, int E, int R, int A, const int64_t* idx,
                          int32_t* cnt, int32_t* psum, int32_t* slot) {
    if (T < 0 || k < 1 || E < 1 || R < 1 || A < 1 || E % R != 0) return ORC_ERR_INVALID_ARG;
    const int E_loc = E / R;
    orc_triple* v = (orc_triple*)malloc(sizeof(orc_triple) * (size_t)(T * k + 1));
    int64_t n = 0;
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            slot[t * k + j] = -1;
            int64_t e = idx[t * k + j];
            if (e >= 0 && e < E) { v[n].e = e; v[n].t = t; v[n].j = j; ++n; }
        }
    qsort(v, (size_t)n, sizeof(orc_triple), orc_triple_cmp);
    /* group boundaries give the counts */
    for (int e = 0; e < E; ++e) cnt[e] = 0;
    for (int64_t i = 0; i < n; ++i) cnt[v[i].e]++;
    /* start row of each expert's group inside its rank */
    int32_t* start = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) {
        int32_t s = 0;
        for (int e2 = (e / E_loc) * E_loc; e2 < e; ++e2) s += (int32_t)align_up(cnt[e2], A);
        start[e] = s;
        psum[e] = s + (int32_t)align_up(cnt[e], A);
    }
    int64_t group_begin = 0;
    for (int64_t i = 0; i < n; ++i) {
        if (i > 0 && v[i].e != v[i - 1].e) group_begin = i;
        slot[v[i].t * k + v[i].j] = start[v[i].e] + (int32_t)(i - group_begin);
    }
    free(start);
    free(v);
    return ORC_OK;
}

/* Rows [psum[e] - pad(e), psum[e]) of expert e's rank hold no routed token. */
static void for_each_padding_row(int E, int R, int A, const int32_t* cnt, const int32_t* psum,
                                 void (*fn)(void*, int, int32_t), void* ctx) {
    const int E_loc = E / R;
    for (int e = 0; e < E; ++e) {
        int32_t pad = (int32_t)align_up(cnt[e], A) - cnt[e];
        for (int32_t row = psum[e] - pad; row < psum[e]; ++row) fn(ctx, e / E_loc, row);
    }
}

/* ---------------------------------------------------------------------------------------
 * Dispatch, BF16   [P1 s2.2 dispatch warps load a token once and store it to each
 *                   destination; P1 s2.4 places it in its expert's range; P3 s1 do_expand
 *                   gives one row per (token, expert), do_zero_padding fills the padding]
 * recv_x is [R, cap, H] of bf16 patterns; recv_w is [R, cap] (nullable).
 * ------------------------------------------------------------------------------------- */
typedef struct { uint8_t* base; int64_t cap, row_bytes; float* recv_w; int64_t cap_w; } pad_ctx;

static void zero_row(void* p, int r, int32_t row) {
    pad_ctx* c = (pad_ctx*)p;
    if (row >= c->cap) return;
    memset(c->base + ((int64_t)r * c->cap + row) * c->row_bytes, 0, (size_t)c->row_bytes);
    if (c->recv_w) c->recv_w[(int64_t)r * c->cap + row] = 0.0f;
}

static void zero_weight_only(void* p, int r, int32_t row) {
    pad_ctx* c = (pad_ctx*)p;
    if (row < c->cap) c->recv_w[(int64_t)r * c->cap + row] = 0.0f;
}

int oracle_dispatch_bf16(int64_t T, int k, int E, int R, int A, int64_t H, int64_t cap,
                         const int64_t* idx, const float* w, const int32_t* cnt, const int32_t* psum,
                         const int32_t* slot, const uint16_t* x, uint16_t* recv_x, float* recv_w,
                         int do_zero_padding) {
    const int E_loc = E / R;
    int status = ORC_OK;
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int32_t row = slot[t * k + j];
            if (row < 0) continue;
            int r = (int)(idx[t * k + j] / E_loc);
            if (row >= cap) { status = ORC_ERR_CAPACITY; continue; }
            memcpy(recv_x + ((int64_t)r * cap + row) * H, x + t * H, (size_t)H * 2);
            if (recv_w) recv_w[(int64_t)r * cap + row] = w ? w[t * k + j] : 0.0f;
        }
    pad_ctx c = { (uint8_t*)recv_x, cap, H * 2, recv_w, cap };
    if (do_zero_padding) for_each_padding_row(E, R, A, cnt, psum, zero_row, &c);
    else if (recv_w) for_each_padding_row(E, R, A, cnt, psum, zero_weight_only, &c);
    return status;
}

/* ---------------------------------------------------------------------------------------
 * FP8 block quantisation of one 1x128 block  [P2 "Key techniques": FP8 dispatch; P4: FP8
 * halves the bytes].  The recipe (amax floor, scale form, rounding) is the reading stated in
 * the file header; every operation is one binary32 operation.
 * ------------------------------------------------------------------------------------- */
void oracle_quantize_block(const uint16_t* xb, int n, uint8_t* codes, float* scale) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float v = fabsf(oracle_bf16_to_float(xb[i]));
        if (v > amax) amax = v;
    }
    float a = amax > 1e-4f ? amax : 1e-4f;
    float inv = 448.0f / a;
    *scale = a / 448.0f;
    for (int i = 0; i < n; ++i) codes[i] = oracle_e4m3_from_float(oracle_bf16_to_float(xb[i]) * inv);
}

/* Dispatch, FP8: recv_x is [R, cap, H] E4M3 codes, recv_scales is [R, cap, H/128] fp32. */
int oracle_dispatch_fp8(int64_t T, int k, int E, int R, int A, int64_t H, int64_t cap,
                        const int64_t* idx, const float* w, const int32_t* cnt, const int32_t* psum,
                        const int32_t* slot, const uint16_t* x, uint8_t* recv_x, float* recv_scales,
                        float* recv_w, int do_zero_padding) {
    if (H % 128 != 0) return ORC_ERR_INVALID_ARG;
    const int E_loc = E / R;
    const int64_t nb = H / 128;
    int status = ORC_OK;
    uint8_t* codes = (uint8_t*)malloc((size_t)H);
    float* scales = (float*)malloc(sizeof(float) * (size_t)nb);
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t b = 0; b < nb; ++b) oracle_quantize_block(x + t * H + b * 128, 128, codes + b * 128, scales + b);
        for (int j = 0; j < k; ++j) {
            int32_t row = slot[t * k + j];
            if (row < 0) continue;
            int r = (int)(idx[t * k + j] / E_loc);
            if (row >= cap) { status = ORC_ERR_CAPACITY; continue; }
            memcpy(recv_x + ((int64_t)r * cap + row) * H, codes, (size_t)H);
            memcpy(recv_scales + ((int64_t)r * cap + row) * nb, scales, sizeof(float) * (size_t)nb);
            if (recv_w) recv_w[(int64_t)r * cap + row] = w ? w[t * k + j] : 0.0f;
        }
    }
    free(codes);
    free(scales);
    if (do_zero_padding) {
        pad_ctx c1 = { recv_x, cap, H, recv_w, cap };
        for_each_padding_row(E, R, A, cnt, psum, zero_row, &c1);
        pad_ctx c2 = { (uint8_t*)recv_scales, cap, nb * 4, NULL, cap };
        for_each_padding_row(E, R, A, cnt, psum, zero_row, &c2);
    } else if (recv_w) {
        pad_ctx c = { recv_x, cap, H, recv_w, cap };
        for_each_padding_row(E, R, A, cnt, psum, zero_weight_only, &c);
    }
    return status;
}

/* ---------------------------------------------------------------------------------------
 * Combine  [P1 s2.3 / s2.5: per token, the top-k expert outputs are summed element by
 *           element (reduced += value); P3 s1: the summed rows are already weighted and the
 *           shared expert's output joins as the bias]
 * y is [R, cap, H] bf16; w [T*k] fp32 (nullable: rows already weighted); bias [T, H] bf16
 * (nullable); out [T, H] bf16.  For each element: acc = 0; for j ascending with a valid slot:
 * acc = fma(w, y, acc) or acc + y; then acc + bias; one rounding to bf16.
 * ------------------------------------------------------------------------------------- */
int oracle_combine(int64_t T, int k, int E, int R, int64_t H, int64_t cap, const int64_t* idx,
                   const int32_t* slot, const uint16_t* y, const float* w, const uint16_t* bias,
                   uint16_t* out) {
    const int E_loc = E / R;
    int status = ORC_OK;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int32_t row = slot[t * k + j];
                if (row < 0) continue;
                if (row >= cap) { status = ORC_ERR_CAPACITY; continue; }
                int r = (int)(idx[t * k + j] / E_loc);
                float v = oracle_bf16_to_float(y[((int64_t)r * cap + row) * H + h]);
                acc = w ? fmaf(w[t * k + j], v, acc) : acc + v;
            }
            if (bias) acc = acc + oracle_bf16_to_float(bias[t * H + h]);
            out[t * H + h] = oracle_float_to_bf16(acc);
        }
    return status;
}

/* The same sum in binary64 (every product w*y is exact there; the few additions round at
 * 2^-53, far below the bf16 tolerance), for bounding the fp32 accumulation order against the
 * mathematics.  out64 is [T, H]. */
void oracle_combine_f64(int64_t T, int k, int E, int R, int64_t H, int64_t cap,
                          const int64_t* idx, const int32_t* slot, const uint16_t* y,
                          const float* w, const uint16_t* bias, double* out64) {
    const int E_loc = E / R;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                int32_t row = slot[t * k + j];
                if (row < 0 || row >= cap) continue;
                int r = (int)(idx[t * k + j] / E_loc);
                double v = (double)oracle_bf16_to_float(y[((int64_t)r * cap + row) * H + h]);
                acc += w ? (double)w[t * k + j] * v : v;
            }
            if (bias) acc += (double)oracle_bf16_to_float(bias[t * H + h]);
            out64[t * H + h] = acc;
        }
}

/* ---------------------------------------------------------------------------------------
 * Backward of combine  ["Why MoE gets stuck on communication" s1 and s2: the handle records one
 * dispatch's grouping and counts and training reuses it in the backward pass]
 * For out[t] = sum_j w[t,j] * y[slot(t,j)] (+ bias[t]):
 *   grad_y[slot(t,j)] = bf16(w[t,j] * grad_out[t])   (one fp32 multiply, then bf16 RNE);
 *                     = grad_out[t]                   when the rows were pre-weighted (w NULL);
 *   padding rows of grad_y are zero when do_zero_padding, other rows untouched.
 * grad_y is [R, cap, H] bf16.
 * ------------------------------------------------------------------------------------- */
int oracle_combine_backward(int64_t T, int k, int E, int R, int A, int64_t H, int64_t cap,
                            const int64_t* idx, const int32_t* cnt, const int32_t* psum,
                            const int32_t* slot, const uint16_t* grad_out, const float* w,
                            uint16_t* grad_y, int do_zero_padding) {
    const int E_loc = E / R;
    int status = ORC_OK;
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int32_t row = slot[t * k + j];
            if (row < 0) continue;
            if (row >= cap) { status = ORC_ERR_CAPACITY; continue; }
            int r = (int)(idx[t * k + j] / E_loc);
            uint16_t* dst = grad_y + ((int64_t)r * cap + row) * H;
            for (int64_t h = 0; h < H; ++h) {
                uint16_t g = grad_out[t * H + h];
                dst[h] = w ? oracle_float_to_bf16(w[t * k + j] * oracle_bf16_to_float(g)) : g;
            }
        }
    if (do_zero_padding) {
        pad_ctx c = { (uint8_t*)grad_y, cap, H * 2, NULL, cap };
        for_each_padding_row(E, R, A, cnt, psum, zero_row, &c);
    }
    return status;
}

/* Gradient of the combine with respect to the pair weights: grad_w[t,j] = sum_h grad_out[t,h] *
 * y[slot(t,j), h] in binary64 (0 for masked pairs). */
void oracle_grad_weights_f64(int64_t T, int k, int E, int R, int64_t H, int64_t cap,
                             const int64_t* idx, const int32_t* slot, const uint16_t* grad_out,
                             const uint16_t* y, double* grad_w) {
    const int E_loc = E / R;
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int32_t row = slot[t * k + j];
            double acc = 0.0;
            if (row >= 0 && row < cap) {
                int r = (int)(idx[t * k + j] / E_loc);
                const uint16_t* yr = y + ((int64_t)r * cap + row) * H;
                for (int64_t h = 0; h < H; ++h)
                    acc += (double)oracle_bf16_to_float(grad_out[t * H + h]) * (double)oracle_bf16_to_float(yr[h]);
            }
            grad_w[t * k + j] = acc;
        }
}

/* ---------------------------------------------------------------------------------------
 * Non-expanded (by rank) round trip  ["Why MoE gets stuck on communication" s1: do_expand
 * selects the expert-side expanded layout; without it every destination rank receives a token
 * once; "Chapter 2: repository map" s2.1: layout.cu produces the token -> rank membership]
 *
 * token_row[t*R + r] = row of token t in rank r's buffer (tokens of rank r in ascending token
 * order), -1 when none of t's experts lives on r.  rows_per_rank[r] = number of such tokens.
 * ------------------------------------------------------------------------------------- */
int oracle_layout_by_rank(int64_t T, int k, int E, int R, const int64_t* idx, int32_t* token_row,
                          int32_t* rows_per_rank) {
    if (T < 0 || k < 1 || E < 1 || R < 1 || E % R != 0) return ORC_ERR_INVALID_ARG;
    const int E_loc = E / R;
    int status = ORC_OK;
    for (int r = 0; r < R; ++r) rows_per_rank[r] = 0;
    for (int64_t t = 0; t < T; ++t)
        for (int r = 0; r < R; ++r) {
            int member = 0;
            for (int j = 0; j < k; ++j) {
                int64_t e = idx[t * k + j];
                if (e < -1 || e >= E) status = ORC_ERR_BAD_EXPERT;
                else if (e >= 0 && e / E_loc == r) member = 1;
            }
            token_row[t * R + r] = member ? rows_per_rank[r]++ : -1;
        }
    return status;
}

/* By-rank dispatch: recv[r, token_row[t,r]] = x[t] (BF16 copy, or FP8 codes + 1x128 scales with
 * the block recipe of oracle_quantize_block).  recv_topk_idx[r, row, j] = e_j - r*E_loc when
 * expert e_j lives on r, else -1; recv_topk_w[r, row, j] = w[t,j] or 0.  Either is nullable.
 * fp8 == 0: recv is uint16 [R, cap, H]; fp8 == 1: recv is uint8 [R, cap, H] and scales
 * [R, cap, H/128]. */
int oracle_dispatch_by_rank(int64_t T, int k, int E, int R, int64_t H, int64_t cap, const int64_t* idx,
                            const float* w, const int32_t* token_row, const uint16_t* x, int fp8, void* recv,
                            float* recv_scales, int32_t* recv_topk_idx, float* recv_topk_w) {
    const int E_loc = E / R;
    const int64_t nb = H / 128;
    int status = ORC_OK;
    uint8_t* codes = (uint8_t*)malloc((size_t)(H > 0 ? H : 1));
    float* scales = (float*)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    for (int64_t t = 0; t < T; ++t) {
        if (fp8)
            for (int64_t b = 0; b < nb; ++b) oracle_quantize_block(x + t * H + b * 128, 128, codes + b * 128, scales + b);
        for (int r = 0; r < R; ++r) {
            int32_t row = token_row[t * R + r];
            if (row < 0) continue;
            if (row >= cap) { status = ORC_ERR_CAPACITY; continue; }
            int64_t g = (int64_t)r * cap + row;
            if (fp8) {
                memcpy((uint8_t*)recv + g * H, codes, (size_t)H);
                memcpy(recv_scales + g * nb, scales, sizeof(float) * (size_t)nb);
            } else {
                memcpy((uint16_t*)recv + g * H, x + t * H, (size_t)H * 2);
            }
            for (int j = 0; j < k; ++j) {
                int64_t e = idx[t * k + j];
                int on_r = e >= 0 && e < E && e / E_loc == r;
                if (recv_topk_idx) recv_topk_idx[g * k + j] = on_r ? (int32_t)(e - (int64_t)r * E_loc) : -1;
                if (recv_topk_w) recv_topk_w[g * k + j] = on_r && w ? w[t * k + j] : 0.0f;
            }
        }
    }
    free(codes);
    free(scales);
    return status;
}

/* By-rank combine: y holds, per (token, rank), the rank's already-weighted partial sum.  For
 * each element: acc = 0 (fp32); for every rank of the token, in the order in which the ranks
 * first appear in topk_idx[t, :], acc += y[r, token_row[t,r]]; then acc + bias; bf16 RNE. */
int oracle_combine_by_rank(int64_t T, int k, int E, int R, int64_t H, int64_t cap, const int64_t* idx,
                           const int32_t* token_row, const uint16_t* y, const uint16_t* bias, uint16_t* out) {
    const int E_loc = E / R;
    int status = ORC_OK;
    int* seen = (int*)malloc(sizeof(int) * (size_t)R);
    for (int64_t t = 0; t < T; ++t)
        for (int64_t h = 0; h < H; ++h) {
            for (int r = 0; r < R; ++r) seen[r] = 0;
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int64_t e = idx[t * k + j];
                if (e < 0 || e >= E) continue;
                int r = (int)(e / E_loc);
                if (seen[r]) continue;
                seen[r] = 1;
                int32_t row = token_row[t * R + r];
                if (row >= cap) { status = ORC_ERR_CAPACITY; continue; }
                acc = acc + oracle_bf16_to_float(y[((int64_t)r * cap + row) * H + h]);
            }
            if (bias) acc = acc + oracle_bf16_to_float(bias[t * H + h]);
            out[t * H + h] = oracle_float_to_bf16(acc);
        }
    free(seen);
    return status;
}

/*
 * Expert GEMM over the dispatch layout ([P1] 3.2 Linear1 and 4.5 GEMM L1 on the expert buffer;
 * [P3] 1: expert_alignment is the grouped GEMM's row alignment).  Inputs are the FP8 dispatch
 * output (codes qx [R, cap, H] and 1x128 scales sx [R, cap, H/128]) and per-expert FP8 weights
 * (codes qw [E, N, H], row n = output column n, and 128x128 block scales sw [E, N/128, H/128]).
 * For every logical rank r, every expert e of r and every row of e's range
 * [psum[e] - align_up(cnt[e], A), psum[e]) (routed rows and padding rows alike), and n < N:
 *   out[r, row, n] = sum over K-blocks b of ( sx[r, row, b] * sw[e, n / 128, b]
 *                    * sum over h in block b of E4M3(qx[r, row, h]) * E4M3(qw[e, n, h]) )
 * in binary64, blocks and columns in ascending order.  Rows outside every range are not
 * written.  Needs H % 128 == 0 and N % 128 == 0; returns -1 otherwise.
 */
int oracle_grouped_gemm_f64(int E, int R, int A, int64_t cap, int64_t H, int64_t N, const int32_t* cnt,
                            const int32_t* psum, const uint8_t* qx, const float* sx, const uint8_t* qw,
                            const float* sw, double* out) {
    if (H % 128 != 0 || N % 128 != 0 || E % R != 0) return -1;
    const int E_loc = E / R;
    const int64_t KB = H / 128, NB = N / 128;
    for (int e = 0; e < E; ++e) {
        const int r = e / E_loc;
        const int64_t end = psum[e], begin = end - align_up(cnt[e], A);
        for (int64_t row = begin; row < end; ++row) {
            const uint8_t* x = qx + ((int64_t)r * cap + row) * H;
            const float* xs = sx + ((int64_t)r * cap + row) * KB;
            for (int64_t n = 0; n < N; ++n) {
                const uint8_t* wr = qw + ((int64_t)e * N + n) * H;
                const float* ws = sw + ((int64_t)e * NB + n / 128) * KB;
                double acc = 0.0;
                for (int64_t b = 0; b < KB; ++b) {
                    double dot = 0.0;
                    for (int64_t h = b * 128; h < b * 128 + 128; ++h)
                        dot += oracle_e4m3_to_double(x[h]) * oracle_e4m3_to_double(wr[h]);
                    acc += (double)xs[b] * (double)ws[b] * dot;
                }
                out[((int64_t)r * cap + row) * N + n] = acc;
            }
        }
    }
    return 0;
}

