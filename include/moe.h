/*
 * moe.h -- C ABI of the single-B200 MoE token round trip: layout -> dispatch -> combine.
 *
 * One MoE layer's token round trip with expert-parallel ranks emulated as logical partitions
 * of one GPU's memory.  Sources (page title, section):
 *   "Why MoE gets stuck on communication -- one expert-parallel round trip, end to end"
 *     (locsic.com), section 1: a long-lived buffer with a uniform per-rank capacity; dispatch
 *     with expert_alignment / do_expand / do_zero_padding / do_cpu_sync; a handle that records
 *     the grouping and counts of one dispatch and is reused by combine; combine sums the
 *     already-weighted expert outputs and adds the shared expert's output as a bias.
 *   "From DeepEP to Mega MoE" (backyes.github.io), sections 2.2-2.5: per-expert counts with
 *     block-local atomics, an inclusive prefix sum psum_num_recv_tokens_per_expert, placement
 *     of every routed row inside its expert's range, element-wise top-k reduction in combine.
 *   "deepep-expert-parallel-dispatch-combine" (phantomic12.github.io), "Arithmetic
 *     intensity": with do_cpu_sync off, outputs are sized to capacity and consumers read the
 *     device-side psum.
 *   "DeepEP expert-parallel communication" (blog.hotdry.top), "Key techniques": num_sms caps
 *     the SMs the data-movement kernels occupy; FP8 dispatch with BF16 combine.
 *
 * Conventions for every call
 *   - T tokens, k = topk, E experts, R logical ranks, E_loc = E / R, A = expert_alignment,
 *     H = hidden, cap = receive capacity in rows per logical rank (uniform over ranks).
 *   - Expert e lives on logical rank e / E_loc.  topk_idx == -1 marks a masked entry.
 *   - Receive buffers are [R, cap, ...] row-major; rank r's rows start at row 0 of block r.
 *     Inside rank r, expert e owns rows [psum[e] - align_up(cnt[e], A), psum[e]); its routed
 *     rows come first, in ascending (token, j) order, then its padding rows.
 *   - Pointers are DEVICE pointers unless the argument says host.  Row pointers (x, recv_x,
 *     recv_scales, y, bias, out) must be 16-byte aligned.  bf16 data is passed as void*.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *     stream-ordered and returns without waiting for the GPU, except where stated.
 *   - Return value: MOE_OK or a negative MOE_ERR_*.  Argument errors are reported before
 *     anything is launched.  Conditions only the GPU can see (an expert id outside [-1, E),
 *     a rank needing more than cap rows) set a status word in the handle; the kernels skip
 *     every write they would make out of range.  They are returned by moe_layout when
 *     do_cpu_sync is set and otherwise by moe_handle_status.
 *   - The library never falls back to the CPU and never allocates memory for the caller's
 *     tensors; the caller owns x, topk_idx, topk_weights, the receive buffers, y, bias, out.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 1

enum moe_status_code {
  MOE_NOT_READY = 1,        /* moe_event_query only: the recorded work has not completed yet */
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1, /* bad size, flag, null or misaligned pointer */
  MOE_ERR_BAD_EXPERT = -2,  /* a topk_idx entry outside [-1, E) */
  MOE_ERR_CAPACITY = -3,    /* some logical rank needs more rows than the given capacity */
  MOE_ERR_CUDA = -4,        /* a CUDA runtime call failed */
  MOE_ERR_OOM = -5,         /* the handle's device memory could not be allocated */
  MOE_ERR_UNSUPPORTED = -6, /* a valid request outside what this build implements */
  MOE_ERR_SCRATCH_LIMIT = -7, /* moe_layout_static_scratch: the problem needs more scratch than
                                 MOE_STATIC_SCRATCH_BYTES */
  MOE_ERR_TIMEOUT = -8        /* a kernel's bounded wait on one of its own shared-memory barriers
                                 expired (2 s); reported by moe_handle_status; internal error */
};

enum moe_dtype { MOE_DTYPE_BF16 = 0, MOE_DTYPE_FP8_E4M3 = 1 };

/* moe_params_t.flags: also build the non-expanded (one row per token and rank) layout that
 * moe_dispatch_by_rank / moe_combine_by_rank / moe_dispatch(do_expand = 0) need (R <= 64). */
#define MOE_LAYOUT_BY_RANK 1

/* moe_params_t.flags, with do_cpu_sync = 1 only: defer the epilogue of the count sync
 * ("Why MoE gets stuck on communication", section 2, issue / drain / epilogue: defer_epilogue
 * moves the host's wait for the receive counts to the wait on the pending work).  moe_layout
 * then enqueues the copy of the counts into pinned memory owned by the handle and returns at
 * once, without blocking the host; moe_handle_wait blocks for them and reports the device
 * conditions.  The handle's device arrays are usable by later stream-ordered calls at once. */
#define MOE_DEFER_EPILOGUE 2

/* Problem description for moe_layout.  All fields are read once; the handle keeps a copy. */
typedef struct moe_params {
  int64_t num_tokens;         /* T >= 0 */
  int32_t num_logical_ranks;  /* R >= 1, E % R == 0 */
  int32_t num_experts;        /* E, 1 <= E <= 4096 */
  int32_t topk;               /* k, 1 <= k <= 32 */
  int32_t hidden;             /* H >= 8, H % 8 == 0 (BF16) and H % 128 == 0 for FP8 */
  int32_t expert_alignment;   /* A >= 1; T*k + E*A < 2^31 */
  int32_t num_sms;            /* SMs the layout kernels may occupy; 0 = all */
  int32_t do_cpu_sync;        /* 1: moe_layout waits for the counts and copies them to host */
  int32_t flags;              /* 0 or MOE_LAYOUT_BY_RANK | MOE_DEFER_EPILOGUE */
  int64_t recv_capacity_rows; /* cap per rank for the handle's row maps; 0 only with
                                 do_cpu_sync=1 (the rows are then sized from the counts) */
} moe_params_t;

typedef struct moe_handle moe_handle_t; /* opaque; owns its device arrays */

/*
 * Rows one logical rank may need when every rank sends it at most max_tokens_per_rank tokens:
 * R * max_tokens_per_rank * min(k, E_loc) + E_loc * (A - 1).  Host only; no GPU work.
 * Returns -1 on invalid parameters.  (The buffer size hint of the round-trip page, section 1.)
 */
int64_t moe_recv_capacity_hint(const moe_params_t* params, int64_t max_tokens_per_rank);

/*
 * Layout ("From DeepEP to Mega MoE" 2.2 and 2.4; "Why MoE gets stuck on communication" 1).
 *   topk_idx      int64 [T, k], device.
 *   topk_weights  fp32 [T, k], device, nullable (row weights then read 0).
 *   out_handle    receives a new handle on MOE_OK (NULL otherwise).  Its device arrays are
 *                 allocated stream-ordered on `stream` and freed by moe_handle_free.
 *   host_rows_per_rank  int32 [R], host, nullable; filled when do_cpu_sync = 1.
 * Fills, in the handle: cnt[E], psum[E] (aligned inclusive prefix per rank), rows_per_rank[R],
 * tokens_per_rank[R], token_in_rank[T, R] (uint8), slot[T, k] (row inside its rank, -1 if
 * masked), row_src[R, row_cap] (source token, -1 for padding rows), row_w[R, row_cap].
 * With do_cpu_sync = 1 the call blocks until the counts reach the host and returns
 * MOE_ERR_BAD_EXPERT / MOE_ERR_CAPACITY directly (no handle is returned then).  The counts are
 * handed over as soon as they are final, through mapped pinned memory, so the call can return
 * while the slot assignment still runs; it is stream-ordered before every later use of the
 * handle.  With MOE_DEFER_EPILOGUE as well it does not block: host_rows_per_rank is not
 * written, the handle is returned, and moe_handle_wait later delivers the counts and those two
 * conditions.
 */
int moe_layout(const moe_params_t* params, const int64_t* topk_idx, const float* topk_weights,
               void* stream, moe_handle_t** out_handle, int32_t* host_rows_per_rank);

/*
 * Dispatch ("From DeepEP to Mega MoE" 2.2 dispatch warps and 2.4 copy epilogue; "Why MoE gets
 * stuck on communication" 1: do_expand, do_zero_padding; FP8 per "DeepEP expert-parallel
 * communication", key techniques).
 *   x             bf16 [T, H], device.
 *   out_dtype     MOE_DTYPE_BF16: recv_x is bf16 [R, cap, H], a copy of x[t] per routed row.
 *                 MOE_DTYPE_FP8_E4M3: recv_x is E4M3 [R, cap, H]; for each 1x128 block,
 *                 a = max(amax, 1e-4), code = E4M3_rne_satfinite(x * (448 / a)) and
 *                 recv_scales[r, row, b] = a / 448 (fp32 [R, cap, H/128]).
 *   recv_weights  fp32 [R, cap], nullable: the pair's topk weight (0 on padding rows).
 *   cap           rows per logical rank in recv_x / recv_scales / recv_weights.
 *   do_expand     1: one row per (token, expert), the layout above.  0: one row per (token,
 *                 rank), see moe_dispatch_by_rank (recv_weights is then [R, cap, k]).
 *   do_zero_padding  1: padding rows are written as zero bytes (codes, scales and bf16).
 *   num_sms       SMs the kernel may occupy (0 = all).
 * Rows beyond rows_per_rank[r] are never written.
 */
int moe_dispatch(const moe_handle_t* handle, const void* x, int out_dtype, void* recv_x,
                 float* recv_scales, float* recv_weights, int64_t cap, int do_expand,
                 int do_zero_padding, int num_sms, void* stream);

/*
 * Layout and expanded dispatch in one call ("From DeepEP to Mega MoE" 2.2: the dispatch kernel
 * runs its notify warps, which count the routing and build psum, beside the dispatch warps that
 * move the tokens; "deepep-expert-parallel-dispatch-combine", arithmetic intensity:
 * do_cpu_sync = False sizes the outputs to capacity and consumers read the device-side psum).
 * Computes exactly moe_layout followed by moe_dispatch(do_expand = 1) with
 * cap = params->recv_capacity_rows and num_sms = params->num_sms, and returns the handle as
 * moe_layout does.  params->do_cpu_sync must be 0 and params->flags 0 (MOE_ERR_INVALID_ARG
 * otherwise); the other arguments are those of moe_layout and moe_dispatch.  A bad expert id or
 * a capacity overflow is reported by moe_handle_status.  Small batches (chunks of at most 8
 * tokens, one per SM of the budget, T * k < 65536, and shared memory for E experts) run as one
 * kernel in which no CTA waits for another: each CTA's layout warps count the whole routing table
 * and assign its own chunk's rows while its dispatch warps load and quantise that chunk's tokens.
 * Other batches run the layout's launches and then the dispatch kernel.
 */
int moe_layout_dispatch(const moe_params_t* params, const int64_t* topk_idx, const float* topk_weights,
                        const void* x, int out_dtype, void* recv_x, float* recv_scales, float* recv_weights,
                        int do_zero_padding, void* stream, moe_handle_t** out_handle);

/*
 * Non-expanded dispatch ("Why MoE gets stuck on communication" 1: without do_expand a destination
 * rank receives each token once; "Chapter 2: repository map" 2.1: token -> rank membership).
 * Rank r receives one row per token that has at least one expert on r, in ascending token order
 * (row = moe_handle_token_rows(handle)[t, r]); cap is the capacity in TOKENS per rank
 * (tokens_per_rank[r] rows are used).  No alignment padding exists in this layout.
 *   recv_x / recv_scales  as for moe_dispatch (BF16 copy or FP8 codes + 1x128 scales).
 *   recv_topk_idx      int32 [R, cap, k], nullable (then topk_idx may be NULL): the local expert
 *                      index (e - r*E_loc) of the token's j-th choice when it lives on r, else -1.
 *   recv_topk_weights  fp32 [R, cap, k], nullable: the matching topk weight, else 0.
 *   topk_idx           int64 [T, k]: the routing given to moe_layout (needed for recv_topk_idx).
 * Needs a handle laid out with MOE_LAYOUT_BY_RANK and R <= 64 (MOE_ERR_UNSUPPORTED otherwise).
 * moe_dispatch with do_expand = 0 calls this with
 * recv_topk_idx = NULL and recv_topk_weights = its recv_weights, read as [R, cap, k].
 */
int moe_dispatch_by_rank(const moe_handle_t* handle, const void* x, const int64_t* topk_idx, int out_dtype,
                         void* recv_x, float* recv_scales, int32_t* recv_topk_idx, float* recv_topk_weights,
                         int64_t cap, int num_sms, void* stream);

/*
 * Non-expanded combine: y is bf16 [R, cap, H] with, for every (token, rank), the rank's
 * already-weighted partial sum over its experts; out[t] = bf16(fp32 sum over the token's ranks in
 * the order in which they first appear in topk_idx[t, :], then + bias[t]).  Needs R <= 64.
 */
int moe_combine_by_rank(const moe_handle_t* handle, const void* y, const void* bias, void* out, int64_t cap,
                        int num_sms, void* stream);

/*
 * Combine ("From DeepEP to Mega MoE" 2.3 and 2.5: element-wise top-k reduction; "Why MoE gets
 * stuck on communication" 1: already-weighted rows, shared-expert output as bias).
 *   y             bf16 [R, cap, H], device: the expert outputs in the dispatch layout.
 *   topk_weights  fp32 [T, k], nullable.  NULL: y rows are already weighted and are summed.
 *   bias          bf16 [T, H], nullable.
 *   out           bf16 [T, H].
 * For each element: acc = 0 (fp32); for j = 0..k-1 with a valid slot, acc = fma(w, y, acc)
 * (or acc + y); then acc + bias; out = bf16 round-to-nearest-even(acc).
 */
int moe_combine(const moe_handle_t* handle, const void* y, const float* topk_weights,
                const void* bias, void* out, int64_t cap, int num_sms, void* stream);

/*
 * Backward of combine ("Why MoE gets stuck on communication" 1 and 2: the handle of a dispatch is
 * reused by the backward pass).  For out[t] = sum_j w[t,j] * y[row(t,j)] (+ bias[t]):
 *   grad_out      bf16 [T, H], device.
 *   topk_weights  fp32 [T, k], nullable: the weights the combine applied (NULL: pre-weighted rows).
 *   grad_y        bf16 [R, cap, H]: grad_y[row(t,j)] = bf16(w[t,j] * grad_out[t]) (one fp32 multiply)
 *                 or grad_out[t] when topk_weights is NULL; padding rows are zeroed when
 *                 do_zero_padding, other rows beyond rows_per_rank are not written.
 *   y             bf16 [R, cap, H], nullable: the combine's input, needed for grad_weights.
 *   grad_weights  fp32 [T, k], nullable: grad_w[t,j] = <grad_out[t], y[row(t,j)]> (0 if masked),
 *                 fp32 FMA per lane over columns in ascending order, then a fixed 32-lane tree.
 * The gradient of the bias is grad_out itself.  The backward of dispatch is moe_combine with
 * topk_weights = NULL applied to the gradient of the received rows.
 */
int moe_combine_backward(const moe_handle_t* handle, const void* grad_out, const float* topk_weights,
                         void* grad_y, int64_t cap, int do_zero_padding, const void* y,
                         float* grad_weights, int num_sms, void* stream);

/*
 * The deferred epilogue of a MOE_DEFER_EPILOGUE layout ("Why MoE gets stuck on communication",
 * section 2: the host waits for the receive counts at wait time, not at issue).  Blocks the host
 * until the layout's count copy has landed, then returns MOE_ERR_BAD_EXPERT / MOE_ERR_CAPACITY
 * as moe_layout would have, or MOE_OK with host_rows_per_rank (int32 [R], host, nullable) filled
 * with the rows each logical rank receives.  The result is kept: later calls return it again
 * without waiting.  A handle laid out with do_cpu_sync = 1 and no deferral returns MOE_OK (its
 * counts are already on the host); one laid out with do_cpu_sync = 0 returns
 * MOE_ERR_INVALID_ARG (its counts never come to the host: use the device arrays).
 */
int moe_handle_wait(moe_handle_t* handle, int32_t* host_rows_per_rank);

/*
 * Events: the pending-object half of "Why MoE gets stuck on communication", section 1 (dispatch
 * and combine return at once; independent work such as the shared expert runs; wait() orders the
 * consumer after them) and section 2 (wait() makes the current stream wait on the recorded event;
 * that orders only that stream, not the host).  To run the round trip on a communication stream
 * asynchronously to a compute stream: record an event on the compute stream, make the
 * communication stream wait for it, issue moe_layout / moe_dispatch / moe_combine there, record
 * an event after them, and make the compute stream wait for that event before it reads the
 * results.  The handle is freed stream-ordered on its layout stream (moe_handle_free).
 */
typedef struct moe_event moe_event_t; /* opaque */

/* Records a new event at the current end of `stream`; *out_event receives it. */
int moe_event_record(void* stream, moe_event_t** out_event);
/* Makes work enqueued on `stream` after this call wait for the event (device side; returns at once). */
int moe_event_wait(const moe_event_t* event, void* stream);
/* Blocks the host until the event's work has completed. */
int moe_event_synchronize(const moe_event_t* event);
/* MOE_OK when the event's work has completed, MOE_NOT_READY while it has not. */
int moe_event_query(const moe_event_t* event);
/* Destroys the event (pending waits on it stay valid).  NULL is accepted. */
int moe_event_free(moe_event_t* event);

/*
 * The first expert GEMM on the FP8 dispatch layout, on the tensor cores ("From DeepEP to Mega MoE"
 * 3.2 Linear1 and 4.5: dispatch -> expert buffer -> GEMM L1; "Why MoE gets stuck on
 * communication" 1: expert_alignment is the grouped GEMM's row alignment).  For every logical
 * rank r, every expert e of r and every row of e's range [psum[e] - align_up(cnt[e], A), psum[e]):
 *   out[r, row, n] = bf16( sum over K-blocks b of recv_scales[r, row, b] * w_scales[e, n/128, b]
 *                          * sum over h in block b of E4M3(recv_x[r, row, h]) * E4M3(w[e, n, h]) )
 * Each 128-wide K-block is summed on the tensor cores (fp32), then scaled and added in fp32 in
 * ascending b; one rounding to bf16 (nearest even) at the end.
 *   recv_x       E4M3 [R, cap, H] and recv_scales fp32 [R, cap, H/128]: an FP8 moe_dispatch's output
 *                for this handle (do_expand = 1).
 *   w            E4M3 [E, N, H]: row n of expert e is output column n (K contiguous).
 *   w_scales     fp32 [E, N/128, H/128]: one scale per 128 x 128 block of w.
 *   out          bf16 [R, cap, N]: the rows of every expert range are written (padding rows too:
 *                zero when the dispatch zeroed them); other rows are not touched.
 * Needs H % 128 == 0, N % 128 == 0 and expert_alignment % 128 == 0, and R * cap and E * N below
 * 2^31 (MOE_ERR_UNSUPPORTED otherwise); recv_x, w and out 16-byte aligned.  Returns
 * MOE_ERR_CAPACITY when the host counts exceed cap; without host counts, rows beyond cap are not
 * computed (the layout's status reports the overflow).  Stream-ordered after the dispatch.
 */
int moe_expert_gemm_fp8(const moe_handle_t* handle, const void* recv_x, const float* recv_scales, const void* w,
                        const float* w_scales, void* out, int64_t N, int64_t cap, int num_sms, void* stream);

/* Waits for `stream`, then returns the handle's device status (MOE_OK, MOE_ERR_BAD_EXPERT,
 * MOE_ERR_CAPACITY or MOE_ERR_TIMEOUT) as left by every layout / dispatch / combine ordered
 * before it. */
int moe_handle_status(const moe_handle_t* handle, void* stream);

/* Device arrays owned by the handle (valid until moe_handle_free). */
const int32_t* moe_handle_counts(const moe_handle_t* handle);          /* [E] */
const int32_t* moe_handle_psum(const moe_handle_t* handle);            /* [E] */
const int32_t* moe_handle_rows_per_rank(const moe_handle_t* handle);   /* [R] */
const int32_t* moe_handle_tokens_per_rank(const moe_handle_t* handle); /* [R] */
const uint8_t* moe_handle_token_in_rank(const moe_handle_t* handle);   /* [T, R] */
const int32_t* moe_handle_slots(const moe_handle_t* handle);           /* [T, k] */
const int32_t* moe_handle_row_src(const moe_handle_t* handle);         /* [R, row_cap] */
const float* moe_handle_row_weights(const moe_handle_t* handle);       /* [R, row_cap] */
const int32_t* moe_handle_token_rows(const moe_handle_t* handle);      /* [T, R]; NULL without
                                                                          MOE_LAYOUT_BY_RANK */
int64_t moe_handle_row_capacity(const moe_handle_t* handle);           /* row_cap */

/* Releases the handle.  Its device memory is freed stream-ordered on the layout stream, so
 * every dispatch / combine that uses the handle must be ordered before this call on that
 * stream (or already complete).  A deferred count copy still in flight is waited for first
 * (host).  NULL is accepted. */
int moe_handle_free(moe_handle_t* handle);

/* Static description of a status code. */
const char* moe_status_string(int status);

/*
 * moe_layout_static_scratch -- the layout of moe_layout without any memory allocation.
 * The pages have no counterpart: this entry point exists for callers that cannot call
 * cudaMalloc -- code whose device memory is owned by another allocator (a framework caching
 * allocator that has reserved the GPU, a runtime that hands out fixed arenas) and serving loops
 * that forbid allocation calls on their hot path, where a driver allocation may block.
 *
 * Computes exactly what moe_layout computes (params->flags must be 0: the by-rank layout is not
 * built here), into caller-owned device buffers:
 *   counts[E], psum[E], rows_per_rank[R], tokens_per_rank[R], token_in_rank[T, R] (uint8),
 *   slots[T, k], row_src[R, cap] and row_weights[R, cap] with cap = recv_capacity_rows (>= 1).
 * Its temporaries (status word, padding prefix, per-chunk counts, per-pair rank and weight)
 * live in one file-scope device array of MOE_STATIC_SCRATCH_BYTES, which every GPU that loads
 * the library holds until the process exits.  It needs
 *   256 + r(4(E+1)) + r(4*C*E) + 2*r(4*T*k) bytes, C = ceil(T/256), r = round up to 256;
 * larger problems return MOE_ERR_SCRATCH_LIMIT before any GPU work.
 *   device_status  int32, device: receives the device status flags of this call (bit 0: an
 *                  expert id outside [-1, E); bit 1: a rank needs more than cap rows); cleared by
 *                  the call.  Required when do_cpu_sync = 0 (MOE_ERR_INVALID_ARG if NULL), since
 *                  nothing else would report those conditions; may be NULL when do_cpu_sync = 1,
 *                  where the call returns them.
 *   host_rows_per_rank  int32 [R], host, nullable: filled when do_cpu_sync = 1.
 * With do_cpu_sync = 1 the call waits for the counts and returns MOE_ERR_BAD_EXPERT /
 * MOE_ERR_CAPACITY directly; with 0 it returns after launching.
 * All calls share the scratch array and it keeps the last call's contents: calls whose GPU
 * work overlaps on the same device (two streams, two host threads) race.  The first call on a
 * device looks up the array's device address with that device current and caches it per
 * device; make that first call before any stream capture.  The cache belongs to the runtime's
 * primary context: calls after cudaDeviceReset, or under a context created through the driver
 * API, are unsupported.  Kernels: one CTA when T*k <= 8192 and E <= 1024, else count, scan and
 * assign over 256-token chunks; the results equal moe_layout's.  Calls no cudaMalloc, cudaFree
 * or allocating library routine.
 */
#define MOE_STATIC_SCRATCH_BYTES (4u << 20)
int moe_layout_static_scratch(const moe_params_t* params, const int64_t* topk_idx,
                              const float* topk_weights, int32_t* counts, int32_t* psum,
                              int32_t* rows_per_rank, int32_t* tokens_per_rank,
                              uint8_t* token_in_rank, int32_t* slots, int32_t* row_src,
                              float* row_weights, int32_t* device_status,
                              int32_t* host_rows_per_rank, void* stream);

/* Number of kernels launched by this library in this process (all calls, all threads). */
int64_t moe_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
