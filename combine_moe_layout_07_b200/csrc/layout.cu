// layout.cu -- routing -> counts, aligned prefix sums and the token->slot handle.
//
// Follows "From DeepEP to Mega MoE" (backyes.github.io) 2.2 (notify warps: per-expert counts
// with block-local atomics, then an inclusive prefix sum psum_num_recv_tokens_per_expert) and
// 2.4 (every routed row gets a position inside its expert's range), with expert_alignment and
// the per-rank receive buffers of "Why MoE gets stuck on communication" (locsic.com) section 1,
// and the rank count / expert count / membership outputs of layout.cu in "Chapter 2:
// repository map" (bowenzhou.top) 2.1.
//
// The pages place rows with atomicAdd on the psum counter, whose order is undefined; here the
// placement is a stable counting sort so the handle is deterministic:
//   count  : per chunk of 256 tokens, a shared-memory histogram (atomicAdd_block) of expert ids
//            and of token->rank membership;
//   scan   : a CTA per 32 experts scans the chunk counts of its experts over chunks (chunk
//            offsets); the last CTA to finish scans align_up(cnt, A), restarted at every rank;
//   assign : per chunk, each warp takes a contiguous run of (t, j) pairs; per-warp histograms
//            are scanned across warps, and inside a warp __match_any_sync + popc give each pair
//            its rank among equal experts -- so rows keep ascending (t, j) order.
// Batches of at most one chunk per SM take the one-launch layout instead (k_layout_fused).  The
// device code it shares with the one-launch layout + dispatch kernel lives in layout_body.cuh.
#include "layout_body.cuh"

namespace moe {

// Phase 1 of the slot assignment: histogram h[E] of the warp's pairs [wp0, wp1) (h zeroed).
__device__ __forceinline__ void warp_histogram(const LayoutLaunch& L, int64_t wp0, int64_t wp1, int32_t* h) {
  const int lane = threadIdx.x & 31;
  for (int64_t base = wp0; base < wp1; base += 32 * kAssignBatch) {
    int32_t ev[kAssignBatch];
#pragma unroll
    for (int r = 0; r < kAssignBatch; ++r) {
      const int64_t p = base + r * 32 + lane;
      ev[r] = p < wp1 ? max(expert_of(__ldg(L.idx + p), L.E), -1) : -1;
    }
#pragma unroll
    for (int r = 0; r < kAssignBatch; ++r) {
      if (base + r * 32 >= wp1) break;  // warp-uniform: the rest of the batch is empty
      histogram_round(ev[r], h);
    }
  }
}

// Phase 3: walk the warp's pairs in (t, j) order; h[e] holds the warp's next row of expert e.
// Writes slot, pair rank, pair weight and the row maps.  Returns true on a row >= row_cap.
__device__ __forceinline__ bool warp_assign(const LayoutLaunch& L, int64_t wp0, int64_t wp1, int32_t* h) {
  const int lane = threadIdx.x & 31;
  bool overflow = false;
  for (int64_t base = wp0; base < wp1; base += 32 * kAssignBatch) {
    int32_t ev[kAssignBatch];
    float wv[kAssignBatch];
#pragma unroll
    for (int r = 0; r < kAssignBatch; ++r) {
      const int64_t p = base + r * 32 + lane;
      ev[r] = p < wp1 ? max(expert_of(__ldg(L.idx + p), L.E), -1) : -1;
      wv[r] = (p < wp1 && L.w) ? __ldg(L.w + p) : 0.0f;
    }
#pragma unroll
    for (int r = 0; r < kAssignBatch; ++r) {
      if (base + r * 32 >= wp1) break;  // warp-uniform: the rest of the batch is empty
      const int64_t p = base + r * 32 + lane;
      overflow |= assign_round(L, p, p < wp1, ev[r], wv[r], h);
    }
  }
  return overflow;
}

// Non-expanded (by-rank) layout for the block-sized group of tokens [t0, t0 + blockDim):
// token_row[t, r] = base_r[r] + (member tokens of rank r before t in the group), -1 when t has
// no expert on r; base_r[r] (shared) advances by the group's count.  tslot[t, j] = the token's
// row on rank(e_j) for the first j of the token on that rank, else -1.  R <= 64 (rank bitmasks);
// wcnt is shared scratch of [blockDim / 32][kMaxByRankRanks].  Called by the whole block.
__device__ __forceinline__ void token_rows_group(const LayoutLaunch& L, int64_t t0, int64_t t_end, int32_t* base_r,
                                                 int32_t* wcnt) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, W = blockDim.x >> 5;
  const int64_t t = t0 + tid;
  const bool valid = t < t_end;
  const uint32_t lt = lanemask_lt();
  uint64_t mask = 0;
  if (valid)
    for (int j = 0; j < L.k; ++j) {
      const int32_t e = expert_of(__ldg(L.idx + t * L.k + j), L.E);
      if (e >= 0) mask |= 1ull << ((uint32_t)e / (uint32_t)L.E_loc);
    }
  for (int r = 0; r < L.R; ++r) {
    const uint32_t b = __ballot_sync(0xffffffffu, (mask >> r) & 1);
    if (lane == 0) wcnt[warp * kMaxByRankRanks + r] = __popc(b);
  }
  __syncthreads();
  for (int r = tid; r < L.R; r += blockDim.x) {
    int32_t run = base_r[r];
    for (int w = 0; w < W; ++w) {
      const int32_t v = wcnt[w * kMaxByRankRanks + r];
      wcnt[w * kMaxByRankRanks + r] = run;
      run += v;
    }
    base_r[r] = run;
  }
  __syncthreads();
  for (int r = 0; r < L.R; ++r) {
    const uint32_t b = __ballot_sync(0xffffffffu, (mask >> r) & 1);
    if (valid) L.d.token_row[t * L.R + r] = ((mask >> r) & 1) ? wcnt[warp * kMaxByRankRanks + r] + __popc(b & lt) : -1;
  }
  if (valid) {
    uint64_t seen = 0;
    for (int j = 0; j < L.k; ++j) {
      const int32_t e = expert_of(__ldg(L.idx + t * L.k + j), L.E);
      int32_t v = -1;
      if (e >= 0) {
        const int r = (int)((uint32_t)e / (uint32_t)L.E_loc);
        if (!((seen >> r) & 1)) {
          seen |= 1ull << r;
          v = L.d.token_row[t * L.R + r];  // written above by this thread
        }
      }
      L.d.tslot[t * L.k + j] = v;
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------------------------ count
// A thread per token: its k ids are loaded together, counted into the chunk's shared-memory
// histogram (atomicAdd_block), and its rank membership is written and counted.
__global__ void __launch_bounds__(kLayoutThreads) k_layout_count(LayoutLaunch L) {
  extern __shared__ int32_t sm[];
  int32_t* hist = sm;       // [E]
  int32_t* tok = sm + L.E;  // [R]
  const int tid = threadIdx.x;
  bool ok = true;
  grid_dependents_launch();
  for (int c = blockIdx.x; c < L.num_chunks; c += gridDim.x) {
    for (int i = tid; i < L.E + L.R; i += blockDim.x) sm[i] = 0;
    __syncthreads();
    const int64_t t0 = (int64_t)c * L.chunk;
    const int64_t t1 = min(L.T, t0 + L.chunk);
    for (int64_t tb = t0; tb < t1; tb += blockDim.x) {  // same trip count for every thread
      const int64_t t = tb + tid;
      ok &= token_membership(L, t, t < t1, hist, tok);
    }
    __syncthreads();
    for (int e = tid; e < L.E; e += blockDim.x) L.d.chunk_cnt[(int64_t)c * L.E + e] = hist[e];
    for (int r = tid; r < L.R; r += blockDim.x) {
      if (tok[r]) atomicAdd(L.d.tokens_per_rank + r, tok[r]);  // integer sum: order-free
      if (L.by_rank) L.d.chunk_tok[(int64_t)c * L.R + r] = tok[r];
    }
    __syncthreads();
  }
  if (!ok) atomicOr(L.d.status, kStatusBadExpert);
}

// ------------------------------------------------------------------------------------ scan
// ceil(E/32) CTAs of 32 x 32 threads.  CTA b owns experts [32b, 32b + 32): lane = expert (so
// every load of a chunk row is one 128-byte segment), warp w = a contiguous group of chunks.
// (1) each thread sums its chunk group; (2) warp-shuffle exclusive scan of the 32 group sums of
// each expert; (3) each thread rewrites its chunk counts as exclusive offsets; the expert total
// is cnt[e].  The CTA that finishes last (an atomic ticket after a fence; nothing waits) then
// scans align_up(cnt, A) and the padding rows over all experts and restarts psum at every rank.
__global__ void __launch_bounds__(kScanThreads) k_layout_scan(LayoutLaunch L, int64_t cap_check) {
  __shared__ int32_t gsum[32][33];
  __shared__ int32_t is_last;
  extern __shared__ int32_t sm[];
  const int E = L.E;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // CTAs [0, ceil(E/32)) scan expert columns of chunk_cnt; the rest (by-rank) rank columns of
  // chunk_tok, the same way
  const int n_expert_ctas = (E + 31) / 32;
  const bool experts = (int)blockIdx.x < n_expert_ctas;
  const int width = experts ? E : L.R;
  int32_t* counts = experts ? L.d.chunk_cnt : L.d.chunk_tok;
  const int col0 = (experts ? (int)blockIdx.x : (int)blockIdx.x - n_expert_ctas) * 32;
  const int e = col0 + lane;
  const int C = L.num_chunks;
  const int cpw = (C + 31) / 32;  // chunks per warp
  const int c0 = min(C, warp * cpw), c1 = min(C, c0 + cpw);
  grid_dependents_launch();
  grid_dependency_wait();  // chunk counts of the count kernel

  int32_t sum = 0;
  if (e < width)
    for (int c = c0; c < c1; ++c) sum += counts[(int64_t)c * width + e];
  gsum[warp][lane] = sum;
  __syncthreads();
  {  // warp x scans the 32 group sums of expert blockIdx.x*32 + x
    const int32_t v = gsum[lane][warp];
    int32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    __syncwarp();
    gsum[lane][warp] = incl - v;
    const int ex = col0 + warp;
    if (experts && lane == 31 && ex < E) L.d.cnt[ex] = incl;
  }
  __syncthreads();
  if (e < width) {
    int32_t off = gsum[warp][lane];
    for (int c = c0; c < c1; ++c) {
      int32_t* q = counts + (int64_t)c * width + e;
      const int32_t v = *q;
      *q = off;
      off += v;
    }
  }

  // the last CTA to finish sees every cnt[e]
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = atomicAdd(L.d.ticket, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (tid == 0) *L.d.ticket = 0;  // ready for the next layout on this scratch
  block_psum<true>(L, L.d.cnt, cap_check, sm, sm + E, sm + 2 * E, nullptr, nullptr, true, whole_cta());
  publish_host_counts(L, whole_cta());
}

// ------------------------------------------------------------------------------------ assign
// A CTA per chunk of tokens, 8 warps; warp w takes a contiguous run of the chunk's (t, j) pairs.
// Phase 1: per-warp histogram (__match_any_sync groups equal ids inside a round; the group
// leader adds its size).  Phase 2: per expert, exclusive scan across warps based at the
// expert's first row for this chunk.  Phase 3: a pair's row = its warp's running base + its rank
// among equal ids of lower lanes in the round.
__global__ void __launch_bounds__(kLayoutThreads) k_layout_assign(LayoutLaunch L) {
  extern __shared__ int32_t whist[];  // [kLayoutWarps][E]
  __shared__ int32_t base_r[kMaxByRankRanks];
  __shared__ int32_t wcnt[kLayoutWarps * kMaxByRankRanks];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = L.E;
  int32_t* h = whist + warp * E;
  bool overflow = false;
  grid_dependents_launch();
  grid_dependency_wait();  // offsets, counts and psum of the scan kernel

  for (int c = blockIdx.x; c < L.num_chunks; c += gridDim.x) {
    const int64_t t0 = (int64_t)c * L.chunk;
    const int64_t t1 = min(L.T, t0 + L.chunk);
    const int64_t p0 = t0 * L.k, np = (t1 - t0) * L.k;
    const int64_t per = (np + kLayoutWarps - 1) / kLayoutWarps;
    const int64_t wp0 = p0 + min(np, warp * per), wp1 = p0 + min(np, (warp + 1) * per);

    for (int e = lane; e < E; e += 32) h[e] = 0;
    __syncwarp();
    warp_histogram(L, wp0, wp1, h);
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
      int32_t base = L.d.psum[e] - align_up_dev(L.d.cnt[e], L.A) + L.d.chunk_cnt[(int64_t)c * E + e];
      for (int w = 0; w < kLayoutWarps; ++w) {
        const int32_t v = whist[w * E + e];
        whist[w * E + e] = base;
        base += v;
      }
    }
    __syncthreads();
    overflow |= warp_assign(L, wp0, wp1, h);
    __syncthreads();
    if (L.by_rank) {  // chunk <= blockDim tokens: one group, based at the chunk offsets
      for (int r = tid; r < L.R; r += blockDim.x) base_r[r] = L.d.chunk_tok[(int64_t)c * L.R + r];
      __syncthreads();
      token_rows_group(L, t0, t1, base_r, wcnt);
    }
  }
  overflow |= row_map_padding(L, L.d.pad_excl, L.d.psum, (int64_t)blockIdx.x * kLayoutWarps + warp,
                              (int64_t)gridDim.x * kLayoutWarps);
  if (overflow) atomicOr(L.d.status, kStatusCapacity);
}

// ------------------------------------------------------------------------------------ fused
// The one-launch layout (layout_body.cuh, fused_layout_chunk): a CTA of kThreads threads per
// chunk, in one cooperative launch; by rank, then the token rows of the chunk, in groups of
// blockDim tokens based at the chunk's per-rank offsets.  One launch and one global handoff
// instead of three kernels; the results are the same.  Instances: 256 threads with 8 or 16
// register rounds of 32 pairs per warp, and 1024 threads with 4 rounds for the wide chunks of a
// capped SM budget (32 warps take a chunk's pairs in a quarter of the rounds: the rounds' match
// and histogram steps run one after another inside a warp).
constexpr int kFusedWideThreads = 1024;
constexpr int kFusedWideRounds = 4;
constexpr int kFusedWideMaxExperts = 1024;  // 32 per-warp histograms of E counts in shared memory

template <int kRounds, int kThreads>
__global__ void __launch_bounds__(kThreads, 1) k_layout_fused(LayoutLaunch L, int64_t cap_check) {
  extern __shared__ int32_t sm[];
  __shared__ int32_t base_r[kMaxByRankRanks];
  __shared__ int32_t wcnt[(kThreads / 32) * kMaxByRankRanks];
  __shared__ int32_t go;
  grid_dependents_launch();
  if (!fused_layout_chunk<kRounds>(L, cap_check, blockIdx.x, gridDim.x, whole_cta(), sm, base_r, &go)) return;
  if (L.by_rank) {  // groups of blockDim tokens (a chunk may hold several), based at the chunk's offsets
    __syncthreads();
    const int64_t t0 = (int64_t)blockIdx.x * L.chunk, t1 = min(L.T, t0 + L.chunk);
    for (int64_t tg = t0; tg < t1; tg += blockDim.x) token_rows_group(L, tg, t1, base_r, wcnt);
  }
}

// At most one chunk per SM of the budget (so every CTA can be resident), the chunk's pairs in
// the warps' registers, and bounded redundant summing.
bool layout_fits_fused(int num_chunks, int chunk, int k, int E, int sm_budget) {
  return num_chunks >= 1 && num_chunks <= sm_budget && E <= kFusedMaxExperts &&
         (int64_t)chunk * k <= (int64_t)kLayoutThreads * kFusedMaxRounds &&
         (int64_t)num_chunks * E <= kFusedMaxChunkCounts;
}

// ------------------------------------------------------------------------------------ small
// The whole layout in one CTA of 32 warps, for small batches (T * k <= kSmallPairs and
// E <= kSmallMaxExperts): membership and id checks, per-warp histograms of token-aligned pair
// ranges, cross-warp scan, psum, slots and row maps, all through shared memory, in one launch
// and with no scratch beyond the handle's arrays.  The allocation-free entry point uses it; the
// handle path runs the one-launch layout (or count -> scan -> assign), which spreads a small
// batch over more SMs and is faster.  The results are the same.
__global__ void __launch_bounds__(kSmallThreads) k_layout_small(LayoutLaunch L, int64_t cap_check) {
  extern __shared__ int32_t sm[];
  const int E = L.E, tid = threadIdx.x, warp = tid >> 5;
  constexpr int W = kSmallThreads / 32;
  int32_t* whist = sm;                  // [W][E]
  int32_t* al = whist + W * E;          // [E]
  int32_t* pad = al + E;                // [E]
  int32_t* gincl = pad + E;             // [E]
  int32_t* psum_s = gincl + E;          // [E]
  int32_t* pad_s = psum_s + E;          // [E + 1]
  int32_t* cnt_s = pad_s + E + 1;       // [E]
  int32_t* tok = cnt_s + E;             // [R]
  grid_dependents_launch();

  for (int i = tid; i < W * E; i += blockDim.x) whist[i] = 0;
  for (int r = tid; r < L.R; r += blockDim.x) tok[r] = 0;
  __syncthreads();

  bool ok = true;
  for (int64_t tb = 0; tb < L.T; tb += blockDim.x) {  // same trip count for every thread
    const int64_t t = tb + tid;
    ok &= token_membership(L, t, t < L.T, nullptr, tok);
  }
  if (!ok) atomicOr(L.d.status, kStatusBadExpert);

  // token-aligned pair range of this warp
  const int64_t tpw = (L.T + W - 1) / W;
  const int64_t wp0 = min(L.T, warp * tpw) * L.k, wp1 = min(L.T, (warp + 1) * tpw) * L.k;
  int32_t* h = whist + warp * E;
  warp_histogram(L, wp0, wp1, h);
  __syncthreads();

  for (int e = tid; e < E; e += blockDim.x) {  // exclusive scan across warps; cnt = total
    int32_t run = 0;
    for (int w = 0; w < W; ++w) {
      const int32_t v = whist[w * E + e];
      whist[w * E + e] = run;
      run += v;
    }
    cnt_s[e] = run;
    L.d.cnt[e] = run;
  }
  for (int r = tid; r < L.R; r += blockDim.x) L.d.tokens_per_rank[r] = tok[r];
  __syncthreads();
  block_psum<false>(L, cnt_s, cap_check, al, pad, gincl, pad_s, psum_s, true, whole_cta());

  for (int e = tid; e < E; e += blockDim.x) {  // base every warp's rows at the segment start
    const int32_t seg = psum_s[e] - al[e];
    for (int w = 0; w < W; ++w) whist[w * E + e] += seg;
  }
  __syncthreads();
  bool overflow = warp_assign(L, wp0, wp1, h);
  overflow |= row_map_padding(L, pad_s, psum_s, warp, W);
  if (overflow) atomicOr(L.d.status, kStatusCapacity);
  if (L.by_rank) {
    __shared__ int32_t base_r[kMaxByRankRanks];
    __shared__ int32_t wcnt[W * kMaxByRankRanks];
    for (int r = tid; r < L.R; r += blockDim.x) base_r[r] = 0;
    __syncthreads();
    for (int64_t t0 = 0; t0 < L.T; t0 += blockDim.x) token_rows_group(L, t0, L.T, base_r, wcnt);
  }
}

bool layout_fits_one_cta(int64_t T, int k, int E) {
  return T * k <= kSmallPairs && E <= kSmallMaxExperts;
}

size_t small_layout_smem(int E, int R) {
  return sizeof(int32_t) * ((size_t)(kSmallThreads / 32) * E + 6 * (size_t)E + 1 + R);
}

// ------------------------------------------------------------------------------------ launch
// Opt in to the dynamic shared memory the largest supported E needs, once per device.
static cudaError_t ensure_smem_attrs() {
  static unsigned long long done = 0;  // one bit per device ordinal
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && (done >> dev) & 1ull) return cudaSuccess;
  err = cudaFuncSetAttribute(k_layout_scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(sizeof(int32_t) * 3 * kMaxExperts));
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(k_layout_small, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)small_layout_smem(kSmallMaxExperts, kSmallMaxExperts));
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(k_layout_assign, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(sizeof(int32_t) * kLayoutWarps * kMaxExperts));
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(k_layout_fused<kFusedRounds, kLayoutThreads>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)fused_layout_smem(kFusedMaxExperts, kFusedMaxExperts, kLayoutWarps));  // R <= E
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(k_layout_fused<kFusedMaxRounds, kLayoutThreads>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)fused_layout_smem(kFusedMaxExperts, kFusedMaxExperts, kLayoutWarps));
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(k_layout_fused<kFusedWideRounds, kFusedWideThreads>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)fused_layout_smem(kFusedWideMaxExperts, kFusedWideMaxExperts,
                                                      kFusedWideThreads / 32));
  if (err == cudaSuccess && dev < 64) done |= 1ull << dev;
  return err;
}

cudaError_t launch_layout_count(const LayoutLaunch& L, cudaStream_t s) {
  if (L.num_chunks == 0) return cudaSuccess;
  const size_t smem = sizeof(int32_t) * (size_t)(L.E + L.R);
  k_layout_count<<<L.grid_chunks, kLayoutThreads, smem, s>>>(L);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_layout_small(const LayoutLaunch& L, int64_t cap_check, cudaStream_t s) {
  cudaError_t err = ensure_smem_attrs();
  if (err != cudaSuccess) return err;
  k_layout_small<<<1, kSmallThreads, small_layout_smem(L.E, L.R), s>>>(L, cap_check);
  note_launch();
  return cudaGetLastError();
}

// One CTA per chunk, launched cooperatively so that all of them are resident (the grid barrier
// inside waits for every CTA).
cudaError_t launch_layout_fused(const LayoutLaunch& L, int64_t cap_check, cudaStream_t s) {
  cudaError_t err = ensure_smem_attrs();
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(L.num_chunks);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // pairs per warp: ceil(chunk * k / warps), held in rounds of 32
  const int64_t pairs = (int64_t)L.chunk * L.k;
  const int64_t per_warp = (pairs + kLayoutWarps - 1) / kLayoutWarps;
  const int wide_warps = kFusedWideThreads / 32;
  if (per_warp > 32 * kFusedMaxRounds) return cudaErrorInvalidValue;
  if (per_warp <= 32 * kFusedRounds) {
    cfg.blockDim = dim3(kLayoutThreads);
    cfg.dynamicSmemBytes = fused_layout_smem(L.E, L.R, kLayoutWarps);
    err = cudaLaunchKernelEx(&cfg, k_layout_fused<kFusedRounds, kLayoutThreads>, L, cap_check);
  } else if (L.E <= kFusedWideMaxExperts && (pairs + wide_warps - 1) / wide_warps <= 32 * kFusedWideRounds) {
    cfg.blockDim = dim3(kFusedWideThreads);
    cfg.dynamicSmemBytes = fused_layout_smem(L.E, L.R, wide_warps);
    err = cudaLaunchKernelEx(&cfg, k_layout_fused<kFusedWideRounds, kFusedWideThreads>, L, cap_check);
  } else {
    cfg.blockDim = dim3(kLayoutThreads);
    cfg.dynamicSmemBytes = fused_layout_smem(L.E, L.R, kLayoutWarps);
    err = cudaLaunchKernelEx(&cfg, k_layout_fused<kFusedMaxRounds, kLayoutThreads>, L, cap_check);
  }
  note_launch();
  return err;
}

cudaError_t launch_layout_scan(const LayoutLaunch& L, int64_t cap_check, cudaStream_t s) {
  cudaError_t err = ensure_smem_attrs();
  if (err != cudaSuccess) return err;
  const size_t smem = sizeof(int32_t) * 3 * (size_t)L.E;
  const int grid = (L.E + 31) / 32 + (L.by_rank ? (L.R + 31) / 32 : 0);
  err = launch_pdl(k_layout_scan, dim3(grid), dim3(kScanThreads), smem, s, L, cap_check);
  note_launch();
  return err;
}

cudaError_t launch_layout_assign(const LayoutLaunch& L, cudaStream_t s) {
  cudaError_t err = ensure_smem_attrs();
  if (err != cudaSuccess) return err;
  const size_t smem = sizeof(int32_t) * (size_t)kLayoutWarps * L.E;
  const int grid = L.grid_chunks > 0 ? L.grid_chunks : 1;
  err = launch_pdl(k_layout_assign, dim3(grid), dim3(kLayoutThreads), smem, s, L);
  note_launch();
  return err;
}

}  // namespace moe
