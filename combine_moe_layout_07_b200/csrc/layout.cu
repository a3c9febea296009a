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
#include "moe_internal.cuh"

namespace moe {

__device__ __forceinline__ int32_t align_up_dev(int32_t n, int32_t a) { return ((n + a - 1) / a) * a; }

// Expert id of a routing entry as int32: the id if in [0, E), -1 when masked, -2 when the
// entry lies outside [-1, E) (an error the count kernel reports).
__device__ __forceinline__ int32_t expert_of(int64_t e, int E) {
  return (e >= 0 && e < E) ? (int32_t)e : (e == -1 ? -1 : -2);
}

// ------------------------------------------------------------------------------------ helpers
// Membership of token t (when `valid`): writes token_in_rank[t, :] and counts the token for every
// rank holding one of its experts into tok[r] (shared memory).  Called by whole warps: with R <= 64
// the per-rank counts are aggregated over the warp (one ballot per rank, one atomic from lane 0),
// which keeps shared-memory atomics off a handful of hot addresses.  When `hist` is given, every
// valid id is also counted into it.  Returns false if one of the token's ids lies outside [-1, E).
__device__ __forceinline__ bool token_membership(const LayoutLaunch& L, int64_t t, bool valid, int32_t* hist,
                                                 int32_t* tok) {
  bool bad = false;
  const int64_t* ids = L.idx + t * L.k;
  uint8_t* member = L.d.token_in_rank + t * L.R;
  if (L.R <= 64) {
    uint64_t mask = 0;
    if (valid) {
#pragma unroll 4
      for (int j = 0; j < L.k; ++j) {
        const int32_t e = expert_of(__ldg(ids + j), L.E);
        bad |= e == -2;
        if (e >= 0) {
          if (hist) atomicAdd_block(&hist[e], 1);
          mask |= 1ull << ((uint32_t)e / (uint32_t)L.E_loc);
        }
      }
      for (int r = 0; r < L.R; ++r) member[r] = (uint8_t)((mask >> r) & 1);
    }
    const int lane = threadIdx.x & 31;
    for (int r = 0; r < L.R; ++r) {
      const int c = __popc(__ballot_sync(0xffffffffu, (mask >> r) & 1));
      if (lane == 0 && c) atomicAdd_block(&tok[r], c);
    }
  } else if (valid) {
    for (int r = 0; r < L.R; ++r) member[r] = 0;
    for (int j = 0; j < L.k; ++j) {
      const int32_t e = expert_of(__ldg(ids + j), L.E);
      bad |= e == -2;
      if (e < 0) continue;
      if (hist) atomicAdd_block(&hist[e], 1);
      const int r = (int)((uint32_t)e / (uint32_t)L.E_loc);
      bool first = true;  // the token's first id on rank r counts it there
      for (int j2 = 0; j2 < j; ++j2) {
        const int32_t e2 = expert_of(__ldg(ids + j2), L.E);
        if (e2 >= 0 && (int)((uint32_t)e2 / (uint32_t)L.E_loc) == r) first = false;
      }
      if (first) {
        member[r] = 1;
        atomicAdd_block(&tok[r], 1);
      }
    }
  }
  return !bad;
}

constexpr int kAssignBatch = 8;  // rounds of 32 pairs a warp loads before it works on them

// One round of 32 pairs of a warp's run (lane = pair, e = expert id or -1): the group of lanes
// with equal ids adds its size to h[e] through its first lane.
__device__ __forceinline__ void histogram_round(int32_t e, int32_t* h) {
  const int lane = threadIdx.x & 31;
  const uint32_t peers = __match_any_sync(0xffffffffu, e);
  if (e >= 0 && lane == __ffs(peers) - 1) h[e] += __popc(peers);
  __syncwarp();
}

// One round of the assignment: pair p (when in_range) with expert e (or -1) and weight w gets
// row h[e] + (lanes below it with the same id); h[e] advances by the group's size.  Writes slot,
// pair rank, pair weight and the row maps.  Returns true on a row >= row_cap.
__device__ __forceinline__ bool assign_round(const LayoutLaunch& L, int64_t p, bool in_range, int32_t e, float w,
                                             int32_t* h) {
  const int lane = threadIdx.x & 31;
  const uint32_t peers = __match_any_sync(0xffffffffu, e);
  int32_t row = -1;
  if (e >= 0) row = h[e] + __popc(peers & lanemask_lt());
  __syncwarp();
  if (e >= 0 && lane == __ffs(peers) - 1) h[e] += __popc(peers);
  __syncwarp();
  bool overflow = false;
  if (in_range) {
    // 32-bit divisions: e < E and p < T * k < 2^31
    const int rk = e >= 0 ? (int)((uint32_t)e / (uint32_t)L.E_loc) : -1;
    L.d.slot[p] = row;
    L.d.pair_rank[p] = rk;
    L.d.pair_w[p] = w;
    if (e >= 0) {
      if (row < L.row_cap) {
        L.d.row_src[(int64_t)rk * L.row_cap + row] = (int32_t)((uint32_t)p / (uint32_t)L.k);
        L.d.row_w[(int64_t)rk * L.row_cap + row] = w;
      } else {
        overflow = true;
      }
    }
  }
  return overflow;
}

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

// Padding rows of the row maps: warp w0, w0 + wstride, ... takes experts in turn and its lanes
// stride over the expert's padding rows [psum - pad, psum) (pad from pad_excl, psum and pad_excl
// in global or shared memory).  Returns true on a row >= row_cap.
__device__ __forceinline__ bool row_map_padding(const LayoutLaunch& L, const int32_t* pad_excl, const int32_t* psum,
                                                int64_t w0, int64_t wstride) {
  const int lane = threadIdx.x & 31;
  bool overflow = false;
  for (int64_t e = w0; e < L.E; e += wstride) {
    const int32_t pad_e = pad_excl[e + 1] - pad_excl[e];
    if (pad_e == 0) continue;
    const int32_t end = psum[e];
    const int64_t base = (int64_t)((uint32_t)e / (uint32_t)L.E_loc) * L.row_cap;
    for (int32_t row = end - pad_e + lane; row < end; row += 32) {
      if (row < L.row_cap) {
        L.d.row_src[base + row] = -1;
        L.d.row_w[base + row] = 0.0f;
      } else {
        overflow = true;
      }
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

// Block-wide exclusive scan of one value per thread (warp shuffles + one smem pass).
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t* warp_tot, int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t w = lane < nwarps ? warp_tot[lane] : 0;
    int32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < nwarps) warp_tot[lane] = wi - w;  // exclusive warp offsets
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int32_t r = warp_tot[warp] + incl - v;
  __syncthreads();
  return r;
}

// Given cnt[] (global memory written by other CTAs when kCntGlobal, else this CTA's shared
// memory), one CTA computes, with al / pad / gincl / pad_s as [E] or [E + 1] shared arrays:
// align_up(cnt, A), the padding prefix over all experts (to pad_excl and pad_s), psum restarted
// at every rank (to psum and psum_s), rows_per_rank and the capacity flag.  With publish = false
// only the shared arrays are written (CTAs that compute the same values for their own use).
template <bool kCntGlobal>
__device__ __forceinline__ void block_psum(const LayoutLaunch& L, const int32_t* cnt, int64_t cap_check, int32_t* al,
                                           int32_t* pad, int32_t* gincl, int32_t* pad_s, int32_t* psum_s,
                                           bool publish = true) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t totals[2];
  const int E = L.E, tid = threadIdx.x;
  for (int x = tid; x < E; x += blockDim.x) {
    const int32_t n = kCntGlobal ? __ldcg(cnt + x) : cnt[x];  // L2: values other CTAs wrote
    al[x] = align_up_dev(n, L.A);
    pad[x] = al[x] - n;
  }
  __syncthreads();
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
  int32_t sa = 0, sp = 0;
  for (int x = e0; x < e1; ++x) {
    sa += al[x];
    sp += pad[x];
  }
  int32_t ra = block_exclusive_scan(sa, warp_tot, &totals[0]);
  int32_t rp = block_exclusive_scan(sp, warp_tot, &totals[1]);
  for (int x = e0; x < e1; ++x) {
    if (publish) L.d.pad_excl[x] = rp;
    if (pad_s) pad_s[x] = rp;
    rp += pad[x];
    ra += al[x];
    gincl[x] = ra;
  }
  if (tid == 0) {
    if (publish) L.d.pad_excl[E] = totals[1];
    if (pad_s) pad_s[E] = totals[1];
  }
  __syncthreads();
  for (int x = tid; x < E; x += blockDim.x) {
    const int first = (x / L.E_loc) * L.E_loc;
    const int32_t v = gincl[x] - (gincl[first] - al[first]);
    if (publish) L.d.psum[x] = v;
    if (psum_s) psum_s[x] = v;
  }
  for (int r = tid; publish && r < L.R; r += blockDim.x) {
    const int first = r * L.E_loc, last = first + L.E_loc - 1;
    const int32_t nrows = gincl[last] - (gincl[first] - al[first]);
    L.d.rows_per_rank[r] = nrows;
    if (cap_check > 0 && nrows > cap_check) atomicOr(L.d.status, kStatusCapacity);
  }
  __syncthreads();
}

// With do_cpu_sync: hand the status flags and the per-rank counts to the host as soon as they
// are final (after psum), through mapped pinned memory, so the host's wait overlaps the rest of
// the layout.  Words: [0] status flags, [7] ready = 1 (written last, after a system-scope fence),
// [8, 8 + R) tokens_per_rank, [8 + R, 8 + 2R) rows_per_rank.  Called by every thread of the CTA
// that published psum / rows_per_rank, after block_psum.
__device__ __forceinline__ void publish_host_counts(const LayoutLaunch& L) {
  int32_t* hc = L.d.host_counts;
  if (hc == nullptr) return;
  for (int r = threadIdx.x; r < L.R; r += blockDim.x) {
    hc[8 + r] = __ldcg(L.d.tokens_per_rank + r);
    hc[8 + L.R + r] = __ldcg(L.d.rows_per_rank + r);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    hc[0] = atomicOr(L.d.status, 0);
    __threadfence_system();  // the counts reach host memory before the flag
    *reinterpret_cast<volatile int32_t*>(hc + 7) = 1;
  }
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
  block_psum<true>(L, L.d.cnt, cap_check, sm, sm + E, sm + 2 * E, nullptr, nullptr);
  publish_host_counts(L);
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
// Batches of at most one chunk per SM in one cooperative launch (every CTA resident at once), a
// CTA per chunk of 256 threads:
//   1. count: each warp loads its contiguous run of the chunk's pairs into registers (at most
//      kFusedRounds rounds of 32) and histograms it; token membership as k_layout_count; chunk
//      counts to global memory and added atomically into the expert totals cnt; then the CTA
//      arrives at a grid barrier (the ticket word; ticket and cnt cleared before the launch) and
//      waits, bounded, until every CTA has arrived;
//   2. every CTA reads the totals and sums the counts of the chunks before its own (its offsets
//      inside each expert); then align / padding prefix / psum as the scan kernel's last CTA
//      (CTA 0 alone publishes psum, pad_excl, rows_per_rank);
//   3. assign: as k_layout_assign for its chunk (pairs from registers), based at those offsets;
//      padding rows of the row maps over all CTAs' warps; by rank, the token rows based at the
//      chunk's rank offsets.
// One launch and one global handoff instead of three kernels; the results are the same.
__device__ __forceinline__ bool wait_count_reached(const int32_t* p, int32_t target, int32_t* status) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t n = 0;; ++n) {
    int32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    if (v >= target) return true;
    if ((n & 63) == 63 && globaltimer_ns() - t0 > kWaitLimitNs) break;
  }
  atomicOr(status, kStatusTimeout);
  return false;
}

__global__ void __launch_bounds__(kLayoutThreads, 1) k_layout_fused(LayoutLaunch L, int64_t cap_check) {
  extern __shared__ int32_t sm[];
  const int E = L.E, R = L.R, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x, C = gridDim.x;
  int32_t* whist = sm;                        // [kLayoutWarps][E]
  int32_t* hist = whist + kLayoutWarps * E;   // [E]  expert totals
  int32_t* off = hist + E;                    // [E]  rows of each expert in the chunks before c
  int32_t* al = off + E;                      // [E]
  int32_t* pad = al + E;                      // [E]
  int32_t* gincl = pad + E;                   // [E]
  int32_t* psum_s = gincl + E;                // [E]
  int32_t* pad_s = psum_s + E;                // [E + 1]
  int32_t* tok = pad_s + E + 1;               // [R]
  __shared__ int32_t base_r[kMaxByRankRanks];
  __shared__ int32_t wcnt[kLayoutWarps * kMaxByRankRanks];
  __shared__ int32_t go;
  grid_dependents_launch();

  // the warp's contiguous run of the chunk's pairs, held in registers for counting and assigning
  const int64_t t0 = (int64_t)c * L.chunk, t1 = min(L.T, t0 + L.chunk);
  const int64_t p0 = t0 * L.k, np = (t1 - t0) * L.k;
  const int64_t per = (np + kLayoutWarps - 1) / kLayoutWarps;
  const int64_t wp0 = p0 + min(np, warp * per), wp1 = p0 + min(np, (warp + 1) * per);
  int32_t ev[kFusedRounds];
  float wv[kFusedRounds];
  bool ok = true;
#pragma unroll
  for (int r = 0; r < kFusedRounds; ++r) {
    const int64_t p = wp0 + r * 32 + lane;
    const int32_t e = p < wp1 ? expert_of(__ldg(L.idx + p), L.E) : -1;
    ok &= e != -2;
    ev[r] = max(e, -1);
    wv[r] = (p < wp1 && L.w) ? __ldg(L.w + p) : 0.0f;
  }
  int32_t* h = whist + warp * E;
  for (int e = lane; e < E; e += 32) h[e] = 0;
  for (int r = tid; r < R; r += blockDim.x) tok[r] = 0;
  __syncthreads();
  // 1. count: per-warp histograms, token membership (ids now in L1), chunk counts
#pragma unroll
  for (int r = 0; r < kFusedRounds; ++r)
    if (wp0 + r * 32 < wp1) histogram_round(ev[r], h);
  for (int64_t tb = t0; tb < t1; tb += blockDim.x) {  // same trip count for every thread
    const int64_t t = tb + tid;
    ok &= token_membership(L, t, t < t1, nullptr, tok);
  }
  if (!ok) atomicOr(L.d.status, kStatusBadExpert);
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int32_t n = 0;
    for (int w = 0; w < kLayoutWarps; ++w) n += whist[w * E + e];
    L.d.chunk_cnt[(int64_t)c * E + e] = n;
    if (n) atomicAdd(L.d.cnt + e, n);  // expert totals (cleared before the launch): order-free
  }
  for (int r = tid; r < R; r += blockDim.x) {
    if (tok[r]) atomicAdd(L.d.tokens_per_rank + r, tok[r]);  // integer sum: order-free
    if (L.by_rank) L.d.chunk_tok[(int64_t)c * R + r] = tok[r];
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    atomicAdd(L.d.ticket, 1);
    go = wait_count_reached(L.d.ticket, C, L.d.status);
  }
  __syncthreads();
  if (!go) return;

  // 2. the expert totals, and the chunk's offsets from the counts of the chunks before it
  // (kFusedLoads loads in flight); then psum.  CTA 0 needs no offsets, so the counts reach the
  // host right after the barrier.
  for (int e = tid; e < E; e += blockDim.x) {
    const int32_t total = __ldcg(L.d.cnt + e);  // issued first: in flight with the chunk loads
    int32_t before = 0;
    for (int cb = 0; cb < c; cb += kFusedLoads) {
      int32_t v[kFusedLoads];
#pragma unroll
      for (int q = 0; q < kFusedLoads; ++q)
        v[q] = cb + q < c ? __ldcg(L.d.chunk_cnt + (int64_t)(cb + q) * E + e) : 0;
#pragma unroll
      for (int q = 0; q < kFusedLoads; ++q) before += v[q];
    }
    off[e] = before;
    hist[e] = total;
  }
  if (L.by_rank)
    for (int r = tid; r < R; r += blockDim.x) {
      int32_t before = 0;
      for (int cc = 0; cc < c; ++cc) before += __ldcg(L.d.chunk_tok + (int64_t)cc * R + r);
      base_r[r] = before;
    }
  __syncthreads();
  block_psum<false>(L, hist, cap_check, al, pad, gincl, pad_s, psum_s, c == 0);
  if (c == 0) publish_host_counts(L);

  // 3. assign: warp bases (exclusive over warps, from the expert's segment start and the chunk's
  // offset), then the warp's pairs from registers
  for (int e = tid; e < E; e += blockDim.x) {
    int32_t base = psum_s[e] - al[e] + off[e];
    for (int w = 0; w < kLayoutWarps; ++w) {
      const int32_t v = whist[w * E + e];
      whist[w * E + e] = base;
      base += v;
    }
  }
  __syncthreads();
  bool overflow = false;
#pragma unroll
  for (int r = 0; r < kFusedRounds; ++r) {
    const int64_t p = wp0 + r * 32 + lane;
    if (wp0 + r * 32 < wp1) overflow |= assign_round(L, p, p < wp1, ev[r], wv[r], h);
  }
  overflow |= row_map_padding(L, pad_s, psum_s, (int64_t)c * kLayoutWarps + warp, (int64_t)C * kLayoutWarps);
  if (overflow) atomicOr(L.d.status, kStatusCapacity);
  if (L.by_rank) {
    __syncthreads();
    token_rows_group(L, t0, t1, base_r, wcnt);
  }
}

size_t fused_layout_smem(int E, int R) { return sizeof(int32_t) * ((size_t)(kLayoutWarps + 7) * E + 1 + R); }

// At most one chunk per SM of the budget (so every CTA can be resident), the chunk's pairs in
// the warps' registers, and bounded redundant summing.
bool layout_fits_fused(int num_chunks, int chunk, int k, int E, int sm_budget) {
  return num_chunks >= 1 && num_chunks <= sm_budget && E <= kFusedMaxExperts &&
         (int64_t)chunk * k <= (int64_t)kLayoutThreads * kFusedRounds && (int64_t)num_chunks * E <= kFusedMaxChunkCounts;
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
  block_psum<false>(L, cnt_s, cap_check, al, pad, gincl, pad_s, psum_s);

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
    err = cudaFuncSetAttribute(k_layout_fused, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)fused_layout_smem(kFusedMaxExperts, kFusedMaxExperts));  // R <= E
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
  cfg.blockDim = dim3(kLayoutThreads);
  cfg.dynamicSmemBytes = fused_layout_smem(L.E, L.R);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, k_layout_fused, L, cap_check);
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
