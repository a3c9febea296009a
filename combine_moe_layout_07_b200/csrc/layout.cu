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

// ------------------------------------------------------------------------------------ count
// A thread per token: its k ids are loaded together, counted into the chunk's shared-memory
// histogram (atomicAdd_block), and its rank membership is written and counted.
__global__ void __launch_bounds__(kLayoutThreads) k_layout_count(LayoutLaunch L) {
  extern __shared__ int32_t sm[];
  int32_t* hist = sm;       // [E]
  int32_t* tok = sm + L.E;  // [R]
  const int tid = threadIdx.x;
  bool bad = false;
  for (int c = blockIdx.x; c < L.num_chunks; c += gridDim.x) {
    for (int i = tid; i < L.E + L.R; i += blockDim.x) sm[i] = 0;
    __syncthreads();
    const int64_t t0 = (int64_t)c * kChunkTokens;
    const int64_t t1 = min(L.T, t0 + kChunkTokens);
    for (int64_t t = t0 + tid; t < t1; t += blockDim.x) {
      const int64_t* ids = L.idx + t * L.k;
      int32_t ev[kMaxTopk];
#pragma unroll
      for (int j = 0; j < kMaxTopk; ++j) {
        ev[j] = j < L.k ? expert_of(__ldg(ids + j), L.E) : -1;
        if (ev[j] == -2) {
          bad = true;
          ev[j] = -1;
        }
      }
      uint8_t* member = L.d.token_in_rank + t * L.R;
      if (L.R <= 64) {
        uint64_t mask = 0;
#pragma unroll
        for (int j = 0; j < kMaxTopk; ++j)
          if (ev[j] >= 0) {
            atomicAdd_block(&hist[ev[j]], 1);
            mask |= 1ull << (ev[j] / L.E_loc);
          }
        for (int r = 0; r < L.R; ++r) member[r] = (uint8_t)((mask >> r) & 1);
        for (uint64_t m = mask; m; m &= m - 1) atomicAdd_block(&tok[__ffsll((long long)m) - 1], 1);
      } else {
        for (int r = 0; r < L.R; ++r) member[r] = 0;
#pragma unroll
        for (int j = 0; j < kMaxTopk; ++j)
          if (ev[j] >= 0) {
            atomicAdd_block(&hist[ev[j]], 1);
            const int r = ev[j] / L.E_loc;
            bool first = true;
#pragma unroll
            for (int j2 = 0; j2 < j; ++j2)
              if (ev[j2] >= 0 && ev[j2] / L.E_loc == r) first = false;
            if (first) {
              member[r] = 1;
              atomicAdd_block(&tok[r], 1);
            }
          }
      }
    }
    __syncthreads();
    for (int e = tid; e < L.E; e += blockDim.x) L.d.chunk_cnt[(int64_t)c * L.E + e] = hist[e];
    for (int r = tid; r < L.R; r += blockDim.x)
      if (tok[r]) atomicAdd(L.d.tokens_per_rank + r, tok[r]);  // integer sum: order-free
    __syncthreads();
  }
  if (bad) atomicOr(L.d.status, kStatusBadExpert);
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

// ------------------------------------------------------------------------------------ scan
// ceil(E/32) CTAs of 32 x 32 threads.  CTA b owns experts [32b, 32b + 32): lane = expert (so
// every load of a chunk row is one 128-byte segment), warp w = a contiguous group of chunks.
// (1) each thread sums its chunk group; (2) warp-shuffle exclusive scan of the 32 group sums of
// each expert; (3) each thread rewrites its chunk counts as exclusive offsets; the expert total
// is cnt[e].  The CTA that finishes last (an atomic ticket after a fence; nothing waits) then
// (4) scans align_up(cnt, A) and the padding rows over all experts and (5) restarts psum at
// every rank.
__global__ void __launch_bounds__(kScanThreads) k_layout_scan(LayoutLaunch L, int64_t cap_check) {
  __shared__ int32_t gsum[32][33];
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t totals[2];
  __shared__ int32_t is_last;
  extern __shared__ int32_t sm[];
  const int E = L.E;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e = blockIdx.x * 32 + lane;
  const int C = L.num_chunks;
  const int cpw = (C + 31) / 32;  // chunks per warp
  const int c0 = min(C, warp * cpw), c1 = min(C, c0 + cpw);

  int32_t sum = 0;
  if (e < E)
    for (int c = c0; c < c1; ++c) sum += L.d.chunk_cnt[(int64_t)c * E + e];
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
    const int ex = blockIdx.x * 32 + warp;
    if (lane == 31 && ex < E) L.d.cnt[ex] = incl;
  }
  __syncthreads();
  if (e < E) {
    int32_t off = gsum[warp][lane];
    for (int c = c0; c < c1; ++c) {
      int32_t* q = L.d.chunk_cnt + (int64_t)c * E + e;
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

  int32_t* al = sm;             // [E] align_up(cnt, A)
  int32_t* pad = sm + E;        // [E] align_up(cnt, A) - cnt
  int32_t* gincl = sm + 2 * E;  // [E] inclusive prefix of al over all experts
  for (int x = tid; x < E; x += blockDim.x) {
    const int32_t n = __ldcg(L.d.cnt + x);
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
    L.d.pad_excl[x] = rp;
    rp += pad[x];
    ra += al[x];
    gincl[x] = ra;
  }
  if (tid == 0) L.d.pad_excl[E] = totals[1];
  __syncthreads();
  for (int x = tid; x < E; x += blockDim.x) {
    const int first = (x / L.E_loc) * L.E_loc;
    L.d.psum[x] = gincl[x] - (gincl[first] - al[first]);
  }
  for (int r = tid; r < L.R; r += blockDim.x) {
    const int first = r * L.E_loc, last = first + L.E_loc - 1;
    const int32_t nrows = gincl[last] - (gincl[first] - al[first]);
    L.d.rows_per_rank[r] = nrows;
    if (cap_check > 0 && nrows > cap_check) atomicOr(L.d.status, kStatusCapacity);
  }
}

// ------------------------------------------------------------------------------------ assign
// A CTA per chunk of tokens, 8 warps; warp w takes a contiguous run of the chunk's (t, j) pairs
// and loads its expert ids kAssignBatch rounds of 32 at a time.  Phase 1: per-warp histogram
// (__match_any_sync groups equal ids inside a round; the group leader adds its size).  Phase 2:
// per expert, exclusive scan across warps based at the expert's first row for this chunk.
// Phase 3: walk the pairs again; a pair's row = its warp's running base + its rank among equal
// ids of lower lanes in the round.
constexpr int kAssignBatch = 8;

__global__ void __launch_bounds__(kLayoutThreads) k_layout_assign(LayoutLaunch L) {
  extern __shared__ int32_t whist[];  // [kLayoutWarps][E]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = L.E;
  int32_t* h = whist + warp * E;
  const uint32_t lt = lanemask_lt();
  bool overflow = false;

  for (int c = blockIdx.x; c < L.num_chunks; c += gridDim.x) {
    const int64_t t0 = (int64_t)c * kChunkTokens;
    const int64_t t1 = min(L.T, t0 + kChunkTokens);
    const int64_t p0 = t0 * L.k, np = (t1 - t0) * L.k;
    const int64_t per = (np + kLayoutWarps - 1) / kLayoutWarps;
    const int64_t wp0 = p0 + min(np, warp * per), wp1 = p0 + min(np, (warp + 1) * per);

    // phase 1: this warp's histogram of its pairs
    for (int e = lane; e < E; e += 32) h[e] = 0;
    __syncwarp();
    for (int64_t base = wp0; base < wp1; base += 32 * kAssignBatch) {
      int32_t ev[kAssignBatch];
#pragma unroll
      for (int r = 0; r < kAssignBatch; ++r) {
        const int64_t p = base + r * 32 + lane;
        ev[r] = p < wp1 ? max(expert_of(__ldg(L.idx + p), E), -1) : -1;
      }
#pragma unroll
      for (int r = 0; r < kAssignBatch; ++r) {
        const uint32_t peers = __match_any_sync(0xffffffffu, ev[r]);
        if (ev[r] >= 0 && lane == __ffs(peers) - 1) h[ev[r]] += __popc(peers);
        __syncwarp();
      }
    }
    __syncthreads();

    // phase 2: per expert, exclusive scan across warps
    for (int e = tid; e < E; e += blockDim.x) {
      int32_t base = L.d.psum[e] - align_up_dev(L.d.cnt[e], L.A) + L.d.chunk_cnt[(int64_t)c * E + e];
      for (int w = 0; w < kLayoutWarps; ++w) {
        const int32_t v = whist[w * E + e];
        whist[w * E + e] = base;
        base += v;
      }
    }
    __syncthreads();

    // phase 3: rows in (t, j) order
    for (int64_t base = wp0; base < wp1; base += 32 * kAssignBatch) {
      int32_t ev[kAssignBatch];
      float wv[kAssignBatch];
#pragma unroll
      for (int r = 0; r < kAssignBatch; ++r) {
        const int64_t p = base + r * 32 + lane;
        ev[r] = p < wp1 ? max(expert_of(__ldg(L.idx + p), E), -1) : -1;
        wv[r] = (p < wp1 && L.w) ? __ldg(L.w + p) : 0.0f;
      }
#pragma unroll
      for (int r = 0; r < kAssignBatch; ++r) {
        const int64_t p = base + r * 32 + lane;
        const int32_t e = ev[r];
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        int32_t row = -1;
        if (e >= 0) row = h[e] + __popc(peers & lt);
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) h[e] += __popc(peers);
        __syncwarp();
        if (p < wp1) {
          L.d.slot[p] = row;
          L.d.pair_rank[p] = e >= 0 ? e / L.E_loc : -1;
          L.d.pair_w[p] = wv[r];
          if (e >= 0) {
            const int rk = e / L.E_loc;
            if (row < L.row_cap) {
              L.d.row_src[(int64_t)rk * L.row_cap + row] = (int32_t)(p / L.k);
              L.d.row_w[(int64_t)rk * L.row_cap + row] = wv[r];
            } else {
              overflow = true;
            }
          }
        }
      }
    }
    __syncthreads();
  }

  // padding rows of the row maps: global padding index i -> expert by binary search
  const int32_t total_pad = L.d.pad_excl[E];
  for (int32_t i = blockIdx.x * blockDim.x + tid; i < total_pad; i += gridDim.x * blockDim.x) {
    int lo = 0, hi = E;  // largest e with pad_excl[e] <= i
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (L.d.pad_excl[mid] <= i) lo = mid;
      else hi = mid;
    }
    const int e = lo;
    const int32_t pad_e = L.d.pad_excl[e + 1] - L.d.pad_excl[e];
    const int32_t row = L.d.psum[e] - pad_e + (i - L.d.pad_excl[e]);
    const int r = e / L.E_loc;
    if (row < L.row_cap) {
      L.d.row_src[(int64_t)r * L.row_cap + row] = -1;
      L.d.row_w[(int64_t)r * L.row_cap + row] = 0.0f;
    } else {
      overflow = true;
    }
  }
  if (overflow) atomicOr(L.d.status, kStatusCapacity);
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
    err = cudaFuncSetAttribute(k_layout_assign, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(sizeof(int32_t) * kLayoutWarps * kMaxExperts));
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

cudaError_t launch_layout_scan(const LayoutLaunch& L, int64_t cap_check, cudaStream_t s) {
  cudaError_t err = ensure_smem_attrs();
  if (err != cudaSuccess) return err;
  const size_t smem = sizeof(int32_t) * 3 * (size_t)L.E;
  k_layout_scan<<<(L.E + 31) / 32, kScanThreads, smem, s>>>(L, cap_check);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_layout_assign(const LayoutLaunch& L, cudaStream_t s) {
  cudaError_t err = ensure_smem_attrs();
  if (err != cudaSuccess) return err;
  const size_t smem = sizeof(int32_t) * (size_t)kLayoutWarps * L.E;
  const int grid = L.grid_chunks > 0 ? L.grid_chunks : 1;
  k_layout_assign<<<grid, kLayoutThreads, smem, s>>>(L);
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe
