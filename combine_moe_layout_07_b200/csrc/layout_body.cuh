// layout_body.cuh -- device code of the layout shared by the layout kernels (layout.cu) and the
// one-launch layout + dispatch kernel (dispatch.cu): expert-id checks, token membership, the
// warp-level histogram and assignment rounds, block scans and psum over a thread group, and the
// body of the one-launch layout for one chunk.
//
// Follows "From DeepEP to Mega MoE" (backyes.github.io) 2.2 (notify warps: per-expert counts
// with block-local atomics, then an inclusive prefix sum psum_num_recv_tokens_per_expert) and
// 2.4 (every routed row gets a position inside its expert's range), with expert_alignment and
// the per-rank receive buffers of "Why MoE gets stuck on communication" (locsic.com) section 1.
#pragma once

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
// pair rank, pair weight and the row maps (and, when rec_slot is given, the slot and rank into
// rec_slot[rec_i] / rec_rank[rec_i] too).  Returns true on a row >= row_cap.
__device__ __forceinline__ bool assign_round(const LayoutLaunch& L, int64_t p, bool in_range, int32_t e, float w,
                                             int32_t* h, int32_t* rec_slot = nullptr, int32_t* rec_rank = nullptr,
                                             int rec_i = 0) {
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
    if (rec_slot) {
      rec_slot[rec_i] = row;
      rec_rank[rec_i] = rk;
    }
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

// A group of threads that runs the block-level steps together: the whole CTA (bar = 0,
// __syncthreads) or the n threads of a named barrier (bar > 0), tid = the thread's index in it.
struct ThreadGroup {
  int tid;
  int n;
  int bar;
  __device__ __forceinline__ void sync() const {
    if (bar == 0) __syncthreads();
    else asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(n) : "memory");
  }
};

__device__ __forceinline__ ThreadGroup whole_cta() { return ThreadGroup{(int)threadIdx.x, (int)blockDim.x, 0}; }

// Exclusive scans of two values per thread of the group at once (warp shuffles + one smem pass);
// warp_tot holds 2 x 32 entries, total 2.  Returns the two exclusive prefixes.
__device__ __forceinline__ int2 block_exclusive_scan2(int32_t v0, int32_t v1, int32_t* warp_tot, int32_t* total,
                                                      const ThreadGroup& g) {
  const int lane = g.tid & 31, warp = g.tid >> 5, nwarps = g.n >> 5;
  int32_t a = v0, b = v1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t na = __shfl_up_sync(0xffffffffu, a, o);
    const int32_t nb = __shfl_up_sync(0xffffffffu, b, o);
    if (lane >= o) {
      a += na;
      b += nb;
    }
  }
  if (lane == 31) {
    warp_tot[warp] = a;
    warp_tot[32 + warp] = b;
  }
  g.sync();
  if (warp == 0) {
    const int32_t wa = lane < nwarps ? warp_tot[lane] : 0, wb = lane < nwarps ? warp_tot[32 + lane] : 0;
    int32_t ia = wa, ib = wb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t na = __shfl_up_sync(0xffffffffu, ia, o);
      const int32_t nb = __shfl_up_sync(0xffffffffu, ib, o);
      if (lane >= o) {
        ia += na;
        ib += nb;
      }
    }
    if (lane < nwarps) {  // exclusive warp offsets
      warp_tot[lane] = ia - wa;
      warp_tot[32 + lane] = ib - wb;
    }
    if (lane == 31) {
      total[0] = ia;
      total[1] = ib;
    }
  }
  g.sync();
  const int2 r = make_int2(warp_tot[warp] + a - v0, warp_tot[32 + warp] + b - v1);
  g.sync();
  return r;
}

// Given cnt[] (global memory written by other CTAs when kCntGlobal, else this CTA's shared
// memory), the group computes, with al / pad / gincl / pad_s as [E] or [E + 1] shared arrays:
// align_up(cnt, A), the padding prefix over all experts (to pad_excl and pad_s), psum restarted
// at every rank (to psum and psum_s), rows_per_rank and the capacity flag.  With publish = false
// only the shared arrays are written (CTAs that compute the same values for their own use).
template <bool kCntGlobal>
__device__ __forceinline__ void block_psum(const LayoutLaunch& L, const int32_t* cnt, int64_t cap_check, int32_t* al,
                                           int32_t* pad, int32_t* gincl, int32_t* pad_s, int32_t* psum_s,
                                           bool publish, const ThreadGroup& g) {
  __shared__ int32_t warp_tot[64];
  __shared__ int32_t totals[2];
  const int E = L.E, tid = g.tid;
  for (int x = tid; x < E; x += g.n) {
    const int32_t n = kCntGlobal ? __ldcg(cnt + x) : cnt[x];  // L2: values other CTAs wrote
    al[x] = align_up_dev(n, L.A);
    pad[x] = al[x] - n;
  }
  g.sync();
  const int per = (E + g.n - 1) / g.n;
  const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
  int32_t sa = 0, sp = 0;
  for (int x = e0; x < e1; ++x) {
    sa += al[x];
    sp += pad[x];
  }
  const int2 rr = block_exclusive_scan2(sa, sp, warp_tot, totals, g);
  int32_t ra = rr.x, rp = rr.y;
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
  g.sync();
  for (int x = tid; x < E; x += g.n) {
    const int first = (x / L.E_loc) * L.E_loc;
    const int32_t v = gincl[x] - (gincl[first] - al[first]);
    if (publish) L.d.psum[x] = v;
    if (psum_s) psum_s[x] = v;
  }
  for (int r = tid; publish && r < L.R; r += g.n) {
    const int first = r * L.E_loc, last = first + L.E_loc - 1;
    const int32_t nrows = gincl[last] - (gincl[first] - al[first]);
    L.d.rows_per_rank[r] = nrows;
    if (cap_check > 0 && nrows > cap_check) atomicOr(L.d.status, kStatusCapacity);
  }
  g.sync();
}

// With do_cpu_sync: hand the status flags and the per-rank counts to the host as soon as they
// are final (after psum), through mapped pinned memory, so the host's wait overlaps the rest of
// the layout.  Words: [0] status flags, [7] ready = 1 (written last, after a system-scope fence),
// [8, 8 + R) tokens_per_rank, [8 + R, 8 + 2R) rows_per_rank.  Called by every thread of the
// group that published psum / rows_per_rank, after block_psum.
__device__ __forceinline__ void publish_host_counts(const LayoutLaunch& L, const ThreadGroup& g) {
  int32_t* hc = L.d.host_counts;
  if (hc == nullptr) return;
  for (int r = g.tid; r < L.R; r += g.n) {
    hc[8 + r] = __ldcg(L.d.tokens_per_rank + r);
    hc[8 + L.R + r] = __ldcg(L.d.rows_per_rank + r);
  }
  g.sync();
  if (g.tid == 0) {
    hc[0] = atomicOr(L.d.status, 0);
    __threadfence_system();  // the counts reach host memory before the flag
    *reinterpret_cast<volatile int32_t*>(hc + 7) = 1;
  }
}

// Wait, bounded by wall-clock time, until *p >= target (acquire at GPU scope): a grid barrier
// over CTAs that are all resident (cooperative launch).  On expiry records kStatusTimeout.
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

// ------------------------------------------------------------------------------------ one launch
// The one-launch layout, for batches of at most one chunk per SM (C chunks, every CTA that holds
// one resident at once), chunk c by a group of W warps (g.n = 32 W threads):
//   1. count: each warp loads its contiguous run of the chunk's pairs into registers (at most
//      kRounds rounds of 32) and histograms it; token membership as the count kernel; chunk
//      counts to global memory and added atomically into the expert totals cnt; then the group
//      arrives at a grid barrier (the ticket word; ticket and cnt cleared before the launch) and
//      waits, bounded, until all C chunks have arrived;
//   2. the totals, and the sum of the counts of the chunks before c (its offsets inside each
//      expert); then align / padding prefix / psum as the scan kernel's last CTA (chunk 0 alone
//      publishes psum, pad_excl, rows_per_rank and, with do_cpu_sync, the host counts);
//   3. assign: as the assign kernel for its chunk (pairs from registers), based at those offsets;
//      padding rows of the row maps over all chunks' warps.  By rank, base_r receives the chunk's
//      per-rank token offsets (the caller builds the token rows).
// Shared memory: sm = fused_layout_smem(E, R, W) bytes; go = a shared flag.  Returns false, the same
// in every thread of the group, when the grid barrier timed out.
constexpr int kFusedMaxRounds = 16;

__host__ __device__ inline size_t fused_layout_smem(int E, int R, int warps) {
  return sizeof(int32_t) * ((size_t)(warps + 7) * E + 1 + R);
}

template <int kRounds>
__device__ __forceinline__ bool fused_layout_chunk(const LayoutLaunch& L, int64_t cap_check, int c, int C,
                                                   const ThreadGroup& g, int32_t* sm, int32_t* base_r,
                                                   int32_t* go) {
  const int E = L.E, R = L.R, tid = g.tid, lane = tid & 31, warp = tid >> 5, W = g.n >> 5;
  int32_t* whist = sm;                        // [W][E]  per-warp histograms, then bases
  int32_t* hist = whist + W * E;              // [E]  expert totals
  int32_t* off = hist + E;                    // [E]  rows of each expert in the chunks before c
  int32_t* al = off + E;                      // [E]
  int32_t* pad = al + E;                      // [E]
  int32_t* gincl = pad + E;                   // [E]
  int32_t* psum_s = gincl + E;                // [E]
  int32_t* pad_s = psum_s + E;                // [E + 1]
  int32_t* tok = pad_s + E + 1;               // [R]

  // the warp's contiguous run of the chunk's pairs, held in registers for counting and assigning
  const int64_t t0 = (int64_t)c * L.chunk, t1 = min(L.T, t0 + L.chunk);
  const int64_t p0 = t0 * L.k, np = (t1 - t0) * L.k;
  const int64_t per = (np + W - 1) / W;
  const int64_t wp0 = p0 + min(np, warp * per), wp1 = p0 + min(np, (warp + 1) * per);
  int32_t ev[kRounds];
  float wv[kRounds];
  bool ok = true;
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const int64_t p = wp0 + r * 32 + lane;
    const int32_t e = p < wp1 ? expert_of(__ldg(L.idx + p), L.E) : -1;
    ok &= e != -2;
    ev[r] = max(e, -1);
    wv[r] = (p < wp1 && L.w) ? __ldg(L.w + p) : 0.0f;
  }
  int32_t* h = whist + warp * E;
  for (int e = lane; e < E; e += 32) h[e] = 0;
  for (int r = tid; r < R; r += g.n) tok[r] = 0;
  g.sync();
  // 1. count: per-warp histograms, token membership (ids now in L1), chunk counts
#pragma unroll
  for (int r = 0; r < kRounds; ++r)
    if (wp0 + r * 32 < wp1) histogram_round(ev[r], h);
  for (int64_t tb = t0; tb < t1; tb += g.n) {  // same trip count for every thread
    const int64_t t = tb + tid;
    ok &= token_membership(L, t, t < t1, nullptr, tok);
  }
  if (!ok) atomicOr(L.d.status, kStatusBadExpert);
  g.sync();
  for (int e = tid; e < E; e += g.n) {
    int32_t n = 0;
    for (int w = 0; w < W; ++w) n += whist[w * E + e];
    L.d.chunk_cnt[(int64_t)c * E + e] = n;
    if (n) atomicAdd(L.d.cnt + e, n);  // expert totals (cleared before the launch): order-free
  }
  for (int r = tid; r < R; r += g.n) {
    if (tok[r]) atomicAdd(L.d.tokens_per_rank + r, tok[r]);  // integer sum: order-free
    if (L.by_rank) L.d.chunk_tok[(int64_t)c * R + r] = tok[r];
  }
  g.sync();
  if (tid == 0) {
    __threadfence();
    atomicAdd(L.d.ticket, 1);
    *go = wait_count_reached(L.d.ticket, C, L.d.status);
  }
  g.sync();
  if (!*go) return false;

  // 2. the expert totals, and the chunk's offsets from the counts of the chunks before it
  // (kFusedLoads loads in flight); then psum.  Chunk 0 needs no offsets, so the counts reach the
  // host right after the barrier.
  for (int e = tid; e < E; e += g.n) {
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
    for (int r = tid; r < R; r += g.n) {
      int32_t before = 0;
      for (int cc = 0; cc < c; ++cc) before += __ldcg(L.d.chunk_tok + (int64_t)cc * R + r);
      base_r[r] = before;
    }
  g.sync();
  block_psum<false>(L, hist, cap_check, al, pad, gincl, pad_s, psum_s, c == 0, g);
  if (c == 0) publish_host_counts(L, g);

  // 3. assign: warp bases (exclusive over warps, from the expert's segment start and the chunk's
  // offset), then the warp's pairs from registers
  for (int e = tid; e < E; e += g.n) {
    int32_t base = psum_s[e] - al[e] + off[e];
    for (int w = 0; w < W; ++w) {
      const int32_t v = whist[w * E + e];
      whist[w * E + e] = base;
      base += v;
    }
  }
  g.sync();
  bool overflow = false;
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const int64_t p = wp0 + r * 32 + lane;
    if (wp0 + r * 32 < wp1) overflow |= assign_round(L, p, p < wp1, ev[r], wv[r], h);
  }
  overflow |= row_map_padding(L, pad_s, psum_s, (int64_t)c * W + warp, (int64_t)C * W);
  if (overflow) atomicOr(L.d.status, kStatusCapacity);
  return true;
}

// ------------------------------------------------------------------------------------ replicated
// The layout of one chunk with no grid-wide step, for the one-launch layout + dispatch of small
// batches.  Every CTA of the launch counts all T * k pairs of the batch itself (the routing table
// comes from DRAM once, then from L2), packing per expert (pairs << 16) | (pairs before the
// chunk) into one shared-memory atomic, so it knows every expert's total and its chunk's offset
// inside each expert without reading another CTA's counts; psum follows as in block_psum, and
// the chunk's pairs are assigned from there.  The chunk is tokens [t0, t1) with (t1 - t0) * k <=
// g.n (one round of 32 pairs per warp), and T * k < 2^16 for the packed counts.
//   publish  (one CTA) writes cnt, psum, pad_excl, rows_per_rank and the capacity and bad-id flags;
//   every CTA adds its chunk's per-rank token counts to tokens_per_rank (cleared before the
//   launch), writes token_in_rank, slot, pair rank / weight and the row maps of its chunk's pairs
//   (and the slot, rank and weight of chunk pair j into rec_slot[j] / rec_rank[j] / rec_w[j]), and
//   the padding rows' row maps of its share (warps blockIdx.x * W + w over gridDim.x * W).
// Shared memory: sm = fused_layout_smem(E, R, W) bytes; afterwards psum_s (sm + (W + 5) E) and
// pad_s (sm + (W + 6) E) hold psum and pad_excl.
constexpr int kRepLoads = 8;  // loads (of two routing ids each) in flight per thread in the batch-wide count

__device__ __forceinline__ void replicated_layout_chunk(const LayoutLaunch& L, int64_t cap_check, int64_t t0,
                                                        int64_t t1, bool publish, const ThreadGroup& g, int32_t* sm,
                                                        int32_t* rec_slot, int32_t* rec_rank, float* rec_w) {
  const int E = L.E, R = L.R, tid = g.tid, warp = tid >> 5, W = g.n >> 5;
  int32_t* whist = sm;                        // [W][E]  per-warp histograms of the chunk, then bases
  int32_t* hist = whist + W * E;              // [E]  expert totals
  int32_t* off = hist + E;                    // [E]  packed counts, then the pairs before the chunk
  int32_t* al = off + E;                      // [E]
  int32_t* pad = al + E;                      // [E]
  int32_t* gincl = pad + E;                   // [E]
  int32_t* psum_s = gincl + E;                // [E]
  int32_t* pad_s = psum_s + E;                // [E + 1]
  int32_t* tok = pad_s + E + 1;               // [R]

  // the chunk's pairs, one per thread (warp w: pairs p0 + 32 w + lane)
  const int64_t p0 = t0 * L.k, np = (t1 - t0) * L.k;
  const int64_t p = p0 + tid;
  const bool mine = tid < np;
  int32_t ev = -1;
  float wv = 0.0f;
  bool ok = true;
  if (mine) {
    const int32_t e = expert_of(__ldg(L.idx + p), E);
    ok = e != -2;
    ev = max(e, -1);
    wv = L.w ? __ldg(L.w + p) : 0.0f;
  }
  if (mine) rec_w[tid] = wv;
  for (int i = tid; i < W * E; i += g.n) whist[i] = 0;
  for (int e = tid; e < E; e += g.n) off[e] = 0;
  for (int r = tid; r < R; r += g.n) tok[r] = 0;
  g.sync();

  // 1. every pair of the batch: (1 << 16) | (q < p0) into off[e]; two ids per 16-byte load when
  // the table is 16-byte aligned (kRepLoads loads in flight per thread)
  const int64_t NP = L.T * L.k;
  bool bad = false;
  const bool vec = (reinterpret_cast<uintptr_t>(L.idx) & 15u) == 0;
  const int64_t NV = vec ? NP / 2 : 0;  // ids [0, 2 NV) by pairs, the rest one by one
  const longlong2* idx2 = reinterpret_cast<const longlong2*>(L.idx);
  for (int64_t v0 = 0; v0 < NV; v0 += (int64_t)g.n * kRepLoads) {
    longlong2 ii[kRepLoads];
#pragma unroll
    for (int u = 0; u < kRepLoads; ++u) {
      const int64_t v = v0 + (int64_t)u * g.n + tid;
      ii[u] = v < NV ? __ldg(idx2 + v) : make_longlong2(-1, -1);
    }
#pragma unroll
    for (int u = 0; u < kRepLoads; ++u) {
      const int64_t q = 2 * (v0 + (int64_t)u * g.n + tid);
      const int32_t ea = expert_of(ii[u].x, E), eb = expert_of(ii[u].y, E);
      bad |= (ea == -2) | (eb == -2);
      if (ea >= 0) atomicAdd_block(&off[ea], (1 << 16) | (q < p0 ? 1 : 0));
      if (eb >= 0) atomicAdd_block(&off[eb], (1 << 16) | (q + 1 < p0 ? 1 : 0));
    }
  }
  for (int64_t q0 = 2 * NV; q0 < NP; q0 += (int64_t)g.n * kRepLoads) {
    int32_t ee[kRepLoads];
#pragma unroll
    for (int u = 0; u < kRepLoads; ++u) {
      const int64_t q = q0 + (int64_t)u * g.n + tid;
      ee[u] = q < NP ? expert_of(__ldg(L.idx + q), E) : -1;
    }
#pragma unroll
    for (int u = 0; u < kRepLoads; ++u) {
      const int64_t q = q0 + (int64_t)u * g.n + tid;
      bad |= ee[u] == -2;
      if (ee[u] >= 0) atomicAdd_block(&off[ee[u]], (1 << 16) | (q < p0 ? 1 : 0));
    }
  }
  if (publish && bad) atomicOr(L.d.status, kStatusBadExpert);
  // 2. the chunk: per-warp histograms (every warp takes part in the match), token membership
  histogram_round(ev, whist + warp * E);
  for (int64_t tb = t0; tb < t1; tb += g.n) {  // same trip count for every thread
    const int64_t t = tb + tid;
    ok &= token_membership(L, t, t < t1, nullptr, tok);
  }
  if (!ok) atomicOr(L.d.status, kStatusBadExpert);
  g.sync();
  for (int e = tid; e < E; e += g.n) {
    const int32_t v = off[e];
    hist[e] = v >> 16;
    off[e] = v & 0xFFFF;
  }
  for (int r = tid; r < R; r += g.n)
    if (tok[r]) atomicAdd(L.d.tokens_per_rank + r, tok[r]);  // integer sum: order-free
  g.sync();
  block_psum<false>(L, hist, cap_check, al, pad, gincl, pad_s, psum_s, publish, g);
  if (publish)
    for (int e = tid; e < E; e += g.n) L.d.cnt[e] = hist[e];

  // 3. assign: warp bases from the expert's segment start and the chunk's offset, then the pairs
  for (int e = tid; e < E; e += g.n) {
    int32_t base = psum_s[e] - al[e] + off[e];
    for (int w = 0; w < W; ++w) {
      const int32_t v = whist[w * E + e];
      whist[w * E + e] = base;
      base += v;
    }
  }
  g.sync();
  bool overflow = assign_round(L, p, mine, ev, wv, whist + warp * E, rec_slot, rec_rank, tid);
  overflow |= row_map_padding(L, pad_s, psum_s, (int64_t)blockIdx.x * W + warp, (int64_t)gridDim.x * W);
  if (overflow) atomicOr(L.d.status, kStatusCapacity);
}

}  // namespace moe
