// dispatch.cu -- gather each routed token's hidden vector into the expert-major receive
// buffers, optionally quantising BF16 -> FP8 E4M3 with 1x128 block scales on the way.
//
// Follows "From DeepEP to Mega MoE" (backyes.github.io) 2.2 (dispatch warps: a token is loaded
// once with a 1-D TMA copy into shared memory and stored from there to each destination) and
// 2.4 (copy epilogue: the row lands at its position inside its expert's range), with
// do_expand / do_zero_padding of "Why MoE gets stuck on communication" (locsic.com) section 1 and
// FP8 dispatch of "DeepEP expert-parallel communication" (blog.hotdry.top), key techniques.
//
// B200 mapping (HBM-bound data movement, one CTA per SM so num_sms caps SMs).  CTA b of G takes
// tokens b, b + G, b + 2G, ...: at any moment the grid works on neighbouring tokens, so the rows
// it writes into each expert's range lie close together (consecutive tokens of an expert own
// consecutive rows), and x is read front to back.  Two kernels share the producer
// (dispatch_producer):
//   k_dispatch_bulk   every dispatch except the weight-scaled rows of the combine backward.  A
//                     storer warp writes each row to its destinations with cp.async.bulk stores
//                     from shared memory (BF16: straight from the loaded stage; FP8: from an
//                     output stage the quantising consumer warps fill); see its own comment.
//   k_dispatch        the register-store form, for rows that differ per destination
//                     (bf16(w * g) of the backward).  Warp 0 is the producer: per token it
//                     computes the destination rows from the handle and issues one
//                     cp.async.bulk load of the bf16 row into a ring of shared-memory stages
//                     (mbarrier full/empty pairs); warps 1..16 form two consumer groups of 8 warps
//                     that take alternate tokens, read the staged row and write it, from
//                     registers, to each destination with 16-byte evict-first stores.
//   FP8 (both): eight lanes own a 1x128 block, amax by three xor-shuffles, inv = 448/a and a/448
//   as IEEE divisions, codes by cvt.rn.satfinite.e4m3x2.
//   Padding rows: k_dispatch_bulk's consumer groups zero one row of the CTA's share after each
//   token they quantise (the rest after the tokens); k_dispatch zeroes them after the tokens, a
//   warp per row.
// Every wait is an mbarrier try_wait bounded by wall-clock time (status kStatusTimeout on
// expiry); there are no named barriers.
#include "layout_body.cuh"

namespace moe {

constexpr int kDispGroups = 2;        // consumer groups take alternate tokens
constexpr int kDispGroupWarps = 8;    // warps per consumer group
constexpr int kDispConsumerWarps = kDispGroups * kDispGroupWarps;
constexpr int kDispGroupThreads = 32 * kDispGroupWarps;
constexpr int kDispConsumers = 32 * kDispConsumerWarps;
constexpr int kDispThreads = 32 + kDispConsumers;
constexpr int kDispMaxStages = 8;
constexpr uint32_t kSmemBudget = 200 * 1024;

struct DispMeta {
  int64_t row[kMaxTopk];   // destination rows (rank * cap + slot) of the valid pairs, in j order
  float w[kMaxTopk];       // their topk weights
  int32_t rank[kMaxTopk];  // their logical ranks
  int32_t n;
  int32_t pad_[3];
};

struct DispSmem {
  uint32_t full, empty, meta, in, total;
};

__host__ __device__ inline uint32_t round_to(uint32_t n, uint32_t a) { return (n + a - 1) / a * a; }

__host__ __device__ inline DispSmem disp_smem(int64_t H, int stages) {
  DispSmem s;
  uint32_t off = 0;
  s.full = off;
  off += 8 * stages;
  s.empty = off;
  off += 8 * stages;
  off = round_to(off, 16);
  s.meta = off;
  off += (uint32_t)sizeof(DispMeta) * stages;
  off = round_to(off, 128);
  s.in = off;
  off += (uint32_t)(2 * H) * stages;
  s.total = off;
  return s;
}

// A walk over the padding rows of all experts in increasing index i (0 <= i < pad_excl[E], the
// padding prefix over experts): one binary search for the first row, then a step per expert
// crossed.  The arrays are the handle's (global memory, read through L1) or, with kShared, a
// CTA's own copy in shared memory (the one-launch layout + dispatch, which computes them itself).
struct PadCursor {
  int e;                     // expert of the current row
  int32_t begin, end, last;  // pad_excl[e], pad_excl[e + 1], psum[e]
  const int32_t* pad_excl;
  const int32_t* psum;
};

template <bool kShared>
__device__ __forceinline__ int32_t ld_layout(const int32_t* p) {
  if constexpr (kShared) return *p;
  else return __ldg(p);
}

template <bool kShared>
__device__ __forceinline__ PadCursor pad_seek(const DispatchLaunch& L, const int32_t* pad_excl, const int32_t* psum,
                                              int32_t i) {
  int lo = 0, hi = L.E;  // largest e with pad_excl[e] <= i
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ld_layout<kShared>(pad_excl + mid) <= i) lo = mid;
    else hi = mid;
  }
  return PadCursor{lo, ld_layout<kShared>(pad_excl + lo), ld_layout<kShared>(pad_excl + lo + 1),
                   ld_layout<kShared>(psum + lo), pad_excl, psum};
}

// Receive-buffer row (rank * cap + row) of padding row i, at or after the cursor's row; -1 when it
// lies at or beyond cap.  Expert e's padding rows are [psum[e] - pad_e, psum[e]) of its rank.
template <bool kShared>
__device__ __forceinline__ int64_t pad_row(const DispatchLaunch& L, PadCursor& c, int32_t i) {
  while (i >= c.end) {
    ++c.e;
    c.begin = c.end;
    c.end = ld_layout<kShared>(c.pad_excl + c.e + 1);
    c.last = ld_layout<kShared>(c.psum + c.e);
  }
  const int32_t row = c.last - (c.end - c.begin) + (i - c.begin);
  return row < L.cap ? (int64_t)(c.e / L.E_loc) * L.cap + row : -1;
}

// The producer warp of both dispatch kernels: pair metadata for tpb items per warp-wide load,
// prefetched one batch ahead; per item, waits for its stage to be free, writes the destination
// rows into the stage's DispMeta (and, by rank, the per-row top-k views) and issues one bulk load
// of the token's bf16 row.  Stage s of item i is i % S, phase (i / S) & 1.
__device__ __forceinline__ void dispatch_producer(const DispatchLaunch& L, int S, uint32_t full0, uint32_t empty0,
                                                  DispMeta* meta, uint32_t in_smem, int64_t n_items, int lane,
                                                  bool& overflow) {
  const int64_t H = L.H;
  const uint32_t in_bytes = (uint32_t)(2 * H);
  const uint16_t* x = static_cast<const uint16_t*>(L.x);
  const int tpb = 32 / L.k, lanes_used = tpb * L.k;
  const float* wsrc = L.scale_w ? L.scale_w : L.pair_w;
  const bool views = L.recv_topk_idx || L.recv_topk_w;  // by-rank per-row top-k views
  const int64_t* ids = views ? L.topk_idx : nullptr;
  PairBatch cur = load_cta_pairs(L.pair_rank, L.slot, wsrc, 0, n_items, L.k, lane, lanes_used, ids);
  int64_t i = 0;
  int s = 0;
  uint32_t par = 0;  // (i / S) & 1
  bool stop = false;
  for (int64_t ib = 0; ib < n_items && !stop; ib += tpb) {
    const PairBatch nxt = load_cta_pairs(L.pair_rank, L.slot, wsrc, ib + tpb, n_items, L.k, lane, lanes_used, ids);
    const int nt = (int)min((int64_t)tpb, n_items - ib);
    for (int q = 0; q < nt; ++q) {
      const int64_t t = cta_token(ib + q);
      if (i >= S) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(empty0 + 8 * s, par ^ 1u, L.status);
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          stop = true;
          break;
        }
      }
      int64_t row = -1;
      if (lane >= q * L.k && lane < (q + 1) * L.k && cur.rank >= 0 && cur.slot >= 0) {  // by-rank rows: -1 on repeats
        if (cur.slot < L.cap) row = (int64_t)cur.rank * L.cap + cur.slot;
        else overflow = true;
      }
      const uint32_t m = __ballot_sync(0xffffffffu, row >= 0);
      if (row >= 0) {
        const int pos = __popc(m & lanemask_lt());
        meta[s].row[pos] = row;
        meta[s].w[pos] = cur.w;
        meta[s].rank[pos] = cur.rank;
      }
      if (lane == 0) meta[s].n = __popc(m);
      __syncwarp();
      if (views) {  // by-rank: each destination row gets the token's k ids / weights for its rank
        const bool mine = lane >= q * L.k && lane < (q + 1) * L.k;
        const int jj = lane - q * L.k;
        const int n = __popc(m);
        for (int d = 0; d < n; ++d) {
          const int64_t row_d = meta[s].row[d];
          const int r_d = meta[s].rank[d];
          if (mine) {
            const bool on = cur.rank == r_d;  // this choice of the token lives on rank r_d
            if (L.recv_topk_idx) L.recv_topk_idx[row_d * L.k + jj] = on ? cur.e - r_d * L.E_loc : -1;
            if (L.recv_topk_w) L.recv_topk_w[row_d * L.k + jj] = on ? cur.w : 0.0f;
          }
        }
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(full0 + 8 * s, in_bytes);
        if (dbg_ok(t < L.T && s < S, L.status, 201, t))
          bulk_load(in_smem + (uint32_t)s * in_bytes, x + t * H, in_bytes, full0 + 8 * s);
      }
      __syncwarp();
      ++i;
      if (++s == S) {
        s = 0;
        par ^= 1u;
      }
    }
    cur = nxt;
  }
  // no load of this CTA may still be in flight when it exits: wait for the last S tokens
  if (lane == 0) {
    int ss = s;
    uint32_t pp = par;
    for (int64_t j = 0; j < min(i, (int64_t)S); ++j) {
      if (--ss < 0) {
        ss = S - 1;
        pp ^= 1u;
      }
      mbar_wait(full0 + 8 * ss, pp, L.status);
    }
  }
}

// An L2 policy that marks lines for eviction first: the receive rows are written once and read
// only by a later kernel, so their lines go back to HBM soon after they are written, in about
// the order the grid writes them.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void bulk_store_hinted(void* dst, uint32_t src_smem, uint32_t bytes, uint64_t pol) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(dst),
               "r"(src_smem), "r"(bytes), "l"(pol)
               : "memory");
}

// Receive-buffer row grow (a padding row), zeroed by the nth threads gtid of a group: codes or
// bf16 row in 16-byte stores, FP8 scales, receive weight 0.
template <bool kFp8>
__device__ __forceinline__ void zero_padding_row(const DispatchLaunch& L, int64_t grow, int gtid, int nth) {
  const int64_t H = L.H, nblk = H / 128;
  const int64_t row_bytes = kFp8 ? H : 2 * H;
  if (!dbg_ok(grow >= 0 && grow < L.R * L.cap, L.status, 204, grow)) return;
  if (L.zero_padding) {
    uint8_t* dst = static_cast<uint8_t*>(L.recv_x) + grow * row_bytes;
    for (int64_t o = (int64_t)gtid * 16; o < row_bytes; o += (int64_t)nth * 16) st_stream_v4(dst + o, make_uint4(0, 0, 0, 0));
    if (kFp8)
      for (int64_t b = gtid; b < nblk; b += nth) L.recv_scales[grow * nblk + b] = 0.0f;
  }
  if (L.recv_w && gtid == 0) L.recv_w[grow] = 0.0f;
}

// Padding rows (zero_padding: zero codes and scales; recv_w: weight 0), a warp per row: warp gw of
// nw warps in the grid takes the contiguous run [gw * P / nw, (gw + 1) * P / nw) of the P rows.
// A block of zero bytes in shared memory from which padding rows are written by bulk (TMA)
// stores: one instruction per kZeroBytes instead of a 16-byte store per thread and step.
constexpr uint32_t kZeroBytes = 4096;

// Receive-buffer row grow (a padding row), zeroed by one warp: lane 0 issues bulk stores of the
// zero block for the codes or bf16 row and, when the scale row is 16-byte aligned, for the FP8
// scales (else the lanes store them), writes the receive weight 0, and commits one bulk group.
// The zero block stays unchanged, so the stores need no wait until the CTA exits.
template <bool kFp8>
__device__ __forceinline__ void zero_padding_row_bulk(const DispatchLaunch& L, int64_t grow, uint32_t zero_smem,
                                                      int lane) {
  const int64_t H = L.H, nblk = H / 128;
  const int64_t row_bytes = kFp8 ? H : 2 * H;
  if (!dbg_ok(grow >= 0 && grow < L.R * L.cap, L.status, 204, grow)) return;
  const bool bulk_scales = kFp8 && (nblk % 4) == 0 && (reinterpret_cast<uintptr_t>(L.recv_scales) & 15) == 0;
  if (L.zero_padding) {
    if (lane == 0) {
      uint8_t* dst = static_cast<uint8_t*>(L.recv_x) + grow * row_bytes;
      for (int64_t o = 0; o < row_bytes; o += kZeroBytes)
        bulk_store(dst + o, zero_smem, (uint32_t)min((int64_t)kZeroBytes, row_bytes - o));
      if (bulk_scales) bulk_store(L.recv_scales + grow * nblk, zero_smem, (uint32_t)(4 * nblk));
      bulk_commit();
    }
    if (kFp8 && !bulk_scales)
      for (int64_t b = lane; b < nblk; b += 32) L.recv_scales[grow * nblk + b] = 0.0f;
  }
  if (L.recv_w && lane == 0) L.recv_w[grow] = 0.0f;
}

template <bool kFp8>
__device__ __forceinline__ void zero_padding_rows(const DispatchLaunch& L, int64_t gw, int64_t nw, int lane,
                                                  bool& overflow) {
  if (!L.zero_padding && !L.recv_w) return;
  const int64_t P = __ldg(L.pad_excl + L.E);
  const int32_t i0 = (int32_t)(P * gw / nw), i1 = (int32_t)(P * (gw + 1) / nw);
  if (i0 >= i1) return;
  PadCursor c = pad_seek<false>(L, L.pad_excl, L.psum, i0);
  for (int32_t i = i0; i < i1; ++i) {
    const int64_t grow = pad_row<false>(L, c, i);
    if (grow < 0) overflow = true;
    else zero_padding_row<kFp8>(L, grow, lane, 32);
  }
}

// FP8 E4M3 codes of the 16 bf16 values of unit u (bytes 32u .. 32u + 31) of a staged row.  Eight
// consecutive lanes hold one 1x128 block: amax over the block by three xor-shuffles, a =
// max(amax, 1e-4), inv = 448 / a and scale = a / 448 as IEEE divisions, codes =
// satfinite(v * inv) rounded to nearest even.  Call with the whole warp; a lane with act = false
// reads nothing and adds zeros to its block's amax.
__device__ __forceinline__ uint4 quantize_unit(uint32_t in_s, int64_t u, bool act, float& scale) {
  uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
  if (act) {
    a = lds_v4(in_s + (uint32_t)u * 32);
    b = lds_v4(in_s + (uint32_t)u * 32 + 16);
  }
  const uint32_t wd[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  float v[16];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    v[2 * q] = bf16lo(wd[q]);
    v[2 * q + 1] = bf16hi(wd[q]);
  }
  float amax = 0.0f;
#pragma unroll
  for (int q = 0; q < 16; ++q) amax = fmaxf(amax, fabsf(v[q]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
  const float am = fmaxf(amax, 1e-4f);
  const float inv = __fdiv_rn(448.0f, am);
  scale = __fdiv_rn(am, 448.0f);
  uint32_t qw[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t lo = pack_e4m3x2(__fmul_rn(v[4 * q], inv), __fmul_rn(v[4 * q + 1], inv));
    const uint32_t hi = pack_e4m3x2(__fmul_rn(v[4 * q + 2], inv), __fmul_rn(v[4 * q + 3], inv));
    qw[q] = lo | (hi << 16);
  }
  return make_uint4(qw[0], qw[1], qw[2], qw[3]);
}

template <bool kFp8>
__global__ void __launch_bounds__(kDispThreads, 1) k_dispatch(DispatchLaunch L, int S) {
  extern __shared__ __align__(128) unsigned char smem[];
  const DispSmem lay = disp_smem(L.H, S);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = smem_u32(smem);
  const uint32_t full0 = base + lay.full, empty0 = base + lay.empty;
  DispMeta* meta = reinterpret_cast<DispMeta*>(smem + lay.meta);
  const int64_t H = L.H;
  const uint32_t in_bytes = (uint32_t)(2 * H);
  const int64_t nblk = H / 128;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kDispGroupWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  grid_dependents_launch();
  grid_dependency_wait();  // the handle written by the layout kernels

  const int64_t n_items = cta_tokens(L.T);
  bool overflow = false;

  if (warp == 0) {
    dispatch_producer(L, S, full0, empty0, meta, base + lay.in, n_items, lane, overflow);
  } else {
    // ---------------------------------------------------------------- consumers
    const int ctid = tid - 32;
    const int grp = (warp - 1) / kDispGroupWarps;
    const int gtid = ctid - grp * kDispGroupThreads;
    int s = grp % S;
    uint32_t par = (uint32_t)((grp / S) & 1);
    for (int64_t i = grp; i < n_items; i += kDispGroups) {
      if (!mbar_wait_warp(full0 + 8 * s, par, L.status)) break;
      const DispMeta& M = meta[s];
      const int n = M.n;
      if (!dbg_ok(n >= 0 && n <= L.k, L.status, 205, n)) break;
      const uint32_t in_s = base + lay.in + (uint32_t)s * in_bytes;
      if constexpr (kFp8) {
        const int64_t nunits = H / 16;  // 16 elements per lane and pass; 8 lanes per 1x128 block
        for (int64_t u = gtid; u - gtid < nunits; u += kDispGroupThreads) {
          const bool act = u < nunits;
          float scale;
          const uint4 qv = quantize_unit(in_s, u, act, scale);
          if (act) {
            for (int j = 0; j < n; ++j) {
              const int64_t row = M.row[j];
              if (!dbg_ok(row >= 0 && row < L.R * L.cap && u * 16 + 16 <= H, L.status, 202, row)) continue;
              st_stream_v4(static_cast<uint8_t*>(L.recv_x) + row * H + u * 16, qv);
              if ((gtid & 7) == 0) L.recv_scales[row * nblk + u / 8] = scale;
            }
          }
        }
      } else {
        const int64_t nvec = H / 8;  // 16-byte vectors per bf16 row
        for (int64_t v = gtid; v < nvec; v += kDispGroupThreads) {
          const uint4 d = lds_v4(in_s + (uint32_t)v * 16);
          for (int j = 0; j < n; ++j) {
            if (!dbg_ok(M.row[j] >= 0 && M.row[j] < L.R * L.cap, L.status, 203, M.row[j])) continue;
            uint4 o = d;
            if (L.scale_w) {  // backward of a weighted combine: bf16(w * g), one fp32 multiply
              const float wj = M.w[j];
              o.x = pack_bf16x2(__fmul_rn(wj, bf16lo(d.x)), __fmul_rn(wj, bf16hi(d.x)));
              o.y = pack_bf16x2(__fmul_rn(wj, bf16lo(d.y)), __fmul_rn(wj, bf16hi(d.y)));
              o.z = pack_bf16x2(__fmul_rn(wj, bf16lo(d.z)), __fmul_rn(wj, bf16hi(d.z)));
              o.w = pack_bf16x2(__fmul_rn(wj, bf16lo(d.w)), __fmul_rn(wj, bf16hi(d.w)));
            }
            st_stream_v4(static_cast<uint16_t*>(L.recv_x) + M.row[j] * H + v * 8, o);
          }
        }
      }
      if (L.recv_w && gtid < n) L.recv_w[M.row[gtid]] = M.w[gtid];
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
      s += kDispGroups;
      while (s >= S) {
        s -= S;
        par ^= 1u;
      }
    }

    zero_padding_rows<kFp8>(L, blockIdx.x * kDispConsumerWarps + (ctid >> 5), gridDim.x * kDispConsumerWarps, lane,
                            overflow);
  }
  if (overflow) atomicOr(L.status, kStatusCapacity);
}

// ------------------------------------------------------------------------------------------------
// Bulk-store dispatch: every dispatch except the weight-scaled rows of the combine backward.  The
// rows leave shared memory through cp.async.bulk stores (the TMA unit writes them; no register
// traffic), which keeps more bytes in flight per SM than 16-byte register stores.
//   warp 0      producer (dispatch_producer): metadata + one bulk load per token, input ring of S;
//   warp 1      storer: tokens in order; lanes 0..n-1 each issue one bulk store of the row to
//               their destination (BF16: straight from the input stage; FP8: from the output
//               stage the consumers filled), and write recv_w; every lane commits a bulk group
//               per token, so after cp.async.bulk.wait_group.read kBulkLag the stage of the token
//               kBulkLag places back has been read and is handed back;
//   warps 2..17 FP8: two consumer groups quantise alternate tokens from the input stage into an
//               output stage (ring of O) and write the 1x128 scales with plain stores (a scale
//               row of H / 128 floats need not be 16-byte aligned).  Each group also zeroes its
//               part of the CTA's padding rows, spread evenly between its tokens; BF16 has
//               nothing to compute, so its groups zero their padding rows from the start.
// The row stores carry an L2 evict-first policy.
// Barriers: full[S] (producer expect_tx, count 1); empty[S] (BF16: the storer; FP8: the group's
// warps + the storer, which reads the stage's metadata); ofull[O] (the group's warps, after
// fence.proxy.async so the bulk engine sees their shared-memory writes); oempty[O] (the storer).
constexpr int kBulkThreads = 64 + kDispConsumers;
constexpr int kBulkMaxIn = 12;  // input stages, a multiple of the consumer-group count
constexpr int kBulkOut = 8;     // FP8 output stages, a multiple of the consumer-group count
constexpr int kBulkLag = 2;     // bulk groups a storer lane leaves reading shared memory

struct BulkSmem {
  uint32_t full, empty, ofull, oempty, meta, in, out, zero, total;
};

__host__ __device__ inline BulkSmem bulk_smem(int64_t H, bool fp8, int S) {
  const int O = fp8 ? kBulkOut : 0;
  BulkSmem b;
  uint32_t off = 0;
  b.full = off;
  off += 8 * S;
  b.empty = off;
  off += 8 * S;
  b.ofull = off;
  off += 8 * O;
  b.oempty = off;
  off += 8 * O;
  off = round_to(off, 16);
  b.meta = off;
  off += (uint32_t)sizeof(DispMeta) * S;
  off = round_to(off, 128);
  b.in = off;
  off += (uint32_t)(2 * H) * S;
  b.out = off;
  off += (uint32_t)H * O;
  off = round_to(off, 128);
  b.zero = off;
  off += kZeroBytes;
  b.total = off;
  return b;
}

template <bool kFp8>
__global__ void __launch_bounds__(kBulkThreads, 1) k_dispatch_bulk(DispatchLaunch L, int S) {
  extern __shared__ __align__(128) unsigned char smem[];
  const BulkSmem lay = bulk_smem(L.H, kFp8, S);
  constexpr int O = kFp8 ? kBulkOut : 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = smem_u32(smem);
  const uint32_t full0 = base + lay.full, empty0 = base + lay.empty;
  const uint32_t ofull0 = base + lay.ofull, oempty0 = base + lay.oempty;
  DispMeta* meta = reinterpret_cast<DispMeta*>(smem + lay.meta);
  const int64_t H = L.H;
  const uint32_t in_bytes = (uint32_t)(2 * H);
  const uint32_t row_bytes = kFp8 ? (uint32_t)H : in_bytes;  // bytes of one destination row

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kFp8 ? kDispGroupWarps + 1 : 1);
    }
    for (int o = 0; o < O; ++o) {
      mbar_init(ofull0 + 8 * o, kDispGroupWarps);
      mbar_init(oempty0 + 8 * o, 1);
    }
    fence_mbar_init();
  }
  for (uint32_t o = (uint32_t)tid * 16; o < kZeroBytes; o += kBulkThreads * 16) sts_v4(base + lay.zero + o, make_uint4(0, 0, 0, 0));
  fence_proxy_async_smem();  // the zero block is read by the bulk engine (async proxy)
  __syncthreads();
  grid_dependents_launch();
  grid_dependency_wait();  // the handle written by the layout kernels

  const int64_t n_items = cta_tokens(L.T);
  bool overflow = false;

  if (warp == 0) {
    dispatch_producer(L, S, full0, empty0, meta, base + lay.in, n_items, lane, overflow);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- storer
    uint8_t* recv = static_cast<uint8_t*>(L.recv_x);
    const uint64_t pol = l2_evict_first_policy();
    int s = 0, o = 0;
    uint32_t par = 0, opar = 0;
    for (int64_t i = 0; i < n_items; ++i) {
      const uint32_t ready = kFp8 ? ofull0 + 8 * o : full0 + 8 * s;
      if (!mbar_wait_warp(ready, kFp8 ? opar : par, L.status)) break;
      const int n = meta[s].n;
      if (!dbg_ok(n >= 0 && n <= L.k, L.status, 206, n)) break;
      const int64_t row = lane < n ? meta[s].row[lane] : -1;
      const float w = lane < n ? meta[s].w[lane] : 0.0f;
      if constexpr (kFp8) {  // the metadata is read: the input stage is the consumers' to release now
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
      }
      if (row >= 0 && dbg_ok(row < L.R * L.cap, L.status, 207, row)) {
        const uint32_t src = kFp8 ? base + lay.out + (uint32_t)o * row_bytes : base + lay.in + (uint32_t)s * in_bytes;
        bulk_store_hinted(recv + row * row_bytes, src, row_bytes, pol);
        if (L.recv_w) L.recv_w[row] = w;
      }
      bulk_commit();
      bulk_wait_read<kBulkLag>();  // the group of token i - kBulkLag has read its stage
      __syncwarp();
      if (lane == 0 && i >= kBulkLag) {
        if constexpr (kFp8) mbar_arrive(oempty0 + 8 * ((o - kBulkLag + O) % O));
        else mbar_arrive(empty0 + 8 * ((s - kBulkLag + S) % S));
      }
      if (++s == S) {
        s = 0;
        par ^= 1u;
      }
      if constexpr (kFp8) {
        if (++o == O) {
          o = 0;
          opar ^= 1u;
        }
      }
    }
    bulk_wait_all();  // no store may still read shared memory when the CTA exits
  } else {
    const int ctid = tid - 64;
    const int grp = (warp - 2) / kDispGroupWarps;
    const int gtid = ctid - grp * kDispGroupThreads;
    // the CTA's share [pb, pe) of the padding rows: FP8, group grp zeroes rows pb + grp, pb + grp +
    // G, .. (G groups), paced over its tokens so that they go out among the token rows; BF16 (no
    // work per token), a warp per row from the start
    const int32_t P = (L.zero_padding || L.recv_w) ? __ldg(L.pad_excl + L.E) : 0;
    const int32_t pb = (int32_t)((int64_t)P * blockIdx.x / gridDim.x);
    const int32_t pe = (int32_t)((int64_t)P * (blockIdx.x + 1) / gridDim.x);
    int32_t pn = pb + grp;
    PadCursor pc{0, 0, 0, 0, L.pad_excl, L.psum};
    if (kFp8 && pn < pe) pc = pad_seek<false>(L, L.pad_excl, L.psum, pn);
    if constexpr (kFp8) {
      // ---------------------------------------------------------------- FP8 consumers
      const int64_t nblk = H / 128, nunits = H / 16;
      const int64_t npad = pn < pe ? (pe - pn + kDispGroups - 1) / kDispGroups : 0;
      const int64_t ntok = n_items > grp ? (n_items - grp + kDispGroups - 1) / kDispGroups : 0;
      int64_t m = 0, pdone = 0;  // tokens and padding rows of this group so far
      int s = grp % S, o = grp % O;
      uint32_t par = (uint32_t)((grp / S) & 1), opar = (uint32_t)((grp / O) & 1);
      for (int64_t i = grp; i < n_items; i += kDispGroups) {
        if (!mbar_wait_warp(full0 + 8 * s, par, L.status)) break;
        if (i >= O && !mbar_wait_warp(oempty0 + 8 * o, opar ^ 1u, L.status)) break;
        const DispMeta& M = meta[s];
        const int n = M.n;
        if (!dbg_ok(n >= 0 && n <= L.k, L.status, 205, n)) break;
        const uint32_t in_s = base + lay.in + (uint32_t)s * in_bytes;
        const uint32_t out_s = base + lay.out + (uint32_t)o * row_bytes;
        for (int64_t u = gtid; u - gtid < nunits; u += kDispGroupThreads) {
          const bool act = u < nunits;
          float scale;
          const uint4 qv = quantize_unit(in_s, u, act, scale);
          if (act) {
            sts_v4(out_s + (uint32_t)u * 16, qv);
            if ((gtid & 7) == 0)
              for (int j = 0; j < n; ++j) {
                const int64_t row = M.row[j];
                if (!dbg_ok(row >= 0 && row < L.R * L.cap, L.status, 202, row)) continue;
                L.recv_scales[row * nblk + u / 8] = scale;
              }
          }
        }
        fence_proxy_async_smem();  // the codes are read next by the bulk engine (async proxy)
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(empty0 + 8 * s);
          mbar_arrive(ofull0 + 8 * o);
        }
        s += kDispGroups;
        while (s >= S) {
          s -= S;
          par ^= 1u;
        }
        o += kDispGroups;
        while (o >= O) {
          o -= O;
          opar ^= 1u;
        }
        for (const int64_t target = ++m * npad / ntok; pdone < target; ++pdone, pn += kDispGroups) {
          const int64_t grow = pad_row<false>(L, pc, pn);
          if (grow < 0) overflow = true;
          else if (gtid < 32) zero_padding_row_bulk<kFp8>(L, grow, base + lay.zero, lane);  // the group's first warp
        }
      }
      for (; pn < pe; pn += kDispGroups) {  // the rows the pacing left
        const int64_t grow = pad_row<false>(L, pc, pn);
        if (grow < 0) overflow = true;
        else if (gtid < 32) zero_padding_row_bulk<kFp8>(L, grow, base + lay.zero, lane);
      }
    } else {  // BF16: warp w of the 16 takes the contiguous run w of the CTA's share
      const int w = ctid >> 5;
      const int32_t i0 = pb + (int32_t)((int64_t)(pe - pb) * w / kDispConsumerWarps);
      const int32_t i1 = pb + (int32_t)((int64_t)(pe - pb) * (w + 1) / kDispConsumerWarps);
      if (i0 < i1) {
        PadCursor c = pad_seek<false>(L, L.pad_excl, L.psum, i0);
        for (int32_t i = i0; i < i1; ++i) {
          const int64_t grow = pad_row<false>(L, c, i);
          if (grow < 0) overflow = true;
          else zero_padding_row_bulk<kFp8>(L, grow, base + lay.zero, lane);
        }
      }
    }
    bulk_wait_all();  // the padding rows' bulk stores read the zero block until they complete
  }
  if (overflow) atomicOr(L.status, kStatusCapacity);
}

// ------------------------------------------------------------------------------------------------
// One-launch layout + dispatch (moe_layout_dispatch without host sync, small batches): the
// layout's notify work and the dispatch in one kernel, as the dispatch kernel of "From DeepEP to
// Mega MoE" 2.2 runs notify warps beside its dispatch warps.  G CTAs of 576 threads, one per SM;
// CTA b owns the chunk of tokens [b * chunk, (b + 1) * chunk) (chunk <= kLdMaxItems, an item and
// a stage per token, no ring).  No CTA waits for another: each computes the layout of its own
// chunk from the whole routing table (replicated_layout_chunk), so the tokens it dispatches are
// the ones whose slots it has just assigned.
//   warp 0       producer: at once, one bulk load of each item's bf16 row (x does not depend on
//                the layout); once the chunk is assigned (the lready barrier), the item's
//                destination rows from the slots the layout recorded in shared memory into its
//                DispMeta, then an arrive on meta[i];
//   warp 1       storer: per item, once its row (BF16: the input stage; FP8: the codes and
//                scales) and its metadata are ready, lanes 0..n-1 each issue one bulk store of
//                the row to a destination and write recv_w; FP8: the lanes copy the scales;
//   warps 2..9   the layout (named barrier 1; CTA 0 publishes the handle's per-expert arrays),
//                then an arrive on lready; then the CTA's share of the padding rows, located from
//                its own psum and padding prefix in shared memory;
//   warps 10..17 FP8: quantise each item into its output stage as soon as its row lands (while
//                the layout runs), the 1x128 scales into shared memory, then exit (the storer
//                writes the scales with the rows).
// Every wait is an mbarrier wait inside the CTA, bounded by wall-clock time.
constexpr int kLdMaxItems = 8;     // items (tokens) per CTA
constexpr int kLdThreads = 576;
constexpr int kLdLayoutBar = 1;    // named barrier of the layout warps

struct LdSmem {
  uint32_t full, qdone, mready, lready, meta, rec, scales, layout, in, out, zero, total;
};

__host__ __device__ inline LdSmem ld_smem(int64_t H, bool fp8, int n, int E, int R) {
  LdSmem l;
  uint32_t off = 0;
  l.full = off;
  off += 8 * n;
  l.qdone = off;
  off += 8 * n;
  l.mready = off;
  off += 8 * n;
  l.lready = off;
  off += 8;
  off = round_to(off, 16);
  l.meta = off;
  off += (uint32_t)sizeof(DispMeta) * n;
  l.rec = off;                          // int32 slot[n * kMaxTopk], rank[n * kMaxTopk], fp32 w[n * kMaxTopk]
  off += 3 * 4 * (uint32_t)(n * kMaxTopk);
  l.scales = off;
  off += fp8 ? (uint32_t)(4 * (H / 128) * n) : 0;
  off = round_to(off, 16);
  l.layout = off;
  off += (uint32_t)fused_layout_smem(E, R, kLayoutWarps);
  off = round_to(off, 128);
  l.in = off;
  off += (uint32_t)(2 * H) * n;
  l.out = off;
  off += fp8 ? (uint32_t)H * n : 0;
  off = round_to(off, 128);
  l.zero = off;
  off += kZeroBytes;
  l.total = off;
  return l;
}

template <bool kFp8>
__global__ void __launch_bounds__(kLdThreads, 1)
    k_layout_dispatch(LayoutLaunch LL, int64_t cap_check, int chunk, DispatchLaunch L) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t H = L.H, nblk = H / 128;
  const int64_t t0 = min((int64_t)blockIdx.x * chunk, L.T), n = min((int64_t)chunk, L.T - t0);
  const LdSmem lay = ld_smem(H, kFp8, kLdMaxItems, LL.E, LL.R);
  const uint32_t base = smem_u32(smem);
  const uint32_t full0 = base + lay.full, qdone0 = base + lay.qdone, mready0 = base + lay.mready;
  const uint32_t lready = base + lay.lready;
  DispMeta* meta = reinterpret_cast<DispMeta*>(smem + lay.meta);
  int32_t* rec_slot = reinterpret_cast<int32_t*>(smem + lay.rec);
  int32_t* rec_rank = rec_slot + kLdMaxItems * kMaxTopk;
  float* rec_w = reinterpret_cast<float*>(rec_rank + kLdMaxItems * kMaxTopk);
  float* scales_s = reinterpret_cast<float*>(smem + lay.scales);
  int32_t* lsm = reinterpret_cast<int32_t*>(smem + lay.layout);
  const uint32_t in_bytes = (uint32_t)(2 * H);
  const uint32_t row_bytes = kFp8 ? (uint32_t)H : in_bytes;

  if (tid == 0) {
    for (int i = 0; i < kLdMaxItems; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(qdone0 + 8 * i, kDispGroupWarps);
      mbar_init(mready0 + 8 * i, 1);
    }
    mbar_init(lready, 1);
    fence_mbar_init();
  }
  for (uint32_t o = (uint32_t)tid * 16; o < kZeroBytes; o += kLdThreads * 16) sts_v4(base + lay.zero + o, make_uint4(0, 0, 0, 0));
  fence_proxy_async_smem();  // the zero block is read by the bulk engine (async proxy)
  __syncthreads();
  grid_dependents_launch();
  grid_dependency_wait();  // the routing and x, and receive buffers earlier kernels may still read
  bool overflow = false;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0)
      for (int64_t i = 0; i < n; ++i) {
        mbar_arrive_expect_tx(full0 + 8 * i, in_bytes);
        if (dbg_ok(i < kLdMaxItems && t0 + i < L.T, L.status, 211, i))
          bulk_load(base + lay.in + (uint32_t)i * in_bytes, static_cast<const uint16_t*>(L.x) + (t0 + i) * H,
                    in_bytes, full0 + 8 * i);
      }
    const bool ok = mbar_wait_warp(lready, 0, L.status);  // the chunk's slots are in rec_*
    for (int64_t i = 0; i < n; ++i) {  // shared memory only
      int64_t row = -1;
      float w = 0.0f;
      if (ok && lane < L.k) {
        const int j = (int)i * L.k + lane;
        const int32_t rk = rec_rank[j], sl = rec_slot[j];
        if (rk >= 0 && sl >= 0) {
          if (sl < L.cap) row = (int64_t)rk * L.cap + sl;
          else overflow = true;
          w = rec_w[j];
        }
      }
      const uint32_t m = __ballot_sync(0xffffffffu, row >= 0);
      if (row >= 0) {
        const int pos = __popc(m & lanemask_lt());
        meta[i].row[pos] = row;
        meta[i].w[pos] = w;
      }
      if (lane == 0) meta[i].n = __popc(m);  // 0 when the layout gave up: nothing is written
      __syncwarp();
      if (lane == 0) mbar_arrive(mready0 + 8 * i);
    }
    // no load of this CTA may still be in flight when it exits
    if (lane == 0)
      for (int64_t i = 0; i < n; ++i) mbar_wait(full0 + 8 * i, 0, L.status);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- storer
    // codes (or bf16 rows): one bulk store per destination; FP8 scales: 16-byte stores by the
    // lanes (4-byte ones when a row of them is not a whole number of 16-byte units or the buffer
    // is not 16-byte aligned), which keeps the bulk-copy queue for the rows
    uint8_t* recv = static_cast<uint8_t*>(L.recv_x);
    const uint64_t pol = l2_evict_first_policy();
    const int64_t sc_units = nblk / 4;  // 16-byte units of a row of scales
    const bool sc_vec = kFp8 && nblk % 4 == 0 && (reinterpret_cast<uintptr_t>(L.recv_scales) & 15u) == 0;
    for (int64_t i = 0; i < n; ++i) {
      if (!mbar_wait_warp(kFp8 ? qdone0 + 8 * i : full0 + 8 * i, 0, L.status)) break;
      if (!mbar_wait_warp(mready0 + 8 * i, 0, L.status)) break;
      const int nd = meta[i].n;
      if (!dbg_ok(nd >= 0 && nd <= L.k, L.status, 212, nd)) break;
      const int64_t row = lane < nd ? meta[i].row[lane] : -1;
      if (row >= 0 && dbg_ok(row < L.R * L.cap, L.status, 213, row)) {
        const uint32_t src = kFp8 ? base + lay.out + (uint32_t)i * row_bytes : base + lay.in + (uint32_t)i * in_bytes;
        bulk_store_hinted(recv + row * row_bytes, src, row_bytes, pol);
        if (L.recv_w) L.recv_w[row] = meta[i].w[lane];
      }
      if (kFp8 && sc_vec)
        for (int64_t x = lane; x < nd * sc_units; x += 32) {
          const int j = (int)(x / sc_units);
          const int64_t u = x - j * sc_units;
          const int64_t r = meta[i].row[j];
          const uint4 v = *reinterpret_cast<const uint4*>(scales_s + i * nblk + 4 * u);
          if (dbg_ok(r >= 0 && r < L.R * L.cap, L.status, 215, r))
            *reinterpret_cast<uint4*>(L.recv_scales + r * nblk + 4 * u) = v;
        }
      else if (kFp8)
        for (int64_t x = lane; x < nd * nblk; x += 32) {
          const int j = (int)(x / nblk);
          const int64_t b = x - j * nblk;
          const int64_t r = meta[i].row[j];
          if (dbg_ok(r >= 0 && r < L.R * L.cap, L.status, 215, r)) L.recv_scales[r * nblk + b] = scales_s[i * nblk + b];
        }
      bulk_commit();
    }
    bulk_wait_all();  // no store may still read shared memory when the CTA exits
  } else if (warp < 10) {
    // ---------------------------------------------------------------- layout, then padding rows
    const ThreadGroup g{tid - 64, kLayoutThreads, kLdLayoutBar};
    replicated_layout_chunk(LL, cap_check, t0, t0 + n, blockIdx.x == 0, g, lsm, rec_slot, rec_rank, rec_w);
    g.sync();  // every pair of the chunk is assigned (its slot recorded) before the arrival
    if (g.tid == 0) mbar_arrive(lready);
    if (L.zero_padding || L.recv_w) {
      const int32_t* pad_s = lsm + (kLayoutWarps + 6) * LL.E;   // pad_excl[E + 1], this CTA's copy
      const int32_t* psum_s = lsm + (kLayoutWarps + 5) * LL.E;  // psum[E]
      const int32_t total = pad_s[LL.E];
      const int32_t pb = (int32_t)((int64_t)total * blockIdx.x / gridDim.x);
      const int32_t pe = (int32_t)((int64_t)total * (blockIdx.x + 1) / gridDim.x);
      const int w = warp - 2;  // warp w of the 8 takes the contiguous run w of the CTA's share
      const int32_t i0 = pb + (int32_t)((int64_t)(pe - pb) * w / kLayoutWarps);
      const int32_t i1 = pb + (int32_t)((int64_t)(pe - pb) * (w + 1) / kLayoutWarps);
      if (i0 < i1) {
        PadCursor c = pad_seek<true>(L, pad_s, psum_s, i0);
        for (int32_t i = i0; i < i1; ++i) {
          const int64_t grow = pad_row<true>(L, c, i);
          if (grow < 0) overflow = true;
          else zero_padding_row_bulk<kFp8>(L, grow, base + lay.zero, lane);
        }
        bulk_wait_all();  // the bulk stores read the zero block until they complete
      }
    }
  } else if (kFp8) {
    // ---------------------------------------------------------------- FP8 quantisers
    const int gtid = tid - 320;
    const int64_t nunits = H / 16;
    for (int64_t i = 0; i < n; ++i) {
      if (!mbar_wait_warp(full0 + 8 * i, 0, L.status)) break;
      const uint32_t in_s = base + lay.in + (uint32_t)i * in_bytes;
      const uint32_t out_s = base + lay.out + (uint32_t)i * row_bytes;
      for (int64_t u = gtid; u - gtid < nunits; u += kDispGroupThreads) {
        const bool act = u < nunits;
        float scale;
        const uint4 qv = quantize_unit(in_s, u, act, scale);
        if (act) {
          sts_v4(out_s + (uint32_t)u * 16, qv);
          if ((gtid & 7) == 0) scales_s[i * nblk + u / 8] = scale;
        }
      }
      fence_proxy_async_smem();  // the codes are read next by the bulk engine (async proxy)
      __syncwarp();
      if (lane == 0) mbar_arrive(qdone0 + 8 * i);
    }
  }
  if (overflow) atomicOr(L.status, kStatusCapacity);
}

// Whether a batch takes the one-launch layout + dispatch: chunks of at most kLdMaxItems tokens,
// one per CTA of the grid, whose pairs fit one round per layout warp (chunk * k <= the layout
// warps' threads), T * k below 2^16 (the packed per-expert counts), and shared memory (the
// layout's arrays, a stage per item) that fits.  Returns the chunk, or 0.
int layout_dispatch_chunk(int64_t T, int64_t H, bool fp8, int E, int R, int grid, int k) {
  if (grid < 1 || T < 1 || T * k >= (int64_t)1 << 16) return 0;
  const int64_t chunk = (T + grid - 1) / grid;
  if (chunk > kLdMaxItems || chunk * k > kLayoutThreads) return 0;
  if (ld_smem(H, fp8, kLdMaxItems, E, R).total > 227u * 1024u - 1024u) return 0;
  return (int)chunk;
}

cudaError_t launch_layout_dispatch(const LayoutLaunch& LL, int64_t cap_check, int chunk, const DispatchLaunch& L,
                                   bool fp8, cudaStream_t st) {
  const uint32_t smem = ld_smem(L.H, fp8, kLdMaxItems, LL.E, LL.R).total;
  if (chunk < 1 || chunk > kLdMaxItems || (int64_t)chunk * LL.k > kLayoutThreads) return cudaErrorInvalidValue;
  auto kern = fp8 ? k_layout_dispatch<true> : k_layout_dispatch<false>;
  static unsigned long long done[2] = {0, 0};
  cudaError_t err = set_smem_limit_once(kern, 227 * 1024 - 1024, &done[fp8 ? 1 : 0]);
  if (err != cudaSuccess) return err;
  const int grid = (int)((L.T + chunk - 1) / chunk);  // every CTA owns a chunk (<= L.grid)
  err = launch_pdl(kern, dim3(grid), dim3(kLdThreads), (size_t)smem, st, LL, cap_check, chunk, L);
  note_launch();
  return err;
}

// The stage count is a multiple of the consumer-group count: stage s is then always consumed by
// group s % G, which observes every phase of its stages in order (a parity wait can only tell
// the current phase from the one before it).
int dispatch_stages(int64_t H) {
  static_assert(kDispMaxStages % kDispGroups == 0, "stages per group");
  for (int s = kDispMaxStages; s >= kDispGroups; s -= kDispGroups)
    if (disp_smem(H, s).total <= kSmemBudget) return s;
  return 0;
}

// Input stages of the bulk-store kernel (a multiple of the group count, more than kBulkLag);
// 0 when not even the smallest ring fits.
int dispatch_bulk_stages(int64_t H, bool fp8) {
  static_assert(kBulkMaxIn % kDispGroups == 0 && kBulkOut % kDispGroups == 0, "stages per group");
  static_assert(kBulkOut > kBulkLag, "the storer hands output stages back kBulkLag tokens late");
  for (int s = kBulkMaxIn; s > kBulkLag; s -= kDispGroups)
    if (bulk_smem(H, fp8, s).total <= kSmemBudget) return s;
  return 0;
}

cudaError_t launch_dispatch(const DispatchLaunch& L, bool fp8, cudaStream_t st) {
  if (!L.scale_w) {
    const int S = dispatch_bulk_stages(L.H, fp8);
    if (S > kBulkLag) {
      const uint32_t smem = bulk_smem(L.H, fp8, S).total;
      static unsigned long long done[2] = {0, 0};
      auto kern = fp8 ? k_dispatch_bulk<true> : k_dispatch_bulk<false>;
      cudaError_t err = set_smem_limit_once(kern, (int)kSmemBudget, &done[fp8 ? 1 : 0]);
      if (err != cudaSuccess) return err;
      err = launch_pdl(kern, dim3(L.grid), dim3(kBulkThreads), smem, st, L, S);
      note_launch();
      return err;
    }
  }
  const int S = dispatch_stages(L.H);
  if (S < kDispGroups) return cudaErrorInvalidValue;
  const uint32_t smem = disp_smem(L.H, S).total;
  static unsigned long long done[2] = {0, 0};
  auto kern = fp8 ? k_dispatch<true> : k_dispatch<false>;
  cudaError_t err = set_smem_limit_once(kern, (int)kSmemBudget, &done[fp8 ? 1 : 0]);
  if (err != cudaSuccess) return err;
  err = launch_pdl(kern, dim3(L.grid), dim3(kDispThreads), smem, st, L, S);
  note_launch();
  return err;
}

}  // namespace moe
