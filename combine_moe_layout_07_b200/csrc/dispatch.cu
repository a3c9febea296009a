// dispatch.cu -- gather each routed token's hidden vector into the expert-major receive
// buffers, optionally quantising BF16 -> FP8 E4M3 with 1x128 block scales on the way.
//
// Follows "From DeepEP to Mega MoE" (backyes.github.io) 2.2 (dispatch warps: a token is loaded
// once with a 1-D TMA copy into shared memory and stored from there to each destination) and
// 2.4 (copy epilogue: the row lands at its position inside its expert's range), with
// do_expand / do_zero_padding of "Why MoE gets stuck on communication" (locsic.com) section 1 and
// FP8 dispatch of "DeepEP expert-parallel communication" (blog.hotdry.top), key techniques.
//
// B200 mapping (HBM-bound data movement, one CTA per SM so num_sms caps SMs):
//   warp 0      producer: per token, computes the destination rows from the handle and issues
//               one cp.async.bulk load of the bf16 row into a ring of shared-memory stages
//               (mbarrier full/empty pairs), so several rows per SM are always in flight;
//   warps 1..16 two consumer groups of 8 warps take alternate tokens; they read the staged row
//               from shared memory and write it, from registers,
//               to each of its k destination rows with 16-byte evict-first stores.  FP8: eight
//               lanes own a 1x128 block, amax by three xor-shuffles, inv = 448/a and a/448 as IEEE
//               divisions, codes by cvt.rn.satfinite.e4m3x2.  Each warp releases the stage on its
//               mbarrier when done.
//   Padding rows are zeroed by the consumer warps after the tokens, a warp per row.
// Every wait is an mbarrier try_wait bounded by wall-clock time (status kStatusTimeout on
// expiry); there are no named barriers.
#include "moe_internal.cuh"

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

__device__ __forceinline__ int find_padding_expert(const int32_t* pad_excl, int E, int32_t i) {
  int lo = 0, hi = E;  // largest e with pad_excl[e] <= i
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(pad_excl + mid) <= i) lo = mid;
    else hi = mid;
  }
  return lo;
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
  const uint16_t* x = static_cast<const uint16_t*>(L.x);

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

  int64_t t_begin, t_end;
  cta_token_range(L.T, t_begin, t_end);
  const int64_t n_items = t_end - t_begin;
  bool overflow = false;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // pair metadata for tpb tokens per warp-wide load, prefetched one batch ahead
    const int tpb = 32 / L.k, lanes_used = tpb * L.k;
    const int64_t p_end = t_end * L.k;
    const float* wsrc = L.scale_w ? L.scale_w : L.pair_w;
    const bool views = L.recv_topk_idx || L.recv_topk_w;  // by-rank per-row top-k views
    const int64_t* ids = views ? L.topk_idx : nullptr;
    PairBatch cur = load_pair_batch(L.pair_rank, L.slot, wsrc, t_begin * L.k, p_end, lane, lanes_used, ids);
    int64_t i = 0;
    int s = 0;
    uint32_t par = 0;  // (i / S) & 1
    bool stop = false;
    for (int64_t tb = t_begin; tb < t_end && !stop; tb += tpb) {
      const PairBatch nxt =
          load_pair_batch(L.pair_rank, L.slot, wsrc, (tb + tpb) * L.k, p_end, lane, lanes_used, ids);
      const int nt = (int)min((int64_t)tpb, t_end - tb);
      for (int q = 0; q < nt; ++q) {
        const int64_t t = tb + q;
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
          if (dbg_ok(t < L.T && lay.in + (uint32_t)(s + 1) * in_bytes <= lay.total, L.status, 201, t))
            bulk_load(base + lay.in + (uint32_t)s * in_bytes, x + t * H, in_bytes, full0 + 8 * s);
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
          const float scale = __fdiv_rn(am, 448.0f);
          uint32_t qw[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t lo = pack_e4m3x2(__fmul_rn(v[4 * q], inv), __fmul_rn(v[4 * q + 1], inv));
            const uint32_t hi = pack_e4m3x2(__fmul_rn(v[4 * q + 2], inv), __fmul_rn(v[4 * q + 3], inv));
            qw[q] = lo | (hi << 16);
          }
          if (act) {
            const uint4 qv = make_uint4(qw[0], qw[1], qw[2], qw[3]);
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

    // ---------------------------------------------------------------- padding rows, a warp per row
    if (L.zero_padding || L.recv_w) {
      const int32_t total_pad = __ldg(L.pad_excl + L.E);
      const int64_t row_bytes = kFp8 ? H : 2 * H;
      const int64_t gw = (int64_t)blockIdx.x * kDispConsumerWarps + (ctid >> 5);
      for (int64_t i = gw; i < total_pad; i += (int64_t)gridDim.x * kDispConsumerWarps) {
        const int e = find_padding_expert(L.pad_excl, L.E, (int32_t)i);
        const int32_t pad_e = __ldg(L.pad_excl + e + 1) - __ldg(L.pad_excl + e);
        const int32_t row = __ldg(L.psum + e) - pad_e + ((int32_t)i - __ldg(L.pad_excl + e));
        if (row >= L.cap) {
          overflow = true;
          continue;
        }
        const int64_t grow = (int64_t)(e / L.E_loc) * L.cap + row;
        if (!dbg_ok(row >= 0 && grow < L.R * L.cap, L.status, 204, grow)) continue;
        if (L.zero_padding) {
          uint8_t* dst = static_cast<uint8_t*>(L.recv_x) + grow * row_bytes;
          for (int64_t o = lane * 16; o < row_bytes; o += 32 * 16) st_stream_v4(dst + o, make_uint4(0, 0, 0, 0));
          if (kFp8)
            for (int64_t b = lane; b < nblk; b += 32) L.recv_scales[grow * nblk + b] = 0.0f;
        }
        if (L.recv_w && lane == 0) L.recv_w[grow] = 0.0f;
      }
    }
  }
  if (overflow) atomicOr(L.status, kStatusCapacity);
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

cudaError_t launch_dispatch(const DispatchLaunch& L, bool fp8, cudaStream_t st) {
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
