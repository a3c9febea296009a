// combine.cu -- gather the expert outputs back to token order and reduce the top-k rows.
//
// Follows "From DeepEP to Mega MoE" (backyes.github.io) 2.3 / 2.5 (combine_reduce: an
// element-wise sum of a token's top-k expert rows, not a GEMM; rows arrive by 1-D TMA loads) and
// "Why MoE gets stuck on communication" (locsic.com) section 1 (the rows are already weighted;
// the shared expert's output is added as the bias).  Optional per-pair weights are applied in
// fp32 when given.
//
// Numerics, fixed so every run is bit-identical: acc = 0 (fp32); for j = 0..k-1 in order,
// skipping masked pairs, acc = fma(w, y, acc) or acc + y; then acc + bias; one rounding to bf16.
//
// B200 mapping (HBM-bound gather, one CTA per SM so num_sms caps SMs).  CTA b of G takes tokens
// b, b + G, b + 2G, ..., so the grid reads neighbouring tokens together and the rows it gathers
// from each expert's range lie close together (3-4 % faster at DeepSeek-V3 prefill than
// contiguous token ranges per CTA).  A work item is one token and one column chunk of CW
// elements (CW <= 2048, chosen so that several stages fit); in the by-rank combine (packed
// items), a token with n source rows takes (k + bias) / (n + bias) chunks per item, so that its
// rows fill the stage's k (+ bias) row slots:
//   warp 0      producer: reads the token's k (rank, slot) pairs from the handle and issues one
//               cp.async.bulk load per valid source row segment (plus the bias segment) into a
//               stage of a shared-memory ring, completed on the stage's mbarrier;
//   warps 1..16 two consumer groups of 8 warps take alternate items; each thread owns 8
//               columns; it reads the k staged segments in j order from shared memory,
//               accumulates in fp32 registers, adds the bias, rounds and writes 16 bytes of the
//               output row with an evict-first store; each warp releases the stage when done.
// Stage index, phase and (token, chunk) advance as counters (no integer division in the loops).
// All waits are mbarrier try_waits bounded by wall-clock time; there are no named barriers.
#include "moe_internal.cuh"

namespace moe {

constexpr int kCombGroups = 2;         // consumer groups reduce alternate items concurrently
constexpr int kCombGroupWarps = 8;     // warps per consumer group
constexpr int kCombConsumerWarps = kCombGroups * kCombGroupWarps;
constexpr int kCombGroupThreads = 32 * kCombGroupWarps;
constexpr int kCombConsumers = 32 * kCombConsumerWarps;
constexpr int kCombThreads = 32 + kCombConsumers;
constexpr int kCombMaxStages = 8;
constexpr uint32_t kCombSmemBudget = 200 * 1024;

struct CombMeta {
  float w[kMaxTopk];  // weights of the valid pairs in j order (weighted combine)
  int32_t n;          // valid pairs (packed items: -1 ends the consumer group's loop)
  int32_t q, c0, width, stride;  // packed items: the CTA's token index, columns, slot stride in bytes
  int32_t pad_[3];
};

struct CombGeom {
  int64_t cw;        // chunk width in elements (multiple of 8)
  int64_t nch;       // chunks per token
  int slots;         // staged rows per item: k (+1 for the bias)
  int stages;
  uint32_t full, empty, meta, data, stage_bytes, total;
};

__host__ __device__ inline uint32_t cround(uint32_t n, uint32_t a) { return (n + a - 1) / a * a; }

__host__ __device__ inline CombGeom comb_geom(int64_t H, int k, bool bias, int stages, int64_t nch) {
  CombGeom g;
  g.cw = ((H + nch - 1) / nch + 7) / 8 * 8;
  g.nch = (H + g.cw - 1) / g.cw;  // every chunk starts inside the row
  g.slots = k + (bias ? 1 : 0);
  g.stages = stages;
  g.stage_bytes = (uint32_t)(g.slots * g.cw * 2);
  uint32_t off = 0;
  g.full = off;
  off += 8 * stages;
  g.empty = off;
  off += 8 * stages;
  off = cround(off, 16);
  g.meta = off;
  off += (uint32_t)sizeof(CombMeta) * stages;
  off = cround(off, 128);
  g.data = off;
  off += g.stage_bytes * stages;
  g.total = off;
  return g;
}

// Chunks as wide as possible (<= 2048 columns) while at least 4 stages fit (2 for huge k).
// The stage count is a multiple of the consumer-group count: stage s is then always consumed
// by group s % G, which observes every phase of its stages in order (a parity wait can only
// tell the current phase from the one before it).
CombGeom combine_geometry(int64_t H, int k, bool bias) {
  static_assert(kCombMaxStages % kCombGroups == 0 && 4 % kCombGroups == 0, "stages per group");
  int64_t nch = (H + 2047) / 2048;
  for (;;) {
    for (int s = kCombMaxStages; s >= 4; s -= kCombGroups) {
      const CombGeom g = comb_geom(H, k, bias, s, nch);
      if (g.total <= kCombSmemBudget) return g;
    }
    if (comb_geom(H, k, bias, 4, nch).cw <= 8) break;
    ++nch;
  }
  CombGeom g = comb_geom(H, k, bias, kCombGroups, nch);
  if (g.total > kCombSmemBudget) g.stages = 0;
  return g;
}

// kPacked (the by-rank combine, whose tokens gather from at most one row per rank): a token with
// n source rows takes mult = (k + bias) / (n + bias) chunks of columns per item, with its row
// segments mult * cw columns wide, so the item fills the stage's k (+ bias) slots of cw columns
// when n is small.  The item's token, columns and slot stride travel in its CombMeta, and after
// the last item the producer sends one item with n = -1 to each consumer group.
template <bool kWeighted, bool kBias, bool kPacked>
__global__ void __launch_bounds__(kCombThreads, 1) k_combine(CombineLaunch L, CombGeom g) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = smem_u32(smem);
  const uint32_t full0 = base + g.full, empty0 = base + g.empty;
  CombMeta* meta = reinterpret_cast<CombMeta*>(smem + g.meta);
  const int S = g.stages;
  const int64_t H = L.H;
  const uint16_t* y = static_cast<const uint16_t*>(L.y);
  const uint16_t* bias = static_cast<const uint16_t*>(L.bias);
  uint16_t* out = static_cast<uint16_t*>(L.out);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kCombGroupWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  grid_dependents_launch();
  grid_dependency_wait();  // the expert outputs and the handle written by earlier kernels

  // CTA b of G takes tokens b, b + G, ... (token index q of this CTA is token b + q * G): the
  // grid reads neighbouring tokens together, so the rows it gathers from each expert's range
  // lie close together
  const int64_t n_tok = cta_tokens(L.T);
  const int64_t n_items = n_tok * g.nch;
  bool overflow = false;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    const int tpb = 32 / L.k, lanes_used = tpb * L.k;
    const uint32_t slot_bytes = (uint32_t)(g.cw * 2);
    PairBatch cur = load_cta_pairs(L.pair_rank, L.slot, kWeighted ? L.w : nullptr, 0, n_tok, L.k, lane, lanes_used);
    int64_t i = 0;
    int s = 0;
    uint32_t par = 0;  // parity of the stage's current use: (i / S) & 1
    bool stop = false;
    for (int64_t qb = 0; qb < n_tok && !stop; qb += tpb) {
      const PairBatch nxt =
          load_cta_pairs(L.pair_rank, L.slot, kWeighted ? L.w : nullptr, qb + tpb, n_tok, L.k, lane, lanes_used);
      const int nt = (int)min((int64_t)tpb, n_tok - qb);
      for (int q = 0; q < nt && !stop; ++q) {
        const int64_t t = cta_token(qb + q);
        int64_t src = -1;
        if (lane >= q * L.k && lane < (q + 1) * L.k && cur.rank >= 0 && cur.slot >= 0) {  // by-rank rows: -1 on repeats
          if (cur.slot < L.cap) src = ((int64_t)cur.rank * L.cap + cur.slot) * H;
          else overflow = true;
        }
        const uint32_t m = __ballot_sync(0xffffffffu, src >= 0);
        const int pos = __popc(m & lanemask_lt());
        const int n = __popc(m);
        const int nb = kBias ? 1 : 0;
        // (a token without rows, n + nb == 0, loads nothing: its items may span the whole stage)
        const int mult = !kPacked ? 1 : (n + nb > 0 ? max(1, (L.k + nb) / (n + nb)) : max(1, L.k + nb));
        const int64_t span = (int64_t)mult * g.cw;              // columns of one item
        const uint32_t stride = (uint32_t)(span * 2);          // bytes between its row segments
        for (int64_t c0 = 0; c0 < H; c0 += span) {
          const uint32_t bytes = (uint32_t)(min(span, H - c0) * 2);
          if (i >= S) {
            bool ok = true;
            if (lane == 0) ok = mbar_wait(empty0 + 8 * s, par ^ 1u, L.status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) {
              stop = true;
              break;
            }
          }
          if (kWeighted && src >= 0) meta[s].w[pos] = cur.w;
          if (lane == 0) {
            meta[s].n = n;
            if constexpr (kPacked) {
              meta[s].q = (int32_t)(qb + q);
              meta[s].c0 = (int32_t)c0;
              meta[s].width = (int32_t)min(span, H - c0);
              meta[s].stride = (int32_t)stride;
            }
          }
          __syncwarp();
          const uint32_t stage = base + g.data + (uint32_t)s * g.stage_bytes;
          const uint32_t bias_off = kPacked ? (uint32_t)n * stride : (uint32_t)L.k * slot_bytes;
          if (lane == 0) {
            mbar_arrive_expect_tx(full0 + 8 * s, bytes * (uint32_t)(n + nb));
            if (kBias && dbg_ok(t * H + c0 + bytes / 2 <= L.T * H && bias_off + bytes <= g.stage_bytes, L.status, 101, t))
              bulk_load(stage + bias_off, bias + t * H + c0, bytes, full0 + 8 * s);
          }
          __syncwarp();
          if (src >= 0 && dbg_ok(src + c0 + bytes / 2 <= L.R * L.cap * H && pos < L.k &&
                                     (uint32_t)pos * stride + bytes <= g.stage_bytes,
                                 L.status, 102, src))
            bulk_load(stage + (uint32_t)pos * stride, y + src + c0, bytes, full0 + 8 * s);
          __syncwarp();
          ++i;
          if (++s == S) {
            s = 0;
            par ^= 1u;
          }
        }
      }
      cur = nxt;
    }
    if constexpr (kPacked) {  // one item with n = -1 per consumer group ends its loop
      for (int gq = 0; gq < kCombGroups && !stop; ++gq) {
        if (i >= S) {
          bool ok = true;
          if (lane == 0) ok = mbar_wait(empty0 + 8 * s, par ^ 1u, L.status);
          if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        }
        if (lane == 0) {
          meta[s].n = -1;
          mbar_arrive(full0 + 8 * s);
        }
        __syncwarp();
        ++i;
        if (++s == S) {
          s = 0;
          par ^= 1u;
        }
      }
    }
    // no load of this CTA may still be in flight when it exits: wait for the last S items
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
    // ---------------------------------------------------------------- consumer groups
    const int cwarp = warp - 1;
    const int grp = cwarp / kCombGroupWarps;
    const int gtid = tid - 32 - grp * kCombGroupThreads;
    const uint32_t slot_bytes = (uint32_t)(g.cw * 2);
    // item i = q * nch + chunk (q: the CTA's token index); this group takes i = grp, grp + G, ...
    int64_t i = grp, q = 0, c = grp;
    while (c >= g.nch) {
      c -= g.nch;
      ++q;
    }
    int s = grp % S;
    uint32_t par = (uint32_t)((grp / S) & 1);
    for (; kPacked || i < n_items; i += kCombGroups) {
      if (!mbar_wait_warp(full0 + 8 * s, par, L.status)) break;
      const int n = meta[s].n;
      if (kPacked && n < 0) break;  // the producer's last item for this group
      if (!dbg_ok(n >= 0 && n <= L.k, L.status, 104, n)) break;
      int64_t c0, width, qi;
      uint32_t stride;
      if constexpr (kPacked) {
        qi = meta[s].q;
        c0 = meta[s].c0;
        width = meta[s].width;
        stride = (uint32_t)meta[s].stride;
      } else {
        qi = q;
        c0 = c * g.cw;
        width = min(g.cw, H - c0);
        stride = slot_bytes;
      }
      const uint32_t stage = base + g.data + (uint32_t)s * g.stage_bytes;
      for (int64_t e = gtid * 8; e < width; e += kCombGroupThreads * 8) {
        float acc[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[v] = 0.0f;
        int j = 0;
        for (; j + 4 <= n; j += 4) {
          uint4 d[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) d[u] = lds_v4(stage + (uint32_t)(j + u) * stride + (uint32_t)e * 2);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t wd[4] = {d[u].x, d[u].y, d[u].z, d[u].w};
            const float wj = kWeighted ? meta[s].w[j + u] : 1.0f;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              if (kWeighted) {
                acc[2 * v] = __fmaf_rn(wj, bf16lo(wd[v]), acc[2 * v]);
                acc[2 * v + 1] = __fmaf_rn(wj, bf16hi(wd[v]), acc[2 * v + 1]);
              } else {
                acc[2 * v] = __fadd_rn(acc[2 * v], bf16lo(wd[v]));
                acc[2 * v + 1] = __fadd_rn(acc[2 * v + 1], bf16hi(wd[v]));
              }
            }
          }
        }
        for (; j < n; ++j) {
          const uint4 d = lds_v4(stage + (uint32_t)j * stride + (uint32_t)e * 2);
          const uint32_t wd[4] = {d.x, d.y, d.z, d.w};
          const float wj = kWeighted ? meta[s].w[j] : 1.0f;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            if (kWeighted) {
              acc[2 * v] = __fmaf_rn(wj, bf16lo(wd[v]), acc[2 * v]);
              acc[2 * v + 1] = __fmaf_rn(wj, bf16hi(wd[v]), acc[2 * v + 1]);
            } else {
              acc[2 * v] = __fadd_rn(acc[2 * v], bf16lo(wd[v]));
              acc[2 * v + 1] = __fadd_rn(acc[2 * v + 1], bf16hi(wd[v]));
            }
          }
        }
        if (kBias) {
          const uint4 b = lds_v4(stage + (kPacked ? (uint32_t)n * stride : (uint32_t)L.k * slot_bytes) + (uint32_t)e * 2);
          const uint32_t wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            acc[2 * v] = __fadd_rn(acc[2 * v], bf16lo(wb[v]));
            acc[2 * v + 1] = __fadd_rn(acc[2 * v + 1], bf16hi(wb[v]));
          }
        }
        const int64_t t = cta_token(qi);
        if (!dbg_ok(qi < n_tok && t < L.T && c0 + e + 8 <= H && n <= L.k &&
                        (uint32_t)(n > 0 ? n - 1 : 0) * stride + (uint32_t)e * 2 + 16 <= g.stage_bytes,
                    L.status, 103, t * 65536 + e))
          continue;
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        st_stream_v4(out + t * H + c0 + e, o);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
      // advance to item i + G
      if constexpr (!kPacked) {
        c += kCombGroups;
        while (c >= g.nch) {
          c -= g.nch;
          ++q;
        }
      }
      s += kCombGroups;
      while (s >= S) {
        s -= S;
        par ^= 1u;
      }
    }
  }
  if (overflow) atomicOr(L.status, kStatusCapacity);
}

cudaError_t launch_combine(const CombineLaunch& L, cudaStream_t st) {
  const bool wgt = L.w != nullptr, has_bias = L.bias != nullptr;
  const CombGeom g = combine_geometry(L.H, L.k, has_bias);
  if (g.stages < kCombGroups || g.stages % kCombGroups != 0) return cudaErrorInvalidValue;
  static unsigned long long done[6] = {0, 0, 0, 0, 0, 0};
  if (L.packed && wgt) return cudaErrorInvalidValue;  // packed items carry no weights
  const int variant = L.packed ? 4 + (has_bias ? 1 : 0) : (wgt ? 2 : 0) + (has_bias ? 1 : 0);
  auto kern = L.packed ? (has_bias ? k_combine<false, true, true> : k_combine<false, false, true>)
              : wgt    ? (has_bias ? k_combine<true, true, false> : k_combine<true, false, false>)
                       : (has_bias ? k_combine<false, true, false> : k_combine<false, false, false>);
  cudaError_t err = set_smem_limit_once(kern, (int)kCombSmemBudget, &done[variant]);
  if (err != cudaSuccess) return err;
  err = launch_pdl(kern, dim3(L.grid), dim3(kCombThreads), (size_t)g.total, st, L, g);
  note_launch();
  return err;
}

}  // namespace moe
