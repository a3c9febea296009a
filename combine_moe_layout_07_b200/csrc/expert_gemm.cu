// expert_gemm.cu -- the first expert GEMM on the FP8 dispatch layout, on the 5th-generation
// tensor cores (tcgen05 MMA, accumulators in tensor memory, TMA-fed shared memory).
//
// Follows "From DeepEP to Mega MoE" (backyes.github.io) 3.2 (Linear1: a TMA load warp stages the
// dispatched tokens and the expert weights, one MMA-issue warp drives the tensor cores, epilogue
// warps read the accumulators from tensor memory) and 4.5 (the separated dataflow: dispatch ->
// expert buffer in HBM -> GEMM L1); "Why MoE gets stuck on communication" (locsic.com) 1:
// expert_alignment is the grouped GEMM's row alignment, so with A % 128 == 0 no 128-row tile
// straddles two experts.
//
//   out[r, row, n] = bf16( sum over K-blocks b of sx[r, row, b] * sw[e, n / 128, b]
//                          * sum over h in block b of qx[r, row, h] * qw[e, n, h] )
// for the rows of every expert range of every logical rank (e = the row's expert).
//
// The dispatch's 1x128 scales are fp32 (a / 448), not the power-of-two factors the block-scaled
// MMA kinds take, so each 128-wide K-block is one plain E4M3 x E4M3 MMA group (4 x K=32) into a
// fresh tensor-memory accumulator, and the epilogue warps promote it: acc += partial * (sx * sw)
// in fp32 registers.  The 512 tensor-memory columns hold 512 / kN accumulator buffers (4 for
// kN = 128, 2 for kN = 256), so the MMAs run up to that many K-blocks ahead of the epilogue.
//
// One CTA per SM, persistent over 128 x kN output tiles (kN = 256 when N % 256 == 0, else 128)
// in m-major order (consecutive tiles share their 128 rows; an expert's weight columns are
// reused across its row tiles from L2).
//   warp 0      TMA producer: per K-block, one 128 x 128-byte tile of rows and one kN x 128-byte
//               tile of weights (128-byte swizzle) into a ring of stages (full/empty mbarriers);
//   warp 1      allocates all 512 tensor-memory columns; one lane issues the MMAs and commits
//               them to the stage's empty barrier and to the accumulator's full barrier;
//   warps 2, 3  set-up only (row tiles per rank, psum into shared memory);
//   warps 4..11 epilogue (warpgroups 1 and 2, which take the registers warpgroup 0 gives back):
//               warp w reads tensor-memory lanes 32 * (w % 4) .. (one output row per thread) and
//               half (w - 4) / 4 of the tile's kN columns (kN / 2 accumulators per thread): per
//               K-block, 32-column loads in rounds of kRoundCols with one wait per round, then
//               the promotions; a bf16 store of its kN / 2 columns per tile.
// Every wait is an mbarrier wait bounded by wall-clock time (status kStatusTimeout).  No TMA
// load here uses cluster multicast.
#include <cuda.h>

#include "moe_internal.cuh"

namespace moe {

constexpr int kGemmM = 128;                            // rows of a tile = the K-block width
constexpr int kGemmEpiWarps = 8;                       // two per tensor-memory lane quarter
constexpr int kGemmEpiWarp0 = 4;                       // the epilogue is warpgroups 1 and 2
constexpr int kGemmThreads = 128 + 32 * kGemmEpiWarps;  // warpgroup 0 (producer, MMA, set-up), epilogue
// Register split (setmaxnreg): warpgroup 0 gives registers back, the epilogue warpgroups take them
// for their 128 accumulators per thread.  The launch holds kGemmThreads x (registers at launch);
// the split needs 128 x kGemmCtlRegs + 256 x kGemmEpiRegs of them, which the host checks against
// the kernel's register count before it launches.
constexpr int kGemmCtlRegs = 112;
constexpr int kGemmEpiRegs = 192;
static_assert(kGemmCtlRegs % 8 == 0 && kGemmEpiRegs % 8 == 0, "setmaxnreg counts are multiples of 8");
constexpr uint32_t kGemmTmemCols = 512;                // all of tensor memory (one CTA per SM)
constexpr uint32_t kGemmStageBudget = 192 * 1024;      // shared memory for the operand ring

// Tile shape: 128 rows x kN output columns (kN = 256 when N allows it: 1.5x fewer operand bytes
// per MMA than kN = 128, which the TMA feed from L2 cannot sustain at full tensor rate).
template <int kN>
struct GemmCfg {
  static constexpr uint32_t kBytesA = kGemmM * 128;           // 128 rows x one 128-byte K-block
  static constexpr uint32_t kBytesB = kN * 128;               // kN weight rows x one K-block
  static constexpr uint32_t kStageBytes = kBytesA + kBytesB;  // a multiple of 1024
  static constexpr int kStages = (int)(kGemmStageBudget / kStageBytes);  // 6 or 4
  static constexpr int kAccBufs = (int)(kGemmTmemCols / kN);  // 4 or 2 accumulators
  static constexpr int kWarpCols = kN / 2;                    // columns an epilogue warp owns
  static constexpr int kRoundCols = kN == 128 ? 64 : 32;      // columns loaded per wait
  static constexpr int kScaleAhead = kN == 128 ? 8 : 4;       // K-blocks of scales loaded ahead (about
                                                              // the same time: a K-block of kN = 256
                                                              // takes twice as long)
  // instruction descriptor: D fp32, A and B E4M3, both K-major, N = kN, M = 128
  static constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(kN >> 3) << 17) | ((uint32_t)(kGemmM >> 4) << 24);
};

struct GemmSmem {
  uint32_t full, empty, tfull, tempty, done, tmem_slot, tiles, psum;  // offsets from the aligned base
  uint32_t stage0, total;
};

template <int kN>
__host__ __device__ inline GemmSmem gemm_smem(int R, int E) {
  using C = GemmCfg<kN>;
  GemmSmem s;
  uint32_t off = 0;
  s.full = off;
  off += 8 * C::kStages;
  s.empty = off;
  off += 8 * C::kStages;
  s.tfull = off;
  off += 8 * C::kAccBufs;
  s.tempty = off;
  off += 8 * C::kAccBufs;
  s.done = off;
  off += 8;
  s.tmem_slot = off;
  off += 8;
  s.tiles = off;                        // int32 [R + 1]: prefix of row tiles per rank
  off += 4 * (uint32_t)(R + 1);
  s.psum = off;                         // int32 [E]: the handle's psum, for the tile -> expert search
  off += 4 * (uint32_t)E;
  off = (off + 1023) / 1024 * 1024;     // 128-byte-swizzled tiles want 1024-byte alignment
  s.stage0 = off;
  off += C::kStageBytes * C::kStages;
  s.total = off;
  return s;
}

// ---------------------------------------------------------------------------- tcgen05 helpers
// Shared-memory matrix descriptor of a K-major operand tile whose 128-byte rows are stored with
// the 128-byte swizzle (as TMA writes them): start address >> 4, leading offset 1 (16 B, unused
// with this swizzle), stride 1024 B between groups of 8 rows, descriptor version 1, swizzle mode 2.
__device__ __forceinline__ uint64_t kmajor_sw128_desc(uint32_t smem_addr) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
}

__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

// Arrive on `bar` once every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_load32(uint32_t taddr, float (&v)[32]) {
  uint32_t u[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
        "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
        "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]),
        "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(u[i]);
}

__device__ __forceinline__ void tmem_wait_load() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// ---------------------------------------------------------------------------- tile map
struct GemmTile {
  int r;          // logical rank
  int64_t row0;   // first row of the tile inside rank r
  int e;          // the tile's expert
  int nb;         // column tile
};

// Tile t of the m-major order: row tile m = t / NT (over all ranks), column tile t % NT.  The
// expert is the first e of rank r whose inclusive aligned prefix psum[e] exceeds the tile's row
// (tiles and psum in shared memory: no global round trip at a tile boundary).
__device__ __forceinline__ GemmTile gemm_tile(int R, int E_loc, int64_t NT, const int32_t* tiles, const int32_t* psum,
                                              int64_t t) {
  GemmTile g;
  const int64_t m = t / NT;
  g.nb = (int)(t - m * NT);
  int lo = 0, hi = R;  // largest r with tiles[r] <= m
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tiles[mid] <= m) lo = mid;
    else hi = mid;
  }
  g.r = lo;
  g.row0 = (m - tiles[lo]) * kGemmM;
  int a = g.r * E_loc, b = a + E_loc - 1;  // first e in [a, b] with psum[e] > row0
  while (a < b) {
    const int mid = (a + b) >> 1;
    if (psum[mid] > g.row0) b = mid;
    else a = mid + 1;
  }
  g.e = a;
  return g;
}

template <int kN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_expert_gemm(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w, GemmLaunch L) {
  using C = GemmCfg<kN>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const GemmSmem lay = gemm_smem<kN>(L.R, L.E);
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base - raw);
  const uint32_t full0 = base + lay.full, empty0 = base + lay.empty;
  const uint32_t tfull0 = base + lay.tfull, tempty0 = base + lay.tempty, done = base + lay.done;
  int32_t* tiles = reinterpret_cast<int32_t*>(smem + lay.tiles);
  int32_t* psum_s = reinterpret_cast<int32_t*>(smem + lay.psum);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + lay.tmem_slot);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t NT = L.N / kN;  // column tiles

  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, kGemmEpiWarps);
    }
    mbar_init(done, 1);
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
  }
  if (warp == 1) {  // the whole warp allocates; the address lands in tmem_slot
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(base + lay.tmem_slot),
                 "r"(kGemmTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  grid_dependents_launch();
  grid_dependency_wait();  // the handle's psum / rows and the dispatched rows
  if (warp == 2) {  // row tiles per rank, prefix over ranks; rows beyond cap (a capacity overflow
                    // the layout has flagged) are never read or written
    int32_t run = 0;
    for (int r0 = 0; r0 < L.R; r0 += 32) {
      const int r = r0 + lane;
      const int32_t v = r < L.R ? (int32_t)(min((int64_t)__ldg(L.rows_per_rank + r), L.cap) / kGemmM) : 0;
      int32_t incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      if (r < L.R) tiles[r] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) tiles[L.R] = run;
  }
  if (warp >= 3)
    for (int e = tid - 96; e < L.E; e += kGemmThreads - 96) psum_s[e] = __ldg(L.psum + e);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t n_tiles = (int64_t)tiles[L.R] * NT;
  const int KB = L.KB;

  if (warp < kGemmEpiWarp0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kGemmCtlRegs));
    if (warp == 0) {
      // ------------------------------------------------------------------ TMA producer
      if (lane == 0) {
        int s = 0;
        uint32_t ph = 0;
        int64_t g = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
          const GemmTile tl = gemm_tile(L.R, L.E_loc, NT, tiles, psum_s, t);
          const int32_t y_rows = (int32_t)((int64_t)tl.r * L.cap + tl.row0);
          const int32_t y_cols = (int32_t)((int64_t)tl.e * L.N + (int64_t)tl.nb * kN);
          for (int kb = 0; kb < KB; ++kb, ++g) {
            if (g >= C::kStages && !(ok = mbar_wait(empty0 + 8 * s, ph ^ 1u, L.status))) break;
            const uint32_t a = base + lay.stage0 + (uint32_t)s * C::kStageBytes;
            mbar_arrive_expect_tx(full0 + 8 * s, C::kStageBytes);
            tma_load_2d(a, &map_x, kb * 128, y_rows, full0 + 8 * s);
            tma_load_2d(a + C::kBytesA, &map_w, kb * 128, y_cols, full0 + 8 * s);
            if (++s == C::kStages) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
        // no load may still be landing when the CTA exits: the last stages must have filled
        for (int64_t j = 0; j < (g < C::kStages ? g : C::kStages); ++j) {
          if (--s < 0) {
            s = C::kStages - 1;
            ph ^= 1u;
          }
          mbar_wait(full0 + 8 * s, ph, L.status);
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        int s = 0;
        uint32_t ph = 0;
        int64_t g = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
          for (int kb = 0; kb < KB; ++kb, ++g) {
            const int b = (int)(g % C::kAccBufs);
            const uint32_t tph = (uint32_t)((g / C::kAccBufs) & 1);
            if (!(ok = mbar_wait(full0 + 8 * s, ph, L.status))) break;
            if (g >= C::kAccBufs && !(ok = mbar_wait(tempty0 + 8 * b, tph ^ 1u, L.status))) break;
            tc_fence_after();
            const uint32_t a = base + lay.stage0 + (uint32_t)s * C::kStageBytes;
            const uint64_t ad = kmajor_sw128_desc(a), bd = kmajor_sw128_desc(a + C::kBytesA);
  #pragma unroll
            for (int k = 0; k < 4; ++k)  // K = 32 E4M3 = 32 bytes = 2 descriptor units per step
              mma_e4m3(tmem + (uint32_t)(b * kN), ad + 2 * k, bd + 2 * k, C::kIdesc, k > 0 ? 1u : 0u);
            mma_commit(empty0 + 8 * s);  // the stage is free once these MMAs have read it
            mma_commit(tfull0 + 8 * b);  // the accumulator is ready for the epilogue
            if (++s == C::kStages) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
        mma_commit(done);  // every MMA of this CTA has completed when `done` flips
        mbar_wait(done, 0, L.status);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kGemmEpiRegs));
    // ------------------------------------------------------------------ epilogue
    constexpr int W = C::kWarpCols;
    const int q = warp & 3;                       // tensor-memory lane quarter of this warp
    const int col0 = ((warp - kGemmEpiWarp0) >> 2) * W;  // the half of the tile's columns it owns
    const int my_row = q * 32 + lane;             // row of the tile this thread owns
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    uint16_t* out = static_cast<uint16_t*>(L.out);
    int64_t g = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      const GemmTile tl = gemm_tile(L.R, L.E_loc, NT, tiles, psum_s, t);
      const int64_t grow = (int64_t)tl.r * L.cap + tl.row0 + my_row;
      const float* sxr = L.sx + grow * KB;
      const float* swr = L.sw + ((int64_t)tl.e * L.NB + ((int64_t)tl.nb * kN + col0) / 128) * KB;
      float acc[W];
#pragma unroll
      for (int i = 0; i < W; ++i) acc[i] = 0.0f;
      // the scales of K-blocks kb0 .. kb0 + A - 1 (products sx * sw), loaded one group ahead
      constexpr int A = C::kScaleAhead;
      float s_cur[A];
#pragma unroll
      for (int j = 0; j < A; ++j) s_cur[j] = j < KB ? __ldg(sxr + j) * __ldg(swr + j) : 0.0f;
      for (int kb0 = 0; kb0 < KB && ok; kb0 += A) {
        float sx_nxt[A], sw_nxt[A];
#pragma unroll
        for (int j = 0; j < A; ++j) {
          const int kn = kb0 + A + j;
          sx_nxt[j] = kn < KB ? __ldg(sxr + kn) : 0.0f;
          sw_nxt[j] = kn < KB ? __ldg(swr + kn) : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < A; ++j) {
          if (kb0 + j >= KB) break;
          const int b = (int)(g % C::kAccBufs);
          const uint32_t tph = (uint32_t)((g / C::kAccBufs) & 1);
          const float scale = s_cur[j];
          if (!(ok = mbar_wait_warp(tfull0 + 8 * b, tph, L.status))) break;
          tc_fence_after();
          const uint32_t ta = tmem + lane_addr + (uint32_t)(b * kN + col0);
#pragma unroll
          for (int c0 = 0; c0 < W; c0 += C::kRoundCols) {  // one wait per round of kRoundCols columns
            float v0[32], v1[32];
            tmem_load32(ta + (uint32_t)c0, v0);
            if constexpr (C::kRoundCols == 64) tmem_load32(ta + (uint32_t)c0 + 32, v1);
            tmem_wait_load();
            if (c0 + C::kRoundCols == W) {  // the whole buffer is in registers: hand it back
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(tempty0 + 8 * b);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[c0 + i] = __fmaf_rn(v0[i], scale, acc[c0 + i]);
            if constexpr (C::kRoundCols == 64) {
#pragma unroll
              for (int i = 0; i < 32; ++i) acc[c0 + 32 + i] = __fmaf_rn(v1[i], scale, acc[c0 + 32 + i]);
            }
          }
          ++g;
        }
#pragma unroll
        for (int j = 0; j < A; ++j) s_cur[j] = sx_nxt[j] * sw_nxt[j];  // landed a group ago
      }
      if (!ok) break;
      uint4* dst = reinterpret_cast<uint4*>(out + grow * L.N + (int64_t)tl.nb * kN + col0);
#pragma unroll
      for (int i = 0; i < W / 8; ++i) {
        uint4 v;
        v.x = pack_bf16x2(acc[8 * i + 0], acc[8 * i + 1]);
        v.y = pack_bf16x2(acc[8 * i + 2], acc[8 * i + 3]);
        v.z = pack_bf16x2(acc[8 * i + 4], acc[8 * i + 5]);
        v.w = pack_bf16x2(acc[8 * i + 6], acc[8 * i + 7]);
        dst[i] = v;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kGemmTmemCols) : "memory");
  }
}

// ---------------------------------------------------------------------------- host side
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiled encode_tiled() {
  static EncodeTiled fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  }
  return fn;
}

// A row-major [rows, cols] E4M3 matrix read in boxes of box_rows x 128 bytes with the 128-byte swizzle.
static bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiled enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};  // bytes between rows (a multiple of 16: cols % 128 == 0)
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int kN>
static cudaError_t launch_gemm_n(const GemmLaunch& L, const void* x, const void* w, cudaStream_t st) {
  CUtensorMap mx, mw;
  if (!make_map(&mx, x, (uint64_t)L.R * (uint64_t)L.cap, (uint64_t)L.KB * 128, kGemmM) ||
      !make_map(&mw, w, (uint64_t)L.E * (uint64_t)L.N, (uint64_t)L.KB * 128, kN))
    return cudaErrorInvalidValue;
  const uint32_t smem = gemm_smem<kN>(L.R, L.E).total + 1024;  // + slack to align the base to 1024 B
  if (smem > 227u * 1024u) return cudaErrorInvalidValue;
  static unsigned long long done = 0;
  cudaError_t err = set_smem_limit_once(k_expert_gemm<kN>, 227 * 1024, &done);
  if (err != cudaSuccess) return err;
  // the register split must fit the registers the launch holds (else setmaxnreg.inc would wait)
  cudaFuncAttributes fa{};
  err = cudaFuncGetAttributes(&fa, k_expert_gemm<kN>);
  if (err != cudaSuccess) return err;
  if ((int64_t)fa.numRegs * kGemmThreads < 128 * kGemmCtlRegs + 32 * kGemmEpiWarps * kGemmEpiRegs)
    return cudaErrorInvalidConfiguration;
  err = launch_pdl(k_expert_gemm<kN>, dim3(L.grid), dim3(kGemmThreads), smem, st, mx, mw, L);
  note_launch();
  return err;
}

// 256-column tiles when N allows them, else 128.
cudaError_t launch_expert_gemm(const GemmLaunch& L, const void* x, const void* w, cudaStream_t st) {
  return L.N % 256 == 0 ? launch_gemm_n<256>(L, x, w, st) : launch_gemm_n<128>(L, x, w, st);
}

uint32_t expert_gemm_smem_bytes(int R, int E) {
  const uint32_t a = gemm_smem<128>(R, E).total, b = gemm_smem<256>(R, E).total;
  return (a > b ? a : b) + 1024;
}

}  // namespace moe
