// combine.cu -- gather the expert outputs back to token order and reduce the top-k rows.
//
// Follows "From DeepEP to Mega MoE" (backyes.github.io) 2.3 / 2.5 (combine_reduce: an
// element-wise sum of a token's top-k expert rows, not a GEMM) and "Why MoE gets stuck on
// communication" (locsic.com) section 1 (the rows are already weighted; the shared expert's
// output is added as the bias).  Optional per-pair weights are applied in fp32 when given.
//
// Numerics, fixed so every run is bit-identical: acc = 0 (fp32); for j = 0..k-1 in order,
// skipping masked pairs, acc = fma(w, y, acc) or acc + y; then acc + bias; one rounding to bf16.
//
// B200 mapping: HBM-bound gather.  One 1024-thread CTA per SM, a warp per token; each lane owns
// 8 bf16 columns per step and issues the loads of all (up to 8) source rows before reducing
// them, so 8 x 16 bytes per lane are in flight; streaming loads skip L1, the output row is
// written with evict-first stores.
#include "moe_internal.cuh"

namespace moe {

constexpr int kCombineWarps = kMoveThreads / 32;
constexpr int kGroup = 8;  // source rows loaded before they are reduced

template <bool kWeighted, bool kBias>
__global__ void __launch_bounds__(kMoveThreads, 1) k_combine(CombineLaunch L) {
  __shared__ int64_t tab_off[kCombineWarps][kMaxTopk];  // element offset of the source row
  __shared__ float tab_w[kCombineWarps][kMaxTopk];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t gw = (int64_t)blockIdx.x * kCombineWarps + warp;
  const int64_t nw = (int64_t)gridDim.x * kCombineWarps;
  const int64_t H = L.H;
  const uint16_t* y = static_cast<const uint16_t*>(L.y);
  const uint16_t* bias = static_cast<const uint16_t*>(L.bias);
  uint16_t* out = static_cast<uint16_t*>(L.out);
  bool overflow = false;

  for (int64_t t = gw; t < L.T; t += nw) {
    int64_t off = -1;
    float wv = 0.0f;
    if (lane < L.k) {
      const int64_t p = t * L.k + lane;
      const int32_t r = __ldg(L.pair_rank + p);
      const int32_t s = __ldg(L.slot + p);
      if (r >= 0) {
        if (s < L.cap) off = ((int64_t)r * L.cap + s) * H;
        else overflow = true;
      }
      if (kWeighted) wv = __ldg(L.w + p);
    }
    const uint32_t vmask = __ballot_sync(0xffffffffu, off >= 0);
    tab_off[warp][lane] = off;
    tab_w[warp][lane] = wv;
    __syncwarp();

    for (int64_t c = lane * 8; c < H; c += 32 * 8) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
      for (uint32_t m = vmask; m;) {
        uint4 d[kGroup];
        float wg[kGroup];
        int n = 0;
#pragma unroll
        for (int g = 0; g < kGroup; ++g) {
          if (m) {
            const int j = __ffs(m) - 1;
            m &= m - 1;
            d[g] = ld_stream_v4(y + tab_off[warp][j] + c);
            wg[g] = tab_w[warp][j];
            n = g + 1;
          }
        }
#pragma unroll
        for (int g = 0; g < kGroup; ++g) {
          if (g < n) {
            const uint32_t u[4] = {d[g].x, d[g].y, d[g].z, d[g].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (kWeighted) {
                acc[2 * i] = __fmaf_rn(wg[g], bf16lo(u[i]), acc[2 * i]);
                acc[2 * i + 1] = __fmaf_rn(wg[g], bf16hi(u[i]), acc[2 * i + 1]);
              } else {
                acc[2 * i] = __fadd_rn(acc[2 * i], bf16lo(u[i]));
                acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], bf16hi(u[i]));
              }
            }
          }
        }
      }
      if (kBias) {
        const uint4 b = ld_stream_v4(bias + t * H + c);
        const uint32_t u[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = __fadd_rn(acc[2 * i], bf16lo(u[i]));
          acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], bf16hi(u[i]));
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      st_stream_v4(out + t * H + c, o);
    }
    __syncwarp();
  }
  if (overflow) atomicOr(L.status, kStatusCapacity);
}

cudaError_t launch_combine(const CombineLaunch& L, cudaStream_t s) {
  const bool wgt = L.w != nullptr, bias = L.bias != nullptr;
  if (wgt && bias) k_combine<true, true><<<L.grid, kMoveThreads, 0, s>>>(L);
  else if (wgt) k_combine<true, false><<<L.grid, kMoveThreads, 0, s>>>(L);
  else if (bias) k_combine<false, true><<<L.grid, kMoveThreads, 0, s>>>(L);
  else k_combine<false, false><<<L.grid, kMoveThreads, 0, s>>>(L);
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe
