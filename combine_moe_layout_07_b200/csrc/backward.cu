// backward.cu -- gradient of the combine with respect to the pair weights.
//
// The handle of one dispatch is reused by the backward pass ("Why MoE gets stuck on
// communication" (locsic.com), sections 1 and 2).  For out[t] = sum_j w[t,j] * y[row(t,j)] (+ bias)
// the gradient of the expert outputs is the dispatch of grad_out scaled by w (dispatch.cu, BF16
// path with scale_w); this file computes the gradient of the weights,
//   grad_w[t,j] = <grad_out[t], y[row(t,j)]>   (0 for masked pairs).
//
// A warp per (t, j) pair: lane l accumulates columns l*8 .. l*8+7, then +256, ... in ascending
// order with fp32 FMA, then the 32 partial sums are added by a fixed xor-shuffle tree, so the
// result is the same on every run.  16-byte streaming loads, 4 column steps in flight per lane.
#include "moe_internal.cuh"

namespace moe {

constexpr int kGradWarps = 8;

__global__ void __launch_bounds__(32 * kGradWarps) k_grad_weights(GradWeightsLaunch L) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * kGradWarps + (threadIdx.x >> 5);
  const int64_t nw = (int64_t)gridDim.x * kGradWarps;
  const int64_t H = L.H;
  const uint16_t* go = static_cast<const uint16_t*>(L.grad_out);
  const uint16_t* y = static_cast<const uint16_t*>(L.y);
  grid_dependents_launch();
  grid_dependency_wait();
  for (int64_t p = gw; p < L.T * L.k; p += nw) {
    const int32_t r = __ldg(L.pair_rank + p), s = __ldg(L.slot + p);
    float acc = 0.0f;
    if (r >= 0 && s >= 0 && s < L.cap) {
      const uint16_t* yr = y + ((int64_t)r * L.cap + s) * H;
      const uint16_t* gr = go + (int64_t)((uint32_t)p / (uint32_t)L.k) * H;
      constexpr int U = 4;
      for (int64_t c0 = lane * 8; c0 < H; c0 += 256 * U) {
        uint4 a[U], b[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int64_t c = c0 + u * 256;
          if (c < H) {
            a[u] = ld_stream_v4(gr + c);
            b[u] = ld_stream_v4(yr + c);
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          if (c0 + u * 256 < H) {
            const uint32_t ga[4] = {a[u].x, a[u].y, a[u].z, a[u].w};
            const uint32_t yb[4] = {b[u].x, b[u].y, b[u].z, b[u].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              acc = __fmaf_rn(bf16lo(ga[q]), bf16lo(yb[q]), acc);
              acc = __fmaf_rn(bf16hi(ga[q]), bf16hi(yb[q]), acc);
            }
          }
        }
      }
    } else if (r >= 0 && s >= 0) {
      atomicOr(L.status, kStatusCapacity);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
    if (lane == 0) L.grad_w[p] = acc;
  }
}

cudaError_t launch_grad_weights(const GradWeightsLaunch& L, cudaStream_t s) {
  cudaError_t err = launch_pdl(k_grad_weights, dim3(L.grid), dim3(32 * kGradWarps), 0, s, L);
  note_launch();
  return err;
}

}  // namespace moe
