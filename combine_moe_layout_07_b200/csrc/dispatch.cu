// dispatch.cu -- gather each routed token's hidden vector into the expert-major receive
// buffers, optionally quantising BF16 -> FP8 E4M3 with 1x128 block scales on the way.
//
// Follows "From DeepEP to Mega MoE" (backyes.github.io) 2.2 (dispatch warps: a token is loaded
// once and stored to each destination; no arithmetic beyond the copy) and 2.4 (copy epilogue:
// the row lands at its position inside its expert's range of the receive buffer), with
// do_expand / do_zero_padding of "Why MoE gets stuck on communication" (locsic.com) section 1 and
// FP8 dispatch of "DeepEP expert-parallel communication" (blog.hotdry.top), key techniques.
//
// B200 mapping: HBM-bound data movement.  One 1024-thread CTA per SM (so num_sms caps SMs), a
// warp per source token: the row is read once with 16-byte streaming loads (no L1 allocation)
// and written to its k destination rows with 16-byte evict-first stores.  FP8: eight lanes own
// one 128-element block; amax is reduced with three xor-shuffles; inv = 448/a and a/448 are
// IEEE divisions; codes come from cvt.rn.satfinite.e4m3x2.  Padding rows are zeroed by the same
// grid after the tokens, a warp per row.
#include "moe_internal.cuh"

namespace moe {

constexpr int kWarpsPerMoveCta = kMoveThreads / 32;

__device__ __forceinline__ int find_padding_expert(const int32_t* pad_excl, int E, int32_t i) {
  int lo = 0, hi = E;  // largest e with pad_excl[e] <= i
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(pad_excl + mid) <= i) lo = mid; else hi = mid;
  }
  return lo;
}

template <bool kFp8>
__global__ void __launch_bounds__(kMoveThreads, 1) k_dispatch(DispatchLaunch L) {
  __shared__ int64_t tab[kWarpsPerMoveCta][kMaxTopk];  // destination row (r * cap + slot)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t gw = (int64_t)blockIdx.x * kWarpsPerMoveCta + warp;
  const int64_t nw = (int64_t)gridDim.x * kWarpsPerMoveCta;
  const int64_t H = L.H;
  bool overflow = false;

  for (int64_t t = gw; t < L.T; t += nw) {
    int64_t my_row = -1;
    if (lane < L.k) {
      const int64_t p = t * L.k + lane;
      const int32_t r = __ldg(L.pair_rank + p);
      const int32_t s = __ldg(L.slot + p);
      if (r >= 0) {
        if (s < L.cap) my_row = (int64_t)r * L.cap + s;
        else overflow = true;
      }
      if (my_row >= 0 && L.recv_w) L.recv_w[my_row] = __ldg(L.pair_w + p);
    }
    const uint32_t vmask = __ballot_sync(0xffffffffu, my_row >= 0);
    tab[warp][lane] = my_row;
    __syncwarp();

    if constexpr (!kFp8) {
      // BF16: copy the row (2H bytes) to every destination, 4 vectors per lane in flight
      constexpr int U = 4;
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(L.x) + t * H);
      const int nvec = (int)(H / 8);
      for (int v0 = 0; v0 < nvec; v0 += 32 * U) {
        uint4 d[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + u * 32 + lane;
          if (v < nvec) d[u] = ld_stream_v4(src + v);
        }
        for (uint32_t m = vmask; m; m &= m - 1) {
          const int j = __ffs(m) - 1;
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(L.recv_x) + tab[warp][j] * H);
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int v = v0 + u * 32 + lane;
            if (v < nvec) st_stream_v4(dst + v, d[u]);
          }
        }
      }
    } else {
      // FP8: lane owns 16 consecutive elements; 8 lanes = one 1x128 block; 512 elements per pass
      const uint16_t* src = static_cast<const uint16_t*>(L.x) + t * H;
      const int64_t nblk = H / 128;
      for (int64_t e0 = lane * 16; e0 - lane * 16 < H; e0 += 512) {
        const bool act = e0 < H;
        uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
        if (act) {
          a = ld_stream_v4(src + e0);
          b = ld_stream_v4(src + e0 + 8);
        }
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        float v[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[2 * i] = bf16lo(w[i]);
          v[2 * i + 1] = bf16hi(w[i]);
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        const float am = fmaxf(amax, 1e-4f);
        const float inv = __fdiv_rn(448.0f, am);
        const float scale = __fdiv_rn(am, 448.0f);
        uint32_t q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t lo = pack_e4m3x2(__fmul_rn(v[4 * i], inv), __fmul_rn(v[4 * i + 1], inv));
          const uint32_t hi = pack_e4m3x2(__fmul_rn(v[4 * i + 2], inv), __fmul_rn(v[4 * i + 3], inv));
          q[i] = lo | (hi << 16);
        }
        const uint4 qv = make_uint4(q[0], q[1], q[2], q[3]);
        if (act) {
          for (uint32_t m = vmask; m; m &= m - 1) {
            const int64_t row = tab[warp][__ffs(m) - 1];
            st_stream_v4(static_cast<uint8_t*>(L.recv_x) + row * H + e0, qv);
            if ((lane & 7) == 0) L.recv_scales[row * nblk + e0 / 128] = scale;
          }
        }
      }
    }
    __syncwarp();
  }

  // padding rows: [psum[e] - pad(e), psum[e]) of expert e's rank
  if (L.zero_padding || L.recv_w) {
    const int32_t total_pad = __ldg(L.pad_excl + L.E);
    const int64_t row_bytes = kFp8 ? H : 2 * H;
    const int64_t nblk = H / 128;
    for (int64_t i = gw; i < total_pad; i += nw) {
      const int e = find_padding_expert(L.pad_excl, L.E, (int32_t)i);
      const int32_t pad_e = __ldg(L.pad_excl + e + 1) - __ldg(L.pad_excl + e);
      const int32_t row = __ldg(L.psum + e) - pad_e + ((int32_t)i - __ldg(L.pad_excl + e));
      if (row >= L.cap) {
        overflow = true;
        continue;
      }
      const int64_t grow = (int64_t)(e / L.E_loc) * L.cap + row;
      if (L.zero_padding) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(L.recv_x) + grow * row_bytes);
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int64_t v = lane; v < row_bytes / 16; v += 32) st_stream_v4(dst + v, z);
        if (kFp8)
          for (int64_t b = lane; b < nblk; b += 32) L.recv_scales[grow * nblk + b] = 0.0f;
      }
      if (L.recv_w && lane == 0) L.recv_w[grow] = 0.0f;
    }
  }
  if (overflow) atomicOr(L.status, kStatusCapacity);
}

cudaError_t launch_dispatch(const DispatchLaunch& L, bool fp8, cudaStream_t s) {
  if (fp8) k_dispatch<true><<<L.grid, kMoveThreads, 0, s>>>(L);
  else k_dispatch<false><<<L.grid, kMoveThreads, 0, s>>>(L);
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe
