// moe_internal.cuh -- shared definitions of the CUDA library (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "moe.h"

namespace moe {

// Device status word bits (the handle's status[0]).
constexpr int32_t kStatusBadExpert = 1;
constexpr int32_t kStatusCapacity = 2;

// Layout tiling: a chunk of tokens per CTA; 8 warps per layout CTA.
constexpr int kChunkTokens = 512;
constexpr int kLayoutThreads = 256;
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr int kScanThreads = 1024;
constexpr int kMaxExperts = 4096;
constexpr int kMaxTopk = 32;

// Data-movement kernels: one 1024-thread CTA per SM, so a num_sms cap is an SM cap.
constexpr int kMoveThreads = 1024;

struct DeviceArrays {
  int32_t* status = nullptr;          // [4]
  int32_t* cnt = nullptr;             // [E]
  int32_t* psum = nullptr;            // [E]
  int32_t* pad_excl = nullptr;        // [E + 1]  exclusive prefix of padding rows, all experts
  int32_t* rows_per_rank = nullptr;   // [R]
  int32_t* tokens_per_rank = nullptr; // [R]
  uint8_t* token_in_rank = nullptr;   // [T * R]
  int32_t* slot = nullptr;            // [T * k]  row inside the destination rank, -1 if masked
  int32_t* pair_rank = nullptr;       // [T * k]  destination logical rank, -1 if masked
  float* pair_w = nullptr;            // [T * k]
  int32_t* chunk_cnt = nullptr;       // [C * E]  counts, then exclusive offsets
  int32_t* chunk_tok = nullptr;       // [C * R]
  int32_t* row_src = nullptr;         // [R * row_cap]
  float* row_w = nullptr;             // [R * row_cap]
};

}  // namespace moe

struct moe_handle {
  moe_params_t p{};
  cudaStream_t stream = nullptr;
  int device = 0;
  void* block = nullptr;       // one stream-ordered allocation for the fixed-size arrays
  void* row_block = nullptr;   // row_src / row_w
  int64_t row_cap = 0;
  int num_chunks = 0;
  bool counts_on_host = false;
  std::vector<int32_t> host_rows;  // rows_per_rank, when do_cpu_sync
  int32_t host_total_pad = -1;     // padding rows over all experts, when do_cpu_sync
  moe::DeviceArrays d;
};

namespace moe {

struct LayoutLaunch {
  const int64_t* idx;
  const float* w;
  int64_t T;
  int k, E, R, E_loc, A;
  int num_chunks;
  int grid_chunks;  // CTAs for the per-chunk kernels (<= num_chunks)
  int64_t row_cap;  // 0 -> row maps not written (filled by a later assign launch)
  DeviceArrays d;
};

cudaError_t launch_layout_count(const LayoutLaunch& L, cudaStream_t s);
cudaError_t launch_layout_scan(const LayoutLaunch& L, int64_t cap_check, cudaStream_t s);
cudaError_t launch_layout_assign(const LayoutLaunch& L, cudaStream_t s);

struct DispatchLaunch {
  const void* x;
  void* recv_x;
  float* recv_scales;
  float* recv_w;
  int64_t T, cap, H;
  int k, E, E_loc;
  int zero_padding;
  int grid;
  const int32_t* pair_rank;
  const int32_t* slot;
  const float* pair_w;
  const int32_t* psum;
  const int32_t* pad_excl;
  int32_t* status;
};

cudaError_t launch_dispatch(const DispatchLaunch& L, bool fp8, cudaStream_t s);

struct CombineLaunch {
  const void* y;
  const float* w;
  const void* bias;
  void* out;
  int64_t T, cap, H;
  int k;
  int grid;
  const int32_t* pair_rank;
  const int32_t* slot;
  int32_t* status;
};

cudaError_t launch_combine(const CombineLaunch& L, cudaStream_t s);

void note_launch(int n = 1);
int sm_count(int device);

// ------------------------------------------------------------------------------ device helpers

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Round to nearest even binary32 -> bf16, two values packed low|high.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two binary32 values -> two E4M3 codes (round to nearest even, saturate to +-448),
// `lo` in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return (uint32_t)r;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

}  // namespace moe
