// moe_internal.cuh -- shared definitions of the CUDA library (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>
#include <vector>

#include "moe.h"

namespace moe {

// Device status word bits (the handle's status[0]).
constexpr int32_t kStatusBadExpert = 1;
constexpr int32_t kStatusCapacity = 2;
constexpr int32_t kStatusBounds = 8;  // MOE_DEBUG builds: an index check failed (details in status[1..3])

#ifdef MOE_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

// Layout tiling: a chunk of tokens per CTA (a thread per token in the count kernel); 8 warps per
// layout CTA.
constexpr int kFusedMaxExperts = 2048;      // fused layout: 15 shared arrays of E counts
constexpr int kFusedMaxChunkCounts = 65536; // fused layout: C * E chunk counts (the last CTA sums C - 1 of each E)
constexpr int kFusedRounds = 8;             // fused layout: rounds of 32 pairs a warp holds in registers
constexpr int kFusedLoads = 32;             // fused layout: chunk counts a thread loads at once
constexpr int kChunkTokens = 256;      // largest chunk: one token per thread of the count kernel
constexpr int kLayoutThreads = 256;
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr int kScanThreads = 1024;
constexpr int kSmallThreads = 1024;     // the one-CTA layout for small batches
constexpr int kSmallPairs = 8192;       // ... used when T * k <= kSmallPairs
constexpr int kSmallMaxExperts = 1024;  // ... and E <= kSmallMaxExperts
constexpr int kMaxExperts = 4096;
constexpr int kMaxTopk = 32;
constexpr int kMaxByRankRanks = 64;  // the non-expanded (by-rank) layout keeps rank bitmasks

// Data-movement kernels: one 1024-thread CTA per SM, so a num_sms cap is an SM cap.
constexpr int kMoveThreads = 1024;

struct DeviceArrays {
  int32_t* status = nullptr;          // [4]  flags, then MOE_DEBUG details
  int32_t* ticket = nullptr;          // [1]  CTAs of the scan that have finished (0 between launches)
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
  int32_t* chunk_tok = nullptr;       // [C * R]  by-rank: member tokens per chunk, then offsets
  int32_t* token_row = nullptr;       // [T * R]  by-rank: row of token t on rank r, -1 if none
  int32_t* tslot = nullptr;           // [T * k]  by-rank: token row on the pair's rank for the
                                      //          first pair of the token on that rank, else -1
  int32_t* row_src = nullptr;         // [R * row_cap]
  float* row_w = nullptr;             // [R * row_cap]
  int32_t* host_counts = nullptr;     // do_cpu_sync: mapped host memory [status, .., ready at 7]
                                      // [tokens_per_rank R][rows_per_rank R], written once the
                                      // counts are final (layout.cu, publish_host_counts)
};

}  // namespace moe

struct moe_handle {
  moe_params_t p{};
  cudaStream_t stream = nullptr;
  int device = 0;
  void* block = nullptr;       // one stream-ordered allocation for every device array
  int64_t row_cap = 0;
  int num_chunks = 0;
  bool counts_on_host = false;
  std::vector<int32_t> host_rows;    // rows_per_rank, when do_cpu_sync
  std::vector<int32_t> host_tokens;  // tokens_per_rank, when do_cpu_sync
  // MOE_DEFER_EPILOGUE: the count copy lands in epi_stage (pinned, owned until free) and
  // epi_event marks its completion; moe_handle_wait finishes the epilogue.
  int32_t* host_block = nullptr;     // mapped pinned block behind d.host_counts (do_cpu_sync)
  size_t host_block_bytes = 0;
  int32_t* epi_stage = nullptr;
  size_t epi_bytes = 0;
  cudaEvent_t epi_event = nullptr;
  bool epi_pending = false;
  int epi_rc = 0;                    // the epilogue's result once run (sticky)
  moe::DeviceArrays d;
};

// A recorded point on a stream (moe_event_record).
struct moe_event {
  cudaEvent_t ev = nullptr;
};

namespace moe {

struct LayoutLaunch {
  const int64_t* idx;
  const float* w;
  int64_t T;
  int k, E, R, E_loc, A;
  int chunk;        // tokens per chunk of the count / assign kernels (<= kChunkTokens)
  int num_chunks;   // ceil(T / chunk)
  int grid_chunks;  // CTAs for the per-chunk kernels (<= num_chunks)
  int64_t row_cap;  // 0 -> row maps not written (filled by a later assign launch)
  int by_rank;      // also build the non-expanded layout (R <= kMaxByRankRanks)
  DeviceArrays d;
};

cudaError_t launch_layout_count(const LayoutLaunch& L, cudaStream_t s);
cudaError_t launch_layout_scan(const LayoutLaunch& L, int64_t cap_check, cudaStream_t s);
cudaError_t launch_layout_assign(const LayoutLaunch& L, cudaStream_t s);
cudaError_t launch_layout_small(const LayoutLaunch& L, int64_t cap_check, cudaStream_t s);
cudaError_t launch_layout_fused(const LayoutLaunch& L, int64_t cap_check, cudaStream_t s);
bool layout_fits_one_cta(int64_t T, int k, int E);
bool layout_fits_fused(int num_chunks, int chunk, int k, int E, int sm_budget);

struct DispatchLaunch {
  const void* x;
  void* recv_x;
  float* recv_scales;
  float* recv_w;
  int64_t T, cap, H;
  int64_t R;  // logical ranks (receive buffers hold R * cap rows)
  int k, E, E_loc;
  int zero_padding;
  int grid;
  const int32_t* pair_rank;
  const int32_t* slot;
  const float* pair_w;
  const float* scale_w;  // BF16 rows only, nullable: each destination row is bf16(w[t,j] * x[t])
  const int64_t* topk_idx;   // by-rank views, nullable: the routing (for local expert ids)
  int32_t* recv_topk_idx;    // by-rank, nullable: [R, cap, k] local expert id or -1
  float* recv_topk_w;        // by-rank, nullable: [R, cap, k] topk weight or 0
  const int32_t* psum;
  const int32_t* pad_excl;
  int32_t* status;
};

cudaError_t launch_dispatch(const DispatchLaunch& L, bool fp8, cudaStream_t s);
int layout_dispatch_chunk(int64_t T, int64_t H, bool fp8, int E, int R, int grid, int k);
cudaError_t launch_layout_dispatch(const LayoutLaunch& LL, int64_t cap_check, int chunk, const DispatchLaunch& L,
                                   bool fp8, cudaStream_t st);

struct CombineLaunch {
  const void* y;
  const float* w;
  const void* bias;
  void* out;
  int64_t T, cap, H;
  int64_t R;  // logical ranks (y holds R * cap rows)
  int k;
  int grid;
  const int32_t* pair_rank;
  const int32_t* slot;
  int32_t* status;
  bool packed;  // items sized by the token's source rows (the by-rank combine), no weights
};

cudaError_t launch_combine(const CombineLaunch& L, cudaStream_t s);

struct GradWeightsLaunch {
  const void* grad_out;  // bf16 [T, H]
  const void* y;         // bf16 [R, cap, H]
  float* grad_w;         // [T, k]
  int64_t T, cap, H;
  int k;
  int grid;
  const int32_t* pair_rank;
  const int32_t* slot;
  int32_t* status;
};

cudaError_t launch_grad_weights(const GradWeightsLaunch& L, cudaStream_t s);

struct GemmLaunch {
  const int32_t* psum;           // handle: inclusive aligned prefix per rank [E]
  const int32_t* rows_per_rank;  // handle [R]
  const float* sx;               // [R, cap, KB] row scales of the dispatched rows
  const float* sw;               // [E, NB, KB] weight block scales
  void* out;                     // bf16 [R, cap, N]
  int64_t cap, N;
  int R, E, E_loc, NB, KB;
  int grid;
  int32_t* status;
};

cudaError_t launch_expert_gemm(const GemmLaunch& L, const void* x, const void* w, cudaStream_t s);
uint32_t expert_gemm_smem_bytes(int R, int E);

void note_launch(int n = 1);
int sm_count(int device);

// Raise a kernel's dynamic shared-memory limit once per device (the attribute is per function).
template <typename Kernel>
cudaError_t set_smem_limit_once(Kernel kernel, int bytes, unsigned long long* done_mask) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && ((*done_mask >> dev) & 1ull)) return cudaSuccess;
  err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err == cudaSuccess && dev < 64) *done_mask |= 1ull << dev;
  return err;
}

// Launch with programmatic stream serialization: the kernel may be scheduled while the
// previous kernel in the stream finishes; it calls grid_dependency_wait() before it reads
// anything that kernel wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

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

// MOE_DEBUG builds: returns `cond`; on the first failure records (code, detail) in status[1..3]
// so the host can report it, and the caller skips the access.  Release builds: always true.
__device__ __forceinline__ bool dbg_ok(bool cond, int32_t* status, int32_t code, int64_t detail) {
  if (!kDebugChecks || cond) return true;
  if ((atomicOr(status, kStatusBounds) & kStatusBounds) == 0) {
    status[1] = code;
    status[2] = (int32_t)(detail & 0xffffffff);
    status[3] = (int32_t)(detail >> 32);
  }
  return false;
}

// Wait until the previous kernel in the stream has completed and its writes are visible (a no-op
// when the kernel was not launched as a programmatic dependent).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Allow the next kernel in the stream to be scheduled (it still waits for this one to finish
// before reading its results).
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

}  // namespace moe

// ------------------------------------------------------------------------------ TMA bulk copies
// 1-D bulk copies (cp.async.bulk) between global and shared memory, completed on an mbarrier
// (loads) or a bulk-group (stores).  Every address is 16-byte aligned and every size a multiple
// of 16 bytes; no multicast.
namespace moe {

constexpr int32_t kStatusTimeout = 4;                  // a bounded wait on an mbarrier gave up
constexpr uint64_t kWaitLimitNs = 2000000000ull;        // 2 s of wall-clock time per wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase of `bar` with the given parity to complete.  Bounded by wall-clock time:
// after kWaitLimitNs it records kStatusTimeout and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 63) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) break;
  }
  atomicOr(status, kStatusTimeout);
  return false;
}

// Warp-wide wait: lane 0 waits (bounded), the result is broadcast, and every lane then observes
// the completed phase itself (acquire).  Call with the whole warp.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, int32_t* status) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, status);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) mbar_try_wait(bar, parity);
  return ok;
}

__device__ __forceinline__ void bulk_load(uint32_t dst_smem, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dst_smem),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void bulk_store(void* dst, uint32_t src_smem, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src_smem), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

}  // namespace moe

// ------------------------------------------------------------------------------ pair metadata
namespace moe {

// The (rank, slot, weight[, expert]) of one (token, j) pair.
struct PairBatch {
  int32_t rank, slot;
  float w;
  int32_t e;  // expert id (only when `ids` is given), else -1
};

// Tokens of CTA b of G in the dispatch and combine kernels: its q-th token is b + q * G, so the
// grid works on neighbouring tokens at any moment.  cta_tokens = how many the CTA has.
__device__ __forceinline__ int64_t cta_tokens(int64_t T) {
  return (int64_t)blockIdx.x < T ? (T - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
}

__device__ __forceinline__ int64_t cta_token(int64_t q) { return (int64_t)blockIdx.x + q * gridDim.x; }

// One warp-wide load of the pairs of the CTA's tokens q0 .. q0 + 32 / k - 1 (lane l: token q0 +
// l / k, pair l % k; lanes_used = (32 / k) * k), for token indices below n_tok.
__device__ __forceinline__ PairBatch load_cta_pairs(const int32_t* pair_rank, const int32_t* slot, const float* w,
                                                    int64_t q0, int64_t n_tok, int k, int lane, int lanes_used,
                                                    const int64_t* ids = nullptr) {
  PairBatch b{-1, -1, 0.0f, -1};
  const int q = lane / k, j = lane - q * k;
  if (lane < lanes_used && q0 + q < n_tok) {
    const int64_t p = cta_token(q0 + q) * k + j;
    b.rank = __ldg(pair_rank + p);
    b.slot = __ldg(slot + p);
    if (w) b.w = __ldg(w + p);
    if (ids && b.rank >= 0) b.e = (int32_t)__ldg(ids + p);
  }
  return b;
}

}  // namespace moe
