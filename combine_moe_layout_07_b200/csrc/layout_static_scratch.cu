// layout_static_scratch.cu -- moe_layout_static_scratch: the same layout as moe_layout, for
// callers that cannot allocate device memory.
//
// Who needs it: code whose GPU memory belongs to another allocator (a framework's caching
// allocator that has reserved nearly all of HBM, or an arena handed out by an embedding
// runtime), and serving loops that forbid allocation calls on their hot path because a driver
// allocation can block on other work.  moe_layout allocates a handle per call; this entry point
// writes into buffers the caller owns and keeps its temporaries in one file-scope device array.
//
// The array (MOE_STATIC_SCRATCH_BYTES) is part of the library's device image: every GPU that
// loads the library holds it until the process exits.  All calls share it and it keeps the last
// call's contents, so the status word and the scan's ticket counter are cleared at the start of
// every call (all other scratch regions are fully rewritten before they are read; the caller's
// tokens_per_rank, which the kernels sum into, is cleared too).  Calls whose GPU work overlaps -- on two
// streams, or from two host threads, on the same device -- race on the array.
//
// Host code cannot use the array's name as a device address: the first call on each device,
// with that device current, asks the runtime for the address (cudaGetSymbolAddress) and caches
// it by device ordinal.  That first call should come before any stream capture.  The cache
// assumes the runtime's primary context: after cudaDeviceReset, or from a context the caller
// created through the driver API, the cached address is stale, and neither case is supported.
//
// Kernels: the one-CTA layout (k_layout_small) when T * k <= 8192 and E <= 1024, otherwise
// count -> scan -> assign over 256-token chunks.  moe_layout picks its kernels by other rules
// (the one-launch cooperative layout, adaptive chunks), but the layout is integer work with one
// correct result, so the outputs are the same.
//
// Nothing here calls cudaMalloc, cudaMallocAsync, cudaMallocHost, cudaFree or any allocating
// library routine.
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

__device__ __align__(256) unsigned char g_layout_scratch[MOE_STATIC_SCRATCH_BYTES];

cudaError_t scratch_address(int device, void** out) {
  static void* addr[64] = {};
  static std::mutex mu;
  if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[device]) {
    void* p = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&p, g_layout_scratch);
    if (err != cudaSuccess) return err;
    addr[device] = p;
  }
  *out = addr[device];
  return cudaSuccess;
}

int64_t round256(int64_t n) { return ((n + 255) / 256) * 256; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_layout_static_scratch(const moe_params_t* p, const int64_t* topk_idx,
                                         const float* topk_weights, int32_t* counts, int32_t* psum,
                                         int32_t* rows_per_rank, int32_t* tokens_per_rank,
                                         uint8_t* token_in_rank, int32_t* slots, int32_t* row_src,
                                         float* row_weights, int32_t* device_status,
                                         int32_t* host_rows_per_rank, void* stream) {
  // argument checks: the same limits as moe_layout, plus caller-owned row maps
  if (!p) return MOE_ERR_INVALID_ARG;
  if (p->num_tokens < 0 || p->num_logical_ranks < 1 || p->num_experts < 1 || p->topk < 1 ||
      p->expert_alignment < 1 || p->hidden < 8 || p->hidden % 8 != 0 || p->num_sms < 0 || p->flags != 0 ||
      (p->do_cpu_sync != 0 && p->do_cpu_sync != 1) || p->recv_capacity_rows < 1 ||
      p->num_experts % p->num_logical_ranks != 0)
    return MOE_ERR_INVALID_ARG;
  if (p->topk > kMaxTopk || p->num_experts > kMaxExperts || p->recv_capacity_rows >= (int64_t)1 << 31 ||
      p->num_tokens * (int64_t)p->topk + (int64_t)p->num_experts * p->expert_alignment >= (int64_t)1 << 31)
    return MOE_ERR_UNSUPPORTED;
  const int64_t T = p->num_tokens, k = p->topk, E = p->num_experts, R = p->num_logical_ranks;
  if (!counts || !psum || !rows_per_rank || !tokens_per_rank || !row_src || !row_weights ||
      (T > 0 && (!topk_idx || !token_in_rank || !slots)))
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(topk_idx) & 7u) || (reinterpret_cast<uintptr_t>(topk_weights) & 3u) ||
      (reinterpret_cast<uintptr_t>(device_status) & 3u))
    return MOE_ERR_INVALID_ARG;
  // without the host wait, device_status is the only place a bad id or an overflow can be read
  if (!p->do_cpu_sync && !device_status) return MOE_ERR_INVALID_ARG;

  // scratch regions: status and scan ticket | pad prefix | chunk counts | pair rank | pair weight
  const int64_t C = (T + kChunkTokens - 1) / kChunkTokens;
  const int64_t o_status = 0, o_pad = o_status + 256, o_ccnt = o_pad + round256(4 * (E + 1)),
                o_prank = o_ccnt + round256(4 * C * E), o_pw = o_prank + round256(4 * T * k),
                end = o_pw + round256(4 * T * k);
  if (end > (int64_t)MOE_STATIC_SCRATCH_BYTES) return MOE_ERR_SCRATCH_LIMIT;

  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return MOE_ERR_CUDA;
  void* base = nullptr;
  if (scratch_address(device, &base) != cudaSuccess) return MOE_ERR_CUDA;
  char* b = static_cast<char*>(base);

  DeviceArrays d{};
  d.status = device_status ? device_status : reinterpret_cast<int32_t*>(b + o_status);
  d.ticket = reinterpret_cast<int32_t*>(b + o_status + 64);
  d.cnt = counts;
  d.psum = psum;
  d.pad_excl = reinterpret_cast<int32_t*>(b + o_pad);
  d.rows_per_rank = rows_per_rank;
  d.tokens_per_rank = tokens_per_rank;
  d.token_in_rank = token_in_rank;
  d.slot = slots;
  d.pair_rank = reinterpret_cast<int32_t*>(b + o_prank);
  d.pair_w = reinterpret_cast<float*>(b + o_pw);
  d.chunk_cnt = reinterpret_cast<int32_t*>(b + o_ccnt);
  d.row_src = row_src;
  d.row_w = row_weights;

  LayoutLaunch L{};
  L.idx = topk_idx;
  L.w = topk_weights;
  L.T = T;
  L.k = (int)k;
  L.E = (int)E;
  L.R = (int)R;
  L.E_loc = (int)(E / R);
  L.A = p->expert_alignment;
  L.chunk = kChunkTokens;
  L.num_chunks = (int)C;
  L.grid_chunks = (int)C;
  if (p->num_sms > 0 && L.grid_chunks > p->num_sms) L.grid_chunks = p->num_sms;
  L.row_cap = p->recv_capacity_rows;
  L.d = d;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool one_cta = layout_fits_one_cta(T, (int)k, (int)E);
  cudaError_t err = cudaMemsetAsync(d.status, 0, sizeof(int32_t), s);
  if (err == cudaSuccess) err = cudaMemsetAsync(d.ticket, 0, sizeof(int32_t), s);
  if (err == cudaSuccess) err = cudaMemsetAsync(tokens_per_rank, 0, sizeof(int32_t) * (size_t)R, s);  // summed atomically
  if (one_cta) {
    if (err == cudaSuccess) err = launch_layout_small(L, p->recv_capacity_rows, s);
  } else {
    if (err == cudaSuccess) err = launch_layout_count(L, s);
    if (err == cudaSuccess) err = launch_layout_scan(L, p->recv_capacity_rows, s);
  }
  if (err != cudaSuccess) return MOE_ERR_CUDA;

  if (p->do_cpu_sync) {
    int32_t flags = 0;  // pageable host copies: the runtime stages them, nothing is allocated here
    err = cudaMemcpyAsync(&flags, d.status, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
    if (err == cudaSuccess && host_rows_per_rank)
      err = cudaMemcpyAsync(host_rows_per_rank, rows_per_rank, sizeof(int32_t) * (size_t)R,
                            cudaMemcpyDeviceToHost, s);
    if (err == cudaSuccess) err = cudaStreamSynchronize(s);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    if (flags & kStatusBadExpert) return MOE_ERR_BAD_EXPERT;
    if (flags & kStatusCapacity) return MOE_ERR_CAPACITY;
  }
  if (one_cta) return MOE_OK;
  return launch_layout_assign(L, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
