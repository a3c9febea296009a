// moe_api.cu -- the C ABI declared in include/moe.h: argument checks, the handle's device
// memory, and the order of kernel launches for layout, dispatch and combine.
//
// The handle follows "Why MoE gets stuck on communication" (locsic.com) section 1 and 2: it
// records one dispatch's grouping and counts, combine reuses it, and it must outlive every
// operation that uses it.  do_cpu_sync follows the same page and "deepep-expert-parallel-
// dispatch-combine" (phantomic12.github.io): with it, the counts are copied to the host and
// the call waits; without it, nothing waits and consumers read the device-side psum.
#include <atomic>
#include <chrono>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>

#include "moe_internal.cuh"
#include "trace.cuh"

namespace moe {

static std::atomic<int64_t> g_launches{0};
void note_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int sm_count(int device) {
  static int cache[64] = {0};
  if (device >= 0 && device < 64 && cache[device] > 0) return cache[device];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0) n = 1;
  if (device >= 0 && device < 64) cache[device] = n;
  return n;
}

static int grid_for(int num_sms, int device) {
  const int n = sm_count(device);
  return (num_sms > 0 && num_sms < n) ? num_sms : n;
}

// The handle's arrays come from a library-owned stream-ordered pool per device whose release
// threshold keeps freed blocks mapped, so a layout -> free -> layout cycle reuses memory instead
// of returning it to the driver at every synchronisation.
static cudaError_t handle_pool(int device, cudaMemPool_t* out) {
  static cudaMemPool_t pools[64] = {};
  static std::mutex mu;
  if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!pools[device]) {
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = device;
    cudaMemPool_t pool;
    cudaError_t err = cudaMemPoolCreate(&pool, &props);
    if (err != cudaSuccess) return err;
    uint64_t keep = ~0ull;
    err = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (err != cudaSuccess) return err;
    pools[device] = pool;
  }
  *out = pools[device];
  return cudaSuccess;
}

static cudaError_t pool_alloc(void** p, size_t bytes, int device, cudaStream_t s) {
  cudaMemPool_t pool;
  cudaError_t err = handle_pool(device, &pool);
  if (err != cudaSuccess) return err;
  return cudaMallocFromPoolAsync(p, bytes, pool, s);
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
static int64_t align_up64(int64_t n, int64_t a) { return ((n + a - 1) / a) * a; }

// Pinned host staging for the do_cpu_sync copy, one per host thread.
struct PinnedStage {
  void* p = nullptr;
  size_t n = 0;
  ~PinnedStage() {
    if (p) cudaFreeHost(p);
  }
  void* get(size_t need) {
    if (need <= n) return p;
    if (p) cudaFreeHost(p);
    p = nullptr;
    n = 0;
    if (cudaMallocHost(&p, need) != cudaSuccess) return nullptr;
    n = need;
    return p;
  }
};
static thread_local PinnedStage g_stage;

// Pinned blocks for deferred count copies: a handle holds one until it is freed, then it goes
// back to this list for the next deferred layout (no cudaMallocHost on the steady path).
static std::mutex g_pin_mu;
static std::vector<std::pair<size_t, void*>> g_pin_free;

static void* pinned_take(size_t need, size_t* got) {
  need = (need + 4095) / 4096 * 4096;
  {
    std::lock_guard<std::mutex> lock(g_pin_mu);
    for (size_t i = 0; i < g_pin_free.size(); ++i)
      if (g_pin_free[i].first >= need) {
        void* p = g_pin_free[i].second;
        *got = g_pin_free[i].first;
        g_pin_free.erase(g_pin_free.begin() + (long)i);
        return p;
      }
  }
  void* p = nullptr;
  if (cudaMallocHost(&p, need) != cudaSuccess) return nullptr;
  *got = need;
  return p;
}

static void pinned_give(void* p, size_t n) {
  if (!p) return;
  std::lock_guard<std::mutex> lock(g_pin_mu);
  g_pin_free.emplace_back(n, p);
}

// Mapped pinned blocks through which the layout kernels hand the counts to a waiting host
// (do_cpu_sync); a handle holds one until it is freed.
static std::mutex g_map_mu;
static std::vector<std::pair<size_t, int32_t*>> g_map_free;

static int32_t* mapped_take(size_t need, size_t* got) {
  need = (need + 4095) / 4096 * 4096;
  {
    std::lock_guard<std::mutex> lock(g_map_mu);
    for (size_t i = 0; i < g_map_free.size(); ++i)
      if (g_map_free[i].first >= need) {
        int32_t* p = g_map_free[i].second;
        *got = g_map_free[i].first;
        g_map_free.erase(g_map_free.begin() + (long)i);
        return p;
      }
  }
  void* p = nullptr;
  if (cudaHostAlloc(&p, need, cudaHostAllocMapped | cudaHostAllocPortable) != cudaSuccess) return nullptr;
  *got = need;
  return static_cast<int32_t*>(p);
}

static void mapped_give(int32_t* p, size_t n) {
  if (!p) return;
  std::lock_guard<std::mutex> lock(g_map_mu);
  g_map_free.emplace_back(n, p);
}

// The do_cpu_sync copy: the handle keeps [status 4, ticket, pad 3][tokens_per_rank R]
// [rows_per_rank R] adjacent, so one copy brings flags and counts to the host.
static size_t count_stage_bytes(int64_t R) { return sizeof(int32_t) * (size_t)(8 + 2 * R); }

static cudaError_t enqueue_count_copy(const moe_handle_t* h, int32_t* stage, cudaStream_t s) {
  return cudaMemcpyAsync(stage, h->d.status, count_stage_bytes(h->p.num_logical_ranks), cudaMemcpyDeviceToHost, s);
}

// The do_cpu_sync epilogue once the copy into `stage` is complete: the status flags decide the
// result; on success the host counts are kept on the handle (and copied to host_rows_per_rank).
static int count_epilogue(moe_handle_t* h, const int32_t* stage, int32_t* host_rows_per_rank) {
  const int64_t R = h->p.num_logical_ranks;
  const int32_t flags = stage[0];
  if (flags & kStatusBadExpert) return MOE_ERR_BAD_EXPERT;
  if (flags & kStatusCapacity) return MOE_ERR_CAPACITY;
  const int32_t* tokens = stage + 8;
  const int32_t* rows = tokens + R;
  h->host_rows.assign(rows, rows + R);
  h->host_tokens.assign(tokens, tokens + R);
  h->counts_on_host = true;
  if (host_rows_per_rank) std::memcpy(host_rows_per_rank, rows, sizeof(int32_t) * (size_t)R);
  return MOE_OK;
}

static int check_params(const moe_params_t* p) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (p->num_tokens < 0 || p->num_logical_ranks < 1 || p->num_experts < 1 || p->topk < 1 ||
      p->expert_alignment < 1 || p->hidden < 8 || p->hidden % 8 != 0 || p->num_sms < 0 ||
      (p->flags & ~(MOE_LAYOUT_BY_RANK | MOE_DEFER_EPILOGUE)) != 0 ||
      (p->do_cpu_sync != 0 && p->do_cpu_sync != 1) || ((p->flags & MOE_DEFER_EPILOGUE) && !p->do_cpu_sync) ||
      p->recv_capacity_rows < 0)
    return MOE_ERR_INVALID_ARG;
  if (p->num_experts % p->num_logical_ranks != 0) return MOE_ERR_INVALID_ARG;
  if (p->topk > kMaxTopk || p->num_experts > kMaxExperts) return MOE_ERR_UNSUPPORTED;
  // every row index and prefix sum must fit in int32
  if (p->num_tokens * (int64_t)p->topk + (int64_t)p->num_experts * p->expert_alignment >= (int64_t)1 << 31)
    return MOE_ERR_UNSUPPORTED;
  if (p->recv_capacity_rows >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  if (p->recv_capacity_rows == 0 && p->do_cpu_sync == 0) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

static void release(moe_handle_t* h) {
  if (!h) return;
  if (h->block) cudaFreeAsync(h->block, h->stream);
  if (h->epi_event) cudaEventDestroy(h->epi_event);
  pinned_give(h->epi_stage, h->epi_bytes);
  mapped_give(h->host_block, h->host_block_bytes);
  delete h;
}

// Host side of publish_host_counts: spin until the layout marks the counts ready.  Bounded: a
// stream error, a stream that finished without publishing, or 10 s return false.
static bool wait_host_counts(const moe_handle_t* h, cudaStream_t s) {
  volatile int32_t* ready = h->host_block + 7;
  const auto t0 = std::chrono::steady_clock::now();
  for (uint32_t n = 1; *ready == 0; ++n) {
    if ((n & 1023) != 0) continue;
    const cudaError_t q = cudaStreamQuery(s);
    if (q == cudaSuccess) return *ready != 0;
    if (q != cudaErrorNotReady) return false;
    if (std::chrono::steady_clock::now() - t0 > std::chrono::seconds(10)) return false;
  }
  std::atomic_thread_fence(std::memory_order_acquire);
  return true;
}

// Everything moe_layout does before its launches: the handle and its arrays (one stream-ordered
// allocation), the mapped count block under do_cpu_sync, the chunking and the launch description.
// The arguments are checked by the caller.  On failure nothing is left allocated.
static int layout_prepare(const moe_params_t* p, const int64_t* topk_idx, const float* topk_weights, cudaStream_t s,
                          moe_handle_t** out_handle, LayoutLaunch* out_launch, bool* out_fused) {
  moe_handle_t* h = new (std::nothrow) moe_handle_t();
  if (!h) return MOE_ERR_OOM;
  h->p = *p;
  h->stream = s;
  if (cudaGetDevice(&h->device) != cudaSuccess) {
    delete h;
    return MOE_ERR_CUDA;
  }
  const int64_t T = p->num_tokens, k = p->topk, E = p->num_experts, R = p->num_logical_ranks;
  // Chunks.  The one-launch layout takes the smallest chunk of 32..256 tokens that leaves at most
  // one chunk per SM the layout may use, if its other limits hold (layout_fits_fused).  Under a
  // num_sms cap, when 256-token chunks still outnumber the SMs, it takes one chunk per SM of
  // ceil(T / SMs) tokens rounded up to a warp, if the pairs still fit the warps' registers.
  // Otherwise the count / assign kernels halve the chunk from kChunkTokens down to 32 tokens
  // while the batch gives fewer than two chunks per SM, so it still spreads over many CTAs
  // (a warp's run of pairs, chunk * k / 8, sets the assign kernel's serial work).
  const int sm_budget = grid_for(p->num_sms, h->device);
  int chunk = 32;
  while ((T + chunk - 1) / chunk > sm_budget && chunk < kChunkTokens) chunk *= 2;
  bool fused = layout_fits_fused((int)((T + chunk - 1) / chunk), chunk, (int)k, (int)E, sm_budget);
  if (!fused && sm_budget < sm_count(h->device) && (T + chunk - 1) / chunk > sm_budget) {
    const int64_t wide = align_up64((T + sm_budget - 1) / sm_budget, 32);
    if (wide < ((int64_t)1 << 30) &&
        layout_fits_fused((int)((T + wide - 1) / wide), (int)wide, (int)k, (int)E, sm_budget)) {
      chunk = (int)wide;
      fused = true;
    }
  }
  if (!fused) {
    const int64_t want_chunks = 2 * (int64_t)sm_count(h->device);
    chunk = kChunkTokens;
    while (chunk > 32 && (T + chunk - 1) / chunk < want_chunks) chunk /= 2;
  }
  h->num_chunks = (int)((T + chunk - 1) / chunk);
  const int64_t C = h->num_chunks;

  // One allocation for every array (256-byte aligned sub-arrays).  Without a capacity the row
  // maps are sized for the worst case of this batch: T * min(k, E_loc) + E_loc * (A - 1) rows.
  const int64_t E_loc = E / R;
  h->row_cap = p->recv_capacity_rows > 0
                   ? p->recv_capacity_rows
                   : T * (k < E_loc ? k : E_loc) + E_loc * (p->expert_alignment - 1);
  int64_t off = 0;
  auto take = [&](int64_t bytes) {
    const int64_t at = off;
    off = align_up64(off + bytes, 256);
    return at;
  };
  // status[4], the scan ticket, tokens_per_rank[R], rows_per_rank[R] and cnt[E] are adjacent: one
  // memset clears them all (the one-launch layout sums cnt atomically), one copy reads the first
  // four back
  const int64_t o_status = take(32 + 8 * R + 4 * E), o_psum = take(4 * E),
                o_pad = take(4 * (E + 1)), o_tir = take(T * R), o_slot = take(4 * T * k),
                o_prank = take(4 * T * k), o_pw = take(4 * T * k), o_ccnt = take(4 * C * E),
                o_rsrc = take(4 * R * h->row_cap), o_rw = take(4 * R * h->row_cap);
  // the non-expanded (by-rank) layout, on request and for R <= kMaxByRankRanks
  const bool by_rank = (p->flags & MOE_LAYOUT_BY_RANK) && R <= kMaxByRankRanks;
  const int64_t o_ctok = by_rank ? take(4 * C * R) : 0, o_trow = by_rank ? take(4 * T * R) : 0,
                o_tslot = by_rank ? take(4 * T * k) : 0;
  if (pool_alloc(&h->block, (size_t)off, h->device, s) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return MOE_ERR_OOM;
  }
  char* b = static_cast<char*>(h->block);
  DeviceArrays& d = h->d;
  d.status = reinterpret_cast<int32_t*>(b + o_status);
  d.ticket = d.status + 4;
  d.tokens_per_rank = d.status + 8;
  d.rows_per_rank = d.tokens_per_rank + R;
  d.cnt = d.rows_per_rank + R;
  d.psum = reinterpret_cast<int32_t*>(b + o_psum);
  d.pad_excl = reinterpret_cast<int32_t*>(b + o_pad);
  d.token_in_rank = reinterpret_cast<uint8_t*>(b + o_tir);
  d.slot = reinterpret_cast<int32_t*>(b + o_slot);
  d.pair_rank = reinterpret_cast<int32_t*>(b + o_prank);
  d.pair_w = reinterpret_cast<float*>(b + o_pw);
  d.chunk_cnt = reinterpret_cast<int32_t*>(b + o_ccnt);
  d.row_src = reinterpret_cast<int32_t*>(b + o_rsrc);
  d.row_w = reinterpret_cast<float*>(b + o_rw);
  if (by_rank) {
    d.chunk_tok = reinterpret_cast<int32_t*>(b + o_ctok);
    d.token_row = reinterpret_cast<int32_t*>(b + o_trow);
    d.tslot = reinterpret_cast<int32_t*>(b + o_tslot);
  }

  // do_cpu_sync without deferral: the kernels publish the counts into a mapped pinned block
  const bool publish = p->do_cpu_sync && !(p->flags & MOE_DEFER_EPILOGUE);
  if (publish) {
    h->host_block = mapped_take(count_stage_bytes(R), &h->host_block_bytes);
    void* dev_view = nullptr;
    if (!h->host_block || cudaHostGetDevicePointer(&dev_view, h->host_block, 0) != cudaSuccess) {
      cudaGetLastError();
      release(h);
      return MOE_ERR_OOM;
    }
    reinterpret_cast<volatile int32_t*>(h->host_block)[7] = 0;
    d.host_counts = static_cast<int32_t*>(dev_view);
  }

  LayoutLaunch L{};
  L.idx = topk_idx;
  L.w = topk_weights;
  L.T = T;
  L.k = (int)k;
  L.E = (int)E;
  L.R = (int)R;
  L.E_loc = (int)E_loc;
  L.A = p->expert_alignment;
  L.chunk = chunk;
  L.num_chunks = h->num_chunks;
  L.grid_chunks = h->num_chunks;
  if (p->num_sms > 0 && L.grid_chunks > p->num_sms) L.grid_chunks = p->num_sms;
  L.row_cap = h->row_cap;
  L.by_rank = by_rank ? 1 : 0;
  L.d = d;

  *out_handle = h;
  *out_launch = L;
  *out_fused = fused;
  return MOE_OK;
}

// The layout's launches: the status block cleared, then the one-launch layout or count -> scan ->
// assign.  (Small batches take 32-token chunks over many CTAs: faster than one CTA whose warps
// each walk hundreds of pairs.)
static cudaError_t layout_enqueue(const moe_params_t* p, const LayoutLaunch& L, bool fused, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(L.d.status, 0, (size_t)(32 + 8 * (int64_t)L.R + 4 * (int64_t)L.E), s);
  if (fused) {
    if (err == cudaSuccess) err = launch_layout_fused(L, p->recv_capacity_rows, s);
  } else {
    if (err == cudaSuccess) err = launch_layout_count(L, s);
    if (err == cudaSuccess) err = launch_layout_scan(L, p->recv_capacity_rows, s);
    if (err == cudaSuccess) err = launch_layout_assign(L, s);
  }
  return err;
}

// The launch description of an expanded dispatch on handle h.
static DispatchLaunch expanded_dispatch(const moe_handle_t* h, const void* x, void* recv_x, float* recv_scales,
                                        float* recv_weights, int64_t cap, int do_zero_padding, int num_sms) {
  const moe_params_t& p = h->p;
  DispatchLaunch L{};
  L.x = x;
  L.recv_x = recv_x;
  L.recv_scales = recv_scales;
  L.recv_w = recv_weights;
  L.T = p.num_tokens;
  L.cap = cap;
  L.H = p.hidden;
  L.k = p.topk;
  L.E = p.num_experts;
  L.E_loc = p.num_experts / p.num_logical_ranks;
  L.zero_padding = do_zero_padding;
  L.R = p.num_logical_ranks;
  L.grid = grid_for(num_sms, h->device);
  L.pair_rank = h->d.pair_rank;
  L.slot = h->d.slot;
  L.pair_w = h->d.pair_w;
  L.psum = h->d.psum;
  L.pad_excl = h->d.pad_excl;
  L.status = h->d.status;
  return L;
}

}  // namespace moe

using namespace moe;

extern "C" {

int64_t moe_recv_capacity_hint(const moe_params_t* p, int64_t max_tokens_per_rank) {
  if (check_params(p) == MOE_ERR_INVALID_ARG || max_tokens_per_rank < 0) return -1;
  const int64_t e_loc = p->num_experts / p->num_logical_ranks;
  const int64_t per_token = p->topk < e_loc ? p->topk : e_loc;
  return (int64_t)p->num_logical_ranks * max_tokens_per_rank * per_token + e_loc * (p->expert_alignment - 1);
}

int moe_layout(const moe_params_t* p, const int64_t* topk_idx, const float* topk_weights, void* stream,
               moe_handle_t** out_handle, int32_t* host_rows_per_rank) {
  TraceRange trace("moe_layout");
  if (!out_handle) return MOE_ERR_INVALID_ARG;
  *out_handle = nullptr;
  int rc = check_params(p);
  if (rc != MOE_OK) return rc;
  if (!topk_idx && p->num_tokens > 0) return MOE_ERR_INVALID_ARG;
  if (!aligned4(topk_weights)) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(topk_idx) & 7u) != 0) return MOE_ERR_INVALID_ARG;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  moe_handle_t* h = nullptr;
  LayoutLaunch L{};
  bool fused = false;
  rc = layout_prepare(p, topk_idx, topk_weights, s, &h, &L, &fused);
  if (rc != MOE_OK) return rc;
  const int64_t R = p->num_logical_ranks;
  const bool publish = p->do_cpu_sync && !(p->flags & MOE_DEFER_EPILOGUE);
  cudaError_t err = layout_enqueue(p, L, fused, s);
  if (err != cudaSuccess) {
    release(h);
    return MOE_ERR_CUDA;
  }

  if (p->do_cpu_sync && (p->flags & MOE_DEFER_EPILOGUE)) {
    // the copy is enqueued into the handle's own pinned block; moe_handle_wait waits for it
    h->epi_stage = static_cast<int32_t*>(pinned_take(count_stage_bytes(R), &h->epi_bytes));
    if (!h->epi_stage) {
      release(h);
      return MOE_ERR_OOM;
    }
    err = cudaEventCreateWithFlags(&h->epi_event, cudaEventDisableTiming);
    if (err == cudaSuccess) err = enqueue_count_copy(h, h->epi_stage, s);
    if (err == cudaSuccess) err = cudaEventRecord(h->epi_event, s);
    if (err != cudaSuccess) {
      release(h);
      return MOE_ERR_CUDA;
    }
    h->epi_pending = true;
  } else if (publish) {
    // the host waits only for the counts; the rest of the layout runs on, stream-ordered
    // before every later use of the handle
    if (!wait_host_counts(h, s)) {
      cudaStreamSynchronize(s);
      cudaGetLastError();
      release(h);
      return MOE_ERR_CUDA;
    }
    rc = count_epilogue(h, h->host_block, host_rows_per_rank);
    if (rc != MOE_OK) {
      cudaStreamSynchronize(s);  // the handle goes away: no kernel may still use its memory
      release(h);
      return rc;
    }
  }
  *out_handle = h;
  return MOE_OK;
}

int moe_handle_wait(moe_handle_t* h, int32_t* host_rows_per_rank) {
  TraceRange trace("moe_handle_wait");
  if (!h) return MOE_ERR_INVALID_ARG;
  if (h->epi_pending) {
    if (cudaEventSynchronize(h->epi_event) != cudaSuccess) return MOE_ERR_CUDA;
    h->epi_pending = false;
    h->epi_rc = count_epilogue(h, h->epi_stage, nullptr);
  }
  if (h->epi_rc != MOE_OK) return h->epi_rc;
  if (!h->counts_on_host) return MOE_ERR_INVALID_ARG;  // do_cpu_sync = 0: nothing comes to the host
  if (host_rows_per_rank)
    std::memcpy(host_rows_per_rank, h->host_rows.data(), sizeof(int32_t) * h->host_rows.size());
  return MOE_OK;
}

int moe_dispatch(const moe_handle_t* h, const void* x, int out_dtype, void* recv_x, float* recv_scales,
                 float* recv_weights, int64_t cap, int do_expand, int do_zero_padding, int num_sms,
                 void* stream) {
  TraceRange trace("moe_dispatch");
  if (!h) return MOE_ERR_INVALID_ARG;
  if (do_expand != 0 && do_expand != 1) return MOE_ERR_INVALID_ARG;
  if (do_zero_padding != 0 && do_zero_padding != 1) return MOE_ERR_INVALID_ARG;
  if (out_dtype != MOE_DTYPE_BF16 && out_dtype != MOE_DTYPE_FP8_E4M3) return MOE_ERR_INVALID_ARG;
  if (cap < 0 || cap >= (int64_t)1 << 31 || num_sms < 0) return MOE_ERR_INVALID_ARG;
  const bool fp8 = out_dtype == MOE_DTYPE_FP8_E4M3;
  const moe_params_t& p = h->p;
  if (fp8 && (p.hidden % 128 != 0 || !recv_scales || !aligned4(recv_scales))) return MOE_ERR_INVALID_ARG;
  if (p.num_tokens > 0 && (!x || !recv_x)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(recv_x) || !aligned4(recv_weights)) return MOE_ERR_INVALID_ARG;
  if (!do_expand)  // one row per (token, rank); recv_weights then holds [R, cap, k] weights
    return moe_dispatch_by_rank(h, x, nullptr, out_dtype, recv_x, recv_scales, nullptr, recv_weights, cap, num_sms,
                                stream);
  if (h->counts_on_host) {
    for (int32_t v : h->host_rows)
      if (v > cap) return MOE_ERR_CAPACITY;
  }
  if (p.num_tokens == 0) return MOE_OK;
  const DispatchLaunch L = expanded_dispatch(h, x, recv_x, recv_scales, recv_weights, cap, do_zero_padding, num_sms);
  return launch_dispatch(L, fp8, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_layout_dispatch(const moe_params_t* p, const int64_t* topk_idx, const float* topk_weights, const void* x,
                        int out_dtype, void* recv_x, float* recv_scales, float* recv_weights, int do_zero_padding,
                        void* stream, moe_handle_t** out_handle) {
  TraceRange trace("moe_layout_dispatch");
  if (!out_handle) return MOE_ERR_INVALID_ARG;
  *out_handle = nullptr;
  int rc = check_params(p);
  if (rc != MOE_OK) return rc;
  if (p->do_cpu_sync != 0 || p->flags != 0) return MOE_ERR_INVALID_ARG;
  if (!topk_idx && p->num_tokens > 0) return MOE_ERR_INVALID_ARG;
  if (!aligned4(topk_weights) || (reinterpret_cast<uintptr_t>(topk_idx) & 7u) != 0) return MOE_ERR_INVALID_ARG;
  if (do_zero_padding != 0 && do_zero_padding != 1) return MOE_ERR_INVALID_ARG;
  if (out_dtype != MOE_DTYPE_BF16 && out_dtype != MOE_DTYPE_FP8_E4M3) return MOE_ERR_INVALID_ARG;
  const bool fp8 = out_dtype == MOE_DTYPE_FP8_E4M3;
  if (fp8 && (p->hidden % 128 != 0 || !recv_scales || !aligned4(recv_scales))) return MOE_ERR_INVALID_ARG;
  if (p->num_tokens > 0 && (!x || !recv_x)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(recv_x) || !aligned4(recv_weights)) return MOE_ERR_INVALID_ARG;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  moe_handle_t* h = nullptr;
  LayoutLaunch L{};
  bool fused = false;
  rc = layout_prepare(p, topk_idx, topk_weights, s, &h, &L, &fused);
  if (rc != MOE_OK) return rc;
  cudaError_t err = cudaSuccess;
  if (p->num_tokens > 0) {
    const int64_t cap = p->recv_capacity_rows;
    const DispatchLaunch D =
        expanded_dispatch(h, x, recv_x, recv_scales, recv_weights, cap, do_zero_padding, p->num_sms);
    const int ld_chunk =
        layout_dispatch_chunk(p->num_tokens, p->hidden, fp8, p->num_experts, p->num_logical_ranks, D.grid, L.k);
    if (ld_chunk > 0) {
      err = cudaMemsetAsync(L.d.status, 0, (size_t)(32 + 8 * (int64_t)L.R + 4 * (int64_t)L.E), s);
      if (err == cudaSuccess) err = launch_layout_dispatch(L, cap, ld_chunk, D, fp8, s);
    } else {  // the same results from the layout's launches and the dispatch kernel
      err = layout_enqueue(p, L, fused, s);
      if (err == cudaSuccess) err = launch_dispatch(D, fp8, s);
    }
  } else {
    err = layout_enqueue(p, L, fused, s);
  }
  if (err != cudaSuccess) {
    release(h);
    return MOE_ERR_CUDA;
  }
  *out_handle = h;
  return MOE_OK;
}

int moe_combine(const moe_handle_t* h, const void* y, const float* topk_weights, const void* bias, void* out,
                int64_t cap, int num_sms, void* stream) {
  TraceRange trace("moe_combine");
  if (!h) return MOE_ERR_INVALID_ARG;
  if (cap < 0 || cap >= (int64_t)1 << 31 || num_sms < 0) return MOE_ERR_INVALID_ARG;
  const moe_params_t& p = h->p;
  if (p.num_tokens > 0 && (!y || !out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(out) || !aligned16(bias) || !aligned4(topk_weights)) return MOE_ERR_INVALID_ARG;
  if (h->counts_on_host) {
    for (int32_t v : h->host_rows)
      if (v > cap) return MOE_ERR_CAPACITY;
  }
  if (p.num_tokens == 0) return MOE_OK;
  CombineLaunch L{};
  L.y = y;
  L.w = topk_weights;
  L.bias = bias;
  L.out = out;
  L.T = p.num_tokens;
  L.cap = cap;
  L.H = p.hidden;
  L.k = p.topk;
  L.R = p.num_logical_ranks;
  L.grid = grid_for(num_sms, h->device);
  L.pair_rank = h->d.pair_rank;
  L.slot = h->d.slot;
  L.status = h->d.status;
  return launch_combine(L, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_dispatch_by_rank(const moe_handle_t* h, const void* x, const int64_t* topk_idx, int out_dtype, void* recv_x,
                         float* recv_scales, int32_t* recv_topk_idx, float* recv_topk_weights, int64_t cap,
                         int num_sms, void* stream) {
  TraceRange trace("moe_dispatch_by_rank");
  if (!h) return MOE_ERR_INVALID_ARG;
  if (out_dtype != MOE_DTYPE_BF16 && out_dtype != MOE_DTYPE_FP8_E4M3) return MOE_ERR_INVALID_ARG;
  if (cap < 0 || cap >= (int64_t)1 << 31 || num_sms < 0) return MOE_ERR_INVALID_ARG;
  const bool fp8 = out_dtype == MOE_DTYPE_FP8_E4M3;
  const moe_params_t& p = h->p;
  if (!h->d.tslot) return MOE_ERR_UNSUPPORTED;  // more logical ranks than the by-rank layout keeps
  if (fp8 && (p.hidden % 128 != 0 || !recv_scales || !aligned4(recv_scales))) return MOE_ERR_INVALID_ARG;
  if (p.num_tokens > 0 && (!x || !recv_x)) return MOE_ERR_INVALID_ARG;
  if (recv_topk_idx && !topk_idx) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(recv_x) || !aligned4(recv_topk_idx) || !aligned4(recv_topk_weights) ||
      (reinterpret_cast<uintptr_t>(topk_idx) & 7u))
    return MOE_ERR_INVALID_ARG;
  if (h->counts_on_host) {
    for (int32_t v : h->host_tokens)
      if (v > cap) return MOE_ERR_CAPACITY;
  }
  if (p.num_tokens == 0) return MOE_OK;
  DispatchLaunch L{};
  L.x = x;
  L.recv_x = recv_x;
  L.recv_scales = recv_scales;
  L.T = p.num_tokens;
  L.cap = cap;
  L.H = p.hidden;
  L.R = p.num_logical_ranks;
  L.k = p.topk;
  L.E = p.num_experts;
  L.E_loc = p.num_experts / p.num_logical_ranks;
  L.zero_padding = 0;  // no alignment padding without expansion
  L.grid = grid_for(num_sms, h->device);
  L.pair_rank = h->d.pair_rank;
  L.slot = h->d.tslot;
  L.pair_w = h->d.pair_w;
  L.topk_idx = topk_idx;
  L.recv_topk_idx = recv_topk_idx;
  L.recv_topk_w = recv_topk_weights;
  L.psum = h->d.psum;
  L.pad_excl = h->d.pad_excl;
  L.status = h->d.status;
  return launch_dispatch(L, fp8, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_combine_by_rank(const moe_handle_t* h, const void* y, const void* bias, void* out, int64_t cap, int num_sms,
                        void* stream) {
  TraceRange trace("moe_combine_by_rank");
  if (!h) return MOE_ERR_INVALID_ARG;
  if (cap < 0 || cap >= (int64_t)1 << 31 || num_sms < 0) return MOE_ERR_INVALID_ARG;
  const moe_params_t& p = h->p;
  if (!h->d.tslot) return MOE_ERR_UNSUPPORTED;
  if (p.num_tokens > 0 && (!y || !out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(out) || !aligned16(bias)) return MOE_ERR_INVALID_ARG;
  if (h->counts_on_host) {
    for (int32_t v : h->host_tokens)
      if (v > cap) return MOE_ERR_CAPACITY;
  }
  if (p.num_tokens == 0) return MOE_OK;
  CombineLaunch L{};
  L.y = y;
  L.w = nullptr;  // the per-rank rows are partial sums of already-weighted expert outputs
  L.bias = bias;
  L.out = out;
  L.T = p.num_tokens;
  L.cap = cap;
  L.H = p.hidden;
  L.k = p.topk;
  L.R = p.num_logical_ranks;
  L.grid = grid_for(num_sms, h->device);
  L.pair_rank = h->d.pair_rank;
  L.slot = h->d.tslot;
  L.status = h->d.status;
  L.packed = true;  // a token has at most one row per rank: items sized by its rows
  return launch_combine(L, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_combine_backward(const moe_handle_t* h, const void* grad_out, const float* topk_weights, void* grad_y,
                         int64_t cap, int do_zero_padding, const void* y, float* grad_weights, int num_sms,
                         void* stream) {
  TraceRange trace("moe_combine_backward");
  if (!h) return MOE_ERR_INVALID_ARG;
  if (cap < 0 || cap >= (int64_t)1 << 31 || num_sms < 0) return MOE_ERR_INVALID_ARG;
  if (do_zero_padding != 0 && do_zero_padding != 1) return MOE_ERR_INVALID_ARG;
  const moe_params_t& p = h->p;
  if (p.num_tokens > 0 && (!grad_out || !grad_y)) return MOE_ERR_INVALID_ARG;
  if (grad_weights && !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(grad_out) || !aligned16(grad_y) || !aligned16(y) || !aligned4(topk_weights) ||
      !aligned4(grad_weights))
    return MOE_ERR_INVALID_ARG;
  if (h->counts_on_host) {
    for (int32_t v : h->host_rows)
      if (v > cap) return MOE_ERR_CAPACITY;
  }
  if (p.num_tokens == 0) return MOE_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DispatchLaunch D{};
  D.x = grad_out;
  D.recv_x = grad_y;
  D.T = p.num_tokens;
  D.cap = cap;
  D.H = p.hidden;
  D.R = p.num_logical_ranks;
  D.k = p.topk;
  D.E = p.num_experts;
  D.E_loc = p.num_experts / p.num_logical_ranks;
  D.zero_padding = do_zero_padding;
  D.grid = grid_for(num_sms, h->device);
  D.pair_rank = h->d.pair_rank;
  D.slot = h->d.slot;
  D.pair_w = h->d.pair_w;
  D.scale_w = topk_weights;
  D.psum = h->d.psum;
  D.pad_excl = h->d.pad_excl;
  D.status = h->d.status;
  if (launch_dispatch(D, false, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (grad_weights) {
    GradWeightsLaunch G{};
    G.grad_out = grad_out;
    G.y = y;
    G.grad_w = grad_weights;
    G.T = p.num_tokens;
    G.cap = cap;
    G.H = p.hidden;
    G.k = p.topk;
    G.grid = 4 * grid_for(num_sms, h->device);
    G.pair_rank = h->d.pair_rank;
    G.slot = h->d.slot;
    G.status = h->d.status;
    if (launch_grad_weights(G, s) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int moe_handle_status(const moe_handle_t* h, void* stream) {
  TraceRange trace("moe_handle_status");
  if (!h) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* stage = static_cast<int32_t*>(g_stage.get(16));
  if (!stage) return MOE_ERR_CUDA;
  if (cudaMemcpyAsync(stage, h->d.status, 16, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (stage[0] & kStatusBounds) {
    std::fprintf(stderr, "moe: index check %d failed, detail %lld\n", stage[1],
                 (long long)(((uint64_t)(uint32_t)stage[3] << 32) | (uint32_t)stage[2]));
    return MOE_ERR_CUDA;
  }
  if (stage[0] & kStatusTimeout) return MOE_ERR_TIMEOUT;
  if (stage[0] & kStatusBadExpert) return MOE_ERR_BAD_EXPERT;
  if (stage[0] & kStatusCapacity) return MOE_ERR_CAPACITY;
  return MOE_OK;
}

const int32_t* moe_handle_counts(const moe_handle_t* h) { return h ? h->d.cnt : nullptr; }
const int32_t* moe_handle_psum(const moe_handle_t* h) { return h ? h->d.psum : nullptr; }
const int32_t* moe_handle_rows_per_rank(const moe_handle_t* h) { return h ? h->d.rows_per_rank : nullptr; }
const int32_t* moe_handle_tokens_per_rank(const moe_handle_t* h) { return h ? h->d.tokens_per_rank : nullptr; }
const uint8_t* moe_handle_token_in_rank(const moe_handle_t* h) { return h ? h->d.token_in_rank : nullptr; }
const int32_t* moe_handle_slots(const moe_handle_t* h) { return h ? h->d.slot : nullptr; }
const int32_t* moe_handle_row_src(const moe_handle_t* h) { return h ? h->d.row_src : nullptr; }
const float* moe_handle_row_weights(const moe_handle_t* h) { return h ? h->d.row_w : nullptr; }
const int32_t* moe_handle_token_rows(const moe_handle_t* h) { return h ? h->d.token_row : nullptr; }
int64_t moe_handle_row_capacity(const moe_handle_t* h) { return h ? h->row_cap : -1; }

int moe_handle_free(moe_handle_t* h) {
  TraceRange trace("moe_handle_free");
  if (!h) return MOE_OK;
  int rc = MOE_OK;
  // a deferred count copy still in flight writes into the handle's pinned block: let it land
  if (h->epi_pending && cudaEventSynchronize(h->epi_event) != cudaSuccess) rc = MOE_ERR_CUDA;
  if (h->block && cudaFreeAsync(h->block, h->stream) != cudaSuccess) rc = MOE_ERR_CUDA;
  if (h->epi_event && cudaEventDestroy(h->epi_event) != cudaSuccess) rc = MOE_ERR_CUDA;
  pinned_give(h->epi_stage, h->epi_bytes);
  mapped_give(h->host_block, h->host_block_bytes);  // written only before its ready flag, which the host saw
  delete h;
  return rc;
}

int moe_expert_gemm_fp8(const moe_handle_t* h, const void* recv_x, const float* recv_scales, const void* w,
                        const float* w_scales, void* out, int64_t N, int64_t cap, int num_sms, void* stream) {
  TraceRange trace("moe_expert_gemm_fp8");
  if (!h || !recv_x || !recv_scales || !w || !w_scales || !out) return MOE_ERR_INVALID_ARG;
  if (N <= 0 || cap < 1 || num_sms < 0) return MOE_ERR_INVALID_ARG;
  const moe_params_t& p = h->p;
  const int64_t H = p.hidden, R = p.num_logical_ranks, E = p.num_experts;
  if (H % 128 != 0 || N % 128 != 0 || p.expert_alignment % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (R * cap >= (int64_t)1 << 31 || E * N >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  if (expert_gemm_smem_bytes((int)R, (int)E) > 227u * 1024u) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(recv_x) || !aligned16(w) || !aligned16(out) || !aligned4(recv_scales) || !aligned4(w_scales))
    return MOE_ERR_INVALID_ARG;
  if (h->counts_on_host)
    for (int32_t v : h->host_rows)
      if (v > cap) return MOE_ERR_CAPACITY;
  GemmLaunch L{};
  L.psum = h->d.psum;
  L.rows_per_rank = h->d.rows_per_rank;
  L.sx = recv_scales;
  L.sw = w_scales;
  L.out = out;
  L.cap = cap;
  L.N = N;
  L.R = (int)R;
  L.E = (int)E;
  L.E_loc = (int)(E / R);
  L.NB = (int)(N / 128);
  L.KB = (int)(H / 128);
  L.grid = grid_for(num_sms, h->device);
  L.status = h->d.status;
  return launch_expert_gemm(L, recv_x, w, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_event_record(void* stream, moe_event_t** out_event) {
  if (!out_event) return MOE_ERR_INVALID_ARG;
  *out_event = nullptr;
  moe_event_t* e = new (std::nothrow) moe_event_t();
  if (!e) return MOE_ERR_OOM;
  if (cudaEventCreateWithFlags(&e->ev, cudaEventDisableTiming) != cudaSuccess) {
    delete e;
    return MOE_ERR_CUDA;
  }
  if (cudaEventRecord(e->ev, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaEventDestroy(e->ev);
    delete e;
    return MOE_ERR_CUDA;
  }
  *out_event = e;
  return MOE_OK;
}

int moe_event_wait(const moe_event_t* e, void* stream) {
  if (!e) return MOE_ERR_INVALID_ARG;
  return cudaStreamWaitEvent(static_cast<cudaStream_t>(stream), e->ev, 0) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_event_synchronize(const moe_event_t* e) {
  TraceRange trace("moe_event_synchronize");
  if (!e) return MOE_ERR_INVALID_ARG;
  return cudaEventSynchronize(e->ev) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_event_query(const moe_event_t* e) {
  if (!e) return MOE_ERR_INVALID_ARG;
  const cudaError_t err = cudaEventQuery(e->ev);
  if (err == cudaSuccess) return MOE_OK;
  if (err == cudaErrorNotReady) return MOE_NOT_READY;
  return MOE_ERR_CUDA;
}

int moe_event_free(moe_event_t* e) {
  if (!e) return MOE_OK;
  const int rc = cudaEventDestroy(e->ev) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  delete e;
  return rc;
}

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_NOT_READY: return "not complete yet";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_BAD_EXPERT: return "expert id outside [-1, num_experts)";
    case MOE_ERR_CAPACITY: return "a logical rank needs more rows than the receive capacity";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_OOM: return "device memory allocation failed";
    case MOE_ERR_UNSUPPORTED: return "unsupported by this build";
    case MOE_ERR_TIMEOUT: return "a kernel gave up waiting on a shared-memory barrier (internal error)";
    case MOE_ERR_SCRATCH_LIMIT: return "problem needs more scratch than MOE_STATIC_SCRATCH_BYTES";
    default: return "unknown status";
  }
}

int64_t moe_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
