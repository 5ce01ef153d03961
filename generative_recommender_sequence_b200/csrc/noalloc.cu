// Allocation-free variant of hstu_attn_cached_fwd.
//
// Some callers cannot allocate device memory at the point where they score
// candidates: code running under a memory pool they do not own, a serving
// process whose allocator is frozen after warm-up, or a host runtime that
// forbids cudaMalloc on its request path.  For them the key-split partial sums
// of the candidate path live in one fixed device array that this library
// reserves when it is loaded.
//
// Behaviour:
//  - scratch is a file-scope __device__ array of kNoAllocScratchBytes (32 MiB);
//    every GPU that loads the library keeps it until the process exits;
//  - host code never uses the array's name as an address: the first call on
//    each device (with that device current) asks cudaGetSymbolAddress for it
//    and caches the result, so that first call should happen before any
//    stream capture begins.  The cache assumes the device's primary context
//    lives as long as the process (no cudaDeviceReset in between, which would
//    also invalidate every KV table);
//  - a call whose partial sums would not fit returns HSTU_ERR_UNSUPPORTED;
//  - every call shares the array and it keeps the last call's contents.  No
//    part of it has to start at zero (each partial is written before it is
//    read), but calls that overlap on the GPU race on it, so callers must not
//    run two of these calls concurrently on different streams;
//  - no cudaMalloc, cudaFree or allocating library routine is called.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/hstu.h"
#include "attn.h"

// The argument checks of hstu_attn_cached_fwd (abi.cu): this entry point runs
// them before sizing its scratch, so both report the same status for the same
// arguments.
hstu_status cached_fwd_validate(hstu_kv_table* t, const int64_t* users, int32_t B, const void* q,
                                const void* k_cand, const void* v_cand, const int64_t* q_offsets,
                                int64_t total_q, int32_t max_q, int32_t max_cached,
                                int32_t mask_mode, const hstu_rab* rab, const void* out,
                                bool* nothing_to_do);

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_addr_mutex;
void* g_addr[64] = {};

// Device address of the scratch array on the current device (nullptr on error).
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_addr_mutex);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_addr[dev] = p;
  }
  return g_addr[dev];
}

}  // namespace

extern "C" {

size_t hstu_attn_cached_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

hstu_status hstu_attn_cached_fwd_noalloc(hstu_kv_table* t, const int64_t* users, int32_t B,
                                         const void* q, const void* k_cand, const void* v_cand,
                                         const int64_t* q_offsets, int64_t total_q, int32_t max_q,
                                         int32_t max_cached, int32_t mask_mode,
                                         const hstu_rab* rab, float scale, void* out,
                                         cudaStream_t stream) {
  bool nothing = false;
  const hstu_status st = cached_fwd_validate(t, users, B, q, k_cand, v_cand, q_offsets, total_q,
                                             max_q, max_cached, mask_mode, rab, out, &nothing);
  if (st != HSTU_OK || nothing) return st;
  const size_t need =
      hstu_attn_cached_workspace_size(t, B, total_q, max_q, max_cached, mask_mode);
  if (need > kNoAllocScratchBytes) return HSTU_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (need > 0) {
    ws = scratch_address();
    if (ws == nullptr) return HSTU_ERR_CUDA;
  }
  return hstu_attn_cached_fwd(t, users, B, q, k_cand, v_cand, q_offsets, total_q, max_q,
                              max_cached, mask_mode, rab, scale, out, ws,
                              need > 0 ? kNoAllocScratchBytes : 0, stream);
}

}  // extern "C"
