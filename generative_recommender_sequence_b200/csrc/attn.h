// Internal launch interface of the attention kernels (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "launch.h"

namespace hstu {

// Where the keys/values of a (user, head) come from and which mask applies.
struct AttnProblem {
  int B = 0, H = 0, d = 0;
  int mode = 0;                       // 0: causal suffix, 1: candidates
  bool paged = false;
  const int64_t* q_off = nullptr;     // [B+1] query rows
  const int64_t* kv_off = nullptr;    // [B+1] contiguous K/V rows (not paged)
  const int64_t* users = nullptr;     // [B] (paged)
  const int32_t* page_lists = nullptr;  // [max_users, max_ppu] (paged)
  const int64_t* lengths = nullptr;   // [max_users] cached lengths (paged)
  int64_t max_users = 0;
  int max_ppu = 0;
  int64_t n_pages = 0;                // pool pages; page n_pages is an all-zero page
  const void* pool = nullptr;         // [n_pages+1][2][H][32][d]
  // token-major tensors; strides in elements between consecutive tokens
  const void* q = nullptr;  int64_t q_stride = 0;
  const void* k = nullptr;  int64_t k_stride = 0;   // contiguous K (or candidates' K)
  const void* v = nullptr;  int64_t v_stride = 0;
  int64_t total_q = 0, total_kv = 0;  // rows of q / of k,v (for tensor maps)
  void* out = nullptr;      int64_t out_stride = 0;
  const float* pos_table = nullptr; int n_pos = 0;
  const float* time_table = nullptr; int n_time = 0;
  const int64_t* ts = nullptr;        // [total_kv] (contiguous only)
  float scale = 1.f;
  int max_q = 0;                      // bound on per-user query count
  int max_kv = 0;                     // bound on per-user key count
  bool f32 = false;                   // fp32 tensors (SIMT kernel only)
  // candidate mode: candidates sit at position (cached length + q_pos_offset)
  int q_pos_offset = 0;
  // write the unscaled fp32 partial sums of every key split to the workspace
  // and leave the reduction to the caller (no output, no split reduce)
  bool partial_only = false;
  // callers without a workspace (hstu_attn_fwd, the uncached block) never
  // split keys over CTAs
  bool allow_split = true;
  // launch with programmatic dependent launch (off for the uncached block
  // stack, where the early-scheduled attention CTAs measured slower)
  bool pdl = true;
};

// bf16, d == 128, tcgen05 path.  workspace: fp32 split partials (may be null if
// split_bytes() == 0).
size_t attn_sm100_workspace_bytes(const AttnProblem& p, int num_sms);
// The key-split plan the launch uses: n_split slices of kps key tiles each.
void attn_sm100_split_plan(const AttnProblem& p, int num_sms, int* n_split, int* kps);
cudaError_t attn_sm100_launch(const AttnProblem& p, void* workspace, size_t ws_bytes,
                              int* err_word, cudaStream_t stream);

// SIMT path: fp32 or bf16, d in {32, 64, 128}.
cudaError_t attn_simt_launch(const AttnProblem& p, cudaStream_t stream);

// TMA descriptor helpers (host).
bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                  uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows);
bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                  uint64_t mid_stride_bytes, uint64_t outer_stride_bytes, uint32_t box_inner,
                  uint32_t box_outer);

// 2-D bf16 tensor map [rows, inner] (row stride in bytes) for TMA stores of
// box_rows x box_inner boxes staged in shared memory with the 64-byte swizzle.
bool make_tmap_2d_store(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                        uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows);

int device_sm_count();

}  // namespace hstu
