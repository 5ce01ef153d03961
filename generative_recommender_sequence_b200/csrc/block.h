// Internal launch interface of the HSTU block kernels (not part of the C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "kv_table.h"

namespace hstu {

struct BlockProblem {
  void* x = nullptr;                  // [T, d_model] bf16, updated in place
  const int64_t* seq_offsets = nullptr;
  int B = 0, max_len = 0;
  int64_t T = 0;
  int n_layers = 0, d_model = 0, H = 0, dh = 0;
  const void* const* w_uvqk = nullptr;  // host array of device pointers [d_model, 4*H*dh]
  const void* const* w_o = nullptr;     // host array of device pointers [H*dh, d_model]
  const float* pos_table = nullptr; int n_pos = 0;
  const float* time_table = nullptr; int n_time = 0;
  const int64_t* ts = nullptr;
  float scale = 1.f, ln_eps = 1e-5f;
};

size_t block_workspace_bytes(int64_t T, int d_model, int H, int dh);

// Largest user count of one cached step (the KV append grid's y extent).
constexpr int kMaxCachedStepUsers = 65535;

// One KV-cached serving step over n_layers (see hstu_block_cached_step in
// include/hstu.h).  x holds the new rows (jagged by new_offsets) and then the
// candidate rows (jagged by cand_offsets, relative to the first candidate row).
struct CachedStepProblem {
  const KvTableDev* tables = nullptr;   // host array [n_layers]
  int n_layers = 0;
  const int64_t* users = nullptr;
  int B = 0;
  void* x = nullptr;                    // [T_new + T_cand, d_model] bf16, in place
  const int64_t* new_offsets = nullptr;
  int64_t T_new = 0;
  int max_new = 0;
  const int64_t* cand_offsets = nullptr;
  int64_t T_cand = 0;
  int max_cand = 0;
  int max_cached = 0;                   // bound on any user's cached length after the append
  int d_model = 0, H = 0, dh = 0;
  const void* const* w_uvqk = nullptr;
  const void* const* w_o = nullptr;
  const float* pos_table = nullptr; int n_pos = 0;
  float scale = 1.f, ln_eps = 1e-5f;
};

size_t block_cached_workspace_bytes(const CachedStepProblem& p, int num_sms);
cudaError_t block_cached_step_launch(const CachedStepProblem& p, void* workspace, size_t ws_bytes,
                                     int* err_word, cudaStream_t stream);
cudaError_t block_fwd_launch(const BlockProblem& p, void* workspace, size_t ws_bytes, int* err_word,
                             cudaStream_t stream);

}  // namespace hstu
