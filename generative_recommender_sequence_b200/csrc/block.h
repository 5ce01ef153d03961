// Internal launch interface of the HSTU block kernels (not part of the C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

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
cudaError_t block_fwd_launch(const BlockProblem& p, void* workspace, size_t ws_bytes, int* err_word,
                             cudaStream_t stream);

}  // namespace hstu
