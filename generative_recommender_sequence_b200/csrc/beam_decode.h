// Internal interface of beam-search decode attention (not part of the C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "kv_table.h"

namespace hstu {

struct BeamDecodeProblem {
  KvTableDev table;                  // context K/V, one table user per request
  const int64_t* users = nullptr;    // [B]
  int B = 0;
  const void* q = nullptr;           // [T_beam, H, d] bf16, this step's beam queries
  const int64_t* beam_offsets = nullptr;  // [B+1] beams of each request (same every step)
  int64_t total_beams = 0;
  int max_beams = 0;
  int max_ctx = 0;                   // bound on any request's context length
  int step = 0;                      // decode step s >= 0
  const void* beam_k = nullptr;      // [s+1][T_beam][H][d] bf16 decode-token K of steps 0..s
  const void* beam_v = nullptr;
  const int32_t* beam_parent = nullptr;  // [s+1][T_beam]: parent beam (within the request) at step t-1
  const float* pos_table = nullptr; int n_pos = 0;
  float scale = 1.f;
  void* out = nullptr;               // [T_beam, H, d] bf16
};

size_t beam_decode_workspace_bytes(const BeamDecodeProblem& p, int num_sms);
cudaError_t beam_decode_launch(const BeamDecodeProblem& p, void* workspace, size_t ws_bytes,
                               int* err_word, cudaStream_t stream);

}  // namespace hstu
