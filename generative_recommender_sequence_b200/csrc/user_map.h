// Internal interface of the sparse user-id -> dense slot map (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace hstu {

struct UserMapDev {
  int64_t* keys = nullptr;       // [n_buckets]: -1 empty, -2 erased, else a user id (>= 0)
  int32_t* vals = nullptr;       // [n_buckets] slot of the key
  int32_t* free_stack = nullptr; // [n_slots], top = free_top - 1
  int32_t* free_top = nullptr;
  int32_t* status = nullptr;     // first device-side error since the last read
  int32_t n_slots = 0;
  int32_t n_buckets = 0;         // power of two, >= 2 n_slots
};

cudaError_t user_map_alloc(UserMapDev* m, int32_t n_slots, const int32_t* host_free_order);
void user_map_free(UserMapDev* m);
cudaError_t user_map_lookup_launch(const UserMapDev& m, const int64_t* ids, int B, bool insert,
                                   int64_t* slots_out, cudaStream_t stream);
cudaError_t user_map_erase_launch(const UserMapDev& m, const int64_t* ids, int B,
                                  cudaStream_t stream);

}  // namespace hstu
