// Internal interface of the paged KV table kernels (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace hstu {

// Plain-old-data view of the table's device storage, passed to kernels by value.
struct KvTableDev {
  int64_t n_pages;
  int page_size, H, d, esize;
  int64_t max_users;
  int max_ppu;
  void* pool;
  int32_t* free_stack;
  int32_t* free_top;
  int32_t* page_lists;
  int32_t* n_held;
  int64_t* lengths;
  int32_t* epoch;
  int32_t* alloc_calls;  // device counter of alloc launches (the next call's epoch - 1)
  int32_t* done;
  int32_t* status;
  int32_t* step_done;  // CTAs of a fused step launch that finished (always back to 0)
  int32_t* step_ok;    // the last alloc of a two-launch step succeeded (1) or not (0)
};

cudaError_t kv_table_alloc_storage(KvTableDev* t, const int32_t* host_free_order);
void kv_table_free_storage(KvTableDev* t);
// n_new[b] tokens per user, or (n_new == nullptr) new_offsets[b + 1] - new_offsets[b].
cudaError_t kv_alloc_launch(const KvTableDev& t, const int64_t* users, const int64_t* n_new, int B,
                            int32_t* page_ids_out, int page_ids_cap, cudaStream_t stream,
                            const int64_t* new_offsets = nullptr);
// Evicts whole users: their pages return to the free stack (see kv_table.cu).
cudaError_t kv_release_launch(const KvTableDev& t, const int64_t* users, int B,
                              cudaStream_t stream);
// k_new / v_new rows are src_row_elems elements apart (0: H * d, packed rows).
cudaError_t kv_append_launch(const KvTableDev& t, const int64_t* users, const void* k_new,
                             const void* v_new, const int64_t* new_offsets, int B, int max_new,
                             cudaStream_t stream, int64_t src_row_elems = 0);
// One serving step: alloc (counts from new_offsets), append and lookup rows
// (cached_len_out / page_table_out optional) as one all-or-nothing operation.
cudaError_t kv_step_launch(const KvTableDev& t, const int64_t* users, const void* k_new,
                           const void* v_new, const int64_t* new_offsets, int B, int max_new,
                           int64_t* cached_len_out, int32_t* page_table_out, int max_pages,
                           cudaStream_t stream, int64_t src_row_elems = 0);
cudaError_t kv_lookup_launch(const KvTableDev& t, const int64_t* users, int B,
                             int64_t* cached_len_out, int32_t* page_table_out, int max_pages,
                             void* k_out, void* v_out, const int64_t* out_offsets, int max_len,
                             cudaStream_t stream);

}  // namespace hstu
