// Sparse user-id -> dense slot map ("How Generative Recommenders Are Redefining
// RecSys at Scale", section "Dynamic embedding": sparse ids are hashed to rows
// of dense storage).  The slots name users of the paged KV table.
//
// Open addressing with linear probing over a power-of-two bucket array; keys
// are the ids (>= 0), -1 marks an empty bucket and -2 an erased one (reused by
// later inserts).  Bucket of an id: the splitmix64 finalizer (Steele, Lea and
// Flood, "Fast splittable pseudorandom number generators", 2014) of the id,
// masked.
//
// lookup: all threads of one CTA find the listed ids in parallel; with insert,
// thread 0 then serves the unknown ids in the order listed (a repeated id
// finds the bucket its first occurrence just filled), popping slots from the
// free stack, so the assignment is deterministic.  If the stack runs out, the
// ids inserted by this call are erased again, the stack is left as it was and
// the status word records the shortage.
// erase: thread 0 erases the listed ids in order and pushes their slots.
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "user_map.h"

namespace hstu {

namespace {

constexpr int64_t kEmpty = -1, kErased = -2;
constexpr int kMapThreads = 1024;
constexpr int kMaxIds = 65536;

__device__ __forceinline__ uint64_t mix64(uint64_t x) {
  x ^= x >> 30;
  x *= 0xbf58476d1ce4e5b9ull;
  x ^= x >> 27;
  x *= 0x94d049bb133111ebull;
  x ^= x >> 31;
  return x;
}

// Bucket holding `id`, or -1.
__device__ int find_bucket(const UserMapDev& m, int64_t id) {
  const uint32_t mask = (uint32_t)m.n_buckets - 1;
  uint32_t b = (uint32_t)mix64((uint64_t)id) & mask;
  for (int i = 0; i < m.n_buckets; ++i, b = (b + 1) & mask) {
    const int64_t k = m.keys[b];
    if (k == id) return (int)b;
    if (k == kEmpty) return -1;
  }
  return -1;
}

__global__ void __launch_bounds__(kMapThreads)
    user_map_lookup_kernel(UserMapDev m, const int64_t* ids, int B, int insert, int64_t* out) {
  __shared__ uint32_t s_miss[kMaxIds / 32];
  __shared__ int s_bad, s_any_miss;
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_bad = 0;
    s_any_miss = 0;
  }
  for (int w = tid; w < (B + 31) / 32; w += kMapThreads) s_miss[w] = 0u;
  __syncthreads();
  for (int i = tid; i < B; i += kMapThreads) {
    const int64_t id = ids[i];
    if (id < 0) {
      atomicOr(&s_bad, 1);
      continue;
    }
    const int b = find_bucket(m, id);
    out[i] = b >= 0 ? (int64_t)m.vals[b] : -1;
    if (b < 0) {
      atomicOr(&s_miss[i >> 5], 1u << (i & 31));
      s_any_miss = 1;
    }
  }
  __syncthreads();
  if (s_bad) {
    for (int i = tid; i < B; i += kMapThreads) out[i] = -1;
    if (tid == 0) atomicCAS(m.status, 0, 1 /* HSTU_ERR_INVALID_ARG */);
    return;
  }
  if (!insert || !s_any_miss || tid != 0) return;
  // thread 0: unknown ids in the order listed
  const int top = *m.free_top;
  int popped = 0;
  int failed_at = -1;
  const uint32_t mask = (uint32_t)m.n_buckets - 1;
  for (int i = 0; i < B; ++i) {
    if (!(s_miss[i >> 5] & (1u << (i & 31)))) continue;
    const int64_t id = ids[i];
    int first_erased = -1, empty = -1, found = -1;
    uint32_t b = (uint32_t)mix64((uint64_t)id) & mask;
    for (int p = 0; p < m.n_buckets; ++p, b = (b + 1) & mask) {
      const int64_t k = m.keys[b];
      if (k == id) {
        found = (int)b;
        break;
      }
      if (k == kErased && first_erased < 0) first_erased = (int)b;
      if (k == kEmpty) {
        empty = (int)b;
        break;
      }
    }
    if (found >= 0) {
      out[i] = m.vals[found];
      continue;
    }
    const int dest = first_erased >= 0 ? first_erased : empty;
    if (popped == top || dest < 0) {
      failed_at = i;
      break;
    }
    const int32_t slot = m.free_stack[top - 1 - popped];
    ++popped;
    m.keys[dest] = id;
    m.vals[dest] = slot;
    out[i] = slot;
  }
  if (failed_at < 0) {
    *m.free_top = top - popped;
    return;
  }
  // roll back: erase what this call inserted (the stack top was never moved)
  for (int i = 0; i < failed_at; ++i) {
    if (!(s_miss[i >> 5] & (1u << (i & 31)))) continue;
    const int b = find_bucket(m, ids[i]);
    if (b >= 0) m.keys[b] = kErased;
  }
  for (int i = 0; i < B; ++i) out[i] = -1;
  atomicCAS(m.status, 0, 2 /* HSTU_ERR_OUT_OF_PAGES: no free slot */);
}

__global__ void user_map_erase_kernel(UserMapDev m, const int64_t* ids, int B) {
  if (threadIdx.x != 0) return;
  int top = *m.free_top;
  for (int i = 0; i < B; ++i) {
    const int64_t id = ids[i];
    if (id < 0) continue;
    const int b = find_bucket(m, id);
    if (b < 0) continue;
    m.keys[b] = kErased;
    if (top < m.n_slots) m.free_stack[top++] = m.vals[b];
  }
  *m.free_top = top;
}

}  // namespace

cudaError_t user_map_alloc(UserMapDev* m, int32_t n_slots, const int32_t* host_free_order) {
  int32_t nb = 1;
  while (nb < 2 * n_slots) nb <<= 1;
  m->n_slots = n_slots;
  m->n_buckets = nb;
  cudaError_t e = cudaMalloc(&m->keys, sizeof(int64_t) * (size_t)nb);
  if (e != cudaSuccess) return e;
  e = cudaMemset(m->keys, 0xff, sizeof(int64_t) * (size_t)nb);  // -1 = empty
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&m->vals, sizeof(int32_t) * (size_t)nb);
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&m->free_stack, sizeof(int32_t) * (size_t)n_slots);
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&m->free_top, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&m->status, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  e = cudaMemset(m->status, 0, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  std::vector<int32_t> order((size_t)n_slots);
  for (int32_t i = 0; i < n_slots; ++i) order[i] = host_free_order ? host_free_order[i] : i;
  e = cudaMemcpy(m->free_stack, order.data(), sizeof(int32_t) * order.size(), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return e;
  e = cudaMemcpy(m->free_top, &n_slots, sizeof(int32_t), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return e;
  return cudaDeviceSynchronize();
}

void user_map_free(UserMapDev* m) {
  cudaFree(m->keys);
  cudaFree(m->vals);
  cudaFree(m->free_stack);
  cudaFree(m->free_top);
  cudaFree(m->status);
}

cudaError_t user_map_lookup_launch(const UserMapDev& m, const int64_t* ids, int B, bool insert,
                                   int64_t* slots_out, cudaStream_t stream) {
  if (B <= 0) return cudaSuccess;
  if (B > kMaxIds) return cudaErrorInvalidValue;
  user_map_lookup_kernel<<<1, kMapThreads, 0, stream>>>(m, ids, B, insert ? 1 : 0, slots_out);
  return cudaGetLastError();
}

cudaError_t user_map_erase_launch(const UserMapDev& m, const int64_t* ids, int B,
                                  cudaStream_t stream) {
  if (B <= 0) return cudaSuccess;
  user_map_erase_kernel<<<1, 32, 0, stream>>>(m, ids, B);
  return cudaGetLastError();
}

}  // namespace hstu
