// Paged GPU KV data table: allocation, append and lookup ("NVIDIA Dynamo-Triton
// Gets End-to-End HSTU Generative Recommender Workflow", section "What the
// workflow combines": the GPU cache is a paged KV data table with lookup,
// allocation, append and eviction).
//
// Storage (all device memory, allocated once by hstu_kv_table_create):
//   pool        [(n_pages + 1)][2 (K,V)][H][32 slots][d]; page n_pages stays
//               zero and stands in for missing pages inside the attention
//               kernel's tile loads
//   free_stack  [n_pages] int32, free_top = number of free pages; the top of
//               the stack is free_stack[free_top - 1]
//   page_lists  [max_users][max_ppu] int32 (-1 = none), n_held [max_users]
//   lengths     [max_users] int64 cached tokens
//   epoch       [max_users] int32: last alloc call that listed the user
//               (duplicate detection without clearing)
//   alloc_calls int32 counter of alloc launches; each launch takes the next
//               epoch from it on the device, so a captured and replayed
//               launch still gets a fresh epoch
//   done        [max_users] int32: append chunk counters (always back to 0)
//   status      first device-side error since the last status read
//   step_done   CTAs of a one-launch serving step that finished (back to 0)
//   step_ok     whether the alloc half of a two-launch serving step succeeded
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <vector>

#include "kv_table.h"
#include "launch.h"
#include "sm100.cuh"

namespace hstu {

namespace {

__device__ __forceinline__ void set_status(int32_t* status, int code) {
  atomicCAS(status, 0, code);
}

constexpr int kAllocThreads = 1024;

// Inclusive prefix sum of one value per thread over a kAllocThreads block
// (warp shuffles, then the warp totals): three barriers.  *total gets the sum.
__device__ int64_t block_inclusive_scan(int64_t x, int64_t* s_warp, int64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int64_t w = s_warp[lane];  // kAllocThreads / 32 == 32 warps
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_warp[lane] = w;
  }
  __syncthreads();
  if (warp > 0) x += s_warp[warp - 1];
  *total = s_warp[31];
  __syncthreads();
  return x;
}

// One CTA.  Phase 1: per-user demand and validation.  Phase 2: block-wide
// exclusive scan of the demand in the order users are listed.  Phase 3: pop
// pages from the top of the free stack (user 0 first).
__global__ void __launch_bounds__(kAllocThreads)
    kv_alloc_kernel(KvTableDev t, const int64_t* users, const int64_t* n_new,
                    const int64_t* new_offsets, int B, int32_t* page_ids_out, int page_ids_cap,
                    int32_t* ok_out, int64_t max_count) {
  __shared__ int64_t s_warp[32];
  __shared__ int s_bad;
  __shared__ int s_epoch;
  const int tid = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  // read early: only alloc / release change it, and they are stream-ordered
  const int64_t top = *t.free_top;
  if (tid == 0) {
    s_bad = 0;
    s_epoch = atomicAdd(t.alloc_calls, 1) + 1;
  }
  __syncthreads();
  const int32_t epoch = s_epoch;
  const int per = (B + kAllocThreads - 1) / kAllocThreads;
  const int b0 = tid * per, b1 = min(B, b0 + per);
  // phase 1
  int64_t mysum = 0;
  for (int b = b0; b < b1; ++b) {
    const int64_t u = users[b];
    const int64_t n = n_new ? n_new[b] : new_offsets[b + 1] - new_offsets[b];
    if (u < 0 || u >= t.max_users || n < 0 || (max_count >= 0 && n > max_count)) {
      atomicOr(&s_bad, 1);
      continue;
    }
    if (atomicExch(&t.epoch[u], epoch) == epoch) atomicOr(&s_bad, 1);  // listed twice
    const int64_t want = (t.lengths[u] + n + t.page_size - 1) / t.page_size;
    int64_t need = want - t.n_held[u];
    need = need < 0 ? 0 : need;
    if (t.n_held[u] + need > t.max_ppu) atomicOr(&s_bad, 1);
    mysum += need;
  }
  // phase 2: inclusive scan of the per-thread sums
  int64_t total;
  const int64_t incl = block_inclusive_scan(mysum, s_warp, &total);
  if (s_bad) {
    if (tid == 0) {
      set_status(t.status, 1 /* HSTU_ERR_INVALID_ARG */);
      if (ok_out) *ok_out = 0;
    }
    return;
  }
  if (total > top) {
    if (tid == 0) {
      set_status(t.status, 2 /* HSTU_ERR_OUT_OF_PAGES */);
      if (ok_out) *ok_out = 0;
    }
    return;
  }
  // phase 3
  int64_t pre = incl - mysum;  // exclusive prefix of this thread's first user
  for (int b = b0; b < b1; ++b) {
    const int64_t u = users[b];
    const int64_t n = n_new ? n_new[b] : new_offsets[b + 1] - new_offsets[b];
    const int64_t want = (t.lengths[u] + n + t.page_size - 1) / t.page_size;
    int64_t need = want - t.n_held[u];
    need = need < 0 ? 0 : need;
    const int held = t.n_held[u];
    for (int64_t k = 0; k < need; ++k) {
      const int32_t pid = t.free_stack[top - 1 - (pre + k)];
      t.page_lists[u * (int64_t)t.max_ppu + held + k] = pid;
      if (page_ids_out && pre + k < page_ids_cap) page_ids_out[pre + k] = pid;
    }
    t.n_held[u] = held + (int)need;
    pre += need;
  }
  if (page_ids_out)
    for (int64_t i = total + tid; i < page_ids_cap; i += kAllocThreads) page_ids_out[i] = -1;
  __syncthreads();
  if (tid == 0) {
    *t.free_top = (int32_t)(top - total);
    if (ok_out) *ok_out = 1;
  }
}

// One CTA.  Releases every page of the listed users (eviction of whole users):
// pages go back on the free stack in the order users are listed, each user's
// pages from its last to its first, so its first page ends on top.  Lengths and
// page lists are cleared.  Duplicate or out-of-range users leave the table
// unchanged and set the status word.
__global__ void __launch_bounds__(kAllocThreads)
    kv_release_kernel(KvTableDev t, const int64_t* users, int B) {
  __shared__ int64_t s_warp[32];
  __shared__ int s_bad;
  __shared__ int s_epoch;
  const int tid = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  const int64_t top = *t.free_top;
  if (tid == 0) {
    s_bad = 0;
    s_epoch = atomicAdd(t.alloc_calls, 1) + 1;
  }
  __syncthreads();
  const int32_t epoch = s_epoch;
  const int per = (B + kAllocThreads - 1) / kAllocThreads;
  const int b0 = tid * per, b1 = min(B, b0 + per);
  int64_t mysum = 0;
  for (int b = b0; b < b1; ++b) {
    const int64_t u = users[b];
    if (u < 0 || u >= t.max_users) {
      atomicOr(&s_bad, 1);
      continue;
    }
    if (atomicExch(&t.epoch[u], epoch) == epoch) atomicOr(&s_bad, 1);  // listed twice
    mysum += t.n_held[u];
  }
  int64_t total;
  const int64_t incl = block_inclusive_scan(mysum, s_warp, &total);
  if (s_bad || top + total > t.n_pages) {
    if (tid == 0) set_status(t.status, 1 /* HSTU_ERR_INVALID_ARG */);
    return;
  }
  int64_t pre = incl - mysum;
  for (int b = b0; b < b1; ++b) {
    const int64_t u = users[b];
    const int held = t.n_held[u];
    int32_t* list = t.page_lists + u * (int64_t)t.max_ppu;
    for (int k = 0; k < held; ++k) {
      t.free_stack[top + pre + (held - 1 - k)] = list[k];
      list[k] = -1;
    }
    t.n_held[u] = 0;
    t.lengths[u] = 0;
    pre += held;
  }
  __syncthreads();
  if (tid == 0) *t.free_top = (int32_t)(top + total);
}

// tokens per CTA: at H * d = 512 bf16 elements a token's K and V rows are 128
// 16-byte vectors, so 256 threads copy two tokens with one vector each
constexpr int kAppendTok = 2;
constexpr int kCopyThreads = 256;
// tokens per CTA of a bulk append (a prefill or an onboarding): whole 32-token
// pages' worth of K and V per CTA instead of two tokens
constexpr int kBulkTok = 64;
constexpr int kBulkFromTokens = 256;  // bulk CTAs once some user appends this many
// tokens per CTA of the one-launch serving step (each thread's vectors are
// loaded before the plan resolves); measured: 2 tokens per CTA beat 8 on the
// serving steps (more CTAs in flight outweigh the completion-counter traffic)
constexpr int kStepTok = 2;
constexpr int kStepVec = kStepTok * 2 * 64 / kCopyThreads;  // bf16 H=4 d=128: 16-byte vectors per thread

// Copies ntok consecutive tokens (source rows src_row0.., positions p0..) of
// K and V into their pages (s_page[i] = page of position (first_page + i) *
// page_size ..).  Thread-strided over 16-byte vectors, eight loads in flight
// per thread before their stores.  H_, D_, PS_ != 0 fix the layout at compile
// time (shifts instead of divisions); 0 reads it from the table.
template <int ESZ, int H_, int D_, int PS_>
__device__ __forceinline__ void bulk_copy(const KvTableDev& t, const uint8_t* __restrict__ k_new,
                                          const uint8_t* __restrict__ v_new, int64_t src_row0,
                                          int64_t src_row_bytes, int ntok, int64_t p0,
                                          int64_t first_page, const int32_t* s_page) {
  const int H = H_ ? H_ : t.H, D = D_ ? D_ : t.d, PS = PS_ ? PS_ : t.page_size;
  const int vph = D * ESZ / 16;  // 16-byte vectors per head row
  const int row_vec = H * vph;
  const int total = ntok * row_vec * 2;
  constexpr int U = 8;
  for (int base = threadIdx.x; base < total; base += kCopyThreads * U) {
    uint4 x[U];
    int64_t dst_off[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int i = base + j * kCopyThreads;
      dst_off[j] = -1;
      if (i < total) {
        const int kv = i / (ntok * row_vec);
        const int rem = i - kv * (ntok * row_vec);
        const int tk = rem / row_vec, v = rem - tk * row_vec;
        const int h = v / vph, e16 = v - h * vph;
        const int64_t pos = p0 + tk;
        const int32_t page = s_page[(int)(pos / PS - first_page)];
        const int slot = (int)(pos % PS);
        const uint8_t* src = (kv ? v_new : k_new) + (src_row0 + tk) * src_row_bytes;
        x[j] = reinterpret_cast<const uint4*>(src)[v];
        dst_off[j] = ((((int64_t)page * 2 + kv) * H + h) * PS + slot) * D * ESZ + (int64_t)e16 * 16;
      }
    }
#pragma unroll
    for (int j = 0; j < U; ++j)
      if (dst_off[j] >= 0)
        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(t.pool) + dst_off[j]) = x[j];
  }
}

// grid (chunks, B): CTA (c, b) copies tokens [c*TOK, ...) of user b (TOK =
// kAppendTok for serving-sized appends, kBulkTok for prefills and onboarding).
// The length is read before any copy and advanced by the last CTA of the user.
// A bulk CTA first reads the (at most two) pages its tokens land in, then
// copies with every thread's loads in flight before its stores.
template <int ESZ, int TOK>
__global__ void __launch_bounds__(kCopyThreads)
    kv_append_kernel(KvTableDev t, const int64_t* __restrict__ users,
                     const uint8_t* __restrict__ k_new, const uint8_t* __restrict__ v_new,
                     const int64_t* __restrict__ new_offsets, int64_t src_row_bytes) {
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.y;
  const int64_t u = users[b];
  const int64_t s = new_offsets[b], n = new_offsets[b + 1] - s;
  const int n_chunks = (int)((n + TOK - 1) / TOK);
  if (blockIdx.x >= n_chunks) return;
  if (u < 0 || u >= t.max_users) {
    if (threadIdx.x == 0) set_status(t.status, 1);
    return;
  }
  const int64_t len = t.lengths[u];
  const bool fits = len + n <= (int64_t)t.n_held[u] * t.page_size;
  if (fits) {
    const int row_vec = t.H * t.d * ESZ / 16;     // 16-byte vectors per token row
    const int vec_per_head = t.d * ESZ / 16;
    const int64_t tok0 = (int64_t)blockIdx.x * TOK;
    const int ntok = (int)((n - tok0) < TOK ? (n - tok0) : TOK);
    const int32_t* plist = t.page_lists + u * (int64_t)t.max_ppu;
    if (TOK <= kAppendTok) {
      for (int i = threadIdx.x; i < ntok * row_vec * 2; i += kCopyThreads) {
        const int kv = i / (ntok * row_vec);
        const int rem = i % (ntok * row_vec);
        const int tk = rem / row_vec, v = rem % row_vec;
        const int h = v / vec_per_head, e16 = v % vec_per_head;
        const int64_t src_row = s + tok0 + tk;
        const int64_t pos = len + tok0 + tk;
        const int32_t page = plist[pos / t.page_size];
        const int slot = (int)(pos % t.page_size);
        const uint8_t* src = (kv ? v_new : k_new) + src_row * src_row_bytes;
        const uint4 x = reinterpret_cast<const uint4*>(src)[v];
        uint8_t* dst = reinterpret_cast<uint8_t*>(t.pool) +
                       ((((int64_t)page * 2 + kv) * t.H + h) * t.page_size + slot) * t.d * ESZ;
        reinterpret_cast<uint4*>(dst)[e16] = x;
      }
    } else {
      // the chunk's positions span pages first_page .. first_page + n_pg - 1
      __shared__ int32_t s_page[kBulkTok / 32 + 2];
      const int64_t p0 = len + tok0;
      const int64_t first_page = p0 / t.page_size;
      const int n_pg = (int)((p0 + ntok - 1) / t.page_size - first_page) + 1;
      for (int i = threadIdx.x; i < n_pg; i += kCopyThreads) s_page[i] = plist[first_page + i];
      __syncthreads();
      // the common layout (bf16, 4 heads of 128) gets compile-time strides
      if (ESZ == 2 && t.H == 4 && t.d == 128 && t.page_size == 32)
        bulk_copy<ESZ, 4, 128, 32>(t, k_new, v_new, s + tok0, src_row_bytes, ntok, p0, first_page,
                                   s_page);
      else
        bulk_copy<ESZ, 0, 0, 0>(t, k_new, v_new, s + tok0, src_row_bytes, ntok, p0, first_page,
                                s_page);
    }
  } else if (threadIdx.x == 0 && blockIdx.x == 0) {
    set_status(t.status, 1);
  }
  // the last CTA of this user commits the new length
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int prev = atomicAdd(&t.done[u], 1);
    if (prev == n_chunks - 1) {
      if (fits) t.lengths[u] = len + n;
      t.done[u] = 0;
      __threadfence();
    }
  }
}

// grid (chunks, B).  Chunk 0 also writes the length and the page table row.
template <int ESZ>
__global__ void __launch_bounds__(kCopyThreads)
    kv_lookup_kernel(KvTableDev t, const int64_t* users, int64_t* cached_len_out,
                     int32_t* page_table_out, int max_pages, uint8_t* k_out, uint8_t* v_out,
                     const int64_t* out_offsets) {
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.y;
  const int64_t u = users[b];
  const bool valid_user = u >= 0 && u < t.max_users;
  const int64_t len = valid_user ? t.lengths[u] : 0;
  if (blockIdx.x == 0) {
    if (threadIdx.x == 0) {
      if (cached_len_out) cached_len_out[b] = len;
      if (!valid_user) set_status(t.status, 1);
    }
    if (page_table_out) {
      const int held = valid_user ? t.n_held[u] : 0;
      for (int p = threadIdx.x; p < max_pages; p += kCopyThreads)
        page_table_out[(int64_t)b * max_pages + p] =
            p < held ? t.page_lists[u * (int64_t)t.max_ppu + p] : -1;
    }
  }
  if (!k_out || !valid_user) return;
  const int64_t tok0 = (int64_t)blockIdx.x * kAppendTok;
  if (tok0 >= len) return;
  const int ntok = (int)((len - tok0) < kAppendTok ? (len - tok0) : kAppendTok);
  const int row_vec = t.H * t.d * ESZ / 16;
  const int vec_per_head = t.d * ESZ / 16;
  const int64_t o = out_offsets[b];
  for (int i = threadIdx.x; i < ntok * row_vec * 2; i += kCopyThreads) {
    const int kv = i / (ntok * row_vec);
    const int rem = i % (ntok * row_vec);
    const int tk = rem / row_vec, v = rem % row_vec;
    const int h = v / vec_per_head, e16 = v % vec_per_head;
    const int64_t pos = tok0 + tk;
    const int32_t page = t.page_lists[u * (int64_t)t.max_ppu + pos / t.page_size];
    const int slot = (int)(pos % t.page_size);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(t.pool) +
                         ((((int64_t)page * 2 + kv) * t.H + h) * t.page_size + slot) * t.d * ESZ;
    uint8_t* dst = (kv ? v_out : k_out) + (o + pos) * (int64_t)t.H * t.d * ESZ;
    reinterpret_cast<uint4*>(dst)[v] = reinterpret_cast<const uint4*>(src)[e16];
  }
}

// One serving step: alloc + append + lookup rows, all or nothing.
//
// Small batches (B <= kStepMaxUsers) run as ONE launch of grid (chunks, B).
// Every CTA reads the listed users' lengths and page counts and the free-stack
// top at entry and re-derives the whole batch's allocation from them
// (validation, per-user page demand, exclusive scan in listed order, pages
// popped from the top of the stack), so all CTAs reach the same decision and
// the same page ids without waiting on each other.  CTA (c, b) copies tokens
// [2c, 2c + 2) of user b into their slots; CTA (0, b) also writes user b's new
// page-list entries and its lookup row.  None of the state read at entry is
// written until every CTA has finished: the last CTA to finish (a grid-wide
// counter) commits lengths, page counts and the stack top and resets the
// counter.  An invalid batch or a lack of pages changes nothing (the lookup
// rows then show the unchanged state) and records the status.
//
// Larger batches (PLAN = false) follow the alloc kernel, which records its
// success in step_ok: the tokens are copied and the lengths advanced (last CTA
// of each user) only when it succeeded; the lookup rows are written either way.
constexpr int kStepMaxUsers = 64;

template <int ESZ, bool PLAN>
__global__ void __launch_bounds__(kCopyThreads)
    kv_step_kernel(KvTableDev t, const int64_t* __restrict__ users,
                   const uint8_t* __restrict__ k_new, const uint8_t* __restrict__ v_new,
                   const int64_t* __restrict__ new_offsets, int B, int max_new,
                   int64_t src_row_bytes, int64_t* __restrict__ cached_len_out,
                   int32_t* __restrict__ page_table_out, int max_pages) {
  __shared__ int64_t s_u[kStepMaxUsers];
  __shared__ int64_t s_len[kStepMaxUsers];
  __shared__ int s_held[kStepMaxUsers];
  __shared__ int s_need[kStepMaxUsers];
  __shared__ int s_pre[kStepMaxUsers + 1];
  __shared__ int64_t s_top;
  __shared__ int s_bad, s_ok, s_last;
  const int tid = threadIdx.x, b = blockIdx.y;
  pdl_launch_dependents();
  pdl_wait();
  int64_t u, len, top = 0;
  int held, need = 0, pre = 0;
  const int64_t s0 = new_offsets[b];
  const int64_t n = new_offsets[b + 1] - s0;
  // this thread's first source vectors depend on nothing the plan computes:
  // load them now so their latency overlaps the plan's dependent loads
  const int row_vec = t.H * t.d * ESZ / 16;  // 16-byte vectors per token row
  const int64_t tok0 = (int64_t)blockIdx.x * kStepTok;
  // (a count above max_new makes the batch invalid: nothing is read for it,
  // and the buffers may then be null)
  const int ntok = (int)(tok0 < n && n <= max_new
                             ? ((n - tok0) < kStepTok ? (n - tok0) : kStepTok)
                             : 0);
  uint4 xpre[kStepVec];
#pragma unroll
  for (int j = 0; j < kStepVec; ++j) {
    const int i = tid + j * kCopyThreads;
    xpre[j] = make_uint4(0u, 0u, 0u, 0u);
    if (i < ntok * row_vec * 2) {
      const int kv = i / (ntok * row_vec);
      const int rem = i % (ntok * row_vec);
      const uint8_t* src = (kv ? v_new : k_new) + (s0 + tok0 + rem / row_vec) * src_row_bytes;
      xpre[j] = reinterpret_cast<const uint4*>(src)[rem % row_vec];
    }
  }
  if (PLAN) {
    if (tid == 0) {
      s_bad = 0;
      s_top = *t.free_top;
    }
    if (tid < kStepMaxUsers) s_need[tid] = 0;
    __syncthreads();
    if (tid < B) {
      const int64_t ui = users[tid];
      const int64_t ni = new_offsets[tid + 1] - new_offsets[tid];
      int64_t li = 0;
      int hi = 0, nd = 0;
      if (ui < 0 || ui >= t.max_users) {
        atomicOr(&s_bad, 1);
      } else {
        // read for every known user: a failed step still reports its state
        li = t.lengths[ui];
        hi = t.n_held[ui];
        if (ni < 0 || ni > max_new) {
          atomicOr(&s_bad, 1);
        } else {
          const int64_t want = (li + ni + t.page_size - 1) / t.page_size;
          const int64_t d = want > hi ? want - hi : 0;
          if (hi + d > t.max_ppu)
            atomicOr(&s_bad, 1);
          else
            nd = (int)d;
        }
      }
      s_u[tid] = ui;
      s_len[tid] = li;
      s_held[tid] = hi;
      s_need[tid] = nd;
    }
    __syncthreads();
    if (tid < B) {
      for (int j = 0; j < tid; ++j)
        if (s_u[j] == s_u[tid]) {  // listed twice
          atomicOr(&s_bad, 1);
          break;
        }
    }
    if (tid < 32) {
      // exclusive scan of the demand in listed order: lane l holds users l, 32 + l
      int a = s_need[tid], c = s_need[32 + tid];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, a, o);
        const int yc = __shfl_up_sync(0xffffffffu, c, o);
        if (tid >= o) {
          a += ya;
          c += yc;
        }
      }
      const int ta = __shfl_sync(0xffffffffu, a, 31);
      s_pre[tid + 1] = a;
      s_pre[tid + 33] = c + ta;
      if (tid == 0) s_pre[0] = 0;
    }
    __syncthreads();
    top = s_top;
    const bool bad = s_bad != 0;
    const bool ok = !bad && s_pre[B] <= top;
    if (!ok && blockIdx.x == 0 && b == 0 && tid == 0)
      set_status(t.status, bad ? 1 /* HSTU_ERR_INVALID_ARG */ : 2 /* HSTU_ERR_OUT_OF_PAGES */);
    if (tid == 0) s_ok = ok;
    u = s_u[b];
    len = s_len[b];
    held = s_held[b];
    need = s_need[b];
    pre = s_pre[b];
  } else {
    if (tid == 0) s_ok = *t.step_ok != 0;
    u = users[b];
    const bool known = u >= 0 && u < t.max_users;
    len = known ? t.lengths[u] : 0;
    held = known ? t.n_held[u] : 0;
  }
  __syncthreads();
  const bool ok = s_ok != 0;
  const bool known = u >= 0 && u < t.max_users;
  const int32_t* list = t.page_lists + (known ? u : 0) * (int64_t)t.max_ppu;
  if (ok && tok0 < n) {
    const int vec_per_head = t.d * ESZ / 16;
    const int total = ntok * row_vec * 2;
    // where vector i goes: pages this step pops come straight from the stack
    // (PLAN); the rest are on the user's list
    auto dst_of = [&](int i) -> uint4* {
      const int kv = i / (ntok * row_vec);
      const int rem = i % (ntok * row_vec);
      const int tk = rem / row_vec, v = rem % row_vec;
      const int h = v / vec_per_head, e16 = v % vec_per_head;
      const int64_t pos = len + tok0 + tk;
      const int64_t pi = pos / t.page_size;
      const int32_t page = (PLAN && pi >= held) ? t.free_stack[top - 1 - (pre + (pi - held))]
                                                : list[pi];
      const int slot = (int)(pos % t.page_size);
      uint8_t* dst = reinterpret_cast<uint8_t*>(t.pool) +
                     ((((int64_t)page * 2 + kv) * t.H + h) * t.page_size + slot) * t.d * ESZ;
      return reinterpret_cast<uint4*>(dst) + e16;
    };
#pragma unroll
    for (int j = 0; j < kStepVec; ++j) {
      const int i = tid + j * kCopyThreads;
      if (i < total) *dst_of(i) = xpre[j];
    }
    for (int i = tid + kStepVec * kCopyThreads; i < total; i += kCopyThreads) {
      const int kv = i / (ntok * row_vec);
      const int rem = i % (ntok * row_vec);
      const uint8_t* src = (kv ? v_new : k_new) + (s0 + tok0 + rem / row_vec) * src_row_bytes;
      *dst_of(i) = reinterpret_cast<const uint4*>(src)[rem % row_vec];
    }
  }
  if (blockIdx.x == 0) {
    const int64_t flen = !known ? 0 : (ok ? len + n : len);
    const int fheld = !known ? 0 : ((PLAN && ok) ? held + need : held);
    if (PLAN && ok) {
      int32_t* wlist = t.page_lists + u * (int64_t)t.max_ppu;
      for (int k = tid; k < need; k += kCopyThreads) wlist[held + k] = t.free_stack[top - 1 - (pre + k)];
    }
    if (tid == 0 && cached_len_out) cached_len_out[b] = flen;
    if (page_table_out) {
      for (int p = tid; p < max_pages; p += kCopyThreads) {
        int32_t pg = -1;
        if (p < fheld) pg = (PLAN && p >= held) ? t.free_stack[top - 1 - (pre + (p - held))] : list[p];
        page_table_out[(int64_t)b * max_pages + p] = pg;
      }
    }
  }
  if (!ok) return;  // the same decision in every CTA (every thread of it)
  __syncthreads();
  if (PLAN) {
    if (tid == 0) {
      __threadfence();
      const int prev = atomicAdd(t.step_done, 1);
      s_last = prev == (int)(gridDim.x * gridDim.y) - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tid < B) {
      const int64_t ui = s_u[tid];
      t.lengths[ui] = s_len[tid] + (new_offsets[tid + 1] - new_offsets[tid]);
      t.n_held[ui] = s_held[tid] + s_need[tid];
    }
    if (tid == 0) {
      *t.free_top = (int32_t)(top - s_pre[B]);
      *t.step_done = 0;
    }
    __threadfence();
  } else {
    // the last CTA of this user commits the new length
    const int n_chunks = (int)((n + kStepTok - 1) / kStepTok);
    if (tid == 0 && tok0 < n) {
      __threadfence();
      const int prev = atomicAdd(&t.done[u], 1);
      if (prev == n_chunks - 1) {
        t.lengths[u] = len + n;
        t.done[u] = 0;
        __threadfence();
      }
    }
  }
}

}  // namespace

cudaError_t kv_table_alloc_storage(KvTableDev* t, const int32_t* host_free_order) {
  const size_t page_bytes = (size_t)2 * t->H * t->page_size * t->d * t->esize;
  cudaError_t e;
  e = cudaMalloc(&t->pool, page_bytes * (size_t)(t->n_pages + 1));
  if (e != cudaSuccess) return e;
  e = cudaMemset(t->pool, 0, page_bytes * (size_t)(t->n_pages + 1));
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&t->free_stack, sizeof(int32_t) * (size_t)std::max<int64_t>(t->n_pages, 1));
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&t->free_top, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&t->page_lists, sizeof(int32_t) * (size_t)t->max_users * t->max_ppu);
  if (e != cudaSuccess) return e;
  e = cudaMemset(t->page_lists, 0xff, sizeof(int32_t) * (size_t)t->max_users * t->max_ppu);
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&t->n_held, sizeof(int32_t) * (size_t)t->max_users);
  if (e != cudaSuccess) return e;
  e = cudaMemset(t->n_held, 0, sizeof(int32_t) * (size_t)t->max_users);
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&t->lengths, sizeof(int64_t) * (size_t)t->max_users);
  if (e != cudaSuccess) return e;
  e = cudaMemset(t->lengths, 0, sizeof(int64_t) * (size_t)t->max_users);
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&t->epoch, sizeof(int32_t) * (size_t)t->max_users);
  if (e != cudaSuccess) return e;
  e = cudaMemset(t->epoch, 0, sizeof(int32_t) * (size_t)t->max_users);
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&t->alloc_calls, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  e = cudaMemset(t->alloc_calls, 0, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&t->done, sizeof(int32_t) * (size_t)t->max_users);
  if (e != cudaSuccess) return e;
  e = cudaMemset(t->done, 0, sizeof(int32_t) * (size_t)t->max_users);
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&t->status, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  e = cudaMemset(t->status, 0, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&t->step_done, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  e = cudaMemset(t->step_done, 0, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  e = cudaMalloc(&t->step_ok, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  e = cudaMemset(t->step_ok, 0, sizeof(int32_t));
  if (e != cudaSuccess) return e;
  std::vector<int32_t> order((size_t)t->n_pages);
  for (int64_t i = 0; i < t->n_pages; ++i) order[i] = host_free_order ? host_free_order[i] : (int32_t)i;
  if (t->n_pages > 0) {
    e = cudaMemcpy(t->free_stack, order.data(), sizeof(int32_t) * order.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return e;
  }
  const int32_t top = (int32_t)t->n_pages;
  e = cudaMemcpy(t->free_top, &top, sizeof(int32_t), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return e;
  return cudaDeviceSynchronize();
}

void kv_table_free_storage(KvTableDev* t) {
  cudaFree(t->pool);
  cudaFree(t->free_stack);
  cudaFree(t->free_top);
  cudaFree(t->page_lists);
  cudaFree(t->n_held);
  cudaFree(t->lengths);
  cudaFree(t->epoch);
  cudaFree(t->alloc_calls);
  cudaFree(t->done);
  cudaFree(t->status);
  cudaFree(t->step_done);
  cudaFree(t->step_ok);
}

cudaError_t kv_alloc_launch(const KvTableDev& t, const int64_t* users, const int64_t* n_new, int B,
                            int32_t* page_ids_out, int page_ids_cap, cudaStream_t stream,
                            const int64_t* new_offsets) {
  if (B == 0 && page_ids_out == nullptr) return cudaSuccess;
  if (n_new == nullptr && new_offsets == nullptr) return cudaErrorInvalidValue;
  return launch_dependent(kv_alloc_kernel, dim3(1), dim3(kAllocThreads), 0, stream, t, users, n_new,
                          new_offsets, B, page_ids_out, page_ids_cap, (int32_t*)nullptr,
                          (int64_t)-1);
}

cudaError_t kv_release_launch(const KvTableDev& t, const int64_t* users, int B,
                              cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  return launch_dependent(kv_release_kernel, dim3(1), dim3(kAllocThreads), 0, stream, t, users, B);
}

cudaError_t kv_append_launch(const KvTableDev& t, const int64_t* users, const void* k_new,
                             const void* v_new, const int64_t* new_offsets, int B, int max_new,
                             cudaStream_t stream, int64_t src_row_elems) {
  if (B == 0 || max_new <= 0) return cudaSuccess;
  const int64_t row_elems = src_row_elems > 0 ? src_row_elems : (int64_t)t.H * t.d;
  // 16-byte vector copies: every source row must start on a 16-byte boundary
  if (row_elems < (int64_t)t.H * t.d || (row_elems * t.esize) % 16 != 0)
    return cudaErrorInvalidValue;
  const uint8_t* k = (const uint8_t*)k_new;
  const uint8_t* v = (const uint8_t*)v_new;
  if (max_new >= kBulkFromTokens) {
    const dim3 grid((max_new + kBulkTok - 1) / kBulkTok, B);
    if (t.esize == 2)
      return launch_dependent(kv_append_kernel<2, kBulkTok>, grid, dim3(kCopyThreads), 0, stream, t,
                              users, k, v, new_offsets, row_elems * 2);
    return launch_dependent(kv_append_kernel<4, kBulkTok>, grid, dim3(kCopyThreads), 0, stream, t,
                            users, k, v, new_offsets, row_elems * 4);
  }
  const dim3 grid((max_new + kAppendTok - 1) / kAppendTok, B);
  if (t.esize == 2)
    return launch_dependent(kv_append_kernel<2, kAppendTok>, grid, dim3(kCopyThreads), 0, stream, t,
                            users, k, v, new_offsets, row_elems * 2);
  return launch_dependent(kv_append_kernel<4, kAppendTok>, grid, dim3(kCopyThreads), 0, stream, t,
                          users, k, v, new_offsets, row_elems * 4);
}

cudaError_t kv_lookup_launch(const KvTableDev& t, const int64_t* users, int B,
                             int64_t* cached_len_out, int32_t* page_table_out, int max_pages,
                             void* k_out, void* v_out, const int64_t* out_offsets, int max_len,
                             cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  const int chunks = k_out ? std::max(1, (max_len + kAppendTok - 1) / kAppendTok) : 1;
  dim3 grid(chunks, B);
  if (t.esize == 2)
    return launch_dependent(kv_lookup_kernel<2>, grid, dim3(kCopyThreads), 0, stream, t, users,
                            cached_len_out, page_table_out, max_pages, (uint8_t*)k_out,
                            (uint8_t*)v_out, out_offsets);
  return launch_dependent(kv_lookup_kernel<4>, grid, dim3(kCopyThreads), 0, stream, t, users,
                          cached_len_out, page_table_out, max_pages, (uint8_t*)k_out,
                          (uint8_t*)v_out, out_offsets);
}

cudaError_t kv_step_launch(const KvTableDev& t, const int64_t* users, const void* k_new,
                           const void* v_new, const int64_t* new_offsets, int B, int max_new,
                           int64_t* cached_len_out, int32_t* page_table_out, int max_pages,
                           cudaStream_t stream, int64_t src_row_elems) {
  if (B == 0) return cudaSuccess;
  if (B < 0 || B > 65535 || max_new < 0 || max_pages < 0) return cudaErrorInvalidValue;
  const int64_t row_elems = src_row_elems > 0 ? src_row_elems : (int64_t)t.H * t.d;
  if (row_elems < (int64_t)t.H * t.d || (row_elems * t.esize) % 16 != 0)
    return cudaErrorInvalidValue;
  if (page_table_out == nullptr) max_pages = 0;
  const dim3 grid(std::max(1, (max_new + kStepTok - 1) / kStepTok), B);
  const int64_t rb = row_elems * t.esize;
  const uint8_t* k = (const uint8_t*)k_new;
  const uint8_t* v = (const uint8_t*)v_new;
  if (B <= kStepMaxUsers) {
    if (t.esize == 2)
      return launch_dependent(kv_step_kernel<2, true>, grid, dim3(kCopyThreads), 0, stream, t, users,
                              k, v, new_offsets, B, max_new, rb, cached_len_out, page_table_out,
                              max_pages);
    return launch_dependent(kv_step_kernel<4, true>, grid, dim3(kCopyThreads), 0, stream, t, users, k,
                            v, new_offsets, B, max_new, rb, cached_len_out, page_table_out,
                            max_pages);
  }
  cudaError_t e = launch_dependent(kv_alloc_kernel, dim3(1), dim3(kAllocThreads), 0, stream, t, users,
                                   (const int64_t*)nullptr, new_offsets, B, (int32_t*)nullptr, 0,
                                   t.step_ok, (int64_t)max_new);
  if (e != cudaSuccess) return e;
  if (t.esize == 2)
    return launch_dependent(kv_step_kernel<2, false>, grid, dim3(kCopyThreads), 0, stream, t, users, k,
                            v, new_offsets, B, max_new, rb, cached_len_out, page_table_out,
                            max_pages);
  return launch_dependent(kv_step_kernel<4, false>, grid, dim3(kCopyThreads), 0, stream, t, users, k, v,
                          new_offsets, B, max_new, rb, cached_len_out, page_table_out, max_pages);
}

}  // namespace hstu
