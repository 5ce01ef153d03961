// C ABI of the HSTU hot path (declared in include/hstu.h): argument checks on
// the host, then dispatch to the CUDA kernels.  No exception crosses the ABI;
// every entry point returns an hstu_status.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/hstu.h"
#include "attn.h"
#include "beam_decode.h"
#include "block.h"
#include "kv_table.h"
#include "selftest.h"
#include "user_map.h"

// Device error word written by kernels whose bounded waits ran out.
__device__ int g_hstu_device_error;

struct hstu_kv_table {
  hstu::KvTableDev dev;
  int device;
  hstu_dtype dtype;
};

namespace hstu {

int device_sm_count() {
  static int cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int* device_error_word() {
  static int* cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_hstu_device_error) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < 64) cached[dev] = reinterpret_cast<int*>(p);
  return reinterpret_cast<int*>(p);
}

hstu_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return HSTU_OK;
  if (e == cudaErrorInvalidValue) return HSTU_ERR_INVALID_ARG;
  return HSTU_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool rab_ok(const hstu_rab* rab, bool allow_time) {
  if (!rab) return true;
  if (rab->pos_table && (rab->n_pos_buckets < 1 || rab->n_pos_buckets > 256)) return false;
  if (rab->time_table) {
    if (!allow_time) return false;
    if (rab->n_time_buckets < 1 || rab->n_time_buckets > 256 || !rab->timestamps) return false;
  }
  return true;
}

void fill_rab(AttnProblem& p, const hstu_rab* rab) {
  if (!rab) return;
  p.pos_table = rab->pos_table;
  p.n_pos = rab->pos_table ? rab->n_pos_buckets : 0;
  p.time_table = rab->time_table;
  p.n_time = rab->time_table ? rab->n_time_buckets : 0;
  p.ts = rab->time_table ? rab->timestamps : nullptr;
}

}  // namespace

bool make_tmap_2d_store(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                        uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                  uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                  uint64_t mid_stride_bytes, uint64_t outer_stride_bytes, uint32_t box_inner,
                  uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {mid_stride_bytes, outer_stride_bytes};
  cuuint32_t box[3] = {box_inner, 1, box_outer};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Attention dispatch shared by hstu_attn_fwd and the block: bf16 d=128 runs on
// the tcgen05 kernel, everything else on the SIMT kernel.
hstu_status attn_dispatch(const AttnProblem& p, void* workspace, size_t ws_bytes,
                          cudaStream_t stream) {
  if (!p.f32 && p.d == 128) {
    return from_cuda(attn_sm100_launch(p, workspace, ws_bytes, device_error_word(), stream));
  }
  return from_cuda(attn_simt_launch(p, stream));
}

}  // namespace hstu

using namespace hstu;

extern "C" {

int32_t hstu_version(void) { return 100; }

const char* hstu_status_string(hstu_status s) {
  switch (s) {
    case HSTU_OK: return "ok";
    case HSTU_ERR_INVALID_ARG: return "invalid argument";
    case HSTU_ERR_OUT_OF_PAGES: return "out of KV pages";
    case HSTU_ERR_CUDA: return "CUDA error";
    case HSTU_ERR_UNSUPPORTED: return "unsupported configuration";
    case HSTU_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown";
}

hstu_status hstu_device_check(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HSTU_ERR_CUDA;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return HSTU_ERR_UNSUPPORTED;
  if (!encode_fn()) return HSTU_ERR_CUDA;
  return HSTU_OK;
}

hstu_status hstu_last_device_error(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return HSTU_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_hstu_device_error, sizeof(int)) != cudaSuccess) return HSTU_ERR_CUDA;
  if (v != 0) {
    const int z = 0;
    cudaMemcpyToSymbol(g_hstu_device_error, &z, sizeof(int));
  }
  return (hstu_status)v;
}

hstu_status hstu_wait_timeout_selftest(int32_t timeout_us, cudaStream_t stream) {
  if (timeout_us < 1 || timeout_us > 2000000) return HSTU_ERR_INVALID_ARG;
  return from_cuda(wait_timeout_selftest_launch(device_error_word(), (int64_t)timeout_us * 1000, stream));
}

hstu_status hstu_attn_fwd(const void* q, const void* k, const void* v, const int64_t* seq_offsets,
                          int32_t B, int32_t max_len, int64_t total_tokens, int32_t H, int32_t d_qk,
                          int32_t d_v,
                          hstu_dtype dt, const hstu_rab* rab, float scale, void* out,
                          cudaStream_t stream) {
  if (B < 0 || max_len < 0 || total_tokens < 0 || H <= 0 || d_qk <= 0) return HSTU_ERR_INVALID_ARG;
  if (total_tokens >= (1LL << 31)) return HSTU_ERR_UNSUPPORTED;
  if (B > 0 && (!q || !k || !v || !seq_offsets || !out)) return HSTU_ERR_INVALID_ARG;
  if (d_qk != d_v) return HSTU_ERR_UNSUPPORTED;
  if (d_qk != 32 && d_qk != 64 && d_qk != 128) return HSTU_ERR_UNSUPPORTED;
  if (dt != HSTU_F32 && dt != HSTU_BF16) return HSTU_ERR_INVALID_ARG;
  if (!rab_ok(rab, true)) return HSTU_ERR_INVALID_ARG;
  if (dt == HSTU_BF16 && d_qk == 128) {
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
      return HSTU_ERR_INVALID_ARG;
  }
  if (B == 0 || max_len == 0 || total_tokens == 0) return HSTU_OK;
  AttnProblem p;
  p.B = B;
  p.H = H;
  p.d = d_qk;
  p.mode = 0;
  p.q_off = seq_offsets;
  p.kv_off = seq_offsets;
  p.q = q;
  p.k = k;
  p.v = v;
  p.q_stride = p.k_stride = p.v_stride = p.out_stride = (int64_t)H * d_qk;
  // tile loads past row T read zeros (the tensor maps end at T)
  p.total_q = p.total_kv = total_tokens;
  p.out = out;
  fill_rab(p, rab);
  p.scale = scale;
  p.max_q = p.max_kv = max_len;
  p.f32 = dt == HSTU_F32;
  p.allow_split = false;  // no workspace: every item streams all of its keys
  return attn_dispatch(p, nullptr, 0, stream);
}

hstu_status hstu_kv_table_create(int64_t n_pages, int32_t page_size, int32_t H, int32_t d,
                                 hstu_dtype dtype, int64_t max_users, int32_t max_pages_per_user,
                                 const int32_t* host_free_order, hstu_kv_table** out_table) {
  if (!out_table) return HSTU_ERR_INVALID_ARG;
  *out_table = nullptr;
  if (n_pages < 0 || n_pages >= (1LL << 31) - 1 || page_size != 32 || H <= 0 || max_users <= 0 ||
      max_pages_per_user <= 0)
    return HSTU_ERR_INVALID_ARG;
  if (d != 32 && d != 64 && d != 128) return HSTU_ERR_UNSUPPORTED;
  if (dtype != HSTU_F32 && dtype != HSTU_BF16) return HSTU_ERR_INVALID_ARG;
  if (host_free_order) {  // must be a permutation
    char* seen = new (std::nothrow) char[(size_t)n_pages]();
    if (!seen) return HSTU_ERR_INVALID_ARG;
    bool ok = true;
    for (int64_t i = 0; i < n_pages && ok; ++i) {
      const int64_t x = host_free_order[i];
      if (x < 0 || x >= n_pages || seen[x]) ok = false;
      else seen[x] = 1;
    }
    delete[] seen;
    if (!ok) return HSTU_ERR_INVALID_ARG;
  }
  hstu_kv_table* t = new (std::nothrow) hstu_kv_table();
  if (!t) return HSTU_ERR_CUDA;
  cudaGetDevice(&t->device);
  t->dtype = dtype;
  std::memset(&t->dev, 0, sizeof(t->dev));
  t->dev.n_pages = n_pages;
  t->dev.page_size = page_size;
  t->dev.H = H;
  t->dev.d = d;
  t->dev.esize = dtype == HSTU_BF16 ? 2 : 4;
  t->dev.max_users = max_users;
  t->dev.max_ppu = max_pages_per_user;
  if (kv_table_alloc_storage(&t->dev, host_free_order) != cudaSuccess) {
    kv_table_free_storage(&t->dev);
    delete t;
    return HSTU_ERR_CUDA;
  }
  *out_table = t;
  return HSTU_OK;
}

void hstu_kv_table_destroy(hstu_kv_table* t) {
  if (!t) return;
  kv_table_free_storage(&t->dev);
  delete t;
}

hstu_status hstu_kv_table_status(hstu_kv_table* t, cudaStream_t stream) {
  if (!t) return HSTU_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return HSTU_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, t->dev.status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (v != 0) {
    const int32_t z = 0;
    if (cudaMemcpy(t->dev.status, &z, sizeof(z), cudaMemcpyHostToDevice) != cudaSuccess)
      return HSTU_ERR_CUDA;
  }
  return (hstu_status)v;
}

hstu_status hstu_kv_table_info(hstu_kv_table* t, void** pool, int32_t** page_lists,
                               int64_t** lengths, int32_t** free_stack, int32_t** free_top) {
  if (!t) return HSTU_ERR_INVALID_ARG;
  if (pool) *pool = t->dev.pool;
  if (page_lists) *page_lists = t->dev.page_lists;
  if (lengths) *lengths = t->dev.lengths;
  if (free_stack) *free_stack = t->dev.free_stack;
  if (free_top) *free_top = t->dev.free_top;
  return HSTU_OK;
}

hstu_status hstu_kv_alloc(hstu_kv_table* t, const int64_t* users, const int64_t* n_new_tokens,
                          int32_t B, int32_t* page_ids_out, int32_t page_ids_cap,
                          cudaStream_t stream) {
  if (!t || B < 0 || B > 65536 || page_ids_cap < 0) return HSTU_ERR_INVALID_ARG;
  if (B > 0 && (!users || !n_new_tokens)) return HSTU_ERR_INVALID_ARG;
  if (page_ids_out == nullptr) page_ids_cap = 0;
  if (B == 0 && page_ids_cap == 0) return HSTU_OK;
  return from_cuda(kv_alloc_launch(t->dev, users, n_new_tokens, B, page_ids_cap ? page_ids_out : nullptr,
                                   page_ids_cap, stream));
}

hstu_status hstu_kv_release(hstu_kv_table* t, const int64_t* users, int32_t B,
                            cudaStream_t stream) {
  if (!t || B < 0 || B > 65536) return HSTU_ERR_INVALID_ARG;
  if (B == 0) return HSTU_OK;
  if (!users) return HSTU_ERR_INVALID_ARG;
  return from_cuda(kv_release_launch(t->dev, users, B, stream));
}

hstu_status hstu_kv_append(hstu_kv_table* t, const int64_t* users, const void* k_new,
                           const void* v_new, const int64_t* new_offsets, int32_t B,
                           int32_t max_new, cudaStream_t stream) {
  if (!t || B < 0 || max_new < 0) return HSTU_ERR_INVALID_ARG;
  if (B == 0 || max_new == 0) return HSTU_OK;
  if (!users || !k_new || !v_new || !new_offsets) return HSTU_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new)) return HSTU_ERR_INVALID_ARG;
  if (B > 65535) return HSTU_ERR_UNSUPPORTED;
  return from_cuda(kv_append_launch(t->dev, users, k_new, v_new, new_offsets, B, max_new, stream));
}

hstu_status hstu_kv_lookup(hstu_kv_table* t, const int64_t* users, int32_t B,
                           int64_t* cached_len_out, int32_t* page_table_out, int32_t max_pages,
                           void* k_out, void* v_out, const int64_t* out_offsets, int32_t max_len,
                           cudaStream_t stream) {
  if (!t || B < 0 || max_pages < 0 || max_len < 0) return HSTU_ERR_INVALID_ARG;
  if (B == 0) return HSTU_OK;
  if (!users) return HSTU_ERR_INVALID_ARG;
  if ((k_out != nullptr) != (v_out != nullptr)) return HSTU_ERR_INVALID_ARG;
  if (k_out && (!out_offsets || !aligned16(k_out) || !aligned16(v_out))) return HSTU_ERR_INVALID_ARG;
  if (page_table_out == nullptr) max_pages = 0;
  if (B > 65535) return HSTU_ERR_UNSUPPORTED;
  return from_cuda(kv_lookup_launch(t->dev, users, B, cached_len_out, page_table_out, max_pages,
                                    k_out, v_out, out_offsets, max_len, stream));
}

hstu_status hstu_kv_step(hstu_kv_table* t, const int64_t* users, const void* k_new,
                         const void* v_new, const int64_t* new_offsets, int32_t B, int32_t max_new,
                         int64_t* cached_len_out, int32_t* page_table_out, int32_t max_pages,
                         cudaStream_t stream) {
  if (!t || B < 0 || max_new < 0 || max_pages < 0) return HSTU_ERR_INVALID_ARG;
  if (B == 0) return HSTU_OK;
  if (!users || !new_offsets) return HSTU_ERR_INVALID_ARG;
  if (max_new > 0 && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)))
    return HSTU_ERR_INVALID_ARG;
  if (page_table_out == nullptr) max_pages = 0;
  if (B > 65535) return HSTU_ERR_UNSUPPORTED;
  return from_cuda(kv_step_launch(t->dev, users, k_new, v_new, new_offsets, B, max_new,
                                  cached_len_out, page_table_out, max_pages, stream));
}

static bool cached_problem(hstu_kv_table* t, const int64_t* users, int32_t B, const void* q,
                           const void* k_cand, const void* v_cand, const int64_t* q_offsets,
                           int64_t total_q, int32_t max_q, int32_t max_cached, int32_t mask_mode,
                           AttnProblem* p) {
  p->B = B;
  p->H = t->dev.H;
  p->d = t->dev.d;
  p->mode = mask_mode == HSTU_MASK_CANDIDATES ? 1 : 0;
  p->paged = true;
  p->q_off = q_offsets;
  p->users = users;
  p->page_lists = t->dev.page_lists;
  p->lengths = t->dev.lengths;
  p->max_users = t->dev.max_users;
  p->max_ppu = t->dev.max_ppu;
  p->n_pages = t->dev.n_pages;
  p->pool = t->dev.pool;
  p->q = q;
  p->k = k_cand;
  p->v = v_cand;
  p->q_stride = p->k_stride = p->v_stride = p->out_stride = (int64_t)t->dev.H * t->dev.d;
  p->total_q = total_q;
  p->total_kv = 0;
  p->max_q = max_q;
  p->max_kv = max_cached;
  p->f32 = t->dtype == HSTU_F32;
  return true;
}

size_t hstu_attn_cached_workspace_size(hstu_kv_table* t, int32_t B, int64_t total_q, int32_t max_q,
                                       int32_t max_cached, int32_t mask_mode) {
  if (!t || B <= 0 || max_q <= 0 || t->dtype != HSTU_BF16 || t->dev.d != 128) return 0;
  if (total_q <= 0 || max_cached < 0) return 0;
  if (mask_mode != HSTU_MASK_CANDIDATES && mask_mode != HSTU_MASK_CAUSAL_SUFFIX) return 0;
  AttnProblem p;
  cached_problem(t, nullptr, B, nullptr, nullptr, nullptr, nullptr, total_q, max_q, max_cached,
                 mask_mode, &p);
  return attn_sm100_workspace_bytes(p, device_sm_count());
}

}  // extern "C"

// Host-side argument checks of hstu_attn_cached_fwd (shared with its
// allocation-free variant, so both report the same status for the same
// arguments).  *nothing_to_do is set for a valid call with no query rows.
hstu_status cached_fwd_validate(hstu_kv_table* t, const int64_t* users, int32_t B, const void* q,
                                const void* k_cand, const void* v_cand, const int64_t* q_offsets,
                                int64_t total_q, int32_t max_q, int32_t max_cached,
                                int32_t mask_mode, const hstu_rab* rab, const void* out,
                                bool* nothing_to_do) {
  *nothing_to_do = false;
  if (!t || B < 0 || max_q < 0 || max_cached < 0 || total_q < 0) return HSTU_ERR_INVALID_ARG;
  if (total_q >= (1LL << 31)) return HSTU_ERR_UNSUPPORTED;
  if (mask_mode != HSTU_MASK_CANDIDATES && mask_mode != HSTU_MASK_CAUSAL_SUFFIX)
    return HSTU_ERR_INVALID_ARG;
  if (B == 0 || max_q == 0 || total_q == 0) {
    *nothing_to_do = true;
    return HSTU_OK;
  }
  if (!users || !q || !q_offsets || !out) return HSTU_ERR_INVALID_ARG;
  if (mask_mode == HSTU_MASK_CANDIDATES && (!k_cand || !v_cand)) return HSTU_ERR_INVALID_ARG;
  if (mask_mode == HSTU_MASK_CAUSAL_SUFFIX && (k_cand || v_cand)) return HSTU_ERR_INVALID_ARG;
  if (!rab_ok(rab, false)) return HSTU_ERR_UNSUPPORTED;
  if (t->dtype == HSTU_BF16 && t->dev.d == 128 &&
      (!aligned16(q) || !aligned16(out) || (k_cand && (!aligned16(k_cand) || !aligned16(v_cand)))))
    return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

extern "C" {

hstu_status hstu_attn_cached_fwd(hstu_kv_table* t, const int64_t* users, int32_t B, const void* q,
                                 const void* k_cand, const void* v_cand, const int64_t* q_offsets,
                                 int64_t total_q, int32_t max_q, int32_t max_cached, int32_t mask_mode,
                                 const hstu_rab* rab, float scale, void* out, void* workspace,
                                 size_t ws_bytes, cudaStream_t stream) {
  bool nothing = false;
  const hstu_status st = cached_fwd_validate(t, users, B, q, k_cand, v_cand, q_offsets, total_q,
                                             max_q, max_cached, mask_mode, rab, out, &nothing);
  if (st != HSTU_OK || nothing) return st;
  AttnProblem p;
  cached_problem(t, users, B, q, k_cand, v_cand, q_offsets, total_q, max_q, max_cached, mask_mode,
                 &p);
  p.out = out;
  fill_rab(p, rab);
  p.scale = scale;
  if (!p.f32 && p.d == 128) {
    const size_t need = attn_sm100_workspace_bytes(p, device_sm_count());
    if (need > 0 && (workspace == nullptr || ws_bytes < need)) return HSTU_ERR_INVALID_ARG;
  }
  return attn_dispatch(p, workspace, ws_bytes, stream);
}

}  // extern "C"

extern "C" {

size_t hstu_block_workspace_size(int64_t T, int32_t d_model, int32_t H, int32_t dh) {
  if (T < 0 || d_model <= 0 || H <= 0 || dh <= 0) return 0;
  return block_workspace_bytes(T, d_model, H, dh);
}

hstu_status hstu_block_fwd(void* x, const int64_t* seq_offsets, int32_t B, int32_t max_len,
                           int64_t T, int32_t n_layers, int32_t d_model, int32_t H, int32_t dh,
                           const void* const* w_uvqk, const void* const* w_o, const hstu_rab* rab,
                           float scale, float ln_eps, void* workspace, size_t ws_bytes,
                           cudaStream_t stream) {
  if (B < 0 || max_len < 0 || T < 0 || n_layers < 0 || d_model <= 0 || H <= 0 || dh <= 0)
    return HSTU_ERR_INVALID_ARG;
  if (T >= (1LL << 31)) return HSTU_ERR_UNSUPPORTED;
  if (dh != 128 || H * dh != d_model || d_model % 128 != 0) return HSTU_ERR_UNSUPPORTED;
  if (!rab_ok(rab, true)) return HSTU_ERR_INVALID_ARG;
  if (T == 0 || n_layers == 0 || B == 0) return HSTU_OK;
  if (!x || !seq_offsets || !w_uvqk || !w_o || !aligned16(x)) return HSTU_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if (!w_uvqk[l] || !w_o[l] || !aligned16(w_uvqk[l]) || !aligned16(w_o[l]))
      return HSTU_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < block_workspace_bytes(T, d_model, H, dh) || !aligned16(workspace))
    return HSTU_ERR_INVALID_ARG;
  BlockProblem p;
  p.x = x;
  p.seq_offsets = seq_offsets;
  p.B = B;
  p.max_len = max_len;
  p.T = T;
  p.n_layers = n_layers;
  p.d_model = d_model;
  p.H = H;
  p.dh = dh;
  p.w_uvqk = w_uvqk;
  p.w_o = w_o;
  if (rab) {
    p.pos_table = rab->pos_table;
    p.n_pos = rab->pos_table ? rab->n_pos_buckets : 0;
    p.time_table = rab->time_table;
    p.n_time = rab->time_table ? rab->n_time_buckets : 0;
    p.ts = rab->time_table ? rab->timestamps : nullptr;
  }
  p.scale = scale;
  p.ln_eps = ln_eps;
  const cudaError_t e = block_fwd_launch(p, workspace, ws_bytes, device_error_word(), stream);
  if (e == cudaErrorNotSupported) return HSTU_ERR_UNSUPPORTED;
  return from_cuda(e);
}

}  // extern "C"

// ---------------------------------------------------------------- cached multi-layer step
namespace {

// Host-side view of the per-layer tables; false if any table does not fit the block.
bool cached_step_problem(hstu_kv_table* const* tables, int32_t n_layers, int32_t d_model, int32_t H,
                         int32_t dh, std::vector<hstu::KvTableDev>* devs) {
  if (!tables || n_layers <= 0) return false;
  devs->clear();
  for (int l = 0; l < n_layers; ++l) {
    const hstu_kv_table* t = tables[l];
    if (!t || t->dtype != HSTU_BF16 || t->dev.H != H || t->dev.d != dh || H * dh != d_model)
      return false;
    devs->push_back(t->dev);
  }
  return true;
}

}  // namespace

extern "C" {

size_t hstu_block_cached_workspace_size(hstu_kv_table* const* tables, int32_t n_layers, int32_t B,
                                        int64_t T_new, int64_t T_cand, int32_t max_cand,
                                        int32_t max_cached, int32_t d_model, int32_t H,
                                        int32_t dh) {
  std::vector<hstu::KvTableDev> devs;
  if (B < 0 || T_new < 0 || T_cand < 0 || max_cand < 0 || max_cached < 0) return 0;
  if (!cached_step_problem(tables, n_layers, d_model, H, dh, &devs)) return 0;
  hstu::CachedStepProblem p;
  p.tables = devs.data();
  p.n_layers = n_layers;
  p.B = B;
  p.T_new = T_new;
  p.T_cand = T_cand;
  p.max_cand = max_cand;
  p.max_cached = max_cached;
  p.d_model = d_model;
  p.H = H;
  p.dh = dh;
  return hstu::block_cached_workspace_bytes(p, hstu::device_sm_count());
}

hstu_status hstu_block_cached_step(hstu_kv_table* const* tables, int32_t n_layers,
                                   const int64_t* users, int32_t B, void* x,
                                   const int64_t* new_offsets, int64_t T_new, int32_t max_new,
                                   const int64_t* cand_offsets, int64_t T_cand, int32_t max_cand,
                                   int32_t max_cached, int32_t d_model, int32_t H, int32_t dh,
                                   const void* const* w_uvqk, const void* const* w_o,
                                   const hstu_rab* rab, float scale, float ln_eps, void* workspace,
                                   size_t ws_bytes, cudaStream_t stream) {
  if (n_layers < 0 || B < 0 || T_new < 0 || T_cand < 0 || max_new < 0 || max_cand < 0 ||
      max_cached < 0 || d_model <= 0 || H <= 0 || dh <= 0)
    return HSTU_ERR_INVALID_ARG;
  if (T_new + T_cand >= (1LL << 31)) return HSTU_ERR_UNSUPPORTED;
  if (dh != 128 || H * dh != d_model || d_model != 512) return HSTU_ERR_UNSUPPORTED;
  if (!rab_ok(rab, false)) return HSTU_ERR_UNSUPPORTED;
  if (n_layers == 0 || B == 0 || T_new + T_cand == 0) return HSTU_OK;
  if (B > hstu::kMaxCachedStepUsers) return HSTU_ERR_UNSUPPORTED;
  std::vector<hstu::KvTableDev> devs;
  if (!cached_step_problem(tables, n_layers, d_model, H, dh, &devs)) return HSTU_ERR_INVALID_ARG;
  if (!users || !x || !aligned16(x) || !w_uvqk || !w_o) return HSTU_ERR_INVALID_ARG;
  if ((T_new > 0 && (!new_offsets || max_new <= 0)) || (T_cand > 0 && (!cand_offsets || max_cand <= 0)))
    return HSTU_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if (!w_uvqk[l] || !w_o[l] || !aligned16(w_uvqk[l]) || !aligned16(w_o[l]))
      return HSTU_ERR_INVALID_ARG;
  hstu::CachedStepProblem p;
  p.tables = devs.data();
  p.n_layers = n_layers;
  p.users = users;
  p.B = B;
  p.x = x;
  p.new_offsets = new_offsets;
  p.T_new = T_new;
  p.max_new = max_new;
  p.cand_offsets = cand_offsets;
  p.T_cand = T_cand;
  p.max_cand = max_cand;
  p.max_cached = max_cached;
  p.d_model = d_model;
  p.H = H;
  p.dh = dh;
  p.w_uvqk = w_uvqk;
  p.w_o = w_o;
  if (rab && rab->pos_table) {
    p.pos_table = rab->pos_table;
    p.n_pos = rab->n_pos_buckets;
  }
  p.scale = scale;
  p.ln_eps = ln_eps;
  const size_t need = hstu::block_cached_workspace_bytes(p, hstu::device_sm_count());
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return HSTU_ERR_INVALID_ARG;
  const cudaError_t e =
      hstu::block_cached_step_launch(p, workspace, ws_bytes, device_error_word(), stream);
  if (e == cudaErrorNotSupported) return HSTU_ERR_UNSUPPORTED;
  return from_cuda(e);
}

}  // extern "C"

// ---------------------------------------------------------------- user-id map
struct hstu_user_map {
  hstu::UserMapDev dev;
};

extern "C" {

hstu_status hstu_user_map_create(int32_t n_slots, const int32_t* host_free_order,
                                 hstu_user_map** out_map) {
  if (!out_map || n_slots <= 0 || n_slots > (1 << 28)) return HSTU_ERR_INVALID_ARG;
  *out_map = nullptr;
  if (host_free_order) {
    std::vector<char> seen((size_t)n_slots, 0);
    for (int32_t i = 0; i < n_slots; ++i) {
      const int32_t x = host_free_order[i];
      if (x < 0 || x >= n_slots || seen[x]) return HSTU_ERR_INVALID_ARG;
      seen[x] = 1;
    }
  }
  hstu_user_map* m = new (std::nothrow) hstu_user_map();
  if (!m) return HSTU_ERR_CUDA;
  if (hstu::user_map_alloc(&m->dev, n_slots, host_free_order) != cudaSuccess) {
    hstu::user_map_free(&m->dev);
    delete m;
    return HSTU_ERR_CUDA;
  }
  *out_map = m;
  return HSTU_OK;
}

void hstu_user_map_destroy(hstu_user_map* m) {
  if (!m) return;
  hstu::user_map_free(&m->dev);
  delete m;
}

hstu_status hstu_user_map_lookup(hstu_user_map* m, const int64_t* ids, int32_t B, int32_t insert,
                                 int64_t* slots_out, cudaStream_t stream) {
  if (!m || B < 0 || B > 65536) return HSTU_ERR_INVALID_ARG;
  if (B == 0) return HSTU_OK;
  if (!ids || !slots_out) return HSTU_ERR_INVALID_ARG;
  return from_cuda(hstu::user_map_lookup_launch(m->dev, ids, B, insert != 0, slots_out, stream));
}

hstu_status hstu_user_map_erase(hstu_user_map* m, const int64_t* ids, int32_t B,
                                cudaStream_t stream) {
  if (!m || B < 0) return HSTU_ERR_INVALID_ARG;
  if (B == 0) return HSTU_OK;
  if (!ids) return HSTU_ERR_INVALID_ARG;
  return from_cuda(hstu::user_map_erase_launch(m->dev, ids, B, stream));
}

hstu_status hstu_user_map_status(hstu_user_map* m, cudaStream_t stream) {
  if (!m) return HSTU_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return HSTU_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, m->dev.status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (v != 0) {
    const int32_t z = 0;
    if (cudaMemcpy(m->dev.status, &z, sizeof(z), cudaMemcpyHostToDevice) != cudaSuccess)
      return HSTU_ERR_CUDA;
  }
  return (hstu_status)v;
}

}  // extern "C"

// ---------------------------------------------------------------- beam decode
extern "C" {

static bool beam_problem(hstu_kv_table* t, const int64_t* users, int32_t B, const void* q,
                         const int64_t* beam_offsets, int64_t total_beams, int32_t max_beams,
                         int32_t max_ctx, int32_t step, const void* beam_k, const void* beam_v,
                         const int32_t* beam_parent, const hstu_rab* rab, float scale, void* out,
                         hstu::BeamDecodeProblem* p) {
  p->table = t->dev;
  p->users = users;
  p->B = B;
  p->q = q;
  p->beam_offsets = beam_offsets;
  p->total_beams = total_beams;
  p->max_beams = max_beams;
  p->max_ctx = max_ctx;
  p->step = step;
  p->beam_k = beam_k;
  p->beam_v = beam_v;
  p->beam_parent = beam_parent;
  if (rab && rab->pos_table) {
    p->pos_table = rab->pos_table;
    p->n_pos = rab->n_pos_buckets;
  }
  p->scale = scale;
  p->out = out;
  return true;
}

size_t hstu_attn_beam_decode_workspace_size(hstu_kv_table* t, int32_t B, int64_t total_beams,
                                            int32_t max_beams, int32_t max_ctx, int32_t step) {
  if (!t || B < 0 || total_beams < 0 || max_beams < 0 || max_ctx < 0 || step < 0) return 0;
  hstu::BeamDecodeProblem p;
  beam_problem(t, nullptr, B, nullptr, nullptr, total_beams, max_beams, max_ctx, step, nullptr,
               nullptr, nullptr, nullptr, 1.f, nullptr, &p);
  return hstu::beam_decode_workspace_bytes(p, device_sm_count());
}

hstu_status hstu_attn_beam_decode(hstu_kv_table* t, const int64_t* users, int32_t B, const void* q,
                                  const int64_t* beam_offsets, int64_t total_beams,
                                  int32_t max_beams, int32_t max_ctx, int32_t step,
                                  const void* beam_k, const void* beam_v,
                                  const int32_t* beam_parent, const hstu_rab* rab, float scale,
                                  void* out, void* workspace, size_t ws_bytes,
                                  cudaStream_t stream) {
  if (!t || B < 0 || total_beams < 0 || max_beams < 0 || max_ctx < 0 || step < 0)
    return HSTU_ERR_INVALID_ARG;
  if (t->dtype != HSTU_BF16 || t->dev.d != 128 || t->dev.H > 32) return HSTU_ERR_UNSUPPORTED;
  if ((int64_t)(step + 1) * total_beams >= (1LL << 31)) return HSTU_ERR_UNSUPPORTED;
  if (!rab_ok(rab, false)) return HSTU_ERR_UNSUPPORTED;
  if (B == 0 || total_beams == 0) return HSTU_OK;
  if (!users || !q || !beam_offsets || !beam_k || !beam_v || !out || max_beams <= 0)
    return HSTU_ERR_INVALID_ARG;
  if (step > 0 && !beam_parent) return HSTU_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(beam_k) || !aligned16(beam_v))
    return HSTU_ERR_INVALID_ARG;
  hstu::BeamDecodeProblem p;
  beam_problem(t, users, B, q, beam_offsets, total_beams, max_beams, max_ctx, step, beam_k, beam_v,
               beam_parent, rab, scale, out, &p);
  const size_t need = hstu::beam_decode_workspace_bytes(p, device_sm_count());
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return HSTU_ERR_INVALID_ARG;
  const cudaError_t e = hstu::beam_decode_launch(p, workspace, ws_bytes, device_error_word(), stream);
  if (e == cudaErrorNotSupported) return HSTU_ERR_UNSUPPORTED;
  return from_cuda(e);
}

}  // extern "C"
