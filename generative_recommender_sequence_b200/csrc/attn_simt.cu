// HSTU attention, SIMT (CUDA-core) kernel for fp32 tensors and for bf16 with
// head dim 32 or 64.  Same definition as the tensor-core kernel (section "HSTU"
// of "How Generative Recommenders Are Redefining RecSys at Scale"):
//     O[i] = scale * sum_{j in M(i)} SiLU(q_i . k_j + rab(i, j)) v_j
// computed with fp32 arithmetic throughout and the accurate expf, which is
// what the 1e-5 fp32 contract needs (tensor-core tf32 cannot meet it).
//
// One CTA per (query tile of 64 rows, head, user); 128 threads.  Keys are
// staged 64 at a time in shared memory: S = Q K^T (4x8 scores per thread),
// bias + mask + SiLU into P, then O += P V (8 rows x d/16 columns per thread).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "attn.h"
#include "sm100.cuh"

namespace hstu {
namespace {

constexpr int QT = 64;   // query rows per CTA
constexpr int KT = 64;   // keys per stage
constexpr int NT = 128;  // threads

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

struct SimtParams {
  int B, H, mode;
  bool paged;
  const int64_t* q_off;
  const int64_t* kv_off;
  const int64_t* users;
  const int32_t* page_lists;
  const int64_t* lengths;
  int64_t max_users;
  int max_ppu;
  int64_t n_pages;
  const void* pool;
  const void* q;
  int64_t q_stride;
  const void* k;
  int64_t k_stride;
  const void* v;
  int64_t v_stride;
  void* out;
  int64_t out_stride;
  const float* pos_table;
  int n_pos;
  const float* time_table;
  int n_time;
  const int64_t* ts;
  float scale;
  int64_t total_q, total_kv;
};

__device__ __forceinline__ int floor_log2_p1(long long x) {  // floor(log2(max(x,0)+1))
  x = x < 0 ? 0 : x;
  return 63 - __clzll(x + 1);
}

template <typename T, int D>
__global__ void __launch_bounds__(NT)
    hstu_attn_simt_kernel(const SimtParams P) {
  extern __shared__ float smem[];
  float* sQ = smem;                       // [QT][D+1]
  float* sK = sQ + QT * (D + 1);          // [KT][D+1]
  float* sV = sK + KT * (D + 1);          // [KT][D]
  float* sP = sV + KT * D;                // [QT][KT+1]
  long long* sKts = reinterpret_cast<long long*>(sP + QT * (KT + 1));  // [KT]
  float* sSelf = reinterpret_cast<float*>(sKts + KT);                  // [QT]

  const int b = blockIdx.z, h = blockIdx.y, m = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t qs = P.q_off[b], nq = P.q_off[b + 1] - qs;
  if ((int64_t)m * QT >= nq) return;
  const int64_t q_row0 = qs + (int64_t)m * QT;
  // rows past the tensors' end (inconsistent offsets) are neither read nor written
  const int nvalid = (int)max64(0, min64(min64(QT, nq - (int64_t)m * QT), P.total_q - q_row0));

  int64_t n_k, kv_row0 = 0, user = 0;
  if (P.paged) {
    // an out-of-range user id has no cached tokens (and no page list is read)
    const int64_t u = P.users[b];
    const bool known = u >= 0 && u < P.max_users;
    user = known ? u : 0;
    n_k = known ? P.lengths[u] : 0;
  } else {
    kv_row0 = P.kv_off[b];
    n_k = P.kv_off[b + 1] - kv_row0;
  }
  const bool cand = P.mode == 1;
  const int64_t p0 = cand ? n_k : n_k - nq + (int64_t)m * QT;  // position of query row 0
  const T* qptr = reinterpret_cast<const T*>(P.q);
  const T* kptr = reinterpret_cast<const T*>(P.k);
  const T* vptr = reinterpret_cast<const T*>(P.v);
  const T* pool = reinterpret_cast<const T*>(P.pool);

  for (int i = tid; i < QT * D; i += NT) {
    const int r = i / D, e = i % D;
    sQ[r * (D + 1) + e] = r < nvalid ? to_f(qptr[(q_row0 + r) * P.q_stride + h * D + e]) : 0.f;
  }

  // thread tiles
  const int rg = tid / 16, kg = tid % 16;   // S: rows 8rg..8rg+7, keys 4kg..4kg+3
  constexpr int OC = D / 16;                // O: rows 8rg..8rg+7, cols kg*OC..
  float acc[8][OC];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < OC; ++j) acc[i][j] = 0.f;

  int64_t kend = cand ? n_k : min64(n_k, p0 + nvalid);  // keys ever visible
  if (kend < 0) kend = 0;
  const bool use_time = P.time_table != nullptr && !P.paged && !cand;
  long long ts_q[8];
  if (use_time) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int64_t qp = p0 + rg * 8 + i;
      qp = qp < 0 ? 0 : (qp >= n_k ? n_k - 1 : qp);
      ts_q[i] = (n_k > 0 && kv_row0 + qp < P.total_kv) ? P.ts[kv_row0 + qp] : 0;
    }
  }

  for (int64_t k0 = 0; k0 < kend; k0 += KT) {
    __syncthreads();
    for (int i = tid; i < KT * D; i += NT) {
      const int c = i / D, e = i % D;
      const int64_t kp = k0 + c;
      float kv = 0.f, vv = 0.f;
      if (kp < kend) {
        if (P.paged) {
          const int pi = (int)(kp / 32), slot = (int)(kp % 32);
          const int64_t page = pi < P.max_ppu ? (int64_t)P.page_lists[user * P.max_ppu + pi] : -1;
          if (page >= 0 && page < P.n_pages) {
            const int64_t base = (((page * 2) * P.H + h) * 32 + slot) * D + e;
            kv = to_f(pool[base]);
            vv = to_f(pool[base + (int64_t)P.H * 32 * D]);
          }
        } else if (kv_row0 + kp < P.total_kv) {
          kv = to_f(kptr[(kv_row0 + kp) * P.k_stride + h * D + e]);
          vv = to_f(vptr[(kv_row0 + kp) * P.v_stride + h * D + e]);
        }
      }
      sK[c * (D + 1) + e] = kv;
      sV[c * D + e] = vv;
    }
    if (use_time && tid < KT) {
      const int64_t kp = k0 + tid;
      sKts[tid] = (kp < n_k && kv_row0 + kp < P.total_kv) ? P.ts[kv_row0 + kp] : 0;
    }
    __syncthreads();
    // scores
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = rg * 8 + i;
      const int64_t qp = cand ? p0 : p0 + r;   // candidates share one position
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = kg * 4 + j;
        const int64_t kp = k0 + c;
        float s = 0.f;
#pragma unroll 8
        for (int e = 0; e < D; ++e) s = fmaf(sQ[r * (D + 1) + e], sK[c * (D + 1) + e], s);
        const bool valid = kp < kend && (cand ? true : kp <= qp);
        const int64_t delta = qp - kp;
        if (P.pos_table) {
          const int bk = min(floor_log2_p1(delta < 0 ? -delta : delta), P.n_pos - 1);
          s += P.pos_table[bk];
        }
        if (use_time) s += P.time_table[min(floor_log2_p1(ts_q[i] - sKts[c]), P.n_time - 1)];
        const float w = s / (1.f + expf(-s));
        sP[r * (KT + 1) + c] = valid ? w : 0.f;
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < KT; ++c) {
      float vv[OC];
#pragma unroll
      for (int j = 0; j < OC; ++j) vv[j] = sV[c * D + kg * OC + j];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float p = sP[(rg * 8 + i) * (KT + 1) + c];
#pragma unroll
        for (int j = 0; j < OC; ++j) acc[i][j] = fmaf(p, vv[j], acc[i][j]);
      }
    }
  }

  if (cand) {
    // the candidate's own key/value: one extra visible key at distance 0
    __syncthreads();
    if (tid < QT) {
      const int r = tid;
      float s = 0.f;
      if (r < nvalid) {
        const int64_t row = q_row0 + r;
        for (int e = 0; e < D; ++e)
          s = fmaf(sQ[r * (D + 1) + e], to_f(kptr[row * P.k_stride + h * D + e]), s);
        if (P.pos_table) s += P.pos_table[0];
        s = s / (1.f + expf(-s));
      }
      sSelf[r] = s;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = rg * 8 + i;
      if (r < nvalid) {
        const int64_t row = q_row0 + r;
#pragma unroll
        for (int j = 0; j < OC; ++j)
          acc[i][j] = fmaf(sSelf[r], to_f(vptr[row * P.v_stride + h * D + kg * OC + j]), acc[i][j]);
      }
    }
  }

  T* out = reinterpret_cast<T*>(P.out);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = rg * 8 + i;
    if (r < nvalid) {
#pragma unroll
      for (int j = 0; j < OC; ++j)
        out[(q_row0 + r) * P.out_stride + h * D + kg * OC + j] = from_f<T>(acc[i][j] * P.scale);
    }
  }
}

template <typename T, int D>
cudaError_t launch_t(const SimtParams& sp, const AttnProblem& p, cudaStream_t stream) {
  const size_t smem = sizeof(float) * (QT * (D + 1) + KT * (D + 1) + KT * D + QT * (KT + 1)) +
                      sizeof(long long) * KT + sizeof(float) * QT;
  auto kern = hstu_attn_simt_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int qt = (p.max_q + QT - 1) / QT;
  dim3 grid(qt > 0 ? qt : 1, p.H, p.B);
  kern<<<grid, NT, smem, stream>>>(sp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t attn_simt_launch(const AttnProblem& p, cudaStream_t stream) {
  if (p.B == 0 || p.total_q == 0 || p.max_q == 0) return cudaSuccess;
  SimtParams sp;
  sp.B = p.B;
  sp.H = p.H;
  sp.mode = p.mode;
  sp.paged = p.paged;
  sp.q_off = p.q_off;
  sp.kv_off = p.kv_off;
  sp.users = p.users;
  sp.page_lists = p.page_lists;
  sp.lengths = p.lengths;
  sp.max_users = p.max_users;
  sp.max_ppu = p.max_ppu;
  sp.n_pages = p.n_pages;
  sp.pool = p.pool;
  sp.q = p.q;
  sp.q_stride = p.q_stride;
  sp.k = p.k;
  sp.k_stride = p.k_stride;
  sp.v = p.v;
  sp.v_stride = p.v_stride;
  sp.out = p.out;
  sp.out_stride = p.out_stride;
  sp.pos_table = p.pos_table;
  sp.n_pos = p.n_pos;
  sp.time_table = p.time_table;
  sp.n_time = p.n_time;
  sp.ts = p.ts;
  sp.scale = p.scale;
  sp.total_q = p.total_q;
  sp.total_kv = p.total_kv;
  if (p.f32) {
    if (p.d == 32) return launch_t<float, 32>(sp, p, stream);
    if (p.d == 64) return launch_t<float, 64>(sp, p, stream);
    if (p.d == 128) return launch_t<float, 128>(sp, p, stream);
  } else {
    if (p.d == 32) return launch_t<__nv_bfloat16, 32>(sp, p, stream);
    if (p.d == 64) return launch_t<__nv_bfloat16, 64>(sp, p, stream);
    if (p.d == 128) return launch_t<__nv_bfloat16, 128>(sp, p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hstu
