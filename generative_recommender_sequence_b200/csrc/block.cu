// HSTU block stack on B200 ("How Generative Recommenders Are Redefining RecSys
// at Scale", section "HSTU": pointwise projection, SiLU attention with a
// relative bias, elementwise gating before the output projection):
//
//   per layer:  UVQK = SiLU(X W1)                  tcgen05 GEMM, SiLU epilogue
//               A    = HSTU attention(Q, K, V)     attn_sm100 (reads UVQK in place)
//               G    = LayerNorm(A) * U            one warp per token
//               X    = X + G W2                    tcgen05 GEMM, residual epilogue
//
// bf16 storage, fp32 accumulation; UVQK, A, G and X are the bf16 tensors the
// stack materialises.
//
// GEMM kernel: persistent, one CTA per SM, 320 threads.  Warp 0 issues TMA
// (A tile 128 x 64 K-major, B tile 64 x BN MN-major, 128-byte swizzle),
// warp 1 issues tcgen05.mma (M=128, N=BN, K=16) into one of two TMEM
// accumulators (2 x BN columns), warps 2-9 drain the other accumulator
// (tcgen05.ld -> epilogue -> global; two warps per TMEM lane quarter, BN/2
// columns each) so the epilogue of tile i overlaps the main loop of tile i+1.
// Each epilogue warp stages its 32 x 32 bf16 result boxes in shared memory
// (two alternating 2 KiB buffers, 64-byte swizzle) and writes them with TMA
// stores: a thread holds one row, so direct stores would touch 32 rows per
// instruction (measured: 10 of GEMM1's 33 us went to those stores).  The
// residual epilogue TMA-loads the tile's X boxes into the same two buffers
// while the main loop runs, adds them there and stores the sums back.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "attn.h"
#include "block.h"
#include "sm100.cuh"

namespace hstu {
namespace {

constexpr int GBM = 128, GBK = 64;
constexpr int kGemmThreads = 320;
constexpr int kEpiWarps = 8;                 // warps 2..9
constexpr int kABytes = GBM * GBK * 2;       // 16 KiB
constexpr int kBBoxBytes = GBK * 64 * 2;     // one 64-column B box: 8 KiB

// Tile width BN (256 for the wide projection, 128 for the 512-column output
// projection, whose 128 x 256 tiles would give 148 SMs only 1.4 waves) and the
// TMA ring depth that keeps about 192 KiB of operands in flight.
template <int BN>
struct GemmCfg {
  static constexpr int kBBytes = GBK * BN * 2;
  static constexpr int kStages = BN >= 256 ? 4 : 6;
  static constexpr int kEpiCols = BN / 2;    // columns per epilogue warp
  static constexpr uint32_t kIdesc = idesc_bf16_f32(GBM, BN, true);
};

enum { EPI_SILU = 0, EPI_RESIDUAL = 1 };

constexpr int kStageBoxBytes = 32 * 32 * 2;  // one 32 x 32 bf16 output box

template <int BN>
struct __align__(1024) GemmSmem {
  uint8_t a[GemmCfg<BN>::kStages][kABytes];
  uint8_t b[GemmCfg<BN>::kStages][GemmCfg<BN>::kBBytes];
  uint8_t out[kEpiWarps][2][kStageBoxBytes];  // per epilogue warp, alternating
  uint64_t full[GemmCfg<BN>::kStages], empty[GemmCfg<BN>::kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t x_full[kEpiWarps];  // residual epilogue: X boxes of the tile landed
  uint64_t mma_done;
  uint32_t tmem_base;
};

struct GemmParams {
  int M, N, K;
  __nv_bfloat16* out;        // [M, N] row stride ldo
  int64_t ldo;
  int* err;
};

template <int EPI, int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_out, const GemmParams P) {
  constexpr int GBN = BN;
  constexpr int GST = GemmCfg<BN>::kStages;
  constexpr int kBBytes = GemmCfg<BN>::kBBytes;
  constexpr int kEpiCols = GemmCfg<BN>::kEpiCols;
  constexpr uint32_t kIdescGemm = GemmCfg<BN>::kIdesc;
  extern __shared__ uint8_t smem_raw[];
  GemmSmem<BN>& sm = *reinterpret_cast<GemmSmem<BN>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // dependent launch: barrier set-up and the TMEM allocation overlap the
  // previous kernel's tail; global memory is touched only after the wait.
  // The next kernel is released only at the end (below): released at entry,
  // its CTAs were scheduled onto SMs while this GEMM still ran, measured
  // slower in the cached serving step.
  const int m_tiles = (P.M + GBM - 1) / GBM, n_tiles = P.N / GBN;
  const int tiles = m_tiles * n_tiles;
  const int kblocks = P.K / GBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < GST; ++i) {
      mbar_init(smem_u32(&sm.full[i]), 1);
      mbar_init(smem_u32(&sm.empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.acc_full[i]), 1);
      mbar_init(smem_u32(&sm.acc_empty[i]), kEpiWarps);
    }
    mbar_init(smem_u32(&sm.mma_done), 1);
    for (int i = 0; i < kEpiWarps; ++i) mbar_init(smem_u32(&sm.x_full[i]), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  pdl_wait();  // A (and, with the residual epilogue, the output) come from earlier kernels
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t c = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int mt = t / n_tiles, nt = t % n_tiles;
        for (int kb = 0; kb < kblocks; ++kb, ++c) {
          const uint32_t s = c % GST;
          if (!(ok = mbar_wait(smem_u32(&sm.empty[s]), ((c / GST) & 1) ^ 1))) break;
          const uint32_t bar = smem_u32(&sm.full[s]);
          mbar_arrive_expect_tx(bar, kABytes + kBBytes);
          tma_load_2d(smem_u32(sm.a[s]), &tm_a, bar, kb * GBK, mt * GBM);
#pragma unroll
          for (int j = 0; j < GBN / 64; ++j)
            tma_load_2d(smem_u32(sm.b[s]) + j * kBBoxBytes, &tm_b, bar, nt * GBN + j * 64, kb * GBK);
        }
      }
      if (!ok) {
        atomicExch(P.err, DEV_ERR_TIMEOUT);
        for (uint32_t i = 0; i < GST && i < c; ++i) {
          const uint32_t cc = c - 1 - i;
          mbar_wait(smem_u32(&sm.full[cc % GST]), (cc / GST) & 1);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t c = 0, tcount = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tcount) {
        const uint32_t ab = tcount & 1;
        if (!(ok = mbar_wait(smem_u32(&sm.acc_empty[ab]), ((tcount >> 1) & 1) ^ 1))) break;
        tc_fence_after();
        for (int kb = 0; kb < kblocks; ++kb, ++c) {
          const uint32_t s = c % GST;
          if (!(ok = mbar_wait(smem_u32(&sm.full[s]), (c / GST) & 1))) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(sm.a[s]), b_base = smem_u32(sm.b[s]);
#pragma unroll
          for (int kk = 0; kk < GBK / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(a_base + kk * 32, 16, 1024);
            // B is MN-major: 64-column boxes 8 KiB apart (LBO), 8-row k groups 1 KiB
            // apart (SBO), 16 k-rows = 2 KiB per k-step
            const uint64_t bdesc = smem_desc_sw128(b_base + kk * 2048, kBBoxBytes, 1024);
            umma_ss(tmem + ab * GBN, adesc, bdesc, kIdescGemm, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(smem_u32(&sm.empty[s]));
        }
        if (!ok) break;
        umma_commit(smem_u32(&sm.acc_full[ab]));
      }
      if (!ok) atomicExch(P.err, DEV_ERR_TIMEOUT);
      umma_commit(smem_u32(&sm.mma_done));
      mbar_wait(smem_u32(&sm.mma_done), 0);
    }
    __syncwarp();
  } else {
    // epilogue warps 2..9: TMEM lane quarter = warp % 4, column half by warp
    const int sub = warp & 3;
    const int chalf = (warp - 2) >> 2;
    const uint32_t lane_addr = (uint32_t)(sub * 32) << 16;
    uint8_t(&stage)[2][kStageBoxBytes] = sm.out[warp - 2];
    // row `lane` of a 32 x 32 box: 64-byte rows, 16-byte chunk q stored at
    // chunk q ^ ((row >> 1) & 3) (the TMA's 64-byte swizzle)
    const int swz = (lane >> 1) & 3;
    uint32_t ecount = 0;  // boxes this warp has staged
    uint32_t tcount = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tcount) {
      const int mt = t / n_tiles, nt = t % n_tiles;
      const uint32_t ab = tcount & 1;
      // residual epilogue (kEpiCols = 64: two boxes per warp, one per staging
      // buffer): the tile's X boxes are TMA-loaded into the buffers before the
      // accumulator is ready, once the previous tile's stores have read them
      static_assert(EPI != EPI_RESIDUAL || kEpiCols == 64, "residual epilogue stages two boxes");
      if (EPI == EPI_RESIDUAL) {
        if (lane == 0) {
          bulk_wait_read0();
          const uint32_t xb = smem_u32(&sm.x_full[warp - 2]);
          mbar_arrive_expect_tx(xb, 2 * kStageBoxBytes);
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
            tma_load_2d(smem_u32(stage[ch]), &tm_out, xb, nt * GBN + chalf * kEpiCols + ch * 32,
                        mt * GBM + sub * 32);
        }
        __syncwarp();
      }
      if (!mbar_wait_warp(smem_u32(&sm.acc_full[ab]), (tcount >> 1) & 1) ||
          (EPI == EPI_RESIDUAL && !mbar_wait_warp(smem_u32(&sm.x_full[warp - 2]), tcount & 1))) {
        if (lane == 0) atomicExch(P.err, DEV_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < kEpiCols / 32; ++ch, ++ecount) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_addr + ab * GBN + chalf * kEpiCols + ch * 32, v);
        tmem_wait_ld();
        reg_fence(v);
        if (ch == kEpiCols / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.acc_empty[ab]));
        }
        // rows past M are computed but not stored (the TMA store clips them)
        float x[32];
        if (EPI == EPI_SILU) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float a = __uint_as_float(v[j]);
            const float h = 0.5f * a;
            x[j] = fmaf(h, tanh_approx(h), h);
          }
        } else {
          const uint4* xrow = reinterpret_cast<const uint4*>(stage[ch] + lane * 64);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 u = xrow[q ^ swz];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 p = *reinterpret_cast<const __nv_bfloat162*>(&w[e]);
              x[q * 8 + 2 * e] = __uint_as_float(v[q * 8 + 2 * e]) + __bfloat162float(p.x);
              x[q * 8 + 2 * e + 1] = __uint_as_float(v[q * 8 + 2 * e + 1]) + __bfloat162float(p.y);
            }
          }
        }
        uint8_t* buf = stage[EPI == EPI_RESIDUAL ? ch : (ecount & 1)];
        // the store issued from this buffer two boxes ago must have read it
        if (EPI != EPI_RESIDUAL && ecount >= 2) {
          if (lane == 0) bulk_wait_read1();
          __syncwarp();
        }
        uint4* srow = reinterpret_cast<uint4*>(buf + lane * 64);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 u;
          u.x = pack_bf16x2(x[q * 8 + 0], x[q * 8 + 1]);
          u.y = pack_bf16x2(x[q * 8 + 2], x[q * 8 + 3]);
          u.z = pack_bf16x2(x[q * 8 + 4], x[q * 8 + 5]);
          u.w = pack_bf16x2(x[q * 8 + 6], x[q * 8 + 7]);
          srow[q ^ swz] = u;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_out, smem_u32(buf), nt * GBN + chalf * kEpiCols + ch * 32,
                       mt * GBM + sub * 32);
          bulk_commit();
        }
      }
    }
    // the output is complete (and the staging buffers free) before the CTA ends
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// G[t, :] = LayerNorm(A[t, :]) * U[t, :] over F = 512 features; one warp per
// token, 16 features per lane, two-pass mean / biased variance in fp32.
__global__ void __launch_bounds__(256)
    ln_gate_kernel(const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ u,
                   int64_t ldu, __nv_bfloat16* __restrict__ g, int64_t T, float eps) {
  constexpr int F = 512;
  pdl_launch_dependents();
  pdl_wait();
  const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const uint4* ar = reinterpret_cast<const uint4*>(a + t * F) + lane * 2;
  const uint4* ur = reinterpret_cast<const uint4*>(u + t * ldu) + lane * 2;
  float x[16], w[16];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint4 av = ar[q], uv = ur[q];
    const uint32_t aw[4] = {av.x, av.y, av.z, av.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 pa = *reinterpret_cast<const __nv_bfloat162*>(&aw[e]);
      const __nv_bfloat162 pu = *reinterpret_cast<const __nv_bfloat162*>(&uw[e]);
      x[q * 8 + 2 * e] = __bfloat162float(pa.x);
      x[q * 8 + 2 * e + 1] = __bfloat162float(pa.y);
      w[q * 8 + 2 * e] = __bfloat162float(pu.x);
      w[q * 8 + 2 * e + 1] = __bfloat162float(pu.y);
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) s += x[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s * (1.f / F);
  float v = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) v = fmaf(x[i] - mean, x[i] - mean, v);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const float inv = rsqrtf(v * (1.f / F) + eps);
  uint4* gr = reinterpret_cast<uint4*>(g + t * F) + lane * 2;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    uint4 o;
    o.x = pack_bf16x2((x[q * 8 + 0] - mean) * inv * w[q * 8 + 0], (x[q * 8 + 1] - mean) * inv * w[q * 8 + 1]);
    o.y = pack_bf16x2((x[q * 8 + 2] - mean) * inv * w[q * 8 + 2], (x[q * 8 + 3] - mean) * inv * w[q * 8 + 3]);
    o.z = pack_bf16x2((x[q * 8 + 4] - mean) * inv * w[q * 8 + 4], (x[q * 8 + 5] - mean) * inv * w[q * 8 + 5]);
    o.w = pack_bf16x2((x[q * 8 + 6] - mean) * inv * w[q * 8 + 6], (x[q * 8 + 7] - mean) * inv * w[q * 8 + 7]);
    gr[q] = o;
  }
}

template <int BN>
size_t gemm_smem_bytes() { return sizeof(GemmSmem<BN>) + 1024; }

// out[M, N] (ld ldo) = epi(A[M, K] (ld lda) @ B[K, N] (ld ldb)); residual
// epilogue reads out before writing it.
template <int EPI, int GBN>
cudaError_t gemm_launch(const void* A, int64_t lda, const void* Bw, int64_t ldb, void* out,
                        int64_t ldo, int M, int N, int K, int* err, bool pdl, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  if (N % GBN != 0 || K % GBK != 0) return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2, GBK, GBM))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tb, Bw, (uint64_t)N, (uint64_t)K, (uint64_t)ldb * 2, 64, GBK))
    return cudaErrorInvalidValue;
  CUtensorMap to;
  if (!make_tmap_2d_store(&to, out, (uint64_t)N, (uint64_t)M, (uint64_t)ldo * 2, 32, 32))
    return cudaErrorInvalidValue;
  auto kern = gemm_bf16_kernel<EPI, GBN>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)gemm_smem_bytes<GBN>());
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int tiles = ((M + GBM - 1) / GBM) * (N / GBN);
  const int grid = std::max(1, std::min(tiles, device_sm_count()));
  GemmParams p{M, N, K, reinterpret_cast<__nv_bfloat16*>(out), ldo, err};
  return launch_kernel(pdl, kern, dim3(grid), dim3(kGemmThreads), gemm_smem_bytes<GBN>(), stream, ta,
                       tb, to, p);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t block_workspace_bytes(int64_t T, int d_model, int H, int dh) {
  const size_t F = (size_t)H * dh;
  return align256((size_t)T * 4 * F * 2) + align256((size_t)T * F * 2) * 2;
}

cudaError_t block_fwd_launch(const BlockProblem& p, void* workspace, size_t ws_bytes, int* err_word,
                             cudaStream_t stream) {
  const int F = p.H * p.dh;
  if (p.dh != 128 || F != p.d_model || F != 512) return cudaErrorNotSupported;
  if (ws_bytes < block_workspace_bytes(p.T, p.d_model, p.H, p.dh)) return cudaErrorInvalidValue;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  __nv_bfloat16* uvqk = reinterpret_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* attn = reinterpret_cast<__nv_bfloat16*>(ws + align256((size_t)p.T * 4 * F * 2));
  __nv_bfloat16* gate =
      reinterpret_cast<__nv_bfloat16*>(ws + align256((size_t)p.T * 4 * F * 2) + align256((size_t)p.T * F * 2));
  const int M = (int)p.T;
  // The stack's kernels are launched stream-ordered, without programmatic
  // dependent launch: with it, the attention CTAs scheduled early behind the
  // projection GEMM cost 11-17 us per layer on B200 (8-layer stack 1223-1270
  // vs 1132 us, same box).
  constexpr bool kPdl = false;
  for (int l = 0; l < p.n_layers; ++l) {
    cudaError_t e = gemm_launch<EPI_SILU, 256>(p.x, p.d_model, p.w_uvqk[l], 4 * F, uvqk, 4 * F, M, 4 * F,
                                          p.d_model, err_word, kPdl, stream);
    if (e != cudaSuccess) return e;
    AttnProblem a;
    a.B = p.B;
    a.H = p.H;
    a.d = p.dh;
    a.mode = 0;
    a.q_off = p.seq_offsets;
    a.kv_off = p.seq_offsets;
    a.q = uvqk + 2 * F;
    a.k = uvqk + 3 * F;
    a.v = uvqk + F;
    a.q_stride = a.k_stride = a.v_stride = 4 * F;
    a.total_q = a.total_kv = p.T;
    a.out = attn;
    a.out_stride = F;
    a.pos_table = p.pos_table;
    a.n_pos = p.n_pos;
    a.time_table = p.time_table;
    a.n_time = p.n_time;
    a.ts = p.ts;
    a.scale = p.scale;
    a.max_q = a.max_kv = p.max_len;
    a.allow_split = false;  // the block's workspace holds no split partials
    a.pdl = kPdl;
    e = attn_sm100_launch(a, nullptr, 0, err_word, stream);
    if (e != cudaSuccess) return e;
    e = launch_kernel(kPdl, ln_gate_kernel, dim3((unsigned)((p.T + 7) / 8)), dim3(256), 0, stream,
                      attn, uvqk, 4 * F, gate, p.T, p.ln_eps);
    if (e != cudaSuccess) return e;
    e = gemm_launch<EPI_RESIDUAL, 128>(gate, F, p.w_o[l], p.d_model, p.x, p.d_model, M, p.d_model, F,
                                  err_word, kPdl, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

namespace {

// Paged attention over one layer's table for the rows described by (q, q_off).
AttnProblem cached_attention(const CachedStepProblem& c, const KvTableDev& t, bool candidates,
                             const __nv_bfloat16* rows, const int64_t* q_off, int64_t total_q,
                             int max_q, __nv_bfloat16* out) {
  const int F = c.H * c.dh;
  AttnProblem a;
  a.B = c.B;
  a.H = c.H;
  a.d = c.dh;
  a.mode = candidates ? 1 : 0;
  a.paged = true;
  a.q_off = q_off;
  a.users = c.users;
  a.page_lists = t.page_lists;
  a.lengths = t.lengths;
  a.max_users = t.max_users;
  a.max_ppu = t.max_ppu;
  a.n_pages = t.n_pages;
  a.pool = t.pool;
  // rows hold [U | V | Q | K] blocks of F columns
  a.q = rows + 2 * F;
  a.k = candidates ? rows + 3 * F : nullptr;
  a.v = candidates ? rows + F : nullptr;
  a.q_stride = a.k_stride = a.v_stride = 4 * F;
  a.total_q = total_q;
  a.out = out;
  a.out_stride = F;
  a.pos_table = c.pos_table;
  a.n_pos = c.n_pos;
  a.scale = c.scale;
  a.max_q = max_q;
  a.max_kv = c.max_cached;
  return a;
}

size_t block_part_bytes(int64_t T, int F) {
  return align256((size_t)T * 4 * F * 2) + align256((size_t)T * F * 2) * 2;
}

}  // namespace

size_t block_cached_workspace_bytes(const CachedStepProblem& p, int num_sms) {
  const int F = p.H * p.dh;
  size_t bytes = block_part_bytes(p.T_new + p.T_cand, F);
  // key-split partials of either attention (they run one after the other)
  size_t split = 0;
  if (p.n_layers > 0 && p.tables) {
    if (p.T_new > 0) {
      const AttnProblem a = cached_attention(p, p.tables[0], false, nullptr, p.new_offsets, p.T_new,
                                             p.max_new, nullptr);
      split = std::max(split, attn_sm100_workspace_bytes(a, num_sms));
    }
    if (p.T_cand > 0) {
      const AttnProblem a = cached_attention(p, p.tables[0], true, nullptr, p.cand_offsets,
                                             p.T_cand, p.max_cand, nullptr);
      split = std::max(split, attn_sm100_workspace_bytes(a, num_sms));
    }
  }
  return bytes + align256(split);
}

cudaError_t block_cached_step_launch(const CachedStepProblem& p, void* workspace, size_t ws_bytes,
                                     int* err_word, cudaStream_t stream) {
  const int F = p.H * p.dh;
  if (p.dh != 128 || F != p.d_model || F != 512) return cudaErrorNotSupported;
  const int64_t T = p.T_new + p.T_cand;
  if (T == 0 || p.n_layers == 0) return cudaSuccess;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  __nv_bfloat16* uvqk = reinterpret_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* attn = reinterpret_cast<__nv_bfloat16*>(ws + align256((size_t)T * 4 * F * 2));
  __nv_bfloat16* gate = reinterpret_cast<__nv_bfloat16*>(ws + align256((size_t)T * 4 * F * 2) +
                                                         align256((size_t)T * F * 2));
  uint8_t* split_ws = ws + block_part_bytes(T, F);
  const size_t split_bytes = ws_bytes > block_part_bytes(T, F) ? ws_bytes - block_part_bytes(T, F) : 0;
  __nv_bfloat16* cand_rows = uvqk + p.T_new * 4 * F;
  const int M = (int)T;
  for (int l = 0; l < p.n_layers; ++l) {
    const KvTableDev& t = p.tables[l];
    // [U | V | Q | K] = SiLU(X W1) for the new and the candidate rows at once
    cudaError_t e = gemm_launch<EPI_SILU, 256>(p.x, p.d_model, p.w_uvqk[l], 4 * F, uvqk, 4 * F, M, 4 * F,
                                          p.d_model, err_word, true, stream);
    if (e != cudaSuccess) return e;
    if (p.T_new > 0) {
      // the new tokens' K, V join this layer's cache, then they attend causally
      // over the cached history and themselves
      e = kv_step_launch(t, p.users, uvqk + 3 * F, uvqk + F, p.new_offsets, p.B, p.max_new, nullptr,
                         nullptr, 0, stream, 4 * F);
      if (e != cudaSuccess) return e;
      const AttnProblem a =
          cached_attention(p, t, false, uvqk, p.new_offsets, p.T_new, p.max_new, attn);
      e = attn_sm100_launch(a, split_ws, split_bytes, err_word, stream);
      if (e != cudaSuccess) return e;
    }
    if (p.T_cand > 0) {
      // candidates see the cached history (new tokens included) and themselves
      const AttnProblem a = cached_attention(p, t, true, cand_rows, p.cand_offsets, p.T_cand,
                                             p.max_cand, attn + p.T_new * F);
      e = attn_sm100_launch(a, split_ws, split_bytes, err_word, stream);
      if (e != cudaSuccess) return e;
    }
    e = launch_dependent(ln_gate_kernel, dim3((unsigned)((T + 7) / 8)), dim3(256), 0, stream, attn,
                         uvqk, 4 * F, gate, T, p.ln_eps);
    if (e != cudaSuccess) return e;
    e = gemm_launch<EPI_RESIDUAL, 128>(gate, F, p.w_o[l], p.d_model, p.x, p.d_model, M, p.d_model, F,
                                  err_word, true, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace hstu
