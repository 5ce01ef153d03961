// Beam-search decode attention over a shared context ("How Generative
// Recommenders Are Redefining RecSys at Scale", section "Semantic ID-GR": long
// request context shared by every beam (ContextKV), a short per-beam decode
// history (BeamKV) and the beams' ancestry (BeamPath)).
//
// Beam j of request b at decode step s (position L_b + s, L_b = cached context
// length) attends to the context tokens 0 .. L_b-1, to the decode tokens of its
// ancestors at steps 0 .. s-1 (positions L_b + t) and to its own token.  HSTU
// attention has no normalisation over keys, so those three key sets add up:
//   * context + own token: the tcgen05 attention kernel in candidate mode, the
//     beams of a request being its candidates (query position offset s), its
//     unscaled fp32 partial sums written to the workspace;
//   * ancestors: beam_path_kernel follows the parent links back to step 0,
//     adds SiLU(q.k + rab) v for each ancestor token to the summed partials,
//     and writes (sum) * scale as bf16 - one rounding, as for any other row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "attn.h"
#include "beam_decode.h"
#include "sm100.cuh"

namespace hstu {

namespace {

constexpr int kD = 128;
constexpr int kBN = 128;

struct BeamParams {
  const int64_t* users;
  const int64_t* lengths;
  int64_t max_users;
  int B;
  const __nv_bfloat16* q;
  const int64_t* beam_offsets;
  int64_t total_beams;
  int H;
  int step;
  const __nv_bfloat16* beam_k;
  const __nv_bfloat16* beam_v;
  const int32_t* beam_parent;
  const float* pos_table;
  int n_pos;
  float scale;
  const float* partial;   // [n_split][T_beam][H][d]
  int n_split, kps;
  __nv_bfloat16* out;
};

__device__ __forceinline__ float silu(float x) { return x / (1.f + __expf(-x)); }

// One CTA per beam row, one warp per head, 4 features per lane.
__global__ void beam_path_kernel(BeamParams P) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t r = blockIdx.x;
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (r >= P.total_beams || h >= P.H) return;
  int lo = 0, hi = P.B;  // request of this row
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (P.beam_offsets[mid] <= r) lo = mid;
    else hi = mid;
  }
  const int b = lo;
  const int64_t base = P.beam_offsets[b];
  const int64_t u = P.users[b];
  const int64_t n_ctx = (u >= 0 && u < P.max_users) ? P.lengths[u] : 0;
  // partial sums of the context + own-token part (candidate layout: ctx tiles + 1)
  const int total = (int)((n_ctx + kBN - 1) / kBN) + 1;
  const int n_valid = min(P.n_split, (total + P.kps - 1) / P.kps);
  const int64_t F = (int64_t)P.H * kD;
  const int f = h * kD + lane * 4;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < n_valid; ++s) {
    const float4 x = *reinterpret_cast<const float4*>(P.partial + ((int64_t)s * P.total_beams + r) * F + f);
    acc[0] += x.x;
    acc[1] += x.y;
    acc[2] += x.z;
    acc[3] += x.w;
  }
  // ancestors at steps s-1 .. 0
  float qv[4];
  {
    const __nv_bfloat162* qp = reinterpret_cast<const __nv_bfloat162*>(P.q + r * F + f);
    const float2 a = __bfloat1622float2(qp[0]), c = __bfloat1622float2(qp[1]);
    qv[0] = a.x; qv[1] = a.y; qv[2] = c.x; qv[3] = c.y;
  }
  int64_t beam = r - base;
  const int64_t nb = P.beam_offsets[b + 1] - base;
  for (int t = P.step - 1; t >= 0; --t) {
    beam = P.beam_parent[(int64_t)(t + 1) * P.total_beams + base + beam];
    if (beam < 0 || beam >= nb) break;  // invalid link: the row keeps what it has
    const int64_t row = (int64_t)t * P.total_beams + base + beam;
    const __nv_bfloat162* kp = reinterpret_cast<const __nv_bfloat162*>(P.beam_k + row * F + f);
    const __nv_bfloat162* vp = reinterpret_cast<const __nv_bfloat162*>(P.beam_v + row * F + f);
    const float2 k0 = __bfloat1622float2(kp[0]), k1 = __bfloat1622float2(kp[1]);
    float dot = qv[0] * k0.x + qv[1] * k0.y + qv[2] * k1.x + qv[3] * k1.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (P.pos_table) {
      const int dist = P.step - t;  // position (L + s) - (L + t)
      dot += P.pos_table[min(31 - __clz(dist + 1), P.n_pos - 1)];
    }
    const float w = silu(dot);
    const float2 v0 = __bfloat1622float2(vp[0]), v1 = __bfloat1622float2(vp[1]);
    acc[0] += w * v0.x;
    acc[1] += w * v0.y;
    acc[2] += w * v1.x;
    acc[3] += w * v1.y;
  }
  __nv_bfloat162* op = reinterpret_cast<__nv_bfloat162*>(P.out + r * F + f);
  op[0] = __floats2bfloat162_rn(acc[0] * P.scale, acc[1] * P.scale);
  op[1] = __floats2bfloat162_rn(acc[2] * P.scale, acc[3] * P.scale);
}

AttnProblem context_problem(const BeamDecodeProblem& p) {
  const KvTableDev& t = p.table;
  AttnProblem a;
  a.B = p.B;
  a.H = t.H;
  a.d = t.d;
  a.mode = 1;  // candidates: the beams
  a.paged = true;
  a.q_off = p.beam_offsets;
  a.users = p.users;
  a.page_lists = t.page_lists;
  a.lengths = t.lengths;
  a.max_users = t.max_users;
  a.max_ppu = t.max_ppu;
  a.n_pages = t.n_pages;
  a.pool = t.pool;
  const int64_t F = (int64_t)t.H * t.d;
  a.q = p.q;
  // the beams' own tokens at this step
  a.k = p.beam_k ? static_cast<const __nv_bfloat16*>(p.beam_k) + (int64_t)p.step * p.total_beams * F
                 : nullptr;
  a.v = p.beam_v ? static_cast<const __nv_bfloat16*>(p.beam_v) + (int64_t)p.step * p.total_beams * F
                 : nullptr;
  a.q_stride = a.k_stride = a.v_stride = a.out_stride = F;
  a.total_q = p.total_beams;
  a.max_q = p.max_beams;
  a.max_kv = p.max_ctx;
  a.pos_table = p.pos_table;
  a.n_pos = p.n_pos;
  a.scale = p.scale;
  a.q_pos_offset = p.step;
  a.partial_only = true;
  return a;
}

}  // namespace

size_t beam_decode_workspace_bytes(const BeamDecodeProblem& p, int num_sms) {
  return attn_sm100_workspace_bytes(context_problem(p), num_sms);
}

cudaError_t beam_decode_launch(const BeamDecodeProblem& p, void* workspace, size_t ws_bytes,
                               int* err_word, cudaStream_t stream) {
  if (p.table.d != kD || p.table.esize != 2 || p.table.H > 32) return cudaErrorNotSupported;
  if (p.total_beams == 0 || p.B == 0) return cudaSuccess;
  const AttnProblem a = context_problem(p);
  cudaError_t e = attn_sm100_launch(a, workspace, ws_bytes, err_word, stream);
  if (e != cudaSuccess) return e;
  BeamParams bp;
  bp.users = p.users;
  bp.lengths = p.table.lengths;
  bp.max_users = p.table.max_users;
  bp.B = p.B;
  bp.q = static_cast<const __nv_bfloat16*>(p.q);
  bp.beam_offsets = p.beam_offsets;
  bp.total_beams = p.total_beams;
  bp.H = p.table.H;
  bp.step = p.step;
  bp.beam_k = static_cast<const __nv_bfloat16*>(p.beam_k);
  bp.beam_v = static_cast<const __nv_bfloat16*>(p.beam_v);
  bp.beam_parent = p.beam_parent;
  bp.pos_table = p.pos_table;
  bp.n_pos = p.n_pos;
  bp.scale = p.scale;
  bp.partial = static_cast<const float*>(workspace);
  attn_sm100_split_plan(a, device_sm_count(), &bp.n_split, &bp.kps);
  bp.out = static_cast<__nv_bfloat16*>(p.out);
  return launch_dependent(beam_path_kernel, dim3((unsigned)p.total_beams), dim3(32 * p.table.H), 0,
                          stream, bp);
}

}  // namespace hstu
