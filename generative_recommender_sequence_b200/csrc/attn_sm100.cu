// HSTU attention forward for B200 (sm_100a): bf16 inputs, head dim 128, fp32
// accumulation in tensor memory.
//
// Computes, per user b, head h and query row i (section "HSTU" of "How
// Generative Recommenders Are Redefining RecSys at Scale": SiLU weighting in
// place of softmax plus a relative attention bias):
//     O[i] = scale * sum_{j in M(i)} SiLU(q_i . k_j + rab(i, j)) v_j
// with the causal-suffix mask (queries are the last n_q of the user's n_k
// tokens, key j visible iff pos_j <= pos_i) or the candidate mask (candidate c
// sees every cached token of its user plus itself).  Keys/values come either
// from token-major jagged tensors or, page by page, from the paged KV table
// (the attention kernel reads the cache directly: "Déploiement de
// recommandeurs génératifs avec NVIDIA Dynamo-Triton et HSTU", section
// "Comment cela fonctionne").
//
// Structure (one persistent CTA per SM, 640 threads):
//   warp 0      TMA producer: Q tile (128 x 128), K ring (2 x 128 x 128), Q double buffer,
//               V ring (2 x 128 x 128), all 128-byte swizzled.  Paged keys are
//               four 32-token page boxes per 128-key tile.
//   warp 1      tcgen05 issuer of S = Q K^T into TMEM (three S/P buffers)
//   warp 3      tcgen05 issuer of O += P V, P read from TMEM (bf16 P written over
//               the start of each warpgroup's S columns)
//   warp 2      stages key timestamps for the time-gap bias (mbarrier ring)
//   warps 4-19  16 "pointwise" warps: read S from TMEM, add the biases, mask,
//               SiLU (via tanh), pack P to bf16 in TMEM, then run the item's
//               epilogue (O * scale -> bf16, or the fp32 partial of a key
//               split).  Paged causal launches split them into two pairs that
//               alternate key tiles (the pair that took an item's last tile runs
//               its epilogue while the other starts the next item); the other
//               launches share every tile among all 16.  Causal launches without
//               key splits stage whole 32 x 32 output boxes in the finished
//               item's Q slot and write them with TMA stores.
// There is no softmax, so there is no running max and no rescaling of O, and
// key splits of one query tile add exactly (the candidate path splits keys).
// Work items (user, head, query tile, split) run longest-first: query tiles
// are visited from the highest tile index down, handed to the CTAs in a snake
// order, or (short contiguous causal batches) by the round-balanced plan.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "attn.h"
#include "sm100.cuh"

namespace hstu {
namespace {

constexpr int BM = 128;            // query rows per tile
constexpr int BN = 128;            // keys per tile
constexpr int HD = 128;            // head dim
constexpr int KST = 2;             // K ring depth
constexpr int QST = 2;             // Q double buffer (next item's Q loads early)
constexpr int VST = 2;             // V ring depth
constexpr int kThreads = 640;      // 20 warps: TMA, MMA, timestamps, spare, 16 pointwise
constexpr int kTileBytes = BM * HD * 2;   // 32 KiB
constexpr int kHalfBytes = kTileBytes / 2;  // one 64-column half: 128 rows x 128 B
constexpr int kMaxUsers = 1024;   // per launch; larger batches are split on the host
constexpr int kMaxRab = 256;

constexpr uint32_t TM_O = 0;      // O accumulator, 128 fp32 columns
constexpr uint32_t TM_SP = 128;    // three S/P buffers of 128 columns each
constexpr int NSP = 3;
// P (bf16 pairs) overwrites the first half of each pointwise warp's own S
// columns.  16 warps per tile (32 columns each): keys [32 c, 32 c + 32) ->
// columns [32 c, 32 c + 16), so MMA k-step kk (16 keys) starts at column
// 32 (kk / 2) + 8 (kk % 2).  Two pairs of warpgroups (64 columns per warp):
// keys [64 c, 64 c + 64) -> columns [64 c, 64 c + 32), k-step kk at
// 64 (kk / 4) + 8 (kk % 4).
template <bool PW2>
__host__ __device__ constexpr uint32_t p_col(int kk) {
  return PW2 ? 64 * (kk >> 2) + 8 * (kk & 3) : 32 * (kk >> 1) + 8 * (kk & 1);
}

constexpr uint32_t kIdescQK = idesc_bf16_f32(BM, BN, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, HD, true);

constexpr int NTS = 4;              // key-timestamp ring depth
constexpr int kPagesStaged = 512;  // page ids staged per item (128 key tiles)
// Round-balanced schedule of the contiguous causal launches (plan_rounds)
// items per CTA it plans: short-sequence batches (a few hundred items, 3
// rounds) gain from it, long ones (17 rounds, users of up to 128 query tiles)
// ran 6.5% slower than in the snake order, which they keep
constexpr int kRsMaxRounds = 8;
constexpr int kRsMaxLevels = 128;  // query tiles per user it can order
constexpr int kRsMaxCtas = 160;    // grid size it can rank
constexpr int kRsItemCost = 2;     // fixed cost of an item, in key tiles (fill + epilogue)
constexpr int kRrowQuarters = 64;   // position-bias row per pointwise warp: 32 columns + 31
constexpr int kRrowPairs = 96;      // same for the two-pair layout: 64 columns + 31
constexpr int RROW = kRrowPairs;

// Key timestamps of one key tile, staged by warp 2: exact float offsets from
// the user's first timestamp (when |offset| < 2^23 for every key), plus the
// raw int64 values for the exact integer path.
struct TsSlot {
  float f[BN];
  long long i[BN];
  int exact;     // every offset fits 23 bits (the float path is exact)
  int sorted;    // key timestamps non-decreasing over the valid keys
  int pad[2];
};

struct __align__(1024) Smem {
  uint8_t q[QST][kTileBytes];
  uint8_t k[KST][kTileBytes];
  uint8_t v[VST][kTileBytes];
  float rrow[16][RROW];        // per pointwise warp: pos bias by (row - col), its column half
  float pos_ext[kMaxRab];      // tables with the clamp at n-1 baked in
  float time_ext[kMaxRab];
  TsSlot ts[NTS];
  int m_q[kMaxUsers + 1];      // per user: first query row
  int m_kv[kMaxUsers];         // per user: first key row (contiguous) or user id (paged)
  int m_nk[kMaxUsers];         // per user: number of keys (sequence / cached length)
  TsSlot qts[2];               // query timestamps of the current / next item
  int pages[kPagesStaged];     // producer: page ids of the current item's key tiles
  uint64_t q_full[QST], q_empty[QST];
  // q_done[s]: the 16 pointwise warps have finished with Q slot s after its
  // item (output boxes staged there were read by their TMA stores)
  uint64_t q_done[QST];
  uint64_t k_full[KST], k_empty[KST];
  uint64_t v_full[VST], v_empty[VST];
  // s_full: one per buffer (16-warp layout) or per (pair, buffer) = tile mod 6
  // (two-pair layout), so each waiter sees every phase of its barriers in order;
  // p_full / sp_empty have one in-order waiter
  uint64_t s_full[2 * NSP], p_full[NSP], sp_empty[NSP];
  uint64_t o_full[2], o_empty;  // o_full[1]: second pair of the two-pair layout
  uint64_t ts_full[NTS], ts_empty[NTS];
  uint64_t qts_full[2], qts_empty[2];
  uint64_t mma_done, mma_done2;
  uint32_t tmem_base;
  int abort_flag;
  // balanced key splits: this CTA's one item (valid, user, query tile, head,
  // key-tile range), derived by plan_balanced
  int bal_ok, bal_b, bal_m, bal_h, bal_t0, bal_t1;
  // round-balanced schedule (contiguous causal launches, plan_rounds): the
  // number of rounds (0: the snake order applies), this CTA's item of each
  // round, and the planner's per-CTA loads and per-level first item indices
  int rs_rounds, rs_levels;
  int rs_b[kRsMaxRounds], rs_m[kRsMaxRounds], rs_rem[kRsMaxRounds];
  int rs_load[kRsMaxCtas];
  int rs_first[kRsMaxLevels + 1];
};

struct KParams {
  int B, H, mode, n_split, kps;
  // balanced key splits (the BAL kernels): per-user split counts chosen on
  // the device, one item per CTA; partial sums of item t at
  // partial + t * BM * HD, and the item offsets per user (int32 [B + 1])
  // written to plan for the reduce
  int* plan;
  const int64_t* q_off;
  const int64_t* kv_off;
  const int64_t* users;
  const int32_t* page_lists;
  const int64_t* lengths;
  int64_t max_users;
  int max_ppu;
  int64_t n_pages;
  const float* pos_table;
  int n_pos;
  const float* time_table;
  int n_time;
  const int64_t* ts;
  int q_pos_offset;
  float scale;
  __nv_bfloat16* out;
  int64_t out_stride;
  float* partial;
  int64_t total_q;
  int* err;
  int part_v8;   // partial buffer 32-byte aligned: store whole 32-byte sectors
};

// ------------------------------------------------------------ scheduling
// Query row blocks of user b (bm rows each) from the cached query offsets.
__device__ __forceinline__ int q_tiles(const int* mq, int b, int bm) {
  return (mq[b + 1] - mq[b] + bm - 1) / bm;
}

__device__ __forceinline__ int count_users_above(const int* qt, int B, int lvl, int bm, int lane) {
  int c = 0;
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int b = b0 + lane;
    const bool p = b < B && q_tiles(qt, b, bm) > lvl;
    c += __popc(__ballot_sync(0xffffffffu, p));
  }
  return c;
}

__device__ __forceinline__ int nth_user_above(const int* qt, int B, int lvl, int bm, int n, int lane) {
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int b = b0 + lane;
    const bool p = b < B && q_tiles(qt, b, bm) > lvl;
    unsigned m = __ballot_sync(0xffffffffu, p);
    const int c = __popc(m);
    if (n < c) {
      for (int i = 0; i < n; ++i) m &= m - 1;
      return b0 + __ffs(m) - 1;
    }
    n -= c;
  }
  return -1;
}

// Item order: query-tile level from the highest down; within a level, users in
// order, then heads, then key splits.  Warp-collective (all lanes agree).
template <int bm>
struct Sched {
  int lvl;
  long long base, cnt;
  int B, HS;
  __device__ void init(const int* qt, int B_, int HS_, int lane) {
    B = B_;
    HS = HS_;
    int mx = 0;
    for (int b = lane; b < B; b += 32) mx = max(mx, q_tiles(qt, b, bm));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    lvl = mx - 1;
    base = 0;
    cnt = lvl >= 0 ? (long long)count_users_above(qt, B, lvl, bm, lane) * HS : 0;
  }
  __device__ bool item(long long t, const int* qt, int lane, int& b, int& m, int& rem) {
    while (lvl >= 0 && t >= base + cnt) {
      base += cnt;
      --lvl;
      cnt = lvl >= 0 ? (long long)count_users_above(qt, B, lvl, bm, lane) * HS : 0;
    }
    if (lvl < 0) return false;
    const long long r = t - base;
    rem = (int)(r % HS);
    b = nth_user_above(qt, B, lvl, bm, (int)(r / HS), lane);
    m = lvl;
    return b >= 0;
  }
};

// Items are sorted longest first; round k hands them to the CTAs in forward
// order for even k and in reverse order for odd k (a snake), so the CTA that
// got the longest item of a round gets the shortest of the next.
__device__ __forceinline__ long long snake_item(long long rnd) {
  const long long G = gridDim.x;
  const long long me = blockIdx.x;
  return rnd * G + ((rnd & 1) ? (G - 1 - me) : me);
}

struct Item {
  int b, h, m, s;
  int64_t q_row0;   // global query row of tile row 0
  int nvalid;       // valid query rows in the tile
  int64_t p0;       // position of query row 0
  int64_t n_k;      // keys of the user (cached length / sequence length)
  int64_t kv_row0;  // contiguous: global row of key position 0
  int64_t user;     // paged: user id
  int n_main;       // tiles from the main key source; tile n_main is the candidate tile
  int t0, t1;       // this item's tile range
};

// Item m of user b covers query rows [BM m, BM m + BM).
template <bool PAGED, bool CAND, bool BAL>
__device__ __forceinline__ Item make_item(const KParams& P, const Smem& sm, int b, int m, int rem) {
  Item it;
  it.b = b;
  it.m = m;
  it.h = rem / P.n_split;
  it.s = rem % P.n_split;
  const int64_t bm = BM;
  const int64_t qs = sm.m_q[b], nq = (int64_t)sm.m_q[b + 1] - qs;
  const int64_t blk0 = bm * m;                           // first row of the block
  const int64_t r0 = blk0;
  it.q_row0 = qs + r0;
  it.nvalid = (int)max64(0, min64(BM, nq - r0));
  it.n_k = sm.m_nk[b];
  if (PAGED) {
    it.user = sm.m_kv[b];
    it.kv_row0 = 0;
  } else {
    it.user = 0;
    it.kv_row0 = sm.m_kv[b];
  }
  int total;
  if (CAND) {
    it.p0 = it.n_k + P.q_pos_offset;
    it.n_main = (int)((it.n_k + BN - 1) / BN);
    total = it.n_main + 1;
  } else {
    it.p0 = it.n_k - nq + r0;
    // position of the block's last valid row
    const int64_t last = it.n_k - nq + blk0 + min64(bm, nq - blk0) - 1;
    it.n_main = last >= 0 ? (int)(last / BN) + 1 : 0;
    total = it.n_main;
  }
  if (BAL) {
    it.s = blockIdx.x;  // the item id: where its partial sums go
    it.t0 = sm.bal_t0;
    it.t1 = min(total, sm.bal_t1);
  } else if (P.n_split > 1) {
    it.t0 = it.s * P.kps;
    it.t1 = min(total, it.t0 + P.kps);
  } else {
    it.t0 = 0;
    it.t1 = total;
  }
  return it;
}

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Key tiles of one query tile of user b (the same for every query tile of a
// candidate user; causal runs in this mode have at most one query tile) and
// its number of query tiles.
template <bool CAND>
__device__ __forceinline__ int plan_tiles(const Smem& sm, int b, int& qt) {
  const int nq = sm.m_q[b + 1] - sm.m_q[b];
  const int n_k = sm.m_nk[b];
  qt = nq > 0 ? (nq + BM - 1) / BM : 0;
  if (qt == 0) return 0;
  if (CAND) return (n_k + BN - 1) / BN + 1;
  const int last = n_k - nq + min(BM, nq) - 1;
  return last >= 0 ? last / BN + 1 : 0;
}

// Runs a user's key tiles are cut into for a target run length (round to
// nearest, at least one run, never more runs than tiles).
__device__ __forceinline__ int plan_runs(int tiles, int target) {
  if (tiles <= 0) return 0;
  return max(1, min(tiles, (tiles + target / 2) / target));
}

// Balanced key splits (candidate scoring and short causal runs, when there are
// fewer (user, head, query tile) items than CTAs).  Every CTA derives the same
// plan from the key counts: the target run length is the smallest that is at
// least ceil(total tiles / CTAs) and lets every user's runs fit one wave, user
// b's tiles are cut into plan_runs(tiles_b, target) near-equal runs (the
// first tiles_b mod runs of them one tile longer), and items are numbered user
// by user, then query tile, head and run.  This CTA takes item blockIdx.x; CTA
// 0 also publishes each user's first item for the reduce.  Called by warp 0
// only; 32-bit arithmetic throughout (this runs before any copy is issued, so
// its length is the launch's latency; the host admits this mode only with at
// most num_sms / 2 (user, head, query tile) items).
template <bool CAND>
__device__ void plan_balanced(const KParams& P, Smem& sm, int lane) {
  const int G = gridDim.x;
  int W = 0;
  for (int b = lane; b < P.B; b += 32) {
    int qt = 0;
    const int t = plan_tiles<CAND>(sm, b, qt);
    W += qt * P.H * t;
  }
  W = warp_sum_i(W);
  int target = max(2, (W + G - 1) / G);
  for (int iter = 0;; ++iter) {
    int items = 0;
    for (int b = lane; b < P.B; b += 32) {
      int qt = 0;
      const int t = plan_tiles<CAND>(sm, b, qt);
      items += qt * P.H * plan_runs(t, target);
    }
    items = warp_sum_i(items);
    if (items <= G) break;
    // one run per user always fits (the host chooses this mode only then)
    target = iter < 64 ? target + 1 : (1 << 30);
  }
  // this CTA's item: exclusive prefix of the users' item counts
  const int me = blockIdx.x;
  int base = 0;
  if (lane == 0) sm.bal_ok = 0;
  __syncwarp();
  for (int b0 = 0; b0 < P.B; b0 += 32) {
    const int b = b0 + lane;
    int qt = 0;
    const int t = b < P.B ? plan_tiles<CAND>(sm, b, qt) : 0;
    const int ns = plan_runs(t, target);
    const int cnt = qt * P.H * ns;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int first = base + incl - cnt;
    if (blockIdx.x == 0 && b < P.B) P.plan[b] = first;
    if (b < P.B && cnt > 0 && me >= first && me < first + cnt) {
      const int r = me - first;
      const int per = P.H * ns;
      const int sidx = r % ns;
      const int q = t / ns, rr = t % ns;   // runs of q + 1 tiles, then of q
      sm.bal_b = b;
      sm.bal_m = r / per;
      sm.bal_h = (r % per) / ns;
      sm.bal_t0 = sidx * q + min(sidx, rr);
      sm.bal_t1 = sm.bal_t0 + q + (sidx < rr ? 1 : 0);
      sm.bal_ok = 1;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (blockIdx.x == 0 && lane == 0) P.plan[P.B] = base;
}

// Round-balanced schedule of a contiguous causal launch, planned identically
// by every CTA (all threads call it).  The item list is the longest-first one
// of Sched (query-tile level descending, then users, then heads); item t of
// level m costs m + 1 key tiles plus kRsItemCost.  Round r hands items
// [G r, G r + G) out in that order to the CTAs sorted by the load they already
// carry (ties by CTA index), so the longest item of a round goes to the least
// loaded CTA.  On jagged batches of a few hundred items of 1..26 tiles (8
// users of 256..4096 tokens, 4 heads) this bounds the busiest CTA close to
// the longest-processing-time rule, where the snake order leaves it 13-15%
// above.  Batches with more rounds (long sequences: there the snake order
// measured faster), levels or CTAs than the tables hold keep the snake order
// (sm.rs_rounds = 0, items decoded one at a time by decode_item).
__device__ __noinline__ void plan_rounds(int B, int H, int n_split, Smem& sm, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
  const int HS = H * n_split;
  if (warp == 0) {
    int mx = 0;
    for (int b = lane; b < B; b += 32) mx = max(mx, q_tiles(sm.m_q, b, BM));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    // rs_first[k]: first item index of level mx - 1 - k (also what decode_item
    // searches when the rounds do not fit)
    const bool levels_ok = mx >= 1 && mx <= kRsMaxLevels;
    long long n = 0;
    if (levels_ok) {
      for (int k = 0; k < mx; ++k) {
        if (lane == 0) sm.rs_first[k] = (int)n;
        n += (long long)count_users_above(sm.m_q, B, mx - 1 - k, BM, lane) * HS;
      }
      if (lane == 0) sm.rs_first[mx] = (int)n;
    }
    const long long rounds = (n + G - 1) / G;
    const bool ok = levels_ok && G <= kRsMaxCtas && n > 0 && rounds <= kRsMaxRounds;
    if (lane == 0) {
      sm.rs_rounds = ok ? (int)rounds : 0;
      sm.rs_levels = mx;
    }
  }
  for (int c = tid; c < kRsMaxCtas; c += kThreads) sm.rs_load[c] = 0;
  __syncthreads();
  const int R = sm.rs_rounds;
  if (R == 0) return;
  const int mx = sm.rs_levels;  // rs_first[mx] is the item count
  const int n_items = sm.rs_first[mx];
  // four threads rank each CTA c: thread (c, part) compares against CTAs
  // part, part + 4, ...; the counts are summed over the four lanes
  const int c = tid >> 2, part = tid & 3;
  for (int r = 0; r < R; ++r) {
    int rank = 0;
    if (c < G) {
      const int key = sm.rs_load[c] * 256 + c;
      for (int c2 = part; c2 < G; c2 += 4) rank += (sm.rs_load[c2] * 256 + c2) < key;
    }
    rank += __shfl_xor_sync(0xffffffffu, rank, 1);
    rank += __shfl_xor_sync(0xffffffffu, rank, 2);
    __syncthreads();  // every rank is taken from the loads before this round
    if (c < G && part == 0) {
      const int t = r * G + rank;
      int item = -1;
      if (t < n_items) {
        int k = 0;  // level index of item t: rs_first[k] <= t < rs_first[k + 1]
        while (sm.rs_first[k + 1] <= t) ++k;
        sm.rs_load[c] += (mx - k) + kRsItemCost;
        item = t;
      }
      if (c == (int)blockIdx.x) sm.rs_b[r] = item;
    }
    __syncthreads();
  }
  // decode this CTA's items: level, user and head of item t
  if (warp == 0) {
    for (int r = 0; r < R; ++r) {
      const int t = sm.rs_b[r];
      int b = -1, m = 0, rem = 0;
      if (t >= 0) {
        int k = 0;
        while (sm.rs_first[k + 1] <= t) ++k;
        m = mx - 1 - k;
        const int ri = t - sm.rs_first[k];
        rem = ri % HS;
        b = nth_user_above(sm.m_q, B, m, BM, ri / HS, lane);
      }
      __syncwarp();
      if (lane == 0) {
        sm.rs_b[r] = b;
        sm.rs_m[r] = m;
        sm.rs_rem[r] = rem;
      }
      __syncwarp();
    }
  }
}

// Item t of the longest-first list, decoded without state (warp-collective).
// The round-balanced launches use it when their batch does not fit
// plan_rounds' round tables: with at most kRsMaxLevels levels the per-level
// first items are in rs_first (binary search), otherwise the levels are
// walked from the top.
__device__ __noinline__ bool decode_item(int B, int HS, const Smem& sm, long long t, int lane, int& b,
                                         int& m, int& rem) {
  const int mx = sm.rs_levels;
  if (mx >= 1 && mx <= kRsMaxLevels) {
    if (t >= sm.rs_first[mx]) return false;
    int lo = 0, hi = mx - 1;  // largest k with rs_first[k] <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sm.rs_first[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int r = (int)(t - sm.rs_first[lo]);
    rem = r % HS;
    m = mx - 1 - lo;
    b = nth_user_above(sm.m_q, B, m, BM, r / HS, lane);
    return b >= 0;
  }
  long long base = 0;
  for (int lvl = mx - 1; lvl >= 0; --lvl) {
    const long long cnt = (long long)count_users_above(sm.m_q, B, lvl, BM, lane) * HS;
    if (t < base + cnt) {
      const long long r = t - base;
      rem = (int)(r % HS);
      b = nth_user_above(sm.m_q, B, lvl, BM, (int)(r / HS), lane);
      m = lvl;
      return b >= 0;
    }
    base += cnt;
  }
  return false;
}

// The rnd-th item of this CTA: one fixed item with balanced splits (BAL);
// the round-balanced schedule of plan_rounds (RS); otherwise the snake order
// over the longest-first item list.
template <bool BAL, bool RS>
__device__ __forceinline__ bool next_item(const KParams& P, const Smem& sm, Sched<BM>& sc,
                                          long long rnd, int lane, int& b, int& m, int& rem) {
  if (BAL) {
    if (rnd > 0 || !sm.bal_ok) return false;
    b = sm.bal_b;
    m = sm.bal_m;
    rem = sm.bal_h;
    return true;
  }
  if (RS) {
    if (sm.rs_rounds > 0) {
      if (rnd >= sm.rs_rounds || sm.rs_b[rnd] < 0) return false;
      b = sm.rs_b[rnd];
      m = sm.rs_m[rnd];
      rem = sm.rs_rem[rnd];
      return true;
    }
    return decode_item(P.B, P.H * P.n_split, sm, snake_item(rnd), lane, b, m, rem);
  }
  return sc.item(snake_item(rnd), sm.m_q, lane, b, m, rem);
}

__device__ __forceinline__ void record_timeout(const KParams& P, Smem& sm) {
  atomicExch(P.err, DEV_ERR_TIMEOUT);
  *(volatile int*)&sm.abort_flag = 1;
}

// One 32-column chunk of one score row: add the biases, mask, SiLU, pack to
// bf16 pairs.  MASK: 0 every key visible, 1 causal (c <= qrel), 2 c < kend,
// 3 only the candidate's own key (c == r).  TIME: 0 none, 1 float-exponent
// bucket (exact offsets), 2 int64 bucket.  rlc[-j] is the position bias of
// column cb + j; tx is the time table with its clamp baked in (256 entries).
template <int MASK, int TIME, int W = 16>
__device__ __forceinline__ void pw_chunk(const uint32_t (&sv)[W], uint32_t (&pk)[W / 2], const int cb,
                                         const float* __restrict__ rlc, const int qrel,
                                         const int kend, const int r, const float* ktf,
                                         const long long* kti, const float tq1,
                                         const long long tqi, const float* tx,
                                         const float self_rab) {
#pragma unroll
  for (int j = 0; j < W; j += 4) {
    float4 kt4;
    if (TIME == 1) kt4 = *reinterpret_cast<const float4*>(ktf + cb + j);
    float pv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = cb + j + e;
      float x = __uint_as_float(sv[j + e]);
      x += (MASK == 3) ? self_rab : rlc[-(j + e)];
      if (TIME == 1) {
        const float kt = e == 0 ? kt4.x : (e == 1 ? kt4.y : (e == 2 ? kt4.z : kt4.w));
        const float d1 = fmaxf(tq1 - kt, 1.0f);
        x += tx[(__float_as_uint(d1) >> 23) - 127];
      } else if (TIME == 2) {
        long long dt = tqi - kti[c];
        dt = dt < 0 ? 0 : dt;
        x += tx[63 - __clzll(dt + 1)];
      }
      const float h = 0.5f * x;
      float y = fmaf(h, tanh_approx(h), h);
      if (MASK == 1) y = (c <= qrel) ? y : 0.f;
      if (MASK == 2) y = (c < kend) ? y : 0.f;
      if (MASK == 3) y = (c == r) ? y : 0.f;
      pv[e] = y;
    }
    pk[j >> 1] = pack_bf16x2(pv[0], pv[1]);
    pk[(j >> 1) + 1] = pack_bf16x2(pv[2], pv[3]);
  }
}

// SiLU of a 16-column chunk whose bias is one constant per row: with
// h = (s + c) / 2, SiLU(s + c) = h + h tanh(h); hrow = c / 2.
__device__ __forceinline__ void silu_rowconst(const uint32_t (&sv)[16], uint32_t (&pk)[8],
                                              const float hrow) {
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    const float h0 = fmaf(0.5f, __uint_as_float(sv[j]), hrow);
    const float h1 = fmaf(0.5f, __uint_as_float(sv[j + 1]), hrow);
    pk[j >> 1] = pack_bf16x2(fmaf(h0, tanh_approx(h0), h0), fmaf(h1, tanh_approx(h1), h1));
  }
}

// One 16-column chunk off the constant-row path: picks the mask class of the
// chunk (warp-uniform) and the bias form, then runs the matching pw_chunk.
// tmode: 0 no time bias, 1 float-exponent buckets, 2 integer buckets.
template <bool CAND>
__device__ __forceinline__ void pw_chunk_any(const uint32_t (&sv)[16], uint32_t (&pk)[8],
                                             const int cb, const bool cand_tile, const int sub,
                                             const int qrel0, const int kend, const int tmode,
                                             const float* rlc, const int qrel, const int r,
                                             const TsSlot& ts, const float tq1,
                                             const long long tq_i, const float* tx,
                                             const float self_rab) {
  int cls;  // 0 visible, 1 per-element, 2 none visible
  int mk;   // per-element mask kind
  if (CAND) {
    if (cand_tile) {
      cls = (cb >> 5) == sub ? 1 : 2;
      mk = 3;
    } else {
      cls = (cb + 15 < kend) ? 0 : (cb >= kend ? 2 : 1);
      mk = 2;
    }
  } else {
    cls = (cb + 15 <= qrel0) ? 0 : (cb > qrel0 + 31 ? 2 : 1);
    mk = 1;
  }
  if (cls == 2) {
#pragma unroll
    for (int j = 0; j < 8; ++j) pk[j] = 0u;
  } else if (!CAND && tmode == 1) {
    if (cls == 0)
      pw_chunk<0, 1>(sv, pk, cb, rlc, qrel, kend, r, ts.f, ts.i, tq1, tq_i, tx, self_rab);
    else
      pw_chunk<1, 1>(sv, pk, cb, rlc, qrel, kend, r, ts.f, ts.i, tq1, tq_i, tx, self_rab);
  } else if (!CAND && tmode == 2) {
    if (cls == 0)
      pw_chunk<0, 2>(sv, pk, cb, rlc, qrel, kend, r, ts.f, ts.i, tq1, tq_i, tx, self_rab);
    else
      pw_chunk<1, 2>(sv, pk, cb, rlc, qrel, kend, r, ts.f, ts.i, tq1, tq_i, tx, self_rab);
  } else if (cls == 0) {
    pw_chunk<0, 0>(sv, pk, cb, rlc, qrel, kend, r, nullptr, nullptr, 0.f, 0, nullptr, self_rab);
  } else if (mk == 1) {
    pw_chunk<1, 0>(sv, pk, cb, rlc, qrel, kend, r, nullptr, nullptr, 0.f, 0, nullptr, self_rab);
  } else if (mk == 2) {
    pw_chunk<2, 0>(sv, pk, cb, rlc, qrel, kend, r, nullptr, nullptr, 0.f, 0, nullptr, self_rab);
  } else {
    pw_chunk<3, 0>(sv, pk, cb, rlc, qrel, kend, r, nullptr, nullptr, 0.f, 0, nullptr, self_rab);
  }
}

// ------------------------------------------------------------ the kernel
// BAL: balanced key splits (one item per CTA, compact partial blocks); only
// paged launches split keys.
template <bool PAGED, bool CAND, bool PW2, bool BAL>
__global__ void __launch_bounds__(kThreads, 1)
    hstu_attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const __grid_constant__ CUtensorMap tm_kc,
                           const __grid_constant__ CUtensorMap tm_vc,
                           const __grid_constant__ CUtensorMap tm_out, const KParams P) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~uintptr_t(1023));
  const int tid = threadIdx.x;
  // contiguous causal launches take the round-balanced schedule (plan_rounds)
  constexpr bool RS = !PAGED && !CAND && !BAL;
  // Contiguous and paged causal launches write their bf16 output through TMA
  // stores staged in the finished item's Q slot (16-warp and two-pair
  // layouts respectively)
  constexpr bool OST = RS;
  constexpr bool OST2 = PW2 && !CAND && !BAL;
  const int warp = tid >> 5, lane = tid & 31;
  // dependent launch: the next kernel may start being scheduled.  Barrier
  // initialisation, the descriptor prefetch and the TMEM allocation touch no
  // global memory, so they overlap the previous kernel's tail; every global
  // read comes after the wait for that kernel (which may have written the KV
  // table or this kernel's inputs).
  pdl_launch_dependents();
  if (tid == 0) {
    sm.abort_flag = 0;
    for (int i = 0; i < QST; ++i) {
      mbar_init(smem_u32(&sm.q_full[i]), 1);
      mbar_init(smem_u32(&sm.q_empty[i]), 1);
      mbar_init(smem_u32(&sm.q_done[i]), 16);
    }
    for (int i = 0; i < KST; ++i) {
      mbar_init(smem_u32(&sm.k_full[i]), 1);
      mbar_init(smem_u32(&sm.k_empty[i]), 1);
    }
    for (int i = 0; i < VST; ++i) {
      mbar_init(smem_u32(&sm.v_full[i]), 1);
      mbar_init(smem_u32(&sm.v_empty[i]), 1);
    }
    // P written / O drained: the warps that handle a tile (16, or one pair of
    // 8 in the two-pair layout)
    constexpr uint32_t kTileWarps = PW2 ? 8 : 16;
    for (int i = 0; i < 2 * NSP; ++i) mbar_init(smem_u32(&sm.s_full[i]), 1);
    for (int i = 0; i < NSP; ++i) {
      mbar_init(smem_u32(&sm.p_full[i]), kTileWarps);
      mbar_init(smem_u32(&sm.sp_empty[i]), 1);
    }
    mbar_init(smem_u32(&sm.o_full[0]), 1);
    mbar_init(smem_u32(&sm.o_full[1]), 1);
    mbar_init(smem_u32(&sm.o_empty), kTileWarps);
    for (int i = 0; i < NTS; ++i) {
      mbar_init(smem_u32(&sm.ts_full[i]), 1);
      mbar_init(smem_u32(&sm.ts_empty[i]), PW2 ? 8 : 16);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.qts_full[i]), 1);
      mbar_init(smem_u32(&sm.qts_empty[i]), 16);
    }
    mbar_init(smem_u32(&sm.mma_done), 1);
    mbar_init(smem_u32(&sm.mma_done2), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    if (CAND) {
      tma_prefetch_desc(&tm_kc);
      tma_prefetch_desc(&tm_vc);
    }
    if (OST || OST2) tma_prefetch_desc(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  pdl_wait();

  // ---- setup
  for (int b = tid; b <= P.B; b += kThreads) {
    sm.m_q[b] = (int)P.q_off[b];
    if (b == P.B) continue;
    if (PAGED) {
      // an out-of-range user id has no cached tokens (and no page list is read)
      const int64_t u = P.users[b];
      const bool known = u >= 0 && u < P.max_users;
      if (known) {
        // the producer reads this user's page ids once the items are known:
        // start them towards L2 now, beside the length load
        const int32_t* pl = P.page_lists + u * (int64_t)P.max_ppu;
        const int n = min(P.max_ppu, kPagesStaged);
        for (int i = 0; i < n; i += 32) prefetch_l2(pl + i);
      }
      sm.m_kv[b] = known ? (int)u : 0;
      sm.m_nk[b] = known ? (int)P.lengths[u] : 0;
    } else {
      sm.m_kv[b] = (int)P.kv_off[b];
      sm.m_nk[b] = (int)(P.kv_off[b + 1] - P.kv_off[b]);
    }
  }
  for (int i = tid; i < kMaxRab; i += kThreads) {
    sm.pos_ext[i] = P.pos_table ? P.pos_table[min(i, P.n_pos - 1)] : 0.f;
    sm.time_ext[i] = P.time_table ? P.time_table[min(i, P.n_time - 1)] : 0.f;
  }
  __syncthreads();
  if (RS) plan_rounds(P.B, P.H, P.n_split, sm, tid);
  if (BAL && warp == 0) plan_balanced<CAND>(P, sm, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int HS = P.H * P.n_split;

  if (warp == 0) {
    // =============================================== TMA producer
    Sched<BM> sc;
    if (!BAL && !RS) sc.init(sm.m_q, P.B, HS, lane);  // one fixed item per CTA otherwise
    uint32_t kc = 0, vc = 0, qi = 0;
    bool ok = true;
    for (long long rnd = 0;; ++rnd) {
      int b, m, rem;
      if (!next_item<BAL, RS>(P, sm, sc, rnd, lane, b, m, rem)) break;
      const Item it = make_item<PAGED, CAND, BAL>(P, sm, b, m, rem);
      if (it.t0 >= it.t1) continue;
      if (lane == 0) {
        const uint32_t qs = qi % QST;
        ok = mbar_wait(smem_u32(&sm.q_empty[qs]), ((qi / QST) & 1) ^ 1);
        // the slot also holds the output boxes of the item two before
        if ((OST || OST2) && ok && qi >= QST)
          ok = mbar_wait(smem_u32(&sm.q_done[qs]), ((qi / QST) - 1) & 1);
        if (ok) {
          const uint32_t bar = smem_u32(&sm.q_full[qs]);
          mbar_arrive_expect_tx(bar, kTileBytes);
          tma_load_3d(smem_u32(sm.q[qs]), &tm_q, bar, 0, it.h, (int)it.q_row0);
          tma_load_3d(smem_u32(sm.q[qs]) + kHalfBytes, &tm_q, bar, 64, it.h, (int)it.q_row0);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      ++qi;
      if (PAGED) {
        // page ids of this item's key tiles, staged once (coalesced) instead of
        // one dependent global load per tile
        const int32_t* plist = P.page_lists + it.user * (int64_t)P.max_ppu;
        const int first = it.t0 * 4;
        const int cnt = min((it.t1 - it.t0) * 4, kPagesStaged);
        __syncwarp();
        for (int i = lane; i < cnt; i += 32) {
          const int idx = first + i;
          sm.pages[i] = idx < P.max_ppu ? plist[idx] : -1;
        }
        __syncwarp();
      }
      // Issue order K0, K1, V0, K2, V1, ... keeps K one tile ahead of V.  Lane 0
      // waits for the slot and posts the byte count; the tile's boxes (two
      // 64-column halves, times four pages when paged) are then issued by one
      // lane each so that the per-copy issue cost is paid in parallel.
      const int nt = it.t1 - it.t0;
      for (int i = 0; i <= nt && ok; ++i) {
        for (int which = 0; which < 2; ++which) {
          // which == 0: K of tile i ; which == 1: V of tile i-1
          const int ti = which == 0 ? i : i - 1;
          if (ti < 0 || ti >= nt) continue;
          const int tile = it.t0 + ti;
          const uint32_t c = which == 0 ? kc : vc;
          const uint32_t slot = which == 0 ? c % KST : c % VST;
          const uint32_t par = (which == 0 ? (c / KST) & 1 : (c / VST) & 1) ^ 1;
          const uint32_t bar = smem_u32(which == 0 ? &sm.k_full[slot] : &sm.v_full[slot]);
          const uint32_t dst = smem_u32(which == 0 ? sm.k[slot] : sm.v[slot]);
          if (lane == 0) {
            ok = mbar_wait(smem_u32(which == 0 ? &sm.k_empty[slot] : &sm.v_empty[slot]), par);
            if (ok) mbar_arrive_expect_tx(bar, kTileBytes);
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          if (which == 0) ++kc; else ++vc;
          const int half = lane & 1;
          if (CAND && tile == it.n_main) {
            if (lane < 2)
              tma_load_3d(dst + half * kHalfBytes, which == 0 ? &tm_kc : &tm_vc, bar, half * 64,
                          it.h, (int)it.q_row0);
          } else if (PAGED) {
            if (lane < 8) {
              const int pg = lane >> 1;
              const int idx = tile * 4 + pg;
              const int si = (tile - it.t0) * 4 + pg;
              const int32_t* plist = P.page_lists + it.user * (int64_t)P.max_ppu;
              int64_t page = si < kPagesStaged ? (int64_t)sm.pages[si]
                                               : (idx < P.max_ppu ? (int64_t)plist[idx] : -1);
              if (page < 0 || page >= P.n_pages) page = P.n_pages;  // the zero page
              const int row = (int)(((page * 2 + which) * P.H + it.h) * 32);
              tma_load_2d(dst + half * kHalfBytes + pg * 4096, &tm_k, bar, half * 64, row);
            }
          } else if (lane < 2) {
            const int row = (int)(it.kv_row0 + (int64_t)tile * BN);
            tma_load_3d(dst + half * kHalfBytes, which == 0 ? &tm_k : &tm_v, bar, half * 64, it.h,
                        row);
          }
        }
      }
      if (!ok) break;
    }
    if (!ok && lane == 0) {
      record_timeout(P, sm);
      // let copies already in flight land before the CTA can exit
      for (uint32_t i = 0; i < KST && i < kc; ++i) {
        const uint32_t c = kc - 1 - i;
        mbar_wait(smem_u32(&sm.k_full[c % KST]), (c / KST) & 1);
      }
      for (uint32_t i = 0; i < VST && i < vc; ++i) {
        const uint32_t c = vc - 1 - i;
        mbar_wait(smem_u32(&sm.v_full[c % VST]), (c / VST) & 1);
      }
      for (uint32_t i = 0; i < QST && i < qi; ++i) {
        const uint32_t c = qi - 1 - i;
        mbar_wait(smem_u32(&sm.q_full[c % QST]), (c / QST) & 1);
      }
    }
  } else if (warp == 1 || warp == 3) {
    // =============================================== MMA issuers
    // Warp 1 issues S = Q K^T, warp 3 issues O += P V.  Two issuers keep the
    // tensor pipe fed: while one waits on its barriers the other's MMAs run.
    Sched<BM> sc;
    if (!BAL && !RS) sc.init(sm.m_q, P.B, HS, lane);  // one fixed item per CTA otherwise
    const bool qk_role = warp == 1;
    uint32_t kc = 0, vc = 0, qi = 0, g = 0;
    bool ok = true;
    for (long long rnd = 0; ok; ++rnd) {
      int b, m, rem;
      if (!next_item<BAL, RS>(P, sm, sc, rnd, lane, b, m, rem)) break;
      const Item it = make_item<PAGED, CAND, BAL>(P, sm, b, m, rem);
      if (it.t0 >= it.t1) continue;
      const int nt = it.t1 - it.t0;
      if (lane == 0) {
        if (qk_role) {
          const uint32_t qs = qi % QST;
          const uint32_t q_base = smem_u32(sm.q[qs]);
          ok = mbar_wait(smem_u32(&sm.q_full[qs]), (qi / QST) & 1);
          for (int i = 0; i < nt && ok; ++i, ++g, ++kc) {
            const uint32_t sb = g % NSP;
            const uint32_t slot = kc % KST;
            // the buffer is free once the O += P V that read its P completed
            ok = mbar_wait(smem_u32(&sm.sp_empty[sb]), ((g / NSP) & 1) ^ 1) &&
                 mbar_wait(smem_u32(&sm.k_full[slot]), (kc / KST) & 1);
            if (!ok) break;
            tc_fence_after();
            const uint32_t k_base = smem_u32(sm.k[slot]);
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk) {
              const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
              const uint64_t adesc = smem_desc_sw128(q_base + off, 16, 1024);
              const uint64_t bdesc = smem_desc_sw128(k_base + off, 16, 1024);
              umma_ss(tmem + TM_SP + sb * 128, adesc, bdesc, kIdescQK, kk > 0 ? 1u : 0u);
            }
            umma_commit(smem_u32(&sm.k_empty[slot]));
            umma_commit(smem_u32(&sm.s_full[PW2 ? g % (2 * NSP) : sb]));
            if (i == nt - 1) umma_commit(smem_u32(&sm.q_empty[qs]));
          }
        } else {
          for (int i = 0; i < nt && ok; ++i, ++g, ++vc) {
            const uint32_t pb = g % NSP;
            const uint32_t slot = vc % VST;
            ok = mbar_wait(smem_u32(&sm.p_full[pb]), (g / NSP) & 1) &&
                 mbar_wait(smem_u32(&sm.v_full[slot]), (vc / VST) & 1) &&
                 (i != 0 || mbar_wait(smem_u32(&sm.o_empty), (qi & 1) ^ 1));
            if (!ok) break;
            tc_fence_after();
            const uint32_t v_base = smem_u32(sm.v[slot]);
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
              // V tile is MN-major: 64-column halves 16 KiB apart (LBO), 8-key
              // groups 1 KiB apart (SBO); 16 keys = 2 KiB per k-step.
              const uint64_t bdesc = smem_desc_sw128(v_base + kk * 2048, kHalfBytes, 1024);
              umma_ts(tmem + TM_O, tmem + TM_SP + pb * 128 + p_col<PW2>(kk), bdesc, kIdescPV,
                      (i == 0 && kk == 0) ? 0u : 1u);
            }
            umma_commit(smem_u32(&sm.v_empty[slot]));
            umma_commit(smem_u32(&sm.sp_empty[pb]));
          }
          // two-pair layout: the pair that took the item's last key tile runs its epilogue
          if (ok) umma_commit(smem_u32(&sm.o_full[PW2 ? (g - 1) & 1 : 0]));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      g = __shfl_sync(0xffffffffu, g, 0);
      ++qi;
    }
    if (lane == 0) {
      if (!ok) record_timeout(P, sm);
      // all MMAs issued by this thread must finish before TMEM is released
      const uint32_t done = smem_u32(qk_role ? &sm.mma_done : &sm.mma_done2);
      umma_commit(done);
      mbar_wait(done, 0);
    }
    __syncwarp();
  } else if (warp == 2) {
    // =============================================== key-timestamp producer
    // Stages the key timestamps of every tile (in the MMA's tile order) for the
    // time-gap bias, so the pointwise warps never wait on global loads.
    if (P.time_table != nullptr && !PAGED && !CAND) {
      Sched<BM> sc;
      if (!BAL && !RS) sc.init(sm.m_q, P.B, HS, lane);  // one fixed item per CTA otherwise
      uint32_t g = 0, qitem = 0;
      bool ok = true;
      for (long long rnd = 0; ok; ++rnd) {
        int b, m, rem;
        if (!next_item<BAL, RS>(P, sm, sc, rnd, lane, b, m, rem)) break;
        const Item it = make_item<PAGED, CAND, BAL>(P, sm, b, m, rem);
        if (it.t0 >= it.t1) continue;
        const long long base = it.n_k > 0 ? P.ts[it.kv_row0] : 0;
        // Key timestamps run two tiles ahead of their slots: the loads of tiles
        // i + 1 and i + 2 are in flight while tile i waits for its slot and is
        // converted, so one global-load latency is not paid per tile.  Lanes
        // past the user's keys load nothing and take the base value later.
        long long ka[BN / 32], kb[BN / 32];
        auto load_tile = [&](int tile, long long (&dst)[BN / 32]) {
#pragma unroll
          for (int i = 0; i < BN / 32; ++i) {
            const int64_t kp = (int64_t)tile * BN + lane + 32 * i;
            if (kp < it.n_k) dst[i] = P.ts[it.kv_row0 + kp];
          }
        };
        load_tile(it.t0, ka);
        if (it.t0 + 1 < it.t1) load_tile(it.t0 + 1, kb);
        {  // query timestamps of this item's rows
          const uint32_t qsl = qitem & 1;
          long long qv[BM / 32];
#pragma unroll
          for (int i = 0; i < BM / 32; ++i) {
            const int r = lane + 32 * i;
            if (r < it.nvalid && it.n_k > 0) {
              const int64_t qpc = min64(max64(it.p0 + r, 0), it.n_k - 1);
              qv[i] = P.ts[it.kv_row0 + qpc];
            }
          }
          ok = mbar_wait_warp(smem_u32(&sm.qts_empty[qsl]), ((qitem >> 1) & 1) ^ 1);
          if (!ok) break;
          TsSlot& qs = sm.qts[qsl];
          bool exact = true;
#pragma unroll
          for (int i = 0; i < BM / 32; ++i) {
            const int r = lane + 32 * i;
            const long long v = (r < it.nvalid && it.n_k > 0) ? qv[i] : base;
            const long long rel = v - base;
            exact = exact && rel > -(1LL << 23) && rel < (1LL << 23);
            qs.i[r] = v;
            qs.f[r] = (float)rel;
          }
          exact = __all_sync(0xffffffffu, exact);
          if (lane == 0) {
            qs.exact = exact ? 1 : 0;
            qs.sorted = 0;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.qts_full[qsl]));
          ++qitem;
        }
        for (int tile = it.t0; tile < it.t1; ++tile, ++g) {
          long long cur[BN / 32];
#pragma unroll
          for (int i = 0; i < BN / 32; ++i) {
            cur[i] = ka[i];
            ka[i] = kb[i];
          }
          if (tile + 2 < it.t1) load_tile(tile + 2, kb);
          const uint32_t slot = g % NTS;
          ok = mbar_wait_warp(smem_u32(&sm.ts_empty[slot]), ((g / NTS) & 1) ^ 1);
          if (!ok) break;
          TsSlot& ts = sm.ts[slot];
          bool exact = true;
#pragma unroll
          for (int i = 0; i < BN / 32; ++i) {
            const int c = lane + 32 * i;
            const int64_t kp = (int64_t)tile * BN + c;
            const long long v = kp < it.n_k ? cur[i] : base;
            const long long rel = v - base;
            exact = exact && rel > -(1LL << 23) && rel < (1LL << 23);
            ts.i[c] = v;
            ts.f[c] = (float)rel;
          }
          exact = __all_sync(0xffffffffu, exact);
          __syncwarp();
          bool sorted = true;
#pragma unroll
          for (int i = 0; i < BN / 32; ++i) {
            const int c = lane + 32 * i;
            const int64_t kp = (int64_t)tile * BN + c;
            if (c + 1 < BN && kp + 1 < it.n_k) sorted = sorted && ts.i[c] <= ts.i[c + 1];
          }
          sorted = __all_sync(0xffffffffu, sorted);
          if (lane == 0) {
            ts.exact = exact ? 1 : 0;
            ts.sorted = sorted ? 1 : 0;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.ts_full[slot]));
        }
      }
      if (!ok && lane == 0) record_timeout(P, sm);
    }
  } else if (PW2 && warp >= 4) {
    // =============================================== pointwise + epilogue (two pairs)
    // 16 warps: key tiles alternate between two pairs of warpgroups; within a
    // pair, warpgroup `chalf` takes score columns [64 chalf, 64 chalf + 64).
    const int pwi = warp - 4;                       // 0..15
    const int wg = pwi >> 3;                        // tile parity handled
    const int chalf = (pwi >> 2) & 1;               // column half of the tile
    const int sub = warp & 3;                       // TMEM lane quarter
    const int r = sub * 32 + lane;                  // tile row owned by this thread
    const uint32_t lane_addr = (uint32_t)(sub * 32) << 16;
    const bool use_time = P.time_table != nullptr && !PAGED && !CAND;
    const bool use_pos = P.pos_table != nullptr;
    float* rrow = sm.rrow[pwi];
    const float self_rab = sm.pos_ext[0];
    // last position bucket this thread read, and its bias (tiles far from the
    // diagonal keep the same bucket for long runs, so the shared table is
    // rarely touched on the constant-row path)
    int pb_idx = -1;
    float pb_val = 0.f;
    Sched<BM> sc;
    if (!BAL && !RS) sc.init(sm.m_q, P.B, HS, lane);  // one fixed item per CTA otherwise
    uint32_t qi = 0, g = 0, my_epi = 0;
    // an output box of this warp's last epilogue still being read out of its
    // Q slot by a TMA store (released when the next item begins)
    bool box_pend = false;
    uint32_t box_slot = 0;
    bool ok = true;
    for (long long rnd = 0; ok; ++rnd) {
      int b, m, rem;
      if (!next_item<BAL, RS>(P, sm, sc, rnd, lane, b, m, rem)) break;
      const Item it = make_item<PAGED, CAND, BAL>(P, sm, b, m, rem);
      if (it.t0 >= it.t1) continue;
      // release the previous item's Q slot here, not at this pair's next S
      // tile: that tile may belong to the item after next, whose Q load waits
      // for this release
      if (OST2 && box_pend) {
        if (lane == 0) {
          bulk_wait_read0();
          mbar_arrive(smem_u32(&sm.q_done[box_slot]));
        }
        __syncwarp();
        box_pend = false;
      }
      // this row's query position (every candidate sits at the cached length)
      const int64_t qp = CAND ? it.p0 : it.p0 + r;
      long long tq_i = 0;
      float tq1 = 1.f;
      bool tq_exact = true;
      const uint32_t qsl = qi & 1;
      if (use_time) {  // this row's timestamp, staged by warp 2
        ok = mbar_wait_warp(smem_u32(&sm.qts_full[qsl]), (qi >> 1) & 1);
        if (!ok) break;
        tq_i = sm.qts[qsl].i[r];
        tq1 = sm.qts[qsl].f[r] + 1.f;
        tq_exact = sm.qts[qsl].exact != 0;
      }
      for (int tile = it.t0; tile < it.t1 && ok; ++tile, ++g) {
        if ((int)(g & 1) != wg) continue;
        const uint32_t sb = g % NSP;
        const bool cand_tile = CAND && tile == it.n_main;
        const int64_t k0 = (int64_t)tile * BN;      // key position of column 0
        // int32 tile-relative coordinates: query position minus k0, valid keys
        const int qrel = (int)max64(min64(qp - k0, 1 << 30), -(1 << 30));
        // lane 0 has the warp's smallest query position
        const int64_t qp0 = CAND ? it.p0 : it.p0 + sub * 32;
        const int qrel0 = (int)max64(min64(qp0 - k0, 1 << 30), -(1 << 30));
        const int kend = (int)max64(min64(it.n_k - k0, BN), 0);
        // offset of this warp's column half in its position-bias row
        const int roff = chalf ? 0 : 64;
        // element (row lane, column c) reads rbase[127 - c]
        const int rshift = use_pos ? ((CAND ? 0 : lane) - roff) : 0;
        const float* rtab = use_pos ? rrow : sm.pos_ext;  // zeros without a table
        const uint32_t tslot = g % NTS;
        bool time_fast = false;
        if (use_time) {
          ok = mbar_wait_warp(smem_u32(&sm.ts_full[tslot]), (g / NTS) & 1);
          if (!ok) break;
          time_fast = tq_exact && sm.ts[tslot].exact;
        }
        // Far from the diagonal a row's 64 columns usually share one position
        // bucket (and, with sorted key timestamps, one time bucket): then the
        // whole bias is one constant per row and is folded into the SiLU.
        float crow = 0.f;
        bool rowconst = false;
        if (!cand_tile) {
          const int cbase = 64 * chalf;
          const int dmax = qrel - cbase, dmin = qrel - cbase - 63;
          bool ok_row = dmin >= 0 || CAND;  // every column of both chunks visible
          if (CAND) ok_row = cbase + 63 < kend;
          if (use_pos) {
            const int b_hi = min(31 - __clz(max(dmax, 0) + 1), kMaxRab - 1);
            const int b_lo = min(31 - __clz(max(dmin, 0) + 1), kMaxRab - 1);
            if (b_hi != pb_idx) {
              pb_idx = b_hi;
              pb_val = sm.pos_ext[b_hi];
            }
            ok_row = ok_row && (b_hi == b_lo || pb_val == sm.pos_ext[b_lo]);
            crow = pb_val;
          }
          if (use_time) {
            const TsSlot& ts = sm.ts[tslot];
            long long d_hi = tq_i - ts.i[cbase], d_lo = tq_i - ts.i[cbase + 63];
            d_hi = d_hi < 0 ? 0 : d_hi;
            d_lo = d_lo < 0 ? 0 : d_lo;
            const int t_hi = min(63 - __clzll(d_hi + 1), kMaxRab - 1);
            const int t_lo = min(63 - __clzll(d_lo + 1), kMaxRab - 1);
            ok_row = ok_row && ts.sorted && sm.time_ext[t_hi] == sm.time_ext[t_lo];
            crow += sm.time_ext[t_hi];
          }
          rowconst = __all_sync(0xffffffffu, ok_row);
        }
        // position-bias row of this warp, only needed off the constant-row path:
        // rrow[j] = position bias at delta qrel0 + j + roff - 127; this warp's
        // columns need j in [0, 95)
        if (use_pos && !cand_tile && !rowconst) {
          __syncwarp();
#pragma unroll
          for (int i = 0; i < kRrowPairs / 32; ++i) {
            const int j = lane + 32 * i;
            const int delta = max(qrel0 + j + roff - 127, 0);
            rrow[j] = sm.pos_ext[min(31 - __clz(delta + 1), kMaxRab - 1)];
          }
          __syncwarp();
        }
        ok = mbar_wait_warp(smem_u32(&sm.s_full[g % (2 * NSP)]), (g / (2 * NSP)) & 1);
        if (!ok) break;
        tc_fence_after();

        // this warp's 64 S columns and, over their first half, its 32 P columns
        const uint32_t s_addr = tmem + lane_addr + TM_SP + sb * 128 + chalf * 64;
        const uint32_t p_addr = s_addr;
        const float hrow = 0.5f * crow;
        // Two 16-column chunks per (rolled) iteration: chunk q + 1 loads while
        // chunk q computes.  P of chunk q goes to columns [8q, 8q + 8), which
        // only covers S chunks already loaded into registers.
        uint32_t sa[16], sb2[16], pk[8];
        tmem_ld16(s_addr, sa);
        if (rowconst) {
#pragma unroll 1
          for (int q = 0; q < 4; q += 2) {
            tmem_wait_ld();
            reg_fence(sa);
            tmem_ld16(s_addr + (q + 1) * 16, sb2);
            silu_rowconst(sa, pk, hrow);
            tmem_st8(p_addr + q * 8, pk);
            tmem_wait_ld();
            reg_fence(sb2);
            if (q == 0) tmem_ld16(s_addr + 32, sa);
            silu_rowconst(sb2, pk, hrow);
            tmem_st8(p_addr + (q + 1) * 8, pk);
          }
        } else {
          const int cb0 = chalf * 64;
          const float* rl0 = rtab + (rshift + 127 - cb0);
          const TsSlot& ts = sm.ts[use_time ? tslot : 0];
          const int tmode = use_time ? (time_fast ? 1 : 2) : 0;
#pragma unroll 1
          for (int q = 0; q < 4; q += 2) {
            tmem_wait_ld();
            reg_fence(sa);
            tmem_ld16(s_addr + (q + 1) * 16, sb2);
            pw_chunk_any<CAND>(sa, pk, cb0 + q * 16, cand_tile, sub, qrel0, kend, tmode, rl0 - q * 16,
                               qrel, r, ts, tq1, tq_i, sm.time_ext, self_rab);
            tmem_st8(p_addr + q * 8, pk);
            tmem_wait_ld();
            reg_fence(sb2);
            if (q == 0) tmem_ld16(s_addr + 32, sa);
            pw_chunk_any<CAND>(sb2, pk, cb0 + q * 16 + 16, cand_tile, sub, qrel0, kend, tmode,
                               rl0 - q * 16 - 16, qrel, r, ts, tq1, tq_i, sm.time_ext, self_rab);
            tmem_st8(p_addr + (q + 1) * 8, pk);
          }
        }
        if (use_time) {
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.ts_empty[tslot]));
        }
        if (!ok) break;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[sb]));
      }
      if (!ok) break;
      if (use_time) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.qts_empty[qsl]));
      }
      // ---- epilogue, by the pair that processed the item's last key tile (so
      // the other pair can start the next item at once); this warp stores O
      // columns [64 chalf, 64 chalf + 64) of its 32 rows.
      if ((int)((g - 1) & 1) != wg) {
        // this pair leaves the item's Q slot alone
        if (OST2) {
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.q_done[qi & 1]));
        }
        ++qi;
        continue;
      }
      // each pair has its own o_full barrier and waits every one of its phases
      // in order (a parity wait must never run two phases ahead or behind)
      ok = mbar_wait_warp(smem_u32(&sm.o_full[wg]), my_epi & 1);
      ++my_epi;
      if (!ok) break;
      tc_fence_after();
      const bool row_ok = r < it.nvalid && it.q_row0 + r < P.total_q;
      const int64_t row = it.q_row0 + r;
      // as in the 16-warp layout: whole 32-row boxes go through the item's Q
      // slot (boxes 2 (pwi mod 8) + q of 2 KiB) and TMA stores
      const bool box_ok = OST2 && !P.partial && 32 * sub + 32 <= it.nvalid;
      const uint32_t qslot = qi & 1;
#pragma unroll 1
      for (int q = 0; q < 2; ++q) {
        const int ocol = 64 * chalf + 32 * q;
        uint32_t oa[32];
        tmem_ld32(tmem + lane_addr + TM_O + ocol, oa);
        tmem_wait_ld();
        reg_fence(oa);
        if (q == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.o_empty));
        }
        if (box_ok) {
          uint8_t* buf = sm.q[qslot] + ((pwi & 7) * 2 + q) * 2048;
          const int swz = (lane >> 1) & 3;  // the TMA's 64-byte swizzle
          uint4* srow = reinterpret_cast<uint4*>(buf + lane * 64);
          const float sc2 = P.scale;
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(oa[j]) * sc2, __uint_as_float(oa[j + 1]) * sc2);
            u.y = pack_bf16x2(__uint_as_float(oa[j + 2]) * sc2, __uint_as_float(oa[j + 3]) * sc2);
            u.z = pack_bf16x2(__uint_as_float(oa[j + 4]) * sc2, __uint_as_float(oa[j + 5]) * sc2);
            u.w = pack_bf16x2(__uint_as_float(oa[j + 6]) * sc2, __uint_as_float(oa[j + 7]) * sc2);
            srow[(j >> 3) ^ swz] = u;
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tm_out, smem_u32(buf), it.h * HD + ocol, (int)(it.q_row0 + 32 * sub));
            bulk_commit();
          }
          continue;
        }
        if (!row_ok) continue;
        if (P.partial) {
          // whole 32-byte sectors when the buffer allows: the scattered
          // per-row partial stores drain faster than as 16-byte pieces
          float* dst = BAL ? P.partial + ((int64_t)it.s * BM + r) * HD + ocol
                           : P.partial + ((int64_t)it.s * P.total_q + row) * (int64_t)P.H * HD +
                                 it.h * HD + ocol;
          if (P.part_v8) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) st_global_v8(dst + j, oa + j);
          } else {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              reinterpret_cast<float4*>(dst)[j / 4] =
                  make_float4(__uint_as_float(oa[j]), __uint_as_float(oa[j + 1]),
                              __uint_as_float(oa[j + 2]), __uint_as_float(oa[j + 3]));
          }
        } else {
          __nv_bfloat16* dst = P.out + row * P.out_stride + it.h * HD + ocol;
          const float sc2 = P.scale;
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(oa[j]) * sc2, __uint_as_float(oa[j + 1]) * sc2);
            u.y = pack_bf16x2(__uint_as_float(oa[j + 2]) * sc2, __uint_as_float(oa[j + 3]) * sc2);
            u.z = pack_bf16x2(__uint_as_float(oa[j + 4]) * sc2, __uint_as_float(oa[j + 5]) * sc2);
            u.w = pack_bf16x2(__uint_as_float(oa[j + 6]) * sc2, __uint_as_float(oa[j + 7]) * sc2);
            reinterpret_cast<uint4*>(dst)[j / 8] = u;
          }
        }
      }
      if (box_ok) {
        box_pend = true;
        box_slot = qslot;
      } else if (OST2) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.q_done[qslot]));
      }
      ++qi;
    }
    if (!ok && lane == 0) record_timeout(P, sm);
    if (OST2) {
      // every output box is written before the CTA ends
      if (lane == 0) {
        bulk_wait_all();
        if (box_pend) mbar_arrive(smem_u32(&sm.q_done[box_slot]));
      }
      __syncwarp();
    }
  } else if (warp >= 4) {
    // =============================================== pointwise + epilogue
    // 16 warps share every key tile: warp (cq, sub) takes score columns
    // [32 cq, 32 cq + 32) of tile rows [32 sub, 32 sub + 32), so each tile's
    // SiLU finishes in the shortest time and the three S/P buffers let the
    // tensor pipe run ahead.
    const int pwi = warp - 4;                       // 0..15
    const int cq = pwi >> 2;                        // column quarter of the tile
    const int sub = warp & 3;                       // TMEM lane quarter
    const int r = sub * 32 + lane;                  // tile row owned by this thread
    const int cbase = 32 * cq;                      // first score column of this warp
    const uint32_t lane_addr = (uint32_t)(sub * 32) << 16;
    const bool use_time = P.time_table != nullptr && !PAGED && !CAND;
    const bool use_pos = P.pos_table != nullptr;
    float* rrow = sm.rrow[pwi];
    const float self_rab = sm.pos_ext[0];
    // offset that puts this warp's position-bias row at rrow[0 .. 63)
    const int roff = 96 - cbase;
    // last position bucket this thread read, and its bias (tiles far from the
    // diagonal keep the same bucket for long runs, so the shared table is
    // rarely touched on the constant-row path)
    int pb_idx = -1;
    float pb_val = 0.f;
    Sched<BM> sc;
    if (!BAL && !RS) sc.init(sm.m_q, P.B, HS, lane);  // one fixed item per CTA otherwise
    uint32_t qi = 0, g = 0;
    // an output box of the previous item still being read out of its Q slot
    // by this warp's TMA store (released once the next item has begun)
    bool box_pend = false;
    uint32_t box_slot = 0;
    bool ok = true;
    for (long long rnd = 0; ok; ++rnd) {
      int b, m, rem;
      if (!next_item<BAL, RS>(P, sm, sc, rnd, lane, b, m, rem)) break;
      const Item it = make_item<PAGED, CAND, BAL>(P, sm, b, m, rem);
      if (it.t0 >= it.t1) continue;
      // this row's query position (every candidate sits at the cached length)
      const int64_t qp = CAND ? it.p0 : it.p0 + r;
      long long tq_i = 0;
      float tq1 = 1.f;
      bool tq_exact = true;
      const uint32_t qsl = qi & 1;
      if (use_time) {  // this row's timestamp, staged by warp 2
        ok = mbar_wait_warp(smem_u32(&sm.qts_full[qsl]), (qi >> 1) & 1);
        if (!ok) break;
        tq_i = sm.qts[qsl].i[r];
        tq1 = sm.qts[qsl].f[r] + 1.f;
        tq_exact = sm.qts[qsl].exact != 0;
      }
      for (int tile = it.t0; tile < it.t1 && ok; ++tile, ++g) {
        const uint32_t sb = g % NSP;
        const bool cand_tile = CAND && tile == it.n_main;
        const int64_t k0 = (int64_t)tile * BN;      // key position of column 0
        // int32 tile-relative coordinates: query position minus k0, valid keys
        const int qrel = (int)max64(min64(qp - k0, 1 << 30), -(1 << 30));
        // lane 0 has the warp's smallest query position
        const int64_t qp0 = CAND ? it.p0 : it.p0 + sub * 32;
        const int qrel0 = (int)max64(min64(qp0 - k0, 1 << 30), -(1 << 30));
        const int kend = (int)max64(min64(it.n_k - k0, BN), 0);
        // element (row lane, column c) reads rtab[rshift + 127 - c]
        const int rshift = use_pos ? ((CAND ? 0 : lane) - roff) : 0;
        const float* rtab = use_pos ? rrow : sm.pos_ext;  // zeros without a table
        const uint32_t tslot = g % NTS;
        bool time_fast = false;
        if (use_time) {
          ok = mbar_wait_warp(smem_u32(&sm.ts_full[tslot]), (g / NTS) & 1);
          if (!ok) break;
          time_fast = tq_exact && sm.ts[tslot].exact;
        }
        // Far from the diagonal a row's 32 columns usually share one position
        // bucket (and, with sorted key timestamps, one time bucket): then the
        // whole bias is one constant per row and is folded into the SiLU.
        float crow = 0.f;
        bool rowconst = false;
        if (!cand_tile) {
          const int dmax = qrel - cbase, dmin = qrel - cbase - 31;
          bool ok_row = dmin >= 0 || CAND;  // every column of both chunks visible
          if (CAND) ok_row = cbase + 31 < kend;
          if (use_pos) {
            const int b_hi = min(31 - __clz(max(dmax, 0) + 1), kMaxRab - 1);
            const int b_lo = min(31 - __clz(max(dmin, 0) + 1), kMaxRab - 1);
            if (b_hi != pb_idx) {
              pb_idx = b_hi;
              pb_val = sm.pos_ext[b_hi];
            }
            ok_row = ok_row && (b_hi == b_lo || pb_val == sm.pos_ext[b_lo]);
            crow = pb_val;
          }
          if (use_time) {
            const TsSlot& ts = sm.ts[tslot];
            long long d_hi = tq_i - ts.i[cbase], d_lo = tq_i - ts.i[cbase + 31];
            d_hi = d_hi < 0 ? 0 : d_hi;
            d_lo = d_lo < 0 ? 0 : d_lo;
            const int t_hi = min(63 - __clzll(d_hi + 1), kMaxRab - 1);
            const int t_lo = min(63 - __clzll(d_lo + 1), kMaxRab - 1);
            ok_row = ok_row && ts.sorted && sm.time_ext[t_hi] == sm.time_ext[t_lo];
            crow += sm.time_ext[t_hi];
          }
          rowconst = __all_sync(0xffffffffu, ok_row);
        }
        // position-bias row of this warp, only needed off the constant-row path:
        // rrow[j] = position bias at delta qrel0 + j + roff - 127, j in [0, 63)
        if (use_pos && !cand_tile && !rowconst) {
          __syncwarp();
#pragma unroll
          for (int i = 0; i < kRrowQuarters / 32; ++i) {
            const int j = lane + 32 * i;
            const int delta = max(qrel0 + j + roff - 127, 0);
            rrow[j] = sm.pos_ext[min(31 - __clz(delta + 1), kMaxRab - 1)];
          }
          __syncwarp();
        }
        // every pointwise warp waits every phase of s_full in order
        ok = mbar_wait_warp(smem_u32(&sm.s_full[sb]), (g / NSP) & 1);
        if (!ok) break;
        tc_fence_after();
        if (OST && box_pend) {
          if (lane == 0) {
            bulk_wait_read0();
            mbar_arrive(smem_u32(&sm.q_done[box_slot]));
          }
          __syncwarp();
          box_pend = false;
        }
        // this warp's 32 S columns; its 16 P columns overwrite the first half
        // (chunk q of P goes to columns [8q, 8q + 8), already loaded as S)
        const uint32_t s_addr = tmem + lane_addr + TM_SP + sb * 128 + cbase;
        const uint32_t p_addr = s_addr;
        const float hrow = 0.5f * crow;
        uint32_t sa[16], sb2[16], pk[8];
        tmem_ld16(s_addr, sa);
        tmem_ld16(s_addr + 16, sb2);
        tmem_wait_ld();
        reg_fence(sa);
        reg_fence(sb2);
        if (rowconst) {
          silu_rowconst(sa, pk, hrow);
          tmem_st8(p_addr, pk);
          silu_rowconst(sb2, pk, hrow);
          tmem_st8(p_addr + 8, pk);
        } else {
          const float* rl0 = rtab + (rshift + 127 - cbase);
          const TsSlot& ts = sm.ts[use_time ? tslot : 0];
          const int tmode = use_time ? (time_fast ? 1 : 2) : 0;
          pw_chunk_any<CAND>(sa, pk, cbase, cand_tile, sub, qrel0, kend, tmode, rl0, qrel, r, ts,
                             tq1, tq_i, sm.time_ext, self_rab);
          tmem_st8(p_addr, pk);
          pw_chunk_any<CAND>(sb2, pk, cbase + 16, cand_tile, sub, qrel0, kend, tmode, rl0 - 16,
                             qrel, r, ts, tq1, tq_i, sm.time_ext, self_rab);
          tmem_st8(p_addr + 8, pk);
        }
        if (use_time) {
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.ts_empty[tslot]));
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[sb]));
      }
      if (!ok) break;
      if (use_time) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.qts_empty[qsl]));
      }
      // ---- epilogue: this warp stores O columns [32 cq, 32 cq + 32) of its
      // 32 rows (every warp waits every phase of o_full in order)
      ok = mbar_wait_warp(smem_u32(&sm.o_full[0]), qi & 1);
      if (!ok) break;
      tc_fence_after();
      const bool row_ok = r < it.nvalid && it.q_row0 + r < P.total_q;
      const int64_t row = it.q_row0 + r;
      uint32_t oa[32];
      tmem_ld32(tmem + lane_addr + TM_O + cbase, oa);
      tmem_wait_ld();
      reg_fence(oa);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.o_empty));
      // a warp whose 32 rows all belong to the item writes its 32 x 32 box
      // through the item's Q slot (no longer read: every MMA of the item is
      // done) and one TMA store; per-thread row stores would touch 32 rows per
      // instruction and stall the warp's next shared-memory reads behind them
      const bool box_ok = OST && !P.partial && 32 * sub + 32 <= it.nvalid;
      if (box_ok) {
        uint8_t* buf = sm.q[qsl] + pwi * 2048;
        const int swz = (lane >> 1) & 3;  // the TMA's 64-byte swizzle
        uint4* srow = reinterpret_cast<uint4*>(buf + lane * 64);
        const float sc2 = P.scale;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          uint4 u;
          u.x = pack_bf16x2(__uint_as_float(oa[j]) * sc2, __uint_as_float(oa[j + 1]) * sc2);
          u.y = pack_bf16x2(__uint_as_float(oa[j + 2]) * sc2, __uint_as_float(oa[j + 3]) * sc2);
          u.z = pack_bf16x2(__uint_as_float(oa[j + 4]) * sc2, __uint_as_float(oa[j + 5]) * sc2);
          u.w = pack_bf16x2(__uint_as_float(oa[j + 6]) * sc2, __uint_as_float(oa[j + 7]) * sc2);
          srow[(j >> 3) ^ swz] = u;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_out, smem_u32(buf), it.h * HD + cbase, (int)(it.q_row0 + 32 * sub));
          bulk_commit();
        }
        box_pend = true;
        box_slot = qsl;
      } else if (OST) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.q_done[qsl]));
      }
      if (row_ok && !box_ok) {
        if (P.partial) {
          // whole 32-byte sectors when the buffer allows: the scattered
          // per-row partial stores drain faster than as 16-byte pieces
          float* dst = BAL ? P.partial + ((int64_t)it.s * BM + r) * HD + cbase
                           : P.partial + ((int64_t)it.s * P.total_q + row) * (int64_t)P.H * HD +
                                 it.h * HD + cbase;
          if (P.part_v8) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) st_global_v8(dst + j, oa + j);
          } else {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              reinterpret_cast<float4*>(dst)[j / 4] =
                  make_float4(__uint_as_float(oa[j]), __uint_as_float(oa[j + 1]),
                              __uint_as_float(oa[j + 2]), __uint_as_float(oa[j + 3]));
          }
        } else {
          __nv_bfloat16* dst = P.out + row * P.out_stride + it.h * HD + cbase;
          const float sc2 = P.scale;
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(oa[j]) * sc2, __uint_as_float(oa[j + 1]) * sc2);
            u.y = pack_bf16x2(__uint_as_float(oa[j + 2]) * sc2, __uint_as_float(oa[j + 3]) * sc2);
            u.z = pack_bf16x2(__uint_as_float(oa[j + 4]) * sc2, __uint_as_float(oa[j + 5]) * sc2);
            u.w = pack_bf16x2(__uint_as_float(oa[j + 6]) * sc2, __uint_as_float(oa[j + 7]) * sc2);
            reinterpret_cast<uint4*>(dst)[j / 8] = u;
          }
        }
      }
      ++qi;
    }
    if (!ok && lane == 0) record_timeout(P, sm);
    if (OST) {
      // every output box is written before the CTA ends
      if (lane == 0) {
        bulk_wait_all();
        if (box_pend) mbar_arrive(smem_u32(&sm.q_done[box_slot]));
      }
      __syncwarp();
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Deterministic reduction of the balanced key splits: CTA (x, g) sums, for
// the group g = (user b, query tile m, head h), the runs' partial blocks in run
// order over 8 of the tile's rows (one float4 per thread), then scales and
// rounds to bf16.  The group's items are first + (m H + h) ns .. + ns - 1
// (plan_balanced), each a contiguous fp32 [BM, HD] block; the four metadata
// loads are independent, so the partial loads start one memory latency after
// the kernel does.
constexpr int kReduceRows = 8;
constexpr int kReduceThreads = 256;  // one float4 of one of the 8 rows per thread

__global__ void __launch_bounds__(kReduceThreads) split_reduce_kernel(KParams P, int max_qt) {
  pdl_launch_dependents();
  pdl_wait();
  const int g = blockIdx.y;
  const int b = g / (max_qt * P.H);
  const int m = (g / P.H) % max_qt;
  const int h = g % P.H;
  if (b >= P.B) return;
  const int64_t q0 = P.q_off[b], q1 = P.q_off[b + 1];
  const int first = P.plan[b], next = P.plan[b + 1];
  const int64_t nq = q1 - q0;
  const int qt = (int)((nq + BM - 1) / BM);
  if (m >= qt) return;
  const int ns = (next - first) / (qt * P.H);
  const int item0 = first + (m * P.H + h) * ns;
  const int rr = blockIdx.x * kReduceRows + threadIdx.x / (HD / 4);
  const int c4 = threadIdx.x % (HD / 4);
  if (m * BM + rr >= nq) return;
  const float* src = P.partial + ((int64_t)item0 * BM + rr) * HD + c4 * 4;
  constexpr int64_t kBlk = (int64_t)BM * HD;  // floats between consecutive runs' blocks
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  int sidx = 0;
  // four runs' loads in flight at a time; the sums still go in run order
  for (; sidx + 4 <= ns; sidx += 4) {
    float4 x[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) x[j] = *reinterpret_cast<const float4*>(src + (sidx + j) * kBlk);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc.x += x[j].x;
      acc.y += x[j].y;
      acc.z += x[j].z;
      acc.w += x[j].w;
    }
  }
  for (; sidx < ns; ++sidx) {
    const float4 x = *reinterpret_cast<const float4*>(src + sidx * kBlk);
    acc.x += x.x;
    acc.y += x.y;
    acc.z += x.z;
    acc.w += x.w;
  }
  const int64_t row = q0 + m * BM + rr;
  if (row >= P.total_q) return;
  __nv_bfloat16* dst = P.out + row * P.out_stride + h * HD + c4 * 4;
  uint2 u;
  u.x = pack_bf16x2(acc.x * P.scale, acc.y * P.scale);
  u.y = pack_bf16x2(acc.z * P.scale, acc.w * P.scale);
  *reinterpret_cast<uint2*>(dst) = u;
}

size_t smem_bytes() { return sizeof(Smem) + 1024; }
// the 1 KiB alignment slack included: at most the 227 KiB a CTA may opt into
static_assert(sizeof(Smem) + 1024 <= 232448, "attention shared memory exceeds the per-CTA limit");

template <bool PAGED, bool CAND, bool PW2 = false, bool BAL = false>
cudaError_t launch_impl(const AttnProblem& p, const KParams& kp, long long items, int num_sms,
                        cudaStream_t stream) {
  CUtensorMap tq, tk, tv, tkc, tvc;
  const uint64_t qrows = (uint64_t)std::max<int64_t>(p.total_q, 1);
  if (!make_tmap_3d(&tq, p.q, HD, p.H, qrows, HD * 2, (uint64_t)p.q_stride * 2, 64, BM))
    return cudaErrorInvalidValue;
  if (PAGED) {
    const uint64_t rows = (uint64_t)(p.n_pages + 1) * 2 * p.H * 32;
    if (!make_tmap_2d(&tk, p.pool, HD, rows, HD * 2, 64, 32)) return cudaErrorInvalidValue;
    tv = tk;
  } else {
    const uint64_t krows = (uint64_t)std::max<int64_t>(p.total_kv, 1);
    if (!make_tmap_3d(&tk, p.k, HD, p.H, krows, HD * 2, (uint64_t)p.k_stride * 2, 64, BN))
      return cudaErrorInvalidValue;
    if (!make_tmap_3d(&tv, p.v, HD, p.H, krows, HD * 2, (uint64_t)p.v_stride * 2, 64, BN))
      return cudaErrorInvalidValue;
  }
  if (CAND) {
    if (!make_tmap_3d(&tkc, p.k, HD, p.H, qrows, HD * 2, (uint64_t)p.k_stride * 2, 64, BM))
      return cudaErrorInvalidValue;
    if (!make_tmap_3d(&tvc, p.v, HD, p.H, qrows, HD * 2, (uint64_t)p.v_stride * 2, 64, BM))
      return cudaErrorInvalidValue;
  } else {
    tkc = tq;
    tvc = tq;
  }
  static_assert(PAGED || !BAL, "only paged launches split keys");
  // causal launches without key splits store their bf16 output boxes with TMA
  CUtensorMap tout = tq;
  if (!CAND && !BAL && p.out != nullptr && !p.partial_only &&
      !make_tmap_2d_store(&tout, p.out, (uint64_t)p.H * HD, qrows, (uint64_t)p.out_stride * 2, 32, 32))
    return cudaErrorInvalidValue;
  auto kern = hstu_attn_sm100_kernel<PAGED, CAND, PW2, BAL>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cached = dev >= 0 && dev < 64 && attr_set[dev];
  if (!cached) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes());
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int grid = (int)std::max<long long>(1, std::min<long long>(items, num_sms));
  cudaError_t e = launch_kernel(p.pdl, kern, dim3(grid), dim3(kThreads), smem_bytes(), stream, tq,
                                tk, tv, tkc, tvc, tout, kp);
  if (e != cudaSuccess || kp.partial == nullptr || p.partial_only) return e;
  const int max_qt = std::max(1, (p.max_q + BM - 1) / BM);
  return launch_kernel(p.pdl, split_reduce_kernel,
                       dim3(BM / kReduceRows, (unsigned)(p.B * p.H * max_qt)), dim3(kReduceThreads), 0,
                       stream, kp, max_qt);
}

// Key-split plan: one wave of (user, head, split) items, each streaming a long
// run of key tiles (fewer pipeline start-ups and fewer partial sums than many
// short splits).  Used by the candidate path and by causal runs of at most one
// query tile per user (new tokens over a long cached history).
void split_plan(const AttnProblem& p, int num_sms, int* n_split, int* kps) {
  *n_split = 1;
  *kps = 1 << 30;
  if (!p.allow_split && !p.partial_only) return;
  if (p.mode != 1 && p.max_q > BM) return;
  const int max_tiles = (p.max_kv + BN - 1) / BN + (p.mode == 1 ? 1 : 0);
  const int qt = std::max(1, (p.max_q + BM - 1) / BM);
  const long long base_items = (long long)p.B * p.H * qt;
  if (base_items <= 0) return;
  int want = (int)std::min<long long>(max_tiles, num_sms / base_items);
  if (want <= 1) return;
  int k = (max_tiles + want - 1) / want;
  k = std::max(k, 2);
  *kps = k;
  *n_split = (max_tiles + k - 1) / k;
  if (*n_split <= 1) {
    *n_split = 1;
    *kps = 1 << 30;
  }
}

size_t balanced_plan_bytes(int B) { return ((size_t)(B + 1) * sizeof(int) + 255) & ~size_t(255); }

}  // namespace

void attn_sm100_split_plan(const AttnProblem& p, int num_sms, int* n_split, int* kps) {
  split_plan(p, num_sms, n_split, kps);
}

size_t attn_sm100_workspace_bytes(const AttnProblem& p, int num_sms) {
  if (p.B > kMaxUsers) {
    // batches over kMaxUsers run as chunks of users (attn_sm100_launch), each
    // with its own key-split plan over the same absolute query rows: the
    // workspace must hold the largest chunk's partials.  A short last chunk
    // can split keys where a full one does not.
    AttnProblem c = p;
    c.B = kMaxUsers;
    size_t need = attn_sm100_workspace_bytes(c, num_sms);
    if (p.B % kMaxUsers != 0) {
      c.B = p.B % kMaxUsers;
      need = std::max(need, attn_sm100_workspace_bytes(c, num_sms));
    }
    return need;
  }
  int ns, kps;
  split_plan(p, num_sms, &ns, &kps);
  if (ns <= 1 && !p.partial_only) return 0;
  if (!p.partial_only) {
    // balanced splits: the per-user item offsets, then one fp32 [BM, HD] block
    // per item, at most one item per SM
    return balanced_plan_bytes(p.B) + (size_t)num_sms * BM * HD * sizeof(float);
  }
  return (size_t)ns * (size_t)p.total_q * p.H * HD * sizeof(float);
}

cudaError_t attn_sm100_launch(const AttnProblem& p, void* workspace, size_t ws_bytes,
                              int* err_word, cudaStream_t stream) {
  if (p.d != HD || p.f32) return cudaErrorInvalidValue;
  if (p.B == 0 || p.total_q == 0) return cudaSuccess;
  if (p.B > kMaxUsers) {
    // users are independent and offsets are absolute rows: run chunks of users
    for (int b0 = 0; b0 < p.B; b0 += kMaxUsers) {
      AttnProblem c = p;
      c.B = std::min(kMaxUsers, p.B - b0);
      c.q_off = p.q_off + b0;
      if (p.kv_off) c.kv_off = p.kv_off + b0;
      if (p.users) c.users = p.users + b0;
      const cudaError_t e = attn_sm100_launch(c, workspace, ws_bytes, err_word, stream);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  const int num_sms = device_sm_count();
  KParams kp;
  std::memset(&kp, 0, sizeof(kp));
  kp.B = p.B;
  kp.H = p.H;
  kp.mode = p.mode;
  split_plan(p, num_sms, &kp.n_split, &kp.kps);
  kp.q_off = p.q_off;
  kp.kv_off = p.kv_off;
  kp.users = p.users;
  kp.page_lists = p.page_lists;
  kp.lengths = p.lengths;
  kp.max_users = p.max_users;
  kp.max_ppu = p.max_ppu;
  kp.n_pages = p.n_pages;
  kp.pos_table = p.pos_table;
  kp.n_pos = p.pos_table ? p.n_pos : 1;
  kp.time_table = p.time_table;
  kp.n_time = p.time_table ? p.n_time : 1;
  kp.ts = p.ts;
  kp.scale = p.scale;
  kp.q_pos_offset = p.q_pos_offset;
  kp.out = reinterpret_cast<__nv_bfloat16*>(p.out);
  kp.out_stride = p.out_stride;
  kp.total_q = p.total_q;
  kp.err = err_word;
  long long items_override = -1;
  bool balanced = false;
  if (kp.n_split > 1 || p.partial_only) {
    const size_t need = attn_sm100_workspace_bytes(p, num_sms);
    if (workspace == nullptr || ws_bytes < need) return cudaErrorInvalidValue;
    if (!p.partial_only) {
      // balanced splits, one item per CTA (the kernel chooses the runs)
      balanced = true;
      kp.n_split = 1;
      kp.kps = 1 << 30;
      kp.plan = reinterpret_cast<int*>(workspace);
      kp.partial = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) +
                                            balanced_plan_bytes(p.B));
      items_override = num_sms;
    } else {
      kp.partial = reinterpret_cast<float*>(workspace);
    }
    kp.part_v8 = (reinterpret_cast<uintptr_t>(kp.partial) & 31) == 0 ? 1 : 0;
  }
  const int qt = (p.max_q + BM - 1) / BM;
  const long long items =
      items_override > 0 ? items_override : (long long)p.B * p.H * std::max(qt, 1) * kp.n_split;
  if (p.paged) {
    if (p.mode == 1)
      return balanced ? launch_impl<true, true, false, true>(p, kp, items, num_sms, stream)
                         : launch_impl<true, true, false, false>(p, kp, items, num_sms, stream);
    // paged causal attention (the long-history path) runs the two-pair
    // pointwise layout: measured faster there than 16 warps per tile
    return balanced ? launch_impl<true, false, true, true>(p, kp, items, num_sms, stream)
                       : launch_impl<true, false, true, false>(p, kp, items, num_sms, stream);
  }
  return p.mode == 1 ? launch_impl<false, true>(p, kp, items, num_sms, stream)
                     : launch_impl<false, false>(p, kp, items, num_sms, stream);
}

}  // namespace hstu
