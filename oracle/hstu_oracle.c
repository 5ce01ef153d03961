/*
 * Plain fp64 CPU oracle for the HSTU attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark use it.  It shares no code, header, table or constant with the CUDA
 * library.
 *
 * What it computes (sources: "How Generative Recommenders Are Redefining RecSys
 * at Scale", section "HSTU": softmax is replaced by SiLU weighting, a relative
 * attention bias is added, and an elementwise gate is applied before the output
 * projection; the exact formula A = SiLU(Q K^T + rab) V / N under a causal mask
 * is the one the build specification states):
 *
 *   O[i,h,:] = scale * sum_{j in M(i)} SiLU( q_i . k_j + rab(i,j) ) * v_j
 *   SiLU(x)  = x / (1 + exp(-x))
 *   rab(i,j) = pos_table[ min(floor(log2(|p_i - p_j| + 1)), n_pos - 1) ]
 *            + time_table[ min(floor(log2(max(ts_i - ts_j, 0) + 1)), n_time - 1) ]
 *
 * Masks:
 *   causal     M(i) = { j of the same user : p_j <= p_i }  (diagonal included)
 *   candidate  M(c) = { every cached history token of the user } U { c itself };
 *              every candidate sits at position p = history length.
 *
 * The paged KV table's role ("Déploiement de recommandeurs génératifs avec NVIDIA
 * Dynamo-Triton et HSTU", section "Comment cela fonctionne": the attention kernel
 * consumes cached K/V directly) does not change the arithmetic: the oracle takes
 * the cached history as a plain jagged array.
 *
 * Everything is a straight loop nest in fp64 in the order of the definition;
 * sums run over j in increasing order, dot products over e in increasing order.
 * Work is split across threads only over independent (row, head) outputs.
 */
#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* scalar helpers                                                       */
/* ------------------------------------------------------------------ */

/* floor(log2(x)) for x >= 1, by repeated halving. */
static int floor_log2_u64(uint64_t x) {
    int b = -1;
    while (x) {
        x >>= 1;
        b++;
    }
    return b;
}

int oracle_pos_bucket(int64_t delta, int n_buckets) {
    uint64_t a = (uint64_t)(delta < 0 ? -delta : delta);
    int b = floor_log2_u64(a + 1);
    return b < n_buckets - 1 ? b : n_buckets - 1;
}

int oracle_time_bucket(int64_t dt, int n_buckets) {
    uint64_t a = (uint64_t)(dt < 0 ? 0 : dt);
    int b = floor_log2_u64(a + 1);
    return b < n_buckets - 1 ? b : n_buckets - 1;
}

double oracle_silu(double x) { return x / (1.0 + exp(-x)); }

/* Round an fp64 value to the nearest bfloat16 (ties to even), returned as fp64.
 * bfloat16 keeps 8 significant bits and the fp32 exponent range. */
double oracle_round_bf16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    double m = frexp(x, &e); /* x = m * 2^e, 0.5 <= |m| < 1 */
    int shift = 8;
    if (e - 1 < -126) shift = e + 133; /* subnormal: spacing 2^-133 */
    double r = nearbyint(ldexp(m, shift)); /* default rounding mode: ties to even */
    double y = ldexp(r, e - shift);
    if (fabs(y) > 3.3895313892515355e38) return x > 0 ? INFINITY : -INFINITY;
    return y;
}

/* ------------------------------------------------------------------ */
/* a tiny thread pool over an index range                               */
/* ------------------------------------------------------------------ */

typedef void (*task_fn)(void* ctx, int64_t t);
typedef struct {
    task_fn fn;
    void* ctx;
    int64_t n;
    atomic_llong next;
} pool_t;

static void* pool_worker(void* arg) {
    pool_t* p = (pool_t*)arg;
    for (;;) {
        int64_t t = atomic_fetch_add(&p->next, 1);
        if (t >= p->n) break;
        p->fn(p->ctx, t);
    }
    return NULL;
}

static void run_tasks(task_fn fn, void* ctx, int64_t n, int n_threads) {
    pool_t p;
    p.fn = fn;
    p.ctx = ctx;
    p.n = n;
    atomic_init(&p.next, 0);
    if (n_threads <= 1 || n <= 1) {
        pool_worker(&p);
        return;
    }
    if (n_threads > 256) n_threads = 256;
    pthread_t th[256];
    int started = 0;
    for (int i = 0; i < n_threads; i++)
        if (pthread_create(&th[i], NULL, pool_worker, &p) == 0) started++;
        else break;
    if (started == 0) pool_worker(&p);
    for (int i = 0; i < started; i++) pthread_join(th[i], NULL);
}

static int64_t find_segment(const int64_t* off, int B, int64_t r) {
    int64_t lo = 0, hi = B; /* off[lo] <= r < off[hi] */
    while (hi - lo > 1) {
        int64_t mid = (lo + hi) / 2;
        if (off[mid] <= r) lo = mid;
        else hi = mid;
    }
    return lo;
}

/* ------------------------------------------------------------------ */
/* causal attention; queries are the last n_q tokens of each sequence   */
/* ------------------------------------------------------------------ */

typedef struct {
    int B, H, dqk, dv;
    const int64_t *kv_off, *q_off;
    const double *q, *k, *v;
    int64_t q_stride, k_stride, v_stride; /* elements between consecutive tokens */
    const int64_t* ts;
    const double* pos_table;
    int n_pos;
    const double* time_table;
    int n_time;
    double scale;
    const int64_t* rows;
    int64_t n_rows;
    double* out;
    int64_t out_stride; /* elements between consecutive output rows */
    int magnitude;      /* 0: SiLU(s) * v; 1: |SiLU(s)| * |v|; 2: |s| * |v| */
} causal_ctx;

static void causal_task(void* vctx, int64_t t) {
    const causal_ctx* c = (const causal_ctx*)vctx;
    int64_t ri = t / c->H;
    int h = (int)(t % c->H);
    int64_t r = c->rows ? c->rows[ri] : ri;
    int64_t b = find_segment(c->q_off, c->B, r);
    int64_t nk = c->kv_off[b + 1] - c->kv_off[b];
    int64_t nq = c->q_off[b + 1] - c->q_off[b];
    int64_t pi = nk - nq + (r - c->q_off[b]); /* position of the query */
    const double* qi = c->q + r * c->q_stride + (int64_t)h * c->dqk;
    double* o = c->out + ri * c->out_stride + (int64_t)h * c->dv;
    for (int e = 0; e < c->dv; e++) o[e] = 0.0;
    for (int64_t pj = 0; pj <= pi; pj++) {
        int64_t j = c->kv_off[b] + pj;
        const double* kj = c->k + j * c->k_stride + (int64_t)h * c->dqk;
        const double* vj = c->v + j * c->v_stride + (int64_t)h * c->dv;
        double s = 0.0;
        for (int e = 0; e < c->dqk; e++) s += qi[e] * kj[e];
        if (c->pos_table) s += c->pos_table[oracle_pos_bucket(pi - pj, c->n_pos)];
        if (c->time_table) {
            int64_t ti = c->ts[c->kv_off[b] + pi];
            s += c->time_table[oracle_time_bucket(ti - c->ts[j], c->n_time)];
        }
        double w = c->magnitude == 2 ? fabs(s) : oracle_silu(s);
        if (c->magnitude)
            for (int e = 0; e < c->dv; e++) o[e] += fabs(w) * fabs(vj[e]);
        else
            for (int e = 0; e < c->dv; e++) o[e] += w * vj[e];
    }
    for (int e = 0; e < c->dv; e++) o[e] *= c->magnitude ? fabs(c->scale) : c->scale;
}

/*
 * q: [Tq, H, dqk]; k: [Tk, H, dqk]; v: [Tk, H, dv]; out: [n_rows or Tq, H, dv].
 * kv_offsets/q_offsets: [B+1]; user b has nk = kv_off[b+1]-kv_off[b] keys and
 * nq <= nk queries, which are its last nq tokens (nq == nk: plain causal).
 * timestamps: [Tk] or NULL; pos_table/time_table may be NULL (no term).
 * rows: query rows to compute (NULL: all Tq rows, in order).
 * Returns 0, or -1 on an argument error.
 */
static int attn_causal_impl(int B, int H, int dqk, int dv, const int64_t* kv_offsets,
                            const int64_t* q_offsets, const double* q, const double* k,
                            const double* v, const int64_t* timestamps, const double* pos_table,
                            int n_pos, const double* time_table, int n_time, double scale,
                            const int64_t* rows, int64_t n_rows, double* out, int n_threads,
                            int magnitude) {
    if (B < 0 || H <= 0 || dqk <= 0 || dv <= 0) return -1;
    for (int b = 0; b < B; b++) {
        int64_t nk = kv_offsets[b + 1] - kv_offsets[b];
        int64_t nq = q_offsets[b + 1] - q_offsets[b];
        if (nk < 0 || nq < 0 || nq > nk) return -1;
    }
    if (time_table && !timestamps) return -1;
    causal_ctx c = {B, H, dqk, dv, kv_offsets, q_offsets, q, k, v,
                    (int64_t)H * dqk, (int64_t)H * dqk, (int64_t)H * dv,
                    timestamps, pos_table, n_pos, time_table, n_time, scale,
                    rows, rows ? n_rows : q_offsets[B], out, (int64_t)H * dv, magnitude};
    run_tasks(causal_task, &c, c.n_rows * H, n_threads);
    return 0;
}

int oracle_attn_causal(int B, int H, int dqk, int dv, const int64_t* kv_offsets,
                       const int64_t* q_offsets, const double* q, const double* k,
                       const double* v, const int64_t* timestamps, const double* pos_table,
                       int n_pos, const double* time_table, int n_time, double scale,
                       const int64_t* rows, int64_t n_rows, double* out, int n_threads) {
    return attn_causal_impl(B, H, dqk, dv, kv_offsets, q_offsets, q, k, v, timestamps, pos_table,
                            n_pos, time_table, n_time, scale, rows, n_rows, out, n_threads, 0);
}

/*
 * Magnitudes of the same sum, term by term as above, with s = q_i . k_j + rab(i,j):
 *   kind 1: |scale| * sum_j |SiLU(s)| * |v_j|
 *   kind 2: |scale| * sum_j |s| * |v_j|
 * Not attention results: they size rounding-error bounds (an error relative to
 * every SiLU term, or proportional to every score, is bounded by these).
 */
int oracle_attn_causal_magnitude(int B, int H, int dqk, int dv, const int64_t* kv_offsets,
                                 const int64_t* q_offsets, const double* q, const double* k,
                                 const double* v, const int64_t* timestamps,
                                 const double* pos_table, int n_pos, const double* time_table,
                                 int n_time, double scale, const int64_t* rows, int64_t n_rows,
                                 double* out, int n_threads, int kind) {
    if (kind != 1 && kind != 2) return -1;
    return attn_causal_impl(B, H, dqk, dv, kv_offsets, q_offsets, q, k, v, timestamps, pos_table,
                            n_pos, time_table, n_time, scale, rows, n_rows, out, n_threads, kind);
}

/* ------------------------------------------------------------------ */
/* candidate scoring against a cached history                           */
/* ------------------------------------------------------------------ */

typedef struct {
    int B, H, dqk, dv;
    const int64_t *hist_off, *cand_off;
    const double *hist_k, *hist_v, *q, *k_cand, *v_cand;
    const double* pos_table;
    int n_pos;
    double scale;
    const int64_t* rows;
    int64_t n_rows;
    double* out;
    int magnitude; /* 0: SiLU(s) * v; 1: |SiLU(s)| * |v|; 2: |s| * |v| */
} cand_ctx;

static void cand_task(void* vctx, int64_t t) {
    const cand_ctx* c = (const cand_ctx*)vctx;
    int64_t ri = t / c->H;
    int h = (int)(t % c->H);
    int64_t r = c->rows ? c->rows[ri] : ri;
    int64_t b = find_segment(c->cand_off, c->B, r);
    int64_t nh = c->hist_off[b + 1] - c->hist_off[b];
    int64_t pc = nh; /* every candidate sits one past the last history token */
    const double* qc = c->q + (r * c->H + h) * c->dqk;
    double* o = c->out + (ri * c->H + h) * c->dv;
    for (int e = 0; e < c->dv; e++) o[e] = 0.0;
    for (int64_t pj = 0; pj <= nh; pj++) {
        const double *kj, *vj;
        if (pj < nh) {
            int64_t j = c->hist_off[b] + pj;
            kj = c->hist_k + (j * c->H + h) * c->dqk;
            vj = c->hist_v + (j * c->H + h) * c->dv;
        } else { /* the candidate itself */
            kj = c->k_cand + (r * c->H + h) * c->dqk;
            vj = c->v_cand + (r * c->H + h) * c->dv;
        }
        double s = 0.0;
        for (int e = 0; e < c->dqk; e++) s += qc[e] * kj[e];
        if (c->pos_table) s += c->pos_table[oracle_pos_bucket(pc - (pj < nh ? pj : pc), c->n_pos)];
        double w = c->magnitude == 2 ? fabs(s) : oracle_silu(s);
        if (c->magnitude)
            for (int e = 0; e < c->dv; e++) o[e] += fabs(w) * fabs(vj[e]);
        else
            for (int e = 0; e < c->dv; e++) o[e] += w * vj[e];
    }
    for (int e = 0; e < c->dv; e++) o[e] *= c->magnitude ? fabs(c->scale) : c->scale;
}

/*
 * hist_k/hist_v: [Th, H, d] jagged by hist_offsets[B+1] (the user's cached tokens).
 * q/k_cand/v_cand: [Tc, H, d] jagged by cand_offsets[B+1].  out: [n_rows or Tc, H, dv].
 */
int oracle_attn_candidates(int B, int H, int dqk, int dv, const int64_t* hist_offsets,
                           const double* hist_k, const double* hist_v,
                           const int64_t* cand_offsets, const double* q,
                           const double* k_cand, const double* v_cand,
                           const double* pos_table, int n_pos, double scale,
                           const int64_t* rows, int64_t n_rows, double* out, int n_threads) {
    if (B < 0 || H <= 0 || dqk <= 0 || dv <= 0) return -1;
    cand_ctx c = {B, H, dqk, dv, hist_offsets, cand_offsets, hist_k, hist_v, q, k_cand,
                  v_cand, pos_table, n_pos, scale, rows, rows ? n_rows : cand_offsets[B], out, 0};
    run_tasks(cand_task, &c, c.n_rows * H, n_threads);
    return 0;
}

/* Magnitudes of the candidate sum, term by term (kinds as for
 * oracle_attn_causal_magnitude). */
int oracle_attn_candidates_magnitude(int B, int H, int dqk, int dv, const int64_t* hist_offsets,
                                     const double* hist_k, const double* hist_v,
                                     const int64_t* cand_offsets, const double* q,
                                     const double* k_cand, const double* v_cand,
                                     const double* pos_table, int n_pos, double scale,
                                     const int64_t* rows, int64_t n_rows, double* out,
                                     int n_threads, int kind) {
    if (B < 0 || H <= 0 || dqk <= 0 || dv <= 0 || (kind != 1 && kind != 2)) return -1;
    cand_ctx c = {B, H, dqk, dv, hist_offsets, cand_offsets, hist_k, hist_v, q, k_cand,
                  v_cand, pos_table, n_pos, scale, rows, rows ? n_rows : cand_offsets[B], out, kind};
    run_tasks(cand_task, &c, c.n_rows * H, n_threads);
    return 0;
}

/* ------------------------------------------------------------------ */
/* HSTU block stack                                                     */
/* ------------------------------------------------------------------ */

typedef struct {
    const double* a;   /* [T, K] */
    const double* w;   /* [K, N] */
    double* y;         /* [T, N] */
    int64_t K, N;
    int act_silu;
    int round;
} gemm_ctx;

static void gemm_task(void* vctx, int64_t t) {
    const gemm_ctx* g = (const gemm_ctx*)vctx;
    double* yt = g->y + t * g->N;
    const double* at = g->a + t * g->K;
    for (int64_t n = 0; n < g->N; n++) {
        double s = 0.0;
        for (int64_t kk = 0; kk < g->K; kk++) s += at[kk] * g->w[kk * g->N + n];
        if (g->act_silu) s = oracle_silu(s);
        yt[n] = g->round ? oracle_round_bf16(s) : s;
    }
}

typedef struct {
    const double *a, *u; /* [T, F] each (u: row stride u_stride) */
    int64_t u_stride;
    double* g;           /* [T, F] */
    int64_t F;
    double eps;
    int round;
} lngate_ctx;

static void lngate_task(void* vctx, int64_t t) {
    const lngate_ctx* c = (const lngate_ctx*)vctx;
    const double* a = c->a + t * c->F;
    const double* u = c->u + t * c->u_stride;
    double mean = 0.0, var = 0.0;
    for (int64_t f = 0; f < c->F; f++) mean += a[f];
    mean /= (double)c->F;
    for (int64_t f = 0; f < c->F; f++) var += (a[f] - mean) * (a[f] - mean);
    var /= (double)c->F; /* biased variance */
    double inv = 1.0 / sqrt(var + c->eps);
    for (int64_t f = 0; f < c->F; f++) {
        double y = (a[f] - mean) * inv * u[f];
        c->g[t * c->F + f] = c->round ? oracle_round_bf16(y) : y;
    }
}

/* LayerNorm (no affine, biased variance) of a[T,F] times the gate u[T,F]. */
int oracle_layernorm_gate(int64_t T, int64_t F, const double* a, const double* u, double eps,
                          int round_bf16, double* g, int n_threads) {
    lngate_ctx c = {a, u, F, g, F, eps, round_bf16};
    run_tasks(lngate_task, &c, T, n_threads);
    return 0;
}

/*
 * x: [T, dm] (input, overwritten with the output of the last layer).
 * w_uvqk: [n_layers, dm, 4*H*dh], columns [U | V | Q | K], head-major in each.
 * w_o: [n_layers, H*dh, dm].
 * One layer: UVQK = SiLU(X W1); A = causal attention(Q, K, V) with the rab;
 *            G = LayerNorm(A) * U; X <- X + G W2.
 * With round_bf16 != 0 each materialised tensor (UVQK, A, G, X) is rounded to
 * bf16 (RNE), exactly where the GPU path stores bf16.  round_output == 0 keeps
 * the last layer's X + G W2 unrounded (every other rounding point stays), so a
 * caller can compare a bf16 result against the value before its final rounding.
 * layer_out: optional [n_layers, T, dm], X after every layer.
 */
int oracle_hstu_block(int64_t T, int B, const int64_t* seq_offsets, int n_layers, int dm, int H,
                      int dh, double* x, const double* w_uvqk, const double* w_o,
                      const int64_t* timestamps, const double* pos_table, int n_pos,
                      const double* time_table, int n_time, double scale, double ln_eps,
                      int round_bf16, int round_output, double* layer_out, int n_threads) {
    if (T != seq_offsets[B]) return -1;
    int64_t F = (int64_t)H * dh, N1 = 4 * F;
    double* uvqk = (double*)malloc(sizeof(double) * T * N1);
    double* a = (double*)malloc(sizeof(double) * T * F);
    double* g = (double*)malloc(sizeof(double) * T * F);
    double* d = (double*)malloc(sizeof(double) * T * dm);
    if (!uvqk || !a || !g || !d) {
        free(uvqk); free(a); free(g); free(d);
        return -2;
    }
    for (int l = 0; l < n_layers; l++) {
        gemm_ctx g1 = {x, w_uvqk + (int64_t)l * dm * N1, uvqk, dm, N1, 1, round_bf16};
        run_tasks(gemm_task, &g1, T, n_threads);
        causal_ctx c = {B, H, dh, dh, seq_offsets, seq_offsets,
                        uvqk + 2 * F, uvqk + 3 * F, uvqk + F, N1, N1, N1,
                        timestamps, pos_table, n_pos, time_table, n_time, scale,
                        NULL, T, a, F};
        run_tasks(causal_task, &c, T * H, n_threads);
        if (round_bf16)
            for (int64_t i = 0; i < T * F; i++) a[i] = oracle_round_bf16(a[i]);
        lngate_ctx lc = {a, uvqk, N1, g, F, ln_eps, round_bf16};
        run_tasks(lngate_task, &lc, T, n_threads);
        gemm_ctx g2 = {g, w_o + (int64_t)l * F * dm, d, F, dm, 0, 0};
        run_tasks(gemm_task, &g2, T, n_threads);
        const int round_x = round_bf16 && (round_output || l + 1 < n_layers);
        for (int64_t i = 0; i < T * dm; i++) {
            double y = x[i] + d[i];
            x[i] = round_x ? oracle_round_bf16(y) : y;
        }
        if (layer_out) memcpy(layer_out + (int64_t)l * T * dm, x, sizeof(double) * T * dm);
    }
    free(uvqk); free(a); free(g); free(d);
    return 0;
}
