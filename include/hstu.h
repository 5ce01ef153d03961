/*
 * hstu.h -- C ABI of the B200 (sm_100a) HSTU attention hot path.
 *
 * What is computed.  HSTU attention ("How Generative Recommenders Are Redefining
 * RecSys at Scale", section "HSTU": SiLU weighting in place of softmax, a
 * relative attention bias, and an elementwise gate before the output
 * projection) over jagged per-user sequences:
 *
 *     O[i,h,:] = scale * sum_{j in M(i)} SiLU(q_i . k_j + rab(i,j)) * v_j
 *     rab(i,j) = pos_table[min(floor(log2(|p_i-p_j|+1)), n_pos-1)]
 *              + time_table[min(floor(log2(max(ts_i-ts_j,0)+1)), n_time-1)]
 *
 * with no 1/sqrt(d) factor and with scale = 1/N given by the caller.  Cached
 * history K/V lives in a paged GPU KV data table with lookup, allocation and
 * append ("NVIDIA Dynamo-Triton Gets End-to-End HSTU Generative Recommender
 * Workflow", section "What the workflow combines"), which the attention kernel
 * reads directly ("Déploiement de recommandeurs génératifs avec NVIDIA
 * Dynamo-Triton et HSTU", section "Comment cela fonctionne").
 *
 * Conventions (all entry points):
 *  - Pointers are DEVICE pointers unless the comment says "host".
 *  - Jagged tensors are values [T, H, d] (row-major, token-major, head next,
 *    feature innermost) plus int64 offsets [B+1] in device memory, offsets[0]
 *    == 0, non-decreasing.  The caller owns every buffer; the library allocates
 *    device memory only in hstu_kv_table_create.
 *  - Every call is asynchronous on `stream` and returns an hstu_status for
 *    errors found on the host (null pointers, unsupported sizes, launch
 *    failures).  Errors found on the device (out of pages, duplicate users,
 *    append past the reserved pages) are recorded in the table's status word:
 *    read it with hstu_kv_table_status.  No C++ exception crosses this ABI.
 *  - The CUDA kernels need an sm_100a device (B200).  There is no CPU path.
 */
#ifndef HSTU_H_
#define HSTU_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define HSTU_API __attribute__((visibility("default")))
#else
#define HSTU_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HSTU_OK = 0,
    HSTU_ERR_INVALID_ARG = 1,
    HSTU_ERR_OUT_OF_PAGES = 2,
    HSTU_ERR_CUDA = 3,
    HSTU_ERR_UNSUPPORTED = 4,
    HSTU_ERR_TIMEOUT = 5
} hstu_status;

typedef enum { HSTU_F32 = 0, HSTU_BF16 = 1 } hstu_dtype;

/* Mask of hstu_attn_cached_fwd. */
typedef enum {
    /* Candidate scoring: candidate c of user b attends to all of b's cached
     * tokens and to itself only; every candidate has position = cached length. */
    HSTU_MASK_CANDIDATES = 0,
    /* Causal suffix: the n_q queries of user b are the last n_q of its cached
     * tokens (positions cached_len - n_q .. cached_len - 1), causal. */
    HSTU_MASK_CAUSAL_SUFFIX = 1
} hstu_mask_mode;

/* Relative attention bias, passed by HOST pointer to a struct of DEVICE
 * pointers.  Either table may be NULL (that term is absent); a NULL struct
 * pointer means no bias.  Tables are fp32 and shared by all heads.
 * timestamps: int64 [T] jagged like the queries/keys of hstu_attn_fwd; the
 * time term is supported only by hstu_attn_fwd and hstu_block_fwd. */
typedef struct {
    const float* pos_table;
    int32_t n_pos_buckets;       /* 1..256 when pos_table != NULL */
    const float* time_table;
    int32_t n_time_buckets;      /* 1..256 when time_table != NULL */
    const int64_t* timestamps;
} hstu_rab;

typedef struct hstu_kv_table hstu_kv_table; /* opaque */

/* Library version and a check that an sm_100 device is current. */
HSTU_API int32_t hstu_version(void);
HSTU_API hstu_status hstu_device_check(void);
HSTU_API const char* hstu_status_string(hstu_status s);

/* Synchronises `stream` and returns (then clears) the library-wide device error
 * word: HSTU_ERR_TIMEOUT if a kernel abandoned a bounded wait (its outputs are
 * then undefined), HSTU_OK otherwise. */
HSTU_API hstu_status hstu_last_device_error(cudaStream_t stream);

/* Failure-detection self test: one GPU thread waits, for at most timeout_us
 * microseconds (1 .. 2 000 000), on an mbarrier that nothing completes, then
 * records HSTU_ERR_TIMEOUT in the device error word that hstu_last_device_error
 * reads -- the bounded wait and error path of every kernel in the library.  No
 * fault, trap or unbounded wait is involved and the context stays usable.
 * Returns HSTU_ERR_INVALID_ARG for a limit outside that range. */
HSTU_API hstu_status hstu_wait_timeout_selftest(int32_t timeout_us, cudaStream_t stream);

/*
 * Jagged causal HSTU attention (section "HSTU" of the page cited above): user
 * b owns tokens [seq_offsets[b], seq_offsets[b+1]); token i attends to the
 * tokens j <= i of the same user; positions count from 0 at each user's first
 * token.
 *   q, k: [T, H, d_qk]; v, out: [T, H, d_v]; dtype dt for all four.
 *   B >= 0 users; max_len is an upper bound of the lengths (used for launch
 *   sizing only; lengths are read on the device); total_tokens = T =
 *   seq_offsets[B], the number of rows of every tensor (bounds the tile loads).
 *   dt == HSTU_BF16: needs d_qk == d_v == 128 (tcgen05 kernel) or
 *   d_qk == d_v in {32, 64} (SIMT kernel); fp32 accumulation.
 *   dt == HSTU_F32:  d_qk == d_v in {32, 64, 128}; fp32 SIMT kernel.
 *   scale multiplies the fp32 sum before the store (1/N).
 * Errors: HSTU_ERR_INVALID_ARG for null pointers / bad sizes,
 * HSTU_ERR_UNSUPPORTED for other head dims, HSTU_ERR_CUDA on launch failure.
 */
HSTU_API hstu_status hstu_attn_fwd(const void* q, const void* k, const void* v,
                          const int64_t* seq_offsets, int32_t B, int32_t max_len,
                          int64_t total_tokens, int32_t H, int32_t d_qk, int32_t d_v, hstu_dtype dt,
                          const hstu_rab* rab, float scale, void* out, cudaStream_t stream);

/*
 * Paged KV data table ("What the workflow combines": lookup, allocation,
 * append).  Pool layout: pool[page][kv (0 = K, 1 = V)][head][slot][d] in dtype,
 * page_size slots per page.  Free pages are a stack initialised from
 * host_free_order (a permutation of 0..n_pages-1, top = LAST element; NULL
 * means 0..n_pages-1).  Each user id in [0, max_users) owns a page list of at
 * most max_pages_per_user pages and a cached length.
 * page_size must be 32; d in {32, 64, 128}; dtype bf16 or fp32.
 * This is the only call that allocates device memory (pool, lists, status).
 */
HSTU_API hstu_status hstu_kv_table_create(int64_t n_pages, int32_t page_size, int32_t H, int32_t d,
                                 hstu_dtype dtype, int64_t max_users,
                                 int32_t max_pages_per_user, const int32_t* host_free_order,
                                 hstu_kv_table** out_table);
HSTU_API void hstu_kv_table_destroy(hstu_kv_table* t);

/* Synchronises `stream`, returns and clears the first device-side error
 * recorded since the last call (HSTU_OK if none). */
HSTU_API hstu_status hstu_kv_table_status(hstu_kv_table* t, cudaStream_t stream);

/* Device pointers of the table's storage, for callers that read the pool
 * directly (all host-pointer outputs; any may be NULL). */
HSTU_API hstu_status hstu_kv_table_info(hstu_kv_table* t, void** pool, int32_t** page_lists,
                               int64_t** lengths, int32_t** free_stack, int32_t** free_top);

/*
 * Allocation: user users[b] (int64 [B], unique, in [0, max_users)) will add
 * n_new_tokens[b] tokens; it receives ceil((len + n_new) / page_size) - held
 * more pages (never negative), popped from the top of the free stack in the
 * order users are listed.  page_ids_out (optional, int32, capacity
 * page_ids_cap) receives the new page ids in that order, -1 padded.
 * If the free stack is too short the table is left unchanged and the status
 * word records HSTU_ERR_OUT_OF_PAGES; duplicate / out-of-range users or a page
 * list overflow record HSTU_ERR_INVALID_ARG (also unchanged).  One CTA; B <= 65536.
 */
HSTU_API hstu_status hstu_kv_alloc(hstu_kv_table* t, const int64_t* users, const int64_t* n_new_tokens,
                          int32_t B, int32_t* page_ids_out, int32_t page_ids_cap,
                          cudaStream_t stream);

/*
 * Eviction of whole users (section "What the workflow combines" of the page
 * cited above: older users are evicted LRU-style when the cache is full; the
 * choice of users is the caller's).  Every page of each listed user returns to
 * the free stack - users in the order listed, each user's pages from its last
 * to its first, so its first page ends on top - and its cached length becomes
 * 0.  users: [B] device, unique.  The page bytes are not cleared.  Duplicate
 * or out-of-range users leave the table unchanged and record
 * HSTU_ERR_INVALID_ARG in the status word.  To keep a user's K/V (host tier),
 * gather it with hstu_kv_lookup first; to bring it back, hstu_kv_alloc then
 * hstu_kv_append.
 */
HSTU_API hstu_status hstu_kv_release(hstu_kv_table* t, const int64_t* users, int32_t B,
                                     cudaStream_t stream);

/*
 * Append: token r of user users[b] (rows new_offsets[b] .. new_offsets[b+1]-1
 * of k_new / v_new, [T_new, H, d] in the table dtype) goes to page
 * list[len / page_size], slot len % page_size, then len grows.  Pages must
 * have been reserved by hstu_kv_alloc; otherwise nothing is written and the
 * status word records HSTU_ERR_INVALID_ARG.  max_new bounds every user's
 * token count (launch sizing).
 */
HSTU_API hstu_status hstu_kv_append(hstu_kv_table* t, const int64_t* users, const void* k_new,
                           const void* v_new, const int64_t* new_offsets, int32_t B,
                           int32_t max_new, cudaStream_t stream);

/*
 * Lookup: cached_len_out[b] (int64) = cached length of users[b];
 * page_table_out (int32 [B, max_pages], optional) = its page list, -1 padded.
 * Optionally (k_out, v_out non-NULL, out_offsets int64 [B+1] = prefix sums of
 * the cached lengths) gathers the cached K/V into jagged [T, H, d] buffers;
 * max_len bounds the cached lengths (launch sizing).
 */
HSTU_API hstu_status hstu_kv_lookup(hstu_kv_table* t, const int64_t* users, int32_t B,
                           int64_t* cached_len_out, int32_t* page_table_out, int32_t max_pages,
                           void* k_out, void* v_out, const int64_t* out_offsets, int32_t max_len,
                           cudaStream_t stream);

/*
 * One serving step of the table ("NVIDIA Dynamo-Triton Gets End-to-End HSTU
 * Generative Recommender Workflow", section "What the workflow combines":
 * allocation, append and lookup of the paged KV data table): the effect of
 * hstu_kv_alloc with n_new[b] = new_offsets[b+1] - new_offsets[b], then
 * hstu_kv_append, then hstu_kv_lookup without the K/V gather, in one call.
 *  users: int64 [B] device, unique, in [0, max_users).
 *  k_new, v_new: [T_new, H, d] device, table dtype, 16-byte aligned (may be
 *    NULL when max_new = 0); new_offsets: int64 [B+1] device.
 *  max_new: bound on every user's new-token count (launch sizing); a larger
 *    count is an invalid argument.
 *  cached_len_out: int64 [B] (optional) = cached length after the step;
 *  page_table_out: int32 [B, max_pages] (optional) = page lists, -1 padded.
 * All or nothing: duplicate or out-of-range users, a negative or too large
 * count (HSTU_ERR_INVALID_ARG) or too few free pages (HSTU_ERR_OUT_OF_PAGES)
 * leave the table unchanged and record the status word; the lookup outputs
 * then show the unchanged table.  Pages are popped exactly as hstu_kv_alloc
 * pops them, so page ids match the three separate calls bit for bit.  Up to
 * 64 users run as one kernel launch; larger batches as two.
 */
HSTU_API hstu_status hstu_kv_step(hstu_kv_table* t, const int64_t* users, const void* k_new,
                                  const void* v_new, const int64_t* new_offsets, int32_t B,
                                  int32_t max_new, int64_t* cached_len_out,
                                  int32_t* page_table_out, int32_t max_pages, cudaStream_t stream);

/*
 * Attention whose history K/V comes from the KV table, read page by page inside
 * the kernel (no gather).  users: int64 [B]; q_offsets: int64 [B+1] jagged
 * query rows; q: [Tq, H, d]; out: [Tq, H, d]; the table's dtype.
 *  HSTU_MASK_CANDIDATES: k_cand, v_cand [Tq, H, d] are the candidates' own
 *    K/V; candidate c sees all cached tokens of its user and itself; every
 *    candidate has position cached_len.
 *  HSTU_MASK_CAUSAL_SUFFIX: k_cand = v_cand = NULL; user b's queries are its
 *    last n_q = q_offsets[b+1]-q_offsets[b] cached tokens (n_q <= cached_len).
 * rab: only the position term (time_table must be NULL).
 * total_q = q_offsets[B] (rows of q, k_cand, v_cand, out); max_q / max_cached
 * bound the per-user query count / cached length (launch sizing).
 * workspace: device scratch of hstu_attn_cached_workspace_size() bytes,
 * 256-byte aligned (may be NULL when that size is 0).  It holds fp32 partial
 * sums when the keys are split over several CTAs: always possible with
 * candidates, and in causal-suffix mode when no user has more than 128 query
 * rows (a few new tokens over a long cache); the split partials are reduced in
 * a fixed order, so results do not depend on scheduling.  bf16 needs d=128.
 */
HSTU_API hstu_status hstu_attn_cached_fwd(hstu_kv_table* t, const int64_t* users, int32_t B,
                                 const void* q, const void* k_cand, const void* v_cand,
                                 const int64_t* q_offsets, int64_t total_q, int32_t max_q,
                                 int32_t max_cached,
                                 int32_t mask_mode, const hstu_rab* rab, float scale, void* out,
                                 void* workspace, size_t ws_bytes, cudaStream_t stream);
HSTU_API size_t hstu_attn_cached_workspace_size(hstu_kv_table* t, int32_t B, int64_t total_q,
                                       int32_t max_q, int32_t max_cached, int32_t mask_mode);

/*
 * Allocation-free variant of hstu_attn_cached_fwd (no counterpart on the pages:
 * it exists for callers that cannot allocate device memory on their request
 * path, such as a server whose allocator is frozen after warm-up or code that
 * runs inside someone else's memory pool).  Same arguments and results as
 * hstu_attn_cached_fwd without workspace/ws_bytes: the split partial sums go
 * to a fixed array of hstu_attn_cached_noalloc_max_scratch() bytes (32 MiB)
 * that the library reserves on every GPU where it is loaded, kept until the
 * process exits.  Calls needing more than that return HSTU_ERR_UNSUPPORTED.
 * The first call on a device looks the array's address up (with that device
 * current) and should come before any stream capture; the address is kept for
 * the life of the process, which assumes the device's primary context is never
 * reset (cudaDeviceReset also invalidates every KV table).  All calls share the
 * array: calls that overlap on the GPU race, so do not run two at once.
 * Arguments are checked exactly as hstu_attn_cached_fwd checks them, before the
 * scratch size.  Allocates no memory.
 */
HSTU_API size_t hstu_attn_cached_noalloc_max_scratch(void);
HSTU_API hstu_status hstu_attn_cached_fwd_noalloc(hstu_kv_table* t, const int64_t* users, int32_t B,
                                                  const void* q, const void* k_cand,
                                                  const void* v_cand, const int64_t* q_offsets,
                                                  int64_t total_q, int32_t max_q, int32_t max_cached,
                                                  int32_t mask_mode, const hstu_rab* rab, float scale,
                                                  void* out, cudaStream_t stream);

/*
 * HSTU block stack ("HSTU" section: projection, SiLU, SiLU attention with rab,
 * elementwise gate before the output projection), bf16 with fp32 accumulation:
 *   for each layer l:
 *     [U|V|Q|K] = SiLU(X @ w_uvqk[l])          w_uvqk[l]: [d_model, 4*H*dh]
 *     A = hstu_attn(Q, K, V) (causal, rab, scale)
 *     G = LayerNorm(A) * U  (over H*dh features, biased variance, ln_eps, no affine)
 *     X = X + G @ w_o[l]                        w_o[l]: [H*dh, d_model]
 * x: [T, d_model] bf16, updated in place.  w_uvqk, w_o: HOST arrays of
 * n_layers device pointers.  Needs dh == 128, H*dh == d_model, d_model % 128 == 0.
 * workspace: >= hstu_block_workspace_size(T, d_model, H, dh) bytes.
 */
HSTU_API hstu_status hstu_block_fwd(void* x, const int64_t* seq_offsets, int32_t B, int32_t max_len,
                           int64_t T, int32_t n_layers, int32_t d_model, int32_t H, int32_t dh,
                           const void* const* w_uvqk, const void* const* w_o,
                           const hstu_rab* rab, float scale, float ln_eps, void* workspace,
                           size_t ws_bytes, cudaStream_t stream);
HSTU_API size_t hstu_block_workspace_size(int64_t T, int32_t d_model, int32_t H, int32_t dh);

/*
 * KV-cached serving step of the block stack ("NVIDIA Dynamo-Triton Gets
 * End-to-End HSTU Generative Recommender Workflow", sections "What the workflow
 * combines" and the benchmark: reusable key-value state is cached per layer so
 * long histories are not recomputed when new tokens arrive).  For each layer l:
 *   [U|V|Q|K] = SiLU(X @ w_uvqk[l]) for every row of x (new and candidate rows);
 *   the new rows' K, V are allocated pages in tables[l] and appended after the
 *     user's cached tokens;
 *   new rows attend causally over the user's cached tokens and the new rows
 *     (HSTU_MASK_CAUSAL_SUFFIX); candidate rows attend over the cached tokens
 *     (new ones included) and themselves only (HSTU_MASK_CANDIDATES: every
 *     candidate sits one position past the last cached token);
 *   G = LayerNorm(A) * U;  X = X + G @ w_o[l].
 * The result equals the uncached stack run over each user's whole sequence,
 * each candidate appended last on its own.
 *
 * tables: HOST array of n_layers tables (bf16, H heads of dh, one per layer),
 *   holding the same users with the same cached lengths.  A prefill is a call
 *   with no candidates on empty tables, the history passed as the new rows.
 * users: [B] device.  x: [T_new + T_cand, d_model] bf16, updated in place: the
 *   new rows (jagged by new_offsets, [B+1] device) first, then the candidate
 *   rows (jagged by cand_offsets, [B+1] device, counted from the first
 *   candidate row).  max_new / max_cand: per-user bounds.  max_cached: bound on
 *   any user's cached length after this step's append.
 * rab: position table only (no time term).  scale = 1/N for the attention.
 * Needs dh == 128, H*dh == d_model == 512, B <= 65535.
 * workspace: >= hstu_block_cached_workspace_size(...) bytes (0 = invalid
 *   arguments).  Page shortage or a duplicate user is recorded in the table's
 *   status word (read it with hstu_kv_table_status per layer).
 */
HSTU_API hstu_status hstu_block_cached_step(hstu_kv_table* const* tables, int32_t n_layers,
                                            const int64_t* users, int32_t B, void* x,
                                            const int64_t* new_offsets, int64_t T_new,
                                            int32_t max_new, const int64_t* cand_offsets,
                                            int64_t T_cand, int32_t max_cand, int32_t max_cached,
                                            int32_t d_model, int32_t H, int32_t dh,
                                            const void* const* w_uvqk, const void* const* w_o,
                                            const hstu_rab* rab, float scale, float ln_eps,
                                            void* workspace, size_t ws_bytes, cudaStream_t stream);
HSTU_API size_t hstu_block_cached_workspace_size(hstu_kv_table* const* tables, int32_t n_layers,
                                                 int32_t B, int64_t T_new, int64_t T_cand,
                                                 int32_t max_cand, int32_t max_cached,
                                                 int32_t d_model, int32_t H, int32_t dh);

/*
 * Beam-search decode attention over a shared context ("How Generative
 * Recommenders Are Redefining RecSys at Scale", section "Semantic ID-GR": a
 * request's long context is shared by all its beams (ContextKV), each beam has
 * a short decode history (BeamKV) and an ancestry (BeamPath)).  The attention
 * is the HSTU one used everywhere in this library.  At decode step `step` = s,
 * beam j of request b sits at position L_b + s (L_b = the request's cached
 * context length in table t, user users[b]) and attends to the context tokens
 * (positions 0 .. L_b-1), to the decode tokens of its ancestors at steps
 * 0 .. s-1 (positions L_b + t) and to its own token:
 *   out = scale * sum_j SiLU(q . k_j + rab(|p - p_j|)) v_j.
 * q: [total_beams, H, 128] bf16 device, this step's beam queries; requests'
 *   beams are jagged by beam_offsets ([B+1] device), the same rows every step.
 * beam_k, beam_v: [s+1][total_beams][H][128] bf16 device, the decode tokens' K
 *   and V of steps 0 .. s (row s = this step's own tokens).
 * beam_parent: [s+1][total_beams] int32 device (may be NULL when s == 0):
 *   beam_parent[t][r] = index, within its request, of the step t-1 beam that
 *   row r of step t extends.  max_ctx: bound on L_b.
 * rab: position table only.  workspace: >= hstu_attn_beam_decode_workspace_size.
 */
HSTU_API hstu_status hstu_attn_beam_decode(hstu_kv_table* t, const int64_t* users, int32_t B,
                                           const void* q, const int64_t* beam_offsets,
                                           int64_t total_beams, int32_t max_beams,
                                           int32_t max_ctx, int32_t step, const void* beam_k,
                                           const void* beam_v, const int32_t* beam_parent,
                                           const hstu_rab* rab, float scale, void* out,
                                           void* workspace, size_t ws_bytes, cudaStream_t stream);
HSTU_API size_t hstu_attn_beam_decode_workspace_size(hstu_kv_table* t, int32_t B,
                                                     int64_t total_beams, int32_t max_beams,
                                                     int32_t max_ctx, int32_t step);

/*
 * Sparse user-id -> dense slot map ("How Generative Recommenders Are Redefining
 * RecSys at Scale", section "Dynamic embedding": sparse ids are hashed onto
 * dense storage rows).  The slots (0 .. n_slots-1) name users of a KV table
 * (max_users = n_slots): pass the slots_out array as its `users`.
 *
 * create: slots start free on a LIFO stack initialised from host_free_order (a
 *   permutation of 0..n_slots-1, top = LAST element; NULL = 0..n_slots-1).
 * lookup: ids [B] int64 device, each >= 0; slots_out [B] int64 device.  A
 *   known id gets its slot.  With insert != 0 unknown ids take slots from the
 *   top of the stack in the order listed (a repeated id shares the slot of its
 *   first occurrence); with insert == 0 they get -1.  A negative id, or too
 *   few free slots for the call's new ids, leaves the map unchanged, writes -1
 *   everywhere and records HSTU_ERR_INVALID_ARG / HSTU_ERR_OUT_OF_PAGES (no
 *   free slot) in the map's status word.  B <= 65536.
 * erase: the listed ids' slots return to the stack in the order listed;
 *   unknown ids are ignored.  Pair it with hstu_kv_release of the same slots.
 * status: synchronises the stream, returns and clears the device error.
 */
typedef struct hstu_user_map hstu_user_map;
HSTU_API hstu_status hstu_user_map_create(int32_t n_slots, const int32_t* host_free_order,
                                          hstu_user_map** out_map);
HSTU_API void hstu_user_map_destroy(hstu_user_map* m);
HSTU_API hstu_status hstu_user_map_lookup(hstu_user_map* m, const int64_t* ids, int32_t B,
                                          int32_t insert, int64_t* slots_out, cudaStream_t stream);
HSTU_API hstu_status hstu_user_map_erase(hstu_user_map* m, const int64_t* ids, int32_t B,
                                         cudaStream_t stream);
HSTU_API hstu_status hstu_user_map_status(hstu_user_map* m, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_H_ */
