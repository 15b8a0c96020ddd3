/*
 * qsa.h -- C ABI of the QSA (Qwen Sparse Attention) hot path for NVIDIA B200 (sm_100a).
 *
 * QSA is the micro-block sparse global attention layer described on the page
 * "Qwen3.8-Flash-Next, 1/9의 학습 비용으로 Qwen3.7-Plus(397B-A17B) 수준에 도달한
 * 125B-A6B 모델" (discuss.pytorch.kr), cited below as [PT]; section
 * "QSA: 인덱서 자체의 비용을 줄이는 희소 어텐션" ([PT §QSA]) and its spec table.
 * It runs in three stages:
 *   1. an MQA indexer (4 query heads, one shared 128-dim key head) scores the
 *      causal key micro-blocks of r = 4 tokens for every query micro-block;
 *   2. a top-k step keeps `budget_blocks` = 512 blocks (2048 tokens) per query
 *      block, always including the query block itself and the one before it;
 *   3. GQA softmax attention (24 Q heads, 2 KV heads, head dim 256, RoPE with
 *      theta = 1e7 on dims 0..63) runs over the selected blocks only.
 *
 * Conventions (all calls):
 *   - Every pointer argument is a DEVICE pointer unless marked "host", 16-byte
 *     aligned, to a contiguous row-major array with the layout given.  bf16
 *     values travel as uint16_t bit patterns.
 *   - The caller owns every buffer, the workspace included; the library
 *     allocates no device memory.  Its only global state is the one-time
 *     kernel attribute setup per device and the fixed 64 MiB scratch array
 *     of qsa_decode_noalloc (reserved where that code is loaded).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Arguments are validated on the host before any launch; on an
 *     argument error nothing is launched.
 *   - Errors come back as a qsa_status; nothing aborts or throws.  Errors
 *     detected on the device (a bounded wait that timed out) are recorded in
 *     the workspace's error word and read back by qsa_check_device_error.
 *   - Positions: token t of a prefill sits at position pos0 + t.
 */
#ifndef QSA_H_
#define QSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = 1,         /* null pointer, negative size, bad range */
  QSA_ERR_UNSUPPORTED = 2,         /* shape other than the one this library implements */
  QSA_ERR_MISALIGNED = 3,          /* a pointer is not 16-byte aligned */
  QSA_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes below the *_workspace_size minimum */
  QSA_ERR_CUDA = 5,                /* a CUDA runtime / driver call failed */
  QSA_ERR_DEVICE_TIMEOUT = 6,      /* a device-side bounded wait gave up */
  QSA_ERR_DEVICE_BOUNDS = 7,       /* a device-side index check failed */
  QSA_ERR_ARCH = 8                 /* the current device is not sm_100 */
} qsa_status;

/* Layer shape.  The implemented (and only accepted) values are the ones of
 * [PT] spec table ("Qwen Sparse Attention", "QSA 인덱서", "QSA 예산") and of the
 * rope_parameters listing in [PT] section "100만 토큰까지 늘리기":
 * n_q_heads 24, n_kv_heads 2, head_dim 256, rope_dim 64, rope_theta 1e7,
 * idx_heads 4, idx_dim 128, block_size 4; budget_blocks is free in [2, 4096]
 * (default 512).  softmax_scale 0 means 1/sqrt(head_dim).
 * aggregation picks the block score of stage 1 (default QSA_AGG_TOKEN_MAX):
 *   QSA_AGG_TOKEN_MAX: S(qb, kb) = max over the causal token pairs (t in qb,
 *     j in kb, j <= t) of s(t, j);
 *   QSA_AGG_MEAN_POOL ([PT §QSA]: each micro-block's keys are mean-pooled
 *     into one compressed key k-bar_b, and every query token scores the
 *     compressed keys, O(n^2 / r)): k-bar_kb = bf16 (round to nearest even)
 *     of the mean of block kb's present indexer keys (exact sum, one fp64
 *     division); S(qb, kb) = max over the present tokens t of block qb of
 *     sum_h w_h(t) ReLU(q_idx_h(t) . k-bar_kb) / sqrt(128), for kb <= qb (the
 *     own block's entry uses all its present keys and never decides a
 *     selection: the own block is always kept).  qsa_decode returns
 *     QSA_ERR_UNSUPPORTED for it; decode with it is qsa_decode_mean_pool. */
enum { QSA_AGG_TOKEN_MAX = 0, QSA_AGG_MEAN_POOL = 1 };
typedef struct {
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t rope_dim;
  double rope_theta;
  int32_t idx_heads;
  int32_t idx_dim;
  int32_t block_size;
  int32_t budget_blocks;
  float softmax_scale;
  int32_t aggregation;
  /* Static YaRN on the rotary dims ([PT] "100만 토큰까지 늘리기": rope_type
   * yarn, factor 4.0, original_max_position_embeddings 262144).  yarn_factor
   * <= 1 (the default, 0) is plain RoPE.  With s = yarn_factor > 1 each
   * rotary pair i keeps its frequency f_i = theta^(-i/32) if its wavelength
   * fits more than yarn_beta_fast (default 32) times into
   * yarn_original_max tokens, gets f_i / s if it fits fewer than
   * yarn_beta_slow (default 1) times, and a linear mix in i in between
   * (ends: the indices where the count crosses the two betas, rounded down /
   * up); the rotated dims of q and k are multiplied by 0.1 ln s + 1. */
  double yarn_factor;
  double yarn_original_max;
  double yarn_beta_fast;
  double yarn_beta_slow;
  /* Block-start position of the mean-pooled indexer ([PT §QSA]: the keys of
   * a micro-block are compressed before the positional step and the
   * compressed key gets one block-start position).  0 (default): the indexer
   * has no positional encoding.  1 (only with QSA_AGG_MEAN_POOL): the
   * indexer queries of token t are rotated at t's position and the compressed
   * key of block b at the position of its first token, 4b, with this layer's
   * RoPE (dims 0..63 of the 128, pairs (i, i + 32), theta and YaRN as above);
   * the rotation is computed in fp64 and each rotated operand is rounded to
   * bf16 once (the compressed key after its mean was rounded to bf16).
   * Positions: pos0 + t in qsa_prefill, t in qsa_index_scores and
   * qsa_mean_pool_keys, the cache position in the decode calls.
   * qsa_prefill_cached and qsa_verify return QSA_ERR_UNSUPPORTED with it. */
  int32_t idx_rope;
} qsa_params;

/* Fills *p with the values above (budget 512). */
void qsa_default_params(qsa_params* p);

/* Human-readable name of a status code (static storage). */
const char* qsa_status_string(qsa_status s);

/* Description of the last failing CUDA step of a call made by this thread
 * (e.g. the CUDA error string of a rejected launch); "" if none yet.  Valid
 * until the thread's next failing call. */
const char* qsa_last_error(void);

/* Stage 1 -- indexer block scores ([PT §QSA], eq. I_ib, with the head
 * weights and causal block-max of this library's reading):
 *   s(t, j)   = sum_h w[t][h] * ReLU(q_idx[t][h] . k_idx[j]) / sqrt(idx_dim)
 *   S(qb, kb) = max over tokens t of block qb (t < T) and j of block kb with
 *               j <= t of s(t, j),   for kb <= qb.
 * q_idx [T][4][128] bf16, w [T][4] bf16, k_idx [T][128] bf16.
 * Writes scores[(qb - qb_begin) * ld + kb] (fp32) for qb in [qb_begin, qb_end)
 * and kb <= qb; entries with kb > qb are not written.
 * Requires 0 <= qb_begin <= qb_end <= ceil(T/4), ld >= qb_end, ld % 4 == 0.
 * With p->aggregation == QSA_AGG_MEAN_POOL the scores are the mean-pooled ones
 * (see qsa_params).
 * ws: at least qsa_index_workspace_size bytes (the device error word, and the
 * compressed keys for mean pooling); with the token-pair block score ws may be
 * NULL, and a device-side timeout is then not reported (the kernel still
 * exits). */
qsa_status qsa_index_workspace_size(const qsa_params* p, int64_t T, size_t* bytes);
qsa_status qsa_index_scores(const qsa_params* p, int64_t T, const uint16_t* q_idx, const uint16_t* w,
                            const uint16_t* k_idx, int64_t qb_begin, int64_t qb_end, float* scores, int64_t ld,
                            void* ws, size_t ws_bytes, void* stream);

/* Stage 2 -- block selection ([PT §QSA]: token budget K = 2048, r = 4, so
 * 512 blocks; the tail of the own block is always included).  For query
 * block qb (row qb - qb_begin of `scores`, entries kb <= qb valid):
 *   qb + 1 <= budget: all blocks 0..qb;
 *   otherwise: qb and qb-1, plus the (budget-2) blocks of [0, qb-2] with the
 *   highest score (ties to the lower block index; -0.0 counts as +0.0).
 * sel [qb_end-qb_begin][budget] int32 ascending, padded with -1; cnt [..] int32.
 * ws: at least qsa_select_workspace_size() bytes (holds the error word). */
qsa_status qsa_select_blocks(const qsa_params* p, const float* scores, int64_t ld, int64_t qb_begin,
                             int64_t qb_end, int32_t* sel, int32_t* cnt, void* ws, size_t ws_bytes, void* stream);
qsa_status qsa_select_workspace_size(const qsa_params* p, size_t* bytes);

/* Whole prefill: RoPE on Q and K, stage 1, stage 2 and stage 3 (sparse GQA
 * attention over the selected blocks, causal inside the own block):
 *   out[t][h] = sum_j softmax_j(q_rot[t][h] . k_rot[j][h/12] * scale) v[j][h/12]
 *   over j in the selected blocks of block t/4 with j <= t;
 *   lse[t][h] = log sum_j exp(logit_j).
 * q [T][24][256], k [T][2][256] (not rotated), v [T][2][256], q_idx [T][4][128],
 * w [T][4], k_idx [T][128]: bf16.  out [T][24][256] bf16.
 * Optional (NULL to skip): lse [T][24] fp32; sel_out [ceil(T/4)][budget] and
 * cnt_out [ceil(T/4)] int32; k_rot_out [T][2][256] bf16 (the rotated keys, to
 * seed a decode cache).
 * ws: at least the minimum of qsa_prefill_workspace_size; a larger workspace
 * lets the call score more query blocks per pass (fewer, larger launches). */
qsa_status qsa_prefill(const qsa_params* p, int64_t T, int64_t pos0, const uint16_t* q, const uint16_t* k,
                       const uint16_t* v, const uint16_t* q_idx, const uint16_t* w, const uint16_t* k_idx,
                       uint16_t* out, float* lse, int32_t* sel_out, int32_t* cnt_out, uint16_t* k_rot_out, void* ws,
                       size_t ws_bytes, void* stream);
/* min_bytes: smallest workspace qsa_prefill accepts; pref_bytes: the size
 * that scores every query block in one pass, capped at 16 GiB (either
 * pointer may be NULL). */
qsa_status qsa_prefill_workspace_size(const qsa_params* p, int64_t T, size_t* min_bytes, size_t* pref_bytes);

/* Prefill of T_new new tokens after L_old tokens already in a cache (the
 * prefix-cached serving case of [PT §QSA] "100만 토큰까지 늘리기": most of a
 * long prompt is cached and only the rest is prefilled).  Equals the last
 * T_new rows of qsa_prefill over all L_old + T_new tokens with pos0 = 0:
 * the new tokens' query blocks qb = L_old/4 .. (L_old+T_new-1)/4 are scored
 * over every key block up to their own, selected as in stage 2, and attend
 * over the selected cached and new keys.
 * Caches (bf16, at least L_old + T_new rows, rows [0, L_old) given):
 *   k_cache [..][2][256] rotated keys, v_cache [..][2][256], kidx_cache
 *   [..][128]; rows [L_old, L_old + T_new) are written by this call (the new
 *   keys rotated at positions L_old ..), as a decode append would.
 * qidx_prev [L_old % 4][4][128], w_prev [L_old % 4][4]: indexer queries and
 *   head weights of the tokens 4*(L_old/4) .. L_old-1 that share the first
 *   new query block (NULL allowed when L_old % 4 == 0).
 * New tokens [T_new]: q [..][24][256], k, v [..][2][256] (k not rotated),
 *   q_idx [..][4][128], w [..][4], k_idx [..][128].
 * Outputs: out [T_new][24][256] bf16; lse [T_new][24] fp32 (nullable);
 *   sel_out [nq][budget], cnt_out [nq] (nullable) for the nq new query blocks.
 * ws: at least the minimum of qsa_prefill_cached_workspace_size. */
qsa_status qsa_prefill_cached(const qsa_params* p, int64_t L_old, int64_t T_new, uint16_t* k_cache,
                              uint16_t* v_cache, uint16_t* kidx_cache, const uint16_t* qidx_prev,
                              const uint16_t* w_prev, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                              const uint16_t* q_idx, const uint16_t* w, const uint16_t* k_idx, uint16_t* out,
                              float* lse, int32_t* sel_out, int32_t* cnt_out, void* ws, size_t ws_bytes,
                              void* stream);
qsa_status qsa_prefill_cached_workspace_size(const qsa_params* p, int64_t L_old, int64_t T_new, size_t* min_bytes,
                                             size_t* pref_bytes);

/* One decode step for B sequences.  Sequence b has cache_len[b] (host array)
 * tokens already in its caches; the new token sits at position
 * L = cache_len[b] and is appended: k_cache[b][L] = RoPE(k_new[b], L),
 * v_cache[b][L] = v_new[b], kidx_cache[b][L] = k_idx_new[b],
 * qidx_ring[b][L % 4] = q_idx_new[b], w_ring[b][L % 4] = w_new[b].
 * The new token's query block qb = L / 4 is scored over the present
 * block-mates 4*qb .. L (their indexer queries come from the ring, which the
 * caller seeds for tokens 4*qb .. L-1 when the decode starts mid-block), the
 * blocks are selected as in stage 2, and attention for the new token runs over
 * them -- by construction what a prefill of L+1 tokens gives for its last
 * token ([PT §QSA]; the full KV cache is kept).  The caller increments
 * cache_len afterwards.
 * k_cache, v_cache [B][max_len][2][256] bf16 (keys rotated); kidx_cache
 * [B][max_len][128]; qidx_ring [B][4][4][128]; w_ring [B][4][4];
 * q_new [B][24][256]; k_new, v_new [B][2][256]; q_idx_new [B][4][128];
 * k_idx_new [B][128]; w_new [B][4]  ->  out [B][24][256] bf16;
 * sel_out [B][budget] int32 (nullable), lse_out [B][24] fp32 (nullable).
 * Requires cache_len[b] < max_len, B <= 4096.
 * Attention is split-KV: each (sequence, KV head) is cut into 1..16 ranges of
 * whole 16-block tiles, chosen so the batch fills the GPU's SMs; with more
 * than one range a combine kernel merges the ranges' partial outputs by their
 * log-sum-exp (qsa_set_decode_splits fixes the number of ranges). */
qsa_status qsa_decode(const qsa_params* p, int32_t B, int64_t max_len, const int64_t* cache_len,
                      uint16_t* k_cache, uint16_t* v_cache, uint16_t* kidx_cache, uint16_t* qidx_ring,
                      uint16_t* w_ring, const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new,
                      const uint16_t* q_idx_new, const uint16_t* k_idx_new, const uint16_t* w_new, uint16_t* out,
                      int32_t* sel_out, float* lse_out, void* ws, size_t ws_bytes, void* stream);
qsa_status qsa_decode_workspace_size(const qsa_params* p, int32_t B, int64_t max_len, size_t* bytes);

/* A tuning and test aid with no counterpart on the pages: n in 1..16 fixes
 * the number of split-KV ranges of every later decode-attention launch of
 * this process (all decode calls, verify included); n = 0 restores the
 * automatic choice.  Returns QSA_ERR_INVALID_ARG outside 0..16.  Takes
 * effect at the next call; calls already enqueued keep their split. */
qsa_status qsa_set_decode_splits(int32_t n);

/* qsa_decode for p->aggregation == QSA_AGG_MEAN_POOL.  kbar_cache
 * [B][ceil(max_len/4)][128] bf16 holds the compressed key of every block:
 * block kb's row is bf16 (round to nearest even) of the mean of its present
 * indexer keys (qsa_mean_pool_keys builds it from a k_idx cache).  The call
 * appends the new token as qsa_decode does and rewrites the row of its block
 * L/4 from the block's present keys (the cached ones and k_idx_new), then
 * scores the compressed keys: the decode indexer reads one 256-byte row per
 * block instead of four.  Same workspace as qsa_decode. */
qsa_status qsa_decode_mean_pool(const qsa_params* p, int32_t B, int64_t max_len, const int64_t* cache_len,
                                uint16_t* k_cache, uint16_t* v_cache, uint16_t* kidx_cache, uint16_t* kbar_cache,
                                uint16_t* qidx_ring, uint16_t* w_ring, const uint16_t* q_new, const uint16_t* k_new,
                                const uint16_t* v_new, const uint16_t* q_idx_new, const uint16_t* k_idx_new,
                                const uint16_t* w_new, uint16_t* out, int32_t* sel_out, float* lse_out, void* ws,
                                size_t ws_bytes, void* stream);
/* One draft decode step that reuses an earlier step's top-k ([PT] section
 * "추측 디코딩을 위한 MTP와 그 밖에 유지된 설계": the MTP draft layer keeps the
 * top-k indices across the steps of one speculative round, as GLM-5 does, so
 * the later draft steps pay neither the indexer nor the top-k).  The new token
 * is appended exactly as by qsa_decode (and, with p->aggregation ==
 * QSA_AGG_MEAN_POOL, its block's compressed key is rewritten in kbar_cache as
 * by qsa_decode_mean_pool; kbar_cache must be NULL otherwise).  Stages 1 and 2
 * do not run: the attended blocks of sequence b are the blocks of
 * sel_in[b][0 .. cnt_in[b]) below qb - 1, followed by the forced blocks
 * qb - 1 (when qb >= 1) and qb of the new token (qb = cache_len[b] / 4), so a
 * reused row taken in an earlier query block still attends the token's own
 * block and the one before it; at most cnt_in[b] + 2 blocks.
 * sel_in [B][budget] int32, cnt_in [B] int32 (device; nullable): typically
 * sel_out of the round's first qsa_decode step.  With cnt_in NULL a row ends
 * at its first negative entry (the -1 padding of sel_out), else it holds
 * cnt_in[b] entries.  Each row must be ascending, distinct and causal
 * (entries in 0 .. qb, 0 <= cnt_in[b] <= budget); a row that is not attends
 * nothing and QSA_ERR_DEVICE_BOUNDS is recorded in the workspace.  Other arguments,
 * outputs and the workspace are those of qsa_decode. */
qsa_status qsa_decode_reuse(const qsa_params* p, int32_t B, int64_t max_len, const int64_t* cache_len,
                            uint16_t* k_cache, uint16_t* v_cache, uint16_t* kidx_cache, uint16_t* kbar_cache,
                            uint16_t* qidx_ring, uint16_t* w_ring, const uint16_t* q_new, const uint16_t* k_new,
                            const uint16_t* v_new, const uint16_t* q_idx_new, const uint16_t* k_idx_new,
                            const uint16_t* w_new, const int32_t* sel_in, const int32_t* cnt_in, uint16_t* out,
                            float* lse_out, void* ws, size_t ws_bytes, void* stream);
/* Batched verify of m new tokens per sequence (the target pass of a
 * speculative round, [PT] "추측 디코딩을 위한 MTP와 그 밖에 유지된 설계"):
 * sequence b has cache_len[b] (host array) tokens in its caches and its new
 * tokens sit at positions L = cache_len[b] .. L + m - 1.  The result is, for
 * every sequence, what qsa_prefill_cached gives with L_old = L and
 * T_new = m: each query block the new tokens touch is scored over all its
 * present tokens (prefill semantics: a block's selection sees every present
 * block-mate, later new tokens included), selected as in stage 2, and every
 * new token attends its block's selection causally.
 * The new tokens are appended to the caches at L .. L + m - 1 (k rotated),
 * as m decode steps would; the q_idx / w ring is only read: qidx_prev
 * [B][4][4][128] and w_prev [B][4][4] hold, in slot t % 4, the indexer
 * queries and head weights of the block-mates 4*(L/4) .. L-1 (a decode ring
 * can be passed as is; NULL allowed when every cache_len[b] % 4 == 0).
 * q_new [B][m][24][256], k_new, v_new [B][m][2][256], q_idx_new
 * [B][m][4][128], k_idx_new [B][m][128], w_new [B][m][4]  ->  out
 * [B][m][24][256] bf16, sel_out [B][m][budget] int32 (nullable: each token's
 * block selection, -1 padded), lse_out [B][m][24] fp32 (nullable).
 * Requires 1 <= m <= 16, cache_len[b] + m <= max_len, B <= 4096.
 * With p->aggregation == QSA_AGG_MEAN_POOL, kbar_cache [B][ceil(max_len/4)]
 * [128] is the compressed-key cache (as for qsa_decode_mean_pool): the rows
 * of the blocks the new tokens touch are rewritten from their present keys
 * and the blocks are scored over the compressed keys; kbar_cache must be
 * NULL otherwise.
 * Kernels: the decode append (per new token), the decode indexer over up to
 * (m + 2) / 4 + 1 query blocks per sequence, the select, a per-token copy
 * of the block's selection, and the split-KV decode attention with one row
 * per new token. */
qsa_status qsa_verify(const qsa_params* p, int32_t B, int32_t m, int64_t max_len, const int64_t* cache_len,
                      uint16_t* k_cache, uint16_t* v_cache, uint16_t* kidx_cache, uint16_t* kbar_cache,
                      const uint16_t* qidx_prev,
                      const uint16_t* w_prev, const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new,
                      const uint16_t* q_idx_new, const uint16_t* k_idx_new, const uint16_t* w_new, uint16_t* out,
                      int32_t* sel_out, float* lse_out, void* ws, size_t ws_bytes, void* stream);
qsa_status qsa_verify_workspace_size(const qsa_params* p, int32_t B, int32_t m, int64_t max_len, size_t* bytes);

/* kbar [ceil(T/4)][128] = the compressed keys of k_idx [T][128] (block b: bf16
 * of the mean of rows 4b .. min(4b+4, T)-1); no workspace; asynchronous. */
qsa_status qsa_mean_pool_keys(const qsa_params* p, int64_t T, const uint16_t* k_idx, uint16_t* kbar, void* stream);

/* qsa_decode without a workspace argument; the pages have no counterpart:
 * this exists for callers that cannot allocate device memory where they run
 * a decode step (their device memory belongs to another runtime's budget, or
 * cudaMalloc is not allowed on their request path).  The caller still owns
 * and passes every input, output and cache, exactly as for qsa_decode; the
 * decode scratch instead lives in a 64 MiB array inside this library.
 *   - The array is reserved on a device when the library's decode code is
 *     loaded there: with CUDA's default lazy module loading, at the first
 *     call of this entry point on that device.  That first call maps the
 *     64 MiB (it can fail under memory pressure and can synchronise), so
 *     make it once at initialisation, outside the request path and outside
 *     any stream capture.  Later calls allocate nothing; the array stays
 *     reserved until the process exits.
 *   - Sizes whose qsa_decode_workspace_size exceeds 64 MiB are rejected with
 *     QSA_ERR_WORKSPACE_TOO_SMALL before any launch (64 sequences at 256K
 *     context need about 41 MiB).
 *   - Every call looks up the array's device address for the current device
 *     (cudaGetSymbolAddress, a host-side lookup once the code is loaded).
 *   - All calls share the one array per device: calls whose executions
 *     overlap on the GPU (different streams, or different host threads on the
 *     same device) race on it and must be serialised by the caller.
 *   - Device-side errors are recorded in the array's error word; read them
 *     with qsa_decode_noalloc_check_error. */
qsa_status qsa_decode_noalloc(const qsa_params* p, int32_t B, int64_t max_len, const int64_t* cache_len,
                              uint16_t* k_cache, uint16_t* v_cache, uint16_t* kidx_cache, uint16_t* qidx_ring,
                              uint16_t* w_ring, const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new,
                              const uint16_t* q_idx_new, const uint16_t* k_idx_new, const uint16_t* w_new,
                              uint16_t* out, int32_t* sel_out, float* lse_out, void* stream);
/* The device error word of qsa_decode_noalloc's array on the current device:
 * synchronises `stream` and returns QSA_OK or the device-side error that the
 * most recent qsa_decode_noalloc call on this device recorded (each call
 * clears the word when it starts), then clears it. */
qsa_status qsa_decode_noalloc_check_error(void* stream);

/* Reads (synchronising `stream`) and clears the device error word at the
 * start of a workspace passed to qsa_select_blocks / qsa_prefill /
 * qsa_decode.  Returns QSA_OK or the first device-side error recorded. */
qsa_status qsa_check_device_error(void* ws, void* stream);

/* Launch tracing, a measurement aid with no counterpart on the pages.
 * Between qsa_trace_begin and qsa_trace_end every kernel this library
 * launches (on any stream, in any call) is bracketed by two CUDA events
 * recorded on its launching stream, for up to `capacity` launches (later
 * launches are not traced).  qsa_trace_end waits for the last traced launch,
 * writes up to `capacity` (kernel id, milliseconds) pairs in launch order,
 * sets *n_out to the number written and releases the events.  Not
 * re-entrant: one trace at a time per process.  Kernel ids: */
enum {
  QSA_KERNEL_ROPE_TABLE = 1,
  QSA_KERNEL_ROPE_K = 2,
  QSA_KERNEL_INDEXER = 3,
  QSA_KERNEL_SELECT = 4,
  QSA_KERNEL_ATTENTION = 5,
  QSA_KERNEL_DECODE_APPEND = 6,
  QSA_KERNEL_DECODE_INDEXER = 7,
  QSA_KERNEL_DECODE_ATTENTION = 8,
  QSA_KERNEL_DECODE_COMBINE = 9,
  QSA_KERNEL_KBAR = 10,
  QSA_KERNEL_VERIFY_EXPAND = 11,
  QSA_KERNEL_IDX_ROPE = 12
};
qsa_status qsa_trace_begin(int32_t capacity);
qsa_status qsa_trace_end(int32_t* kernel_ids, float* ms, int32_t capacity, int32_t* n_out);

#ifdef __cplusplus
}
#endif
#endif /* QSA_H_ */
