// Internal launchers of the QSA kernels (not part of the C ABI).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "qsa_debug.h"   // the fault-injection codes of the debug build's tests

namespace qsa {

// Debug build (QSA_DEBUG_HOOKS) only: returns `code` (a QSA_INJECT_* of
// qsa_debug.h) if the fault injection that qsa_debug_inject armed is `code`,
// disarming it (so it applies to one launch); otherwise 0.  Release builds
// return 0 and compile no injection code.
#ifdef QSA_DEBUG_HOOKS
int take_debug_injection(int code);
#else
inline int take_debug_injection(int) { return 0; }
#endif

// RoPE angles of positions pos0 .. pos0+T-1: cs[t][i] = attn_factor * (cos a,
// sin a), a = (pos0 + t) * inv_freq[i], i < 32, angle formed in fp64.
cudaError_t launch_rope_table(int64_t T, int64_t pos0, const double* inv_freq_host, double attn_factor, float2* cs,
                              cudaStream_t s);
// k_rot[t][g] = RoPE(k[t][g]) on dims 0..63, dims 64..255 copied.
cudaError_t launch_rope_k(int64_t T, const uint16_t* k, const float2* cs, uint16_t* k_rot, cudaStream_t s);

// Block scores of query blocks [qb_begin, qb_end) into S (row stride ld, only
// kb <= qb written).  segmax (nullable, row stride ld_seg): per row, the max
// over each segment of 8 key blocks (segment s = blocks 8s .. 8s+7, blocks
// after the row's own block counting as 0).  Keys are tokens [0, T) of tm_k;
// the query rows (tm_q) and w start at token q_tok0 (<= 4 * qb_begin).
// mean_pool: tm_k holds the mean-pooled block keys [ceil(T/4)][128] (launch_kbar)
// and S(qb, kb) = max over the present tokens t of block qb of the score of t
// against kbar[kb]; otherwise tm_k holds the keys [T][128] and S is the max over
// causal token pairs.
cudaError_t launch_indexer_prefill(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const uint16_t* w,
                                   float* S, int64_t ld, float* segmax, int64_t ld_seg, int64_t T, int64_t q_tok0,
                                   int64_t qb_begin, int64_t qb_end, bool mean_pool, float scale, uint32_t* err,
                                   int num_sms, cudaStream_t stream);
// kbar[b] = bf16 round-to-nearest-even of the mean of k_idx rows 4b .. min(4b+4, T)-1.
cudaError_t launch_kbar(const uint16_t* k_idx, int64_t T, uint16_t* kbar, cudaStream_t stream);
// The mean-pooled indexer with block-start positions: kbar as launch_kbar,
// then dims 0..63 rotated at position pos0 + 4b (fp64, rounded to bf16).
cudaError_t launch_kbar_rope(const uint16_t* k_idx, int64_t T, int64_t pos0, const double* inv_freq_host,
                             double attn_factor, uint16_t* kbar, cudaStream_t stream);
// out[t] = q_idx[t] ([T][4][128]) with dims 0..63 of every head rotated at
// position pos0 + t (fp64, rounded to bf16), dims 64..127 copied.
cudaError_t launch_idx_rope_q(int64_t T, int64_t pos0, const double* inv_freq_host, double attn_factor,
                              const uint16_t* q_idx, uint16_t* out, cudaStream_t stream);

// Top-k block selection, one row per query block.  Row r covers query block
// row_qb ? row_qb[r] : qb_begin + r, read from S + r * ld.  segmax (nullable,
// row stride ld_seg): the indexer's maxima over segments of 8 key blocks; with
// it, long rows are filtered from the segment maxima instead of a full pass.
size_t select_smem_bytes(int budget);
cudaError_t launch_select(const float* S, int64_t ld, const float* segmax, int64_t ld_seg, int64_t qb_begin,
                          int64_t n_rows, const int64_t* row_qb, int budget, int32_t* sel, int32_t* cnt, uint32_t* err,
                          cudaStream_t stream);

// Sparse GQA attention for query blocks [qb_begin, qb_end) given their
// selections (sel/cnt indexed from qb_begin): tcgen05 kernel, persistent.
// Keys k_rot / v are tokens [0, T); q, the RoPE table cs, out and lse start at
// token q_tok0 (tokens before it in the first block get no output).
cudaError_t launch_sparse_attn_prefill_tc(int64_t T, const uint16_t* q, const uint16_t* k_rot, const uint16_t* v,
                                          const float2* cs, const int32_t* sel, const int32_t* cnt, int budget,
                                          int64_t qb_begin, int64_t qb_end, int64_t q_tok0, float scale_log2,
                                          uint16_t* out, float* lse, uint32_t* err, int num_sms,
                                          cudaStream_t stream);

// ---------------------------------------------------------------- decode
// Lengths come from the host array L_host (passed to the kernel as launch
// parameters) and are stored to L_dev / qb_dev for the later kernels.
cudaError_t launch_decode_append(int B, int64_t max_len, const int64_t* L_host, int64_t* L_dev, int64_t* qb_dev,
                                 const double* inv_freq_host, double attn_factor,
                                 uint16_t* k_cache, uint16_t* v_cache, uint16_t* kidx_cache, uint16_t* qidx_ring,
                                 uint16_t* w_ring, const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new,
                                 const uint16_t* q_idx_new, const uint16_t* k_idx_new, const uint16_t* w_new,
                                 uint16_t* q_rot, uint16_t* kbar_cache, int64_t kbar_len, const int32_t* sel_in,
                                 const int32_t* cnt_in, int budget, int32_t* sel_r, int sel_r_ld, int32_t* cnt_r,
                                 uint32_t* err, cudaStream_t s, bool idx_rope = false, uint16_t* ring_rot = nullptr);
// kbar_cache (nullable, [B][kbar_len][128]): score the mean-pooled key blocks
// (aggregation = mean pool) instead of the keys.
cudaError_t launch_decode_indexer(int B, int64_t max_len, int64_t max_L, const int64_t* L_dev,
                                  const uint16_t* kidx_cache, const uint16_t* kbar_cache, int64_t kbar_len,
                                  const uint16_t* qidx_ring, const uint16_t* w_ring, float* S, int64_t ld,
                                  float scale, cudaStream_t s);
// Decode attention for B sequences (one new token each, rotated queries
// q_rot [B][24][256]): the tcgen05 attention kernel over the cached K / V.
// Split-KV decode attention: each (sequence, KV head) is cut into n_split
// ranges of 16-block tiles.  n_split == 1 writes out / lse directly; otherwise
// the ranges write part_o [B][2][n_split][12][256] fp32 and part_lse
// [B][2][n_split][12] (base 2) and launch_decode_combine merges them.
cudaError_t launch_decode_attn_tc(int B, int64_t max_len, const int64_t* L_dev, const uint16_t* q_rot,
                                  const uint16_t* k_cache, const uint16_t* v_cache, const int32_t* sel,
                                  const int32_t* cnt, int budget, float scale_log2, int n_split, float* part_o,
                                  float* part_lse, uint16_t* out, float* lse, uint32_t* err, int num_sms,
                                  cudaStream_t stream, int rows_per_seq = 1);
// Verify (m new tokens per sequence at L_b .. L_b + m - 1, nqv query-block
// rows per sequence): append the tokens, score the query blocks they touch
// (block tokens before L_b from the ring), and give each token row its
// block's selection.
cudaError_t launch_verify_append(int B, int m, int nqv, int64_t max_len, const int64_t* L_host, int64_t* Lb_dev,
                                 int64_t* Ls_tok, int64_t* row_qb, const double* inv_freq_host, double attn_factor,
                                 uint16_t* k_cache, uint16_t* v_cache, uint16_t* kidx_cache, const uint16_t* q_new,
                                 const uint16_t* k_new, const uint16_t* v_new, const uint16_t* k_idx_new,
                                 uint16_t* q_rot, cudaStream_t s);
// kbar_cache non-null: mean-pooled scores over the compressed keys.
cudaError_t launch_verify_indexer(int B, int nqv, int m, int64_t max_len, int64_t max_L, const int64_t* Lb_dev,
                                  const int64_t* row_qb, const uint16_t* kidx_cache, const uint16_t* kbar_cache,
                                  int64_t kbar_len, const uint16_t* qidx_ring, const uint16_t* w_ring,
                                  const uint16_t* qidx_new, const uint16_t* w_new, float* S, int64_t ld, float scale,
                                  cudaStream_t s);
cudaError_t launch_verify_kbar(int B, int m, int nqv, int64_t max_len, int64_t kbar_len, const int64_t* Lb,
                               const int64_t* row_qb, const uint16_t* kidx_cache, uint16_t* kbar_cache,
                               cudaStream_t s);
cudaError_t launch_verify_expand(int B, int m, int nqv, int budget, const int64_t* Ls_tok, const int32_t* sel_blk,
                                 const int32_t* cnt_blk, int32_t* sel_tok, int32_t* cnt_tok, cudaStream_t s);
cudaError_t launch_decode_combine(int B, const float* part_o, const float* part_lse, const int32_t* cnt, int n_split,
                                  uint16_t* out, float* lse, cudaStream_t stream);

}  // namespace qsa
