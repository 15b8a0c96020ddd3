// Decode: indexer block scores of the new token's query block over the whole
// indexer-key cache (the decode step's dominant HBM stream).
//
// Same score as prefill (page "Qwen3.8-Flash-Next, 1/9의 학습 비용으로 Qwen3.7-
// Plus(397B-A17B) 수준에 도달한 125B-A6B 모델", section "QSA: 인덱서 자체의 비용을
// 줄이는 희소 어텐션", eq. I_ib with this library's head weights and causal
// block max): for the block qb = L/4 of the new token at position L, the
// query tokens are the present block-mates 4qb .. L (from the ring) and
// S(qb, kb) = max over those tokens t and keys j of block kb, j <= t, of
// sum_h w_h(t) ReLU(q_idx_h(t) . k_idx(j)) / sqrt(128).
//
// Kernel: 16 keys x 16 (token, head) columns per bf16 tensor-core MMA
// (m16n8k16, two n-tiles).  The dot product is a sum over the 128 dims, so
// the dims may be assigned to MMA k-slots in any order as long as A and B
// agree: each thread loads 16 contiguous bytes (8 dims) of a key row straight
// from global memory into its A fragment registers for two k-steps, and the
// query fragments use the same assignment.  No shared memory; every load is a
// full 32-byte sector.  Column n of n-tile nt is (token n/2, head 2*nt + n%2),
// so a thread's accumulators hold all 4 heads of one token for two keys.
#include "qsa_device.cuh"
#include "qsa_kernels.h"

namespace qsa {
namespace {

constexpr int THREADS = 128;
constexpr int KEYS_PER_CTA = 2048;

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// MEAN: the rows are mean-pooled key blocks (kbar_cache [B][kbar_len][128])
// and S(qb, kb) is the max over the present block-mates of their score
// against kbar[kb] (no per-key causal test: kb <= qb); otherwise the rows are
// keys and S is the max over causal token pairs.
// VER (verify, token-pair scores only): S row r scores query block
// row_qb[r] of sequence r / nqv, whose m new tokens sit at L .. L + m - 1
// (L = Ls[b], the length before them); the block's tokens before L take their
// q_idx / w from the ring (slot = position % 4), the new ones from
// qidx_new / w_new [B][m][...].  row_qb[r] < 0: nothing to score.
template <bool MEAN, bool VER>
__global__ void __launch_bounds__(THREADS)
decode_indexer_kernel(int64_t max_len, const int64_t* __restrict__ Ls, const uint16_t* __restrict__ kidx_cache,
                      const uint16_t* __restrict__ kbar_cache, int64_t kbar_len,
                      const uint16_t* __restrict__ qidx_ring, const uint16_t* __restrict__ w_ring,
                      float* __restrict__ S, int64_t ld, float scale, const int64_t* __restrict__ row_qb, int nqv,
                      int m, const uint16_t* __restrict__ qidx_new, const uint16_t* __restrict__ w_new) {
  const int64_t row = blockIdx.y;
  const int64_t b = VER ? row / nqv : row;
  const int64_t L = Ls[b];
  const int64_t qb = VER ? row_qb[row] : L >> 2;
  if (VER && qb < 0) return;
  const int64_t pos_end = VER ? L + m - 1 : L;        // last present token
  const int64_t last_key = 4 * qb + 3 < pos_end ? 4 * qb + 3 : pos_end;
  const int64_t last_row = MEAN ? qb : last_key;       // last row with data
  const int64_t j_begin = (int64_t)blockIdx.x * KEYS_PER_CTA;
  if (j_begin > last_row) return;
  int64_t j_end = j_begin + KEYS_PER_CTA;
  const int64_t rows_end = MEAN ? qb + 1 : 4 * qb + 4;
  if (j_end > rows_end) j_end = rows_end;
  const int present = (int)(last_key - 4 * qb) + 1;   // block-mates 4qb .. last_key

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g8 = lane >> 2, q4 = lane & 3;

  // B fragments: column g8 -> (token g8/2, head 2*nt + g8%2), dims 32*d + 8*q4 .. +7
  uint4 qf[2][4];
  {
    const int tok = g8 >> 1;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int head = 2 * nt + (g8 & 1);
      const int64_t pos = 4 * qb + tok;
      const uint4* src = reinterpret_cast<const uint4*>(
          VER && pos >= L ? qidx_new + ((b * m + (pos - L)) * 4 + head) * 128
                          : qidx_ring + ((b * 4 + tok) * 4 + head) * 128);
#pragma unroll
      for (int d = 0; d < 4; ++d) qf[nt][d] = tok < present ? src[4 * d + q4] : make_uint4(0, 0, 0, 0);
    }
  }
  // head weights of this thread's token q4
  float w[4];
  {
    const bool ok = q4 < present;
    const int64_t pos = 4 * qb + q4;
#pragma unroll
    for (int h = 0; h < 4; ++h)
      w[h] = ok ? bf16_bits_to_f32(VER && pos >= L ? w_new[(b * m + (pos - L)) * 4 + h] : w_ring[(b * 4 + q4) * 4 + h])
                : 0.f;
  }
  const int64_t t_tok = 4 * qb + q4;                 // this thread's query token
  const bool tok_ok = q4 < present;
  const uint16_t* kb_base = MEAN ? kbar_cache + b * kbar_len * 128 : kidx_cache + b * max_len * 128;
  float* Srow = S + row * ld;

  // the next tile's 16 keys are loaded while the current tile is scored
  constexpr int64_t STEP = 16 * (THREADS / 32);
  auto load_tile = [&](int64_t jt, uint4 (&k0)[4], uint4 (&k1)[4]) {
    const int64_t j0 = jt + g8, j1 = jt + g8 + 8;
    const int64_t r0 = j0 <= last_row ? j0 : last_row, r1 = j1 <= last_row ? j1 : last_row;
    const uint4* k0p = reinterpret_cast<const uint4*>(kb_base + r0 * 128);
    const uint4* k1p = reinterpret_cast<const uint4*>(kb_base + r1 * 128);
#pragma unroll
    for (int d = 0; d < 4; ++d) { k0[d] = ldg_stream(k0p + 4 * d + q4); k1[d] = ldg_stream(k1p + 4 * d + q4); }
  };
  uint4 n0[4], n1[4];
  if (j_begin + 16 * warp < j_end) load_tile(j_begin + 16 * warp, n0, n1);
  for (int64_t jt = j_begin + 16 * warp; jt < j_end; jt += STEP) {
    const int64_t j0 = jt + g8, j1 = jt + g8 + 8;
    uint4 k0[4], k1[4];
#pragma unroll
    for (int d = 0; d < 4; ++d) { k0[d] = n0[d]; k1[d] = n1[d]; }
    if (jt + STEP < j_end) load_tile(jt + STEP, n0, n1);
    float acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
    for (int d = 0; d < 4; ++d) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        mma16816(acc[nt], k0[d].x, k1[d].x, k0[d].y, k1[d].y, qf[nt][d].x, qf[nt][d].y);
        mma16816(acc[nt], k0[d].z, k1[d].z, k0[d].w, k1[d].w, qf[nt][d].z, qf[nt][d].w);
      }
    }
    // acc[nt][0..1]: key j0, heads 2nt, 2nt+1 of token q4; acc[nt][2..3]: key j1
    float s0 = w[0] * fmaxf(acc[0][0], 0.f);
    s0 = fmaf(w[1], fmaxf(acc[0][1], 0.f), s0);
    s0 = fmaf(w[2], fmaxf(acc[1][0], 0.f), s0);
    s0 = fmaf(w[3], fmaxf(acc[1][1], 0.f), s0);
    float s1 = w[0] * fmaxf(acc[0][2], 0.f);
    s1 = fmaf(w[1], fmaxf(acc[0][3], 0.f), s1);
    s1 = fmaf(w[2], fmaxf(acc[1][2], 0.f), s1);
    s1 = fmaf(w[3], fmaxf(acc[1][3], 0.f), s1);
    if constexpr (MEAN) {
      s0 = (tok_ok && j0 <= qb) ? s0 : 0.f;
      s1 = (tok_ok && j1 <= qb) ? s1 : 0.f;
      // max over the 4 tokens (lanes q4); rows j0, j1 are key blocks
#pragma unroll
      for (int off = 1; off <= 2; off <<= 1) {
        s0 = fmaxf(s0, __shfl_xor_sync(0xffffffffu, s0, off));
        s1 = fmaxf(s1, __shfl_xor_sync(0xffffffffu, s1, off));
      }
      if (q4 == 0) {
        if (j0 <= qb) Srow[j0] = s0 * scale;
        if (j1 <= qb) Srow[j1] = s1 * scale;
      }
    } else {
      s0 = (tok_ok && j0 <= t_tok) ? s0 : 0.f;
      s1 = (tok_ok && j1 <= t_tok) ? s1 : 0.f;
      // max over the 4 tokens (lanes q4), then over the 4 keys of a block (g8 % 4)
#pragma unroll
      for (int off = 1; off <= 8; off <<= 1) {
        s0 = fmaxf(s0, __shfl_xor_sync(0xffffffffu, s0, off));
        s1 = fmaxf(s1, __shfl_xor_sync(0xffffffffu, s1, off));
      }
      if ((lane & 15) == 0) {
        const int64_t kb0 = (jt >> 2) + (lane >> 4);     // lane 0: blocks +0 / +2, lane 16: +1 / +3
        if (kb0 <= qb) Srow[kb0] = s0 * scale;
        if (kb0 + 2 <= qb) Srow[kb0 + 2] = s1 * scale;
      }
    }
  }
}

// Verify whose new tokens touch two query blocks per sequence (nqv == 2):
// one CTA row per sequence scores both blocks against each key tile it
// loads, so the key cache is read once per call.  Same scores as the
// one-block kernel: rows b * 2 + jb of S for blocks row_qb[b * 2 + jb]
// (row_qb[b * 2 + 1] < 0: the new tokens stay in the first block).
__global__ void __launch_bounds__(THREADS)
verify_indexer2_kernel(int64_t max_len, const int64_t* __restrict__ Ls, const uint16_t* __restrict__ kidx_cache,
                       const uint16_t* __restrict__ qidx_ring, const uint16_t* __restrict__ w_ring,
                       float* __restrict__ S, int64_t ld, float scale, const int64_t* __restrict__ row_qb, int m,
                       const uint16_t* __restrict__ qidx_new, const uint16_t* __restrict__ w_new) {
  const int64_t b = blockIdx.y;
  const int64_t L = Ls[b];
  const int64_t pos_end = L + m - 1;
  const int64_t qbv[2] = {row_qb[2 * b], row_qb[2 * b + 1]};
  const bool two = qbv[1] >= 0;
  const int64_t qb_last = two ? qbv[1] : qbv[0];
  const int64_t last_row = 4 * qb_last + 3 < pos_end ? 4 * qb_last + 3 : pos_end;
  const int64_t j_begin = (int64_t)blockIdx.x * KEYS_PER_CTA;
  if (j_begin > last_row) return;
  int64_t j_end = j_begin + KEYS_PER_CTA;
  if (j_end > 4 * qb_last + 4) j_end = 4 * qb_last + 4;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g8 = lane >> 2, q4 = lane & 3;
  uint4 qf[2][2][4];
  float w[2][4];
  int64_t t_tok[2];
  bool tok_ok[2];
#pragma unroll
  for (int jb = 0; jb < 2; ++jb) {
    const int64_t qb = qbv[jb];
    const int64_t lk = 4 * qb + 3 < pos_end ? 4 * qb + 3 : pos_end;
    const int present = qb < 0 ? 0 : (int)(lk - 4 * qb) + 1;
    const int tok = g8 >> 1;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int head = 2 * nt + (g8 & 1);
      const int64_t pos = 4 * qb + tok;
      const uint4* src = reinterpret_cast<const uint4*>(pos >= L ? qidx_new + ((b * m + (pos - L)) * 4 + head) * 128
                                                                 : qidx_ring + ((b * 4 + tok) * 4 + head) * 128);
#pragma unroll
      for (int d = 0; d < 4; ++d) qf[jb][nt][d] = tok < present ? src[4 * d + q4] : make_uint4(0, 0, 0, 0);
    }
    const int64_t pos = 4 * qb + q4;
#pragma unroll
    for (int h = 0; h < 4; ++h)
      w[jb][h] = q4 < present ? bf16_bits_to_f32(pos >= L ? w_new[(b * m + (pos - L)) * 4 + h]
                                                          : w_ring[(b * 4 + q4) * 4 + h])
                              : 0.f;
    t_tok[jb] = pos;
    tok_ok[jb] = q4 < present;
  }
  const uint16_t* kb_base = kidx_cache + b * max_len * 128;

  constexpr int64_t STEP = 16 * (THREADS / 32);
  auto load_tile = [&](int64_t jt, uint4 (&k0)[4], uint4 (&k1)[4]) {
    const int64_t j0 = jt + g8, j1 = jt + g8 + 8;
    const int64_t r0 = j0 <= last_row ? j0 : last_row, r1 = j1 <= last_row ? j1 : last_row;
    const uint4* k0p = reinterpret_cast<const uint4*>(kb_base + r0 * 128);
    const uint4* k1p = reinterpret_cast<const uint4*>(kb_base + r1 * 128);
#pragma unroll
    for (int d = 0; d < 4; ++d) { k0[d] = ldg_stream(k0p + 4 * d + q4); k1[d] = ldg_stream(k1p + 4 * d + q4); }
  };
  uint4 n0[4], n1[4];
  if (j_begin + 16 * warp < j_end) load_tile(j_begin + 16 * warp, n0, n1);
  for (int64_t jt = j_begin + 16 * warp; jt < j_end; jt += STEP) {
    const int64_t j0 = jt + g8, j1 = jt + g8 + 8;
    uint4 k0[4], k1[4];
#pragma unroll
    for (int d = 0; d < 4; ++d) { k0[d] = n0[d]; k1[d] = n1[d]; }
    if (jt + STEP < j_end) load_tile(jt + STEP, n0, n1);
#pragma unroll
    for (int jb = 0; jb < 2; ++jb) {
      if (jb == 1 && !two) break;
      const int64_t qb = qbv[jb];
      float acc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
      for (int d = 0; d < 4; ++d) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          mma16816(acc[nt], k0[d].x, k1[d].x, k0[d].y, k1[d].y, qf[jb][nt][d].x, qf[jb][nt][d].y);
          mma16816(acc[nt], k0[d].z, k1[d].z, k0[d].w, k1[d].w, qf[jb][nt][d].z, qf[jb][nt][d].w);
        }
      }
      float s0 = w[jb][0] * fmaxf(acc[0][0], 0.f);
      s0 = fmaf(w[jb][1], fmaxf(acc[0][1], 0.f), s0);
      s0 = fmaf(w[jb][2], fmaxf(acc[1][0], 0.f), s0);
      s0 = fmaf(w[jb][3], fmaxf(acc[1][1], 0.f), s0);
      float s1 = w[jb][0] * fmaxf(acc[0][2], 0.f);
      s1 = fmaf(w[jb][1], fmaxf(acc[0][3], 0.f), s1);
      s1 = fmaf(w[jb][2], fmaxf(acc[1][2], 0.f), s1);
      s1 = fmaf(w[jb][3], fmaxf(acc[1][3], 0.f), s1);
      s0 = (tok_ok[jb] && j0 <= t_tok[jb]) ? s0 : 0.f;
      s1 = (tok_ok[jb] && j1 <= t_tok[jb]) ? s1 : 0.f;
#pragma unroll
      for (int off = 1; off <= 8; off <<= 1) {
        s0 = fmaxf(s0, __shfl_xor_sync(0xffffffffu, s0, off));
        s1 = fmaxf(s1, __shfl_xor_sync(0xffffffffu, s1, off));
      }
      if ((lane & 15) == 0) {
        float* Srow = S + (2 * b + jb) * ld;
        const int64_t kb0 = (jt >> 2) + (lane >> 4);
        if (kb0 <= qb) Srow[kb0] = s0 * scale;
        if (kb0 + 2 <= qb) Srow[kb0 + 2] = s1 * scale;
      }
    }
  }
}

}  // namespace

cudaError_t launch_decode_indexer(int B, int64_t max_len, int64_t max_L, const int64_t* L_dev,
                                  const uint16_t* kidx_cache, const uint16_t* kbar_cache, int64_t kbar_len,
                                  const uint16_t* qidx_ring, const uint16_t* w_ring, float* S, int64_t ld,
                                  float scale, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  const int64_t rows = kbar_cache ? max_L / 4 + 1 : max_L + 4;
  const int64_t nx = (rows + KEYS_PER_CTA - 1) / KEYS_PER_CTA;
  dim3 grid((unsigned)nx, (unsigned)B);
  if (kbar_cache)
    decode_indexer_kernel<true, false><<<grid, THREADS, 0, s>>>(max_len, L_dev, kidx_cache, kbar_cache, kbar_len,
                                                                qidx_ring, w_ring, S, ld, scale, nullptr, 1, 1,
                                                                nullptr, nullptr);
  else
    decode_indexer_kernel<false, false><<<grid, THREADS, 0, s>>>(max_len, L_dev, kidx_cache, nullptr, 0, qidx_ring,
                                                                 w_ring, S, ld, scale, nullptr, 1, 1, nullptr, nullptr);
  return cudaGetLastError();
}

cudaError_t launch_verify_indexer(int B, int nqv, int m, int64_t max_len, int64_t max_L, const int64_t* Lb_dev,
                                  const int64_t* row_qb, const uint16_t* kidx_cache, const uint16_t* kbar_cache,
                                  int64_t kbar_len, const uint16_t* qidx_ring, const uint16_t* w_ring,
                                  const uint16_t* qidx_new, const uint16_t* w_new, float* S, int64_t ld, float scale,
                                  cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  if (kbar_cache) {   // mean pool: rows are the compressed key blocks 0 .. qb
    const int64_t nkb = (max_L + m + 3) / 4 + 1;
    const int64_t nxb = (nkb + KEYS_PER_CTA - 1) / KEYS_PER_CTA;
    decode_indexer_kernel<true, true><<<dim3((unsigned)nxb, (unsigned)(B * nqv)), THREADS, 0, s>>>(
        max_len, Lb_dev, kidx_cache, kbar_cache, kbar_len, qidx_ring, w_ring, S, ld, scale, row_qb, nqv, m, qidx_new,
        w_new);
    return cudaGetLastError();
  }
  const int64_t rows = max_L + m + 3;                 // keys up to the last new token's block end
  const int64_t nx = (rows + KEYS_PER_CTA - 1) / KEYS_PER_CTA;
  if (nqv == 2) {
    verify_indexer2_kernel<<<dim3((unsigned)nx, (unsigned)B), THREADS, 0, s>>>(max_len, Lb_dev, kidx_cache, qidx_ring,
                                                                               w_ring, S, ld, scale, row_qb, m,
                                                                               qidx_new, w_new);
    return cudaGetLastError();
  }
  dim3 grid((unsigned)nx, (unsigned)(B * nqv));
  decode_indexer_kernel<false, true><<<grid, THREADS, 0, s>>>(max_len, Lb_dev, kidx_cache, nullptr, 0, qidx_ring,
                                                              w_ring, S, ld, scale, row_qb, nqv, m, qidx_new, w_new);
  return cudaGetLastError();
}

// Compressed keys of the query blocks a verify touches, from the caches after
// the append: row r = (b, j) rewrites kbar[b][row_qb[r]] as the bf16 (round
// to nearest even) of the exact mean of the block's present keys.
__global__ void verify_kbar_kernel(int m, int nqv, int64_t max_len, int64_t kbar_len, const int64_t* __restrict__ Lb,
                                   const int64_t* __restrict__ row_qb, const uint16_t* __restrict__ kidx_cache,
                                   uint16_t* __restrict__ kbar_cache) {
  const int64_t r = blockIdx.x, b = r / nqv;
  const int64_t qb = row_qb[r];
  if (qb < 0) return;
  const int64_t t0 = 4 * qb, t_end = Lb[b] + m;     // present keys t0 .. t_end - 1 (at most 4)
  const int n = (int)(t_end - t0 < 4 ? t_end - t0 : 4);
  const int c = threadIdx.x;
  const uint16_t* kc = kidx_cache + b * max_len * 128;
  double sum = 0.0;
  for (int i = 0; i < n; ++i) sum += (double)__uint_as_float((uint32_t)kc[(t0 + i) * 128 + c] << 16);
  kbar_cache[(b * kbar_len + qb) * 128 + c] = f64_to_bf16_rne(sum / (double)n);
}

cudaError_t launch_verify_kbar(int B, int m, int nqv, int64_t max_len, int64_t kbar_len, const int64_t* Lb,
                               const int64_t* row_qb, const uint16_t* kidx_cache, uint16_t* kbar_cache,
                               cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  verify_kbar_kernel<<<B * nqv, 128, 0, s>>>(m, nqv, max_len, kbar_len, Lb, row_qb, kidx_cache, kbar_cache);
  return cudaGetLastError();
}

// Token row t = (b, i) of a verify takes the selection of its query block:
// row b * nqv + (pos / 4 - L_b / 4) of sel_blk / cnt_blk, pos = Ls_tok[t].
__global__ void verify_expand_kernel(int m, int nqv, int budget, const int64_t* __restrict__ Ls_tok,
                                     const int32_t* __restrict__ sel_blk, const int32_t* __restrict__ cnt_blk,
                                     int32_t* __restrict__ sel_tok, int32_t* __restrict__ cnt_tok) {
  const int64_t t = blockIdx.x;
  const int64_t b = t / m;
  const int64_t j = (Ls_tok[t] >> 2) - (Ls_tok[b * m] >> 2);
  const int64_t r = b * nqv + j;
  for (int e = threadIdx.x; e < budget; e += blockDim.x) sel_tok[t * budget + e] = sel_blk[r * budget + e];
  if (threadIdx.x == 0) cnt_tok[t] = cnt_blk[r];
}

cudaError_t launch_verify_expand(int B, int m, int nqv, int budget, const int64_t* Ls_tok, const int32_t* sel_blk,
                                 const int32_t* cnt_blk, int32_t* sel_tok, int32_t* cnt_tok, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  verify_expand_kernel<<<B * m, 128, 0, s>>>(m, nqv, budget, Ls_tok, sel_blk, cnt_blk, sel_tok, cnt_tok);
  return cudaGetLastError();
}

}  // namespace qsa
