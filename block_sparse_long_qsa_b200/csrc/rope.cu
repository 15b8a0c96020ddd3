// RoPE on the keys (prefill) and the decode append.
//
// Rotary embedding with theta = 1e7 on dims 0..63 of every Q and K head
// (rope_dim 64 = partial_rotary_factor 0.25 of head_dim 256; page "Qwen3.8-
// Flash-Next, 1/9의 학습 비용으로 Qwen3.7-Plus(397B-A17B) 수준에 도달한 125B-A6B
// 모델", spec table and section "100만 토큰까지 늘리기").  Pairs are
// (i, i + 32); angle a = position * f_i with f_i = theta^(-i/32), or its
// static-YaRN version (section "100만 토큰까지 늘리기": rope_type yarn,
// factor 4) computed on the host, formed in fp64 so that positions near 2^20
// keep their phase, then rotated in fp32; with YaRN the rotated dims are also
// multiplied by the attention factor 0.1 ln(factor) + 1.
#include "qsa_device.cuh"
#include "qsa_kernels.h"

namespace qsa {
namespace {

// Frequencies of the 32 rotary pairs and the factor applied to the rotated
// dims (YaRN's attention factor; 1 for plain RoPE).
struct InvFreq { double f[32]; double scale; };

// cs[t][i] = scale * (cos a, sin a) for a = (pos0 + t) * inv_freq[i]
__global__ void rope_table_kernel(int64_t T, int64_t pos0, InvFreq inv, float2* __restrict__ cs) {
  const int64_t n = T * 32;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = e >> 5;
    const int i = (int)(e & 31);
    double sa, ca;
    sincos((double)(pos0 + t) * inv.f[i], &sa, &ca);
    cs[e] = make_float2((float)(inv.scale * ca), (float)(inv.scale * sa));
  }
}

__device__ __forceinline__ void rotate8(const uint4& lo, const uint4& hi, const float2* c8, uint4& olo, uint4& ohi) {
  // lo holds dims i..i+7, hi holds dims i+32..i+39
  const uint32_t* a = reinterpret_cast<const uint32_t*>(&lo);
  const uint32_t* b = reinterpret_cast<const uint32_t*>(&hi);
  uint32_t* oa = reinterpret_cast<uint32_t*>(&olo);
  uint32_t* ob = reinterpret_cast<uint32_t*>(&ohi);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float x0 = bf16lo(a[p]), x1 = bf16hi(a[p]);
    const float y0 = bf16lo(b[p]), y1 = bf16hi(b[p]);
    const float2 c0 = c8[2 * p], c1 = c8[2 * p + 1];
    oa[p] = pack_bf16x2(x0 * c0.x - y0 * c0.y, x1 * c1.x - y1 * c1.y);
    ob[p] = pack_bf16x2(y0 * c0.x + x0 * c0.y, y1 * c1.x + x1 * c1.y);
  }
}

// One thread per (token, kv head, 16-byte chunk slot): slots 0..3 rotate the
// chunk pairs (s, s+4) of dims 0..63, slots 4..27 copy chunks 8..31.
__global__ void rope_k_kernel(int64_t T, const uint4* __restrict__ k, const float2* __restrict__ cs,
                              uint4* __restrict__ k_rot) {
  const int64_t n = T * 2 * 28;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = e / 28;          // t * 2 + g
    const int slot = (int)(e - row * 28);
    const uint4* src = k + row * 32;
    uint4* dst = k_rot + row * 32;
    if (slot < 4) {
      const int64_t t = row >> 1;
      const uint4 lo = __ldg(src + slot), hi = __ldg(src + slot + 4);
      uint4 olo, ohi;
      rotate8(lo, hi, cs + t * 32 + 8 * slot, olo, ohi);
      dst[slot] = olo;
      dst[slot + 4] = ohi;
    } else {
      dst[slot + 4] = __ldg(src + slot + 4);
    }
  }
}

// Indexer queries of the mean-pooled indexer with block-start positions:
// out[t][h] = q_idx[t][h] with dims 0..63 rotated at position pos0 + t
// (pairs (i, i + 32); fp64 angle and rotation, rounded to bf16 once) and
// dims 64..127 copied.  One thread per (token, pair i): the pair's angle
// serves the 4 heads, and the thread copies one of the token's 32 16-byte
// chunks of unrotated dims (head i / 8, chunk i % 8).
__global__ void idx_rope_q_kernel(int64_t T, int64_t pos0, InvFreq inv, const uint16_t* __restrict__ q,
                                  uint16_t* __restrict__ out) {
  const int64_t n = T * 32;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = e >> 5;
    const int i = (int)(e & 31);
    double sa, ca;
    sincos((double)(pos0 + t) * inv.f[i], &sa, &ca);
    ca *= inv.scale;
    sa *= inv.scale;
    const uint16_t* src = q + t * 512;
    uint16_t* dst = out + t * 512;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const double x = (double)bf16_bits_to_f32(src[h * 128 + i]), y = (double)bf16_bits_to_f32(src[h * 128 + i + 32]);
      dst[h * 128 + i] = f64_to_bf16_rne(x * ca - y * sa);
      dst[h * 128 + i + 32] = f64_to_bf16_rne(y * ca + x * sa);
    }
    const int h = i >> 3, c = i & 7;
    reinterpret_cast<uint4*>(dst + h * 128 + 64)[c] = reinterpret_cast<const uint4*>(src + h * 128 + 64)[c];
  }
}

// Compressed keys with block-start positions: kbar[b] = bf16 of the mean of
// k_idx rows 4b .. min(4b + 4, T) - 1 (exact fp64 sum, one division), then
// dims 0..63 rotated at position pos0 + 4b (fp64, rounded to bf16 once
// more).  One thread per (block, j < 96): the pair (j, j + 32) for j < 32,
// else the unrotated dim j + 32.
__device__ __forceinline__ double kbar_mean_bf16(const uint16_t* __restrict__ rows, int n, int c) {
  double sum = 0.0;
  for (int r = 0; r < n; ++r) sum += (double)bf16_bits_to_f32(rows[r * 128 + c]);
  return (double)bf16_bits_to_f32(f64_to_bf16_rne(sum / (double)n));
}
__global__ void kbar_rope_kernel(const uint16_t* __restrict__ k_idx, int64_t T, int64_t nkb, int64_t pos0, InvFreq inv,
                                 uint16_t* __restrict__ kbar) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= nkb * 96) return;
  const int64_t b = e / 96;
  const int j = (int)(e - b * 96);
  const int64_t t0 = 4 * b;
  const int n = (int)(T - t0 < 4 ? T - t0 : 4);
  const uint16_t* rows = k_idx + t0 * 128;
  uint16_t* dst = kbar + b * 128;
  if (j < 32) {
    const double x = kbar_mean_bf16(rows, n, j), y = kbar_mean_bf16(rows, n, j + 32);
    double sa, ca;
    sincos((double)(pos0 + t0) * inv.f[j], &sa, &ca);
    ca *= inv.scale;
    sa *= inv.scale;
    dst[j] = f64_to_bf16_rne(x * ca - y * sa);
    dst[j + 32] = f64_to_bf16_rne(y * ca + x * sa);
  } else {
    dst[j + 32] = f64_to_bf16_rne(kbar_mean_bf16(rows, n, j + 32));
  }
}

// Decode append: one CTA per sequence.
//   k_cache[b][L] = RoPE(k_new[b], L); v_cache[b][L] = v_new[b];
//   kidx_cache[b][L] = k_idx_new[b]; ring slot L % 4 <- (q_idx_new[b], w_new[b]);
//   q_rot[b] = RoPE(q_new[b], L); with kbar_cache (mean pooling, [B][kbar_len][128])
//   the compressed key of block L/4 is recomputed from its present keys.
constexpr int LEN_CHUNK = 1024;
struct LenChunk { int64_t L[LEN_CHUNK]; int32_t b0; };

__global__ void decode_append_kernel(int64_t max_len, LenChunk lens, int64_t* __restrict__ L_dev,
                                     int64_t* __restrict__ qb_dev, InvFreq inv,
                                     uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                     uint4* __restrict__ kidx_cache, uint4* __restrict__ qidx_ring,
                                     uint16_t* __restrict__ w_ring, const uint4* __restrict__ q_new,
                                     const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                     const uint4* __restrict__ q_idx_new, const uint4* __restrict__ k_idx_new,
                                     const uint16_t* __restrict__ w_new, uint4* __restrict__ q_rot,
                                     uint16_t* __restrict__ kbar_cache, int64_t kbar_len,
                                     const int32_t* __restrict__ sel_in, const int32_t* __restrict__ cnt_in,
                                     int budget, int32_t* __restrict__ sel_r, int sel_r_ld,
                                     int32_t* __restrict__ cnt_r, uint32_t* err, int idx_rope,
                                     uint16_t* __restrict__ ring_rot) {
  __shared__ float2 cs[32];
  __shared__ double kmean[128];
  __shared__ int n_keep, first_neg;
  const int b = lens.b0 + blockIdx.x;
  const int64_t L = lens.L[blockIdx.x];
  if (threadIdx.x == 0) {
    L_dev[b] = L;
    qb_dev[b] = L >> 2;
    n_keep = 0;
    first_neg = budget;
  }
  if (sel_in != nullptr) {
    // Reused selection (an earlier step's top-k of this sequence): its blocks
    // below qb - 1, then the forced blocks qb - 1 and qb of this token.  The
    // given row must be ascending, distinct and causal (<= qb); otherwise the
    // step attends nothing and reports QSA_ERR_DEVICE_BOUNDS.  Without
    // counts a row ends at its first negative entry (the -1 padding of
    // sel_out).
    const int64_t qb = L >> 2;
    const int32_t* r = sel_in + (int64_t)b * budget;
    __syncthreads();   // n_keep, first_neg initialised
    if (cnt_in == nullptr) {
      for (int i = threadIdx.x; i < budget; i += blockDim.x)
        if (r[i] < 0) atomicMin(&first_neg, i);
      __syncthreads();
    }
    const int c = cnt_in != nullptr ? cnt_in[b] : first_neg;
    const bool c_ok = c >= 0 && c <= budget;
    int bad = !c_ok, keep = 0;
    for (int i = threadIdx.x; c_ok && i < c; i += blockDim.x) {
      const int32_t v = r[i];
      bad |= v < 0 || v > qb || (i > 0 && v <= r[i - 1]);
      keep += v < qb - 1;
    }
    if (keep) atomicAdd(&n_keep, keep);
    bad = __syncthreads_or(bad);
    const int m = n_keep;   // entries below qb - 1 form a prefix of an ascending row
    int32_t* o = sel_r + (int64_t)b * sel_r_ld;
    for (int i = threadIdx.x; !bad && i < m; i += blockDim.x) o[i] = r[i];
    if (threadIdx.x == 0) {
      if (qb >= 1) o[m] = (int32_t)(qb - 1);
      o[m + (qb >= 1)] = (int32_t)qb;
      cnt_r[b] = bad ? 0 : m + 1 + (qb >= 1);
      if (bad) report_error(err, QSA_ERR_DEVICE_BOUNDS);
    }
  }
  if (threadIdx.x < 32) {
    double sa, ca;
    sincos((double)L * inv.f[threadIdx.x], &sa, &ca);
    cs[threadIdx.x] = make_float2((float)(inv.scale * ca), (float)(inv.scale * sa));
  }
  __syncthreads();
  // rotated rows: 2 kv heads (k) + 24 q heads, 4 rotate slots each; copies of the rest
  const int n_rows = 2 + 24;
  for (int e = threadIdx.x; e < n_rows * 28; e += blockDim.x) {
    const int row = e / 28, slot = e % 28;
    const uint4* src = row < 2 ? k_new + ((int64_t)b * 2 + row) * 32 : q_new + ((int64_t)b * 24 + row - 2) * 32;
    uint4* dst = row < 2 ? k_cache + (((int64_t)b * max_len + L) * 2 + row) * 32
                         : q_rot + ((int64_t)b * 24 + row - 2) * 32;
    if (slot < 4) {
      uint4 olo, ohi;
      rotate8(src[slot], src[slot + 4], cs + 8 * slot, olo, ohi);
      dst[slot] = olo;
      dst[slot + 4] = ohi;
    } else {
      dst[slot + 4] = src[slot + 4];
    }
  }
  for (int e = threadIdx.x; e < 64; e += blockDim.x)            // v: 2 x 512 B
    v_cache[((int64_t)b * max_len + L) * 64 + e] = v_new[(int64_t)b * 64 + e];
  for (int e = threadIdx.x; e < 16; e += blockDim.x)            // k_idx: 256 B
    kidx_cache[((int64_t)b * max_len + L) * 16 + e] = k_idx_new[(int64_t)b * 16 + e];
  const int slot = (int)(L & 3);
  for (int e = threadIdx.x; e < 64; e += blockDim.x)            // q_idx: 4 x 256 B
    qidx_ring[((int64_t)b * 4 + slot) * 64 + e] = q_idx_new[(int64_t)b * 64 + e];
  if (threadIdx.x < 4) w_ring[((int64_t)b * 4 + slot) * 4 + threadIdx.x] = w_new[(int64_t)b * 4 + threadIdx.x];
  const int64_t t0 = L & ~(int64_t)3;     // first token of the new token's block
  if (kbar_cache != nullptr) {
    // mean of keys 4 qb .. L: the earlier ones from the cache, the new one from k_idx_new
    uint16_t* krow = kbar_cache + ((int64_t)b * kbar_len + (L >> 2)) * 128;
    if (threadIdx.x < 128) {
      const int c = threadIdx.x;
      const uint16_t* kc = reinterpret_cast<const uint16_t*>(kidx_cache) + (int64_t)b * max_len * 128;
      const uint16_t* kn = reinterpret_cast<const uint16_t*>(k_idx_new) + (int64_t)b * 128;
      double sum = 0.0;
      for (int64_t t = t0; t < L; ++t) sum += (double)__uint_as_float((uint32_t)kc[t * 128 + c] << 16);
      sum += (double)__uint_as_float((uint32_t)kn[c] << 16);
      const uint16_t m = f64_to_bf16_rne(sum / (double)(L - t0 + 1));
      if (idx_rope) kmean[c] = (double)bf16_bits_to_f32(m);
      else krow[c] = m;
    }
    if (idx_rope) {
      // the block's start position 4 qb: dims 0..63 rotated (fp64, one more rounding)
      __syncthreads();
      if (threadIdx.x < 32) {
        const int i = threadIdx.x;
        double sa, ca;
        sincos((double)t0 * inv.f[i], &sa, &ca);
        ca *= inv.scale;
        sa *= inv.scale;
        krow[i] = f64_to_bf16_rne(kmean[i] * ca - kmean[i + 32] * sa);
        krow[i + 32] = f64_to_bf16_rne(kmean[i + 32] * ca + kmean[i] * sa);
      } else if (threadIdx.x >= 64 && threadIdx.x < 128) {
        krow[threadIdx.x] = f64_to_bf16_rne(kmean[threadIdx.x]);
      }
    }
  }
  if (ring_rot != nullptr) {
    // indexer queries of the block-mates 4 qb .. L rotated at their positions
    // (the mean-pooled indexer with block-start positions): ring slot j holds
    // token 4 qb + j; the new token's own q_idx is read from q_idx_new
    const int present = (int)(L - t0) + 1;
    const uint16_t* ring16 = reinterpret_cast<const uint16_t*>(qidx_ring);
    const uint16_t* new16 = reinterpret_cast<const uint16_t*>(q_idx_new) + (int64_t)b * 512;
    for (int e = threadIdx.x; e < present * 32; e += blockDim.x) {
      const int tok = e >> 5, i = e & 31;
      const uint16_t* src = tok == slot ? new16 : ring16 + ((int64_t)b * 4 + tok) * 512;
      uint16_t* dst = ring_rot + ((int64_t)b * 4 + tok) * 512;
      double sa, ca;
      sincos((double)(t0 + tok) * inv.f[i], &sa, &ca);
      ca *= inv.scale;
      sa *= inv.scale;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const double x = (double)bf16_bits_to_f32(src[h * 128 + i]);
        const double y = (double)bf16_bits_to_f32(src[h * 128 + i + 32]);
        dst[h * 128 + i] = f64_to_bf16_rne(x * ca - y * sa);
        dst[h * 128 + i + 32] = f64_to_bf16_rne(y * ca + x * sa);
      }
      const int h = i >> 3, c = i & 7;
      reinterpret_cast<uint4*>(dst + h * 128 + 64)[c] = reinterpret_cast<const uint4*>(src + h * 128 + 64)[c];
    }
  }
}

// Verify append: block (sequence b, new token i) of a chunk of sequences puts
// token i at position pos = L_b + i: its key rotated at pos into k_cache, its
// value and indexer key into the caches, its queries rotated at pos into
// q_rot[b][i] and pos into Ls_tok[b][i]; block i = 0 also records L_b and the
// query blocks qb = L_b/4 + j (j < nqv; -1 past the last new token) that the
// verify scores.  The q_idx / w ring is left as it is (read-only here).
__global__ void verify_append_kernel(int64_t max_len, int m, int nqv, LenChunk lens, int64_t* __restrict__ Lb_dev,
                                     int64_t* __restrict__ Ls_tok, int64_t* __restrict__ row_qb, InvFreq inv,
                                     uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                     uint4* __restrict__ kidx_cache, const uint4* __restrict__ q_new,
                                     const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                     const uint4* __restrict__ k_idx_new, uint4* __restrict__ q_rot) {
  __shared__ float2 cs[32];
  const int bl = blockIdx.x / m, i = blockIdx.x % m;
  const int64_t b = lens.b0 + bl;
  const int64_t L = lens.L[bl];
  const int64_t pos = L + i;
  const int64_t tok = b * m + i;                       // token row [b][i]
  if (threadIdx.x == 0) {
    Ls_tok[tok] = pos;
    if (i == 0) {
      Lb_dev[b] = L;
      for (int j = 0; j < nqv; ++j) {
        const int64_t qb = (L >> 2) + j;
        row_qb[b * nqv + j] = 4 * qb <= L + m - 1 ? qb : -1;
      }
    }
  }
  if (threadIdx.x < 32) {
    double sa, ca;
    sincos((double)pos * inv.f[threadIdx.x], &sa, &ca);
    cs[threadIdx.x] = make_float2((float)(inv.scale * ca), (float)(inv.scale * sa));
  }
  __syncthreads();
  // rotated rows: 2 kv heads (k) + 24 q heads, 4 rotate slots each; copies of the rest
  for (int e = threadIdx.x; e < 26 * 28; e += blockDim.x) {
    const int row = e / 28, slot = e % 28;
    const uint4* src = row < 2 ? k_new + (tok * 2 + row) * 32 : q_new + (tok * 24 + row - 2) * 32;
    uint4* dst = row < 2 ? k_cache + ((b * max_len + pos) * 2 + row) * 32 : q_rot + (tok * 24 + row - 2) * 32;
    if (slot < 4) {
      uint4 olo, ohi;
      rotate8(src[slot], src[slot + 4], cs + 8 * slot, olo, ohi);
      dst[slot] = olo;
      dst[slot + 4] = ohi;
    } else {
      dst[slot + 4] = src[slot + 4];
    }
  }
  for (int e = threadIdx.x; e < 64; e += blockDim.x)            // v: 2 x 512 B
    v_cache[(b * max_len + pos) * 64 + e] = v_new[tok * 64 + e];
  for (int e = threadIdx.x; e < 16; e += blockDim.x)            // k_idx: 256 B
    kidx_cache[(b * max_len + pos) * 16 + e] = k_idx_new[tok * 16 + e];
}

InvFreq to_struct(const double* f, double scale) {
  InvFreq s;
  for (int i = 0; i < 32; ++i) s.f[i] = f[i];
  s.scale = scale;
  return s;
}

int grid_for(int64_t n, int threads) {
  int64_t g = (n + threads - 1) / threads;
  const int64_t cap = 148LL * 16;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

cudaError_t launch_rope_table(int64_t T, int64_t pos0, const double* inv_freq_host, double attn_factor, float2* cs,
                              cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  rope_table_kernel<<<grid_for(T * 32, 256), 256, 0, s>>>(T, pos0, to_struct(inv_freq_host, attn_factor), cs);
  return cudaGetLastError();
}

cudaError_t launch_rope_k(int64_t T, const uint16_t* k, const float2* cs, uint16_t* k_rot, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  rope_k_kernel<<<grid_for(T * 56, 256), 256, 0, s>>>(T, reinterpret_cast<const uint4*>(k), cs,
                                                        reinterpret_cast<uint4*>(k_rot));
  return cudaGetLastError();
}

cudaError_t launch_idx_rope_q(int64_t T, int64_t pos0, const double* inv_freq_host, double attn_factor,
                              const uint16_t* q_idx, uint16_t* out, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  idx_rope_q_kernel<<<grid_for(T * 32, 256), 256, 0, s>>>(T, pos0, to_struct(inv_freq_host, attn_factor), q_idx, out);
  return cudaGetLastError();
}

cudaError_t launch_kbar_rope(const uint16_t* k_idx, int64_t T, int64_t pos0, const double* inv_freq_host,
                             double attn_factor, uint16_t* kbar, cudaStream_t s) {
  const int64_t nkb = (T + 3) / 4;
  if (nkb <= 0) return cudaSuccess;
  const int64_t n = nkb * 96;
  kbar_rope_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(k_idx, T, nkb, pos0, to_struct(inv_freq_host, attn_factor),
                                                                kbar);
  return cudaGetLastError();
}

cudaError_t launch_decode_append(int B, int64_t max_len, const int64_t* L_host, int64_t* L_dev, int64_t* qb_dev,
                                 const double* inv_freq_host, double attn_factor, uint16_t* k_cache,
                                 uint16_t* v_cache, uint16_t* kidx_cache, uint16_t* qidx_ring, uint16_t* w_ring,
                                 const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new,
                                 const uint16_t* q_idx_new, const uint16_t* k_idx_new, const uint16_t* w_new,
                                 uint16_t* q_rot, uint16_t* kbar_cache, int64_t kbar_len, const int32_t* sel_in,
                                 const int32_t* cnt_in, int budget, int32_t* sel_r, int sel_r_ld, int32_t* cnt_r,
                                 uint32_t* err, cudaStream_t s, bool idx_rope, uint16_t* ring_rot) {
  const InvFreq inv = to_struct(inv_freq_host, attn_factor);
  for (int b0 = 0; b0 < B; b0 += LEN_CHUNK) {
    const int n = B - b0 < LEN_CHUNK ? B - b0 : LEN_CHUNK;
    LenChunk lens;
    lens.b0 = b0;
    for (int i = 0; i < n; ++i) lens.L[i] = L_host[b0 + i];
    decode_append_kernel<<<n, 256, 0, s>>>(
        max_len, lens, L_dev, qb_dev, inv, reinterpret_cast<uint4*>(k_cache), reinterpret_cast<uint4*>(v_cache),
        reinterpret_cast<uint4*>(kidx_cache), reinterpret_cast<uint4*>(qidx_ring), w_ring,
        reinterpret_cast<const uint4*>(q_new), reinterpret_cast<const uint4*>(k_new),
        reinterpret_cast<const uint4*>(v_new), reinterpret_cast<const uint4*>(q_idx_new),
        reinterpret_cast<const uint4*>(k_idx_new), w_new, reinterpret_cast<uint4*>(q_rot), kbar_cache, kbar_len,
        sel_in, cnt_in, budget, sel_r, sel_r_ld, cnt_r, err, idx_rope ? 1 : 0, ring_rot);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_verify_append(int B, int m, int nqv, int64_t max_len, const int64_t* L_host, int64_t* Lb_dev,
                                 int64_t* Ls_tok, int64_t* row_qb, const double* inv_freq_host, double attn_factor,
                                 uint16_t* k_cache, uint16_t* v_cache, uint16_t* kidx_cache, const uint16_t* q_new,
                                 const uint16_t* k_new, const uint16_t* v_new, const uint16_t* k_idx_new,
                                 uint16_t* q_rot, cudaStream_t s) {
  const InvFreq inv = to_struct(inv_freq_host, attn_factor);
  for (int b0 = 0; b0 < B; b0 += LEN_CHUNK) {
    const int n = B - b0 < LEN_CHUNK ? B - b0 : LEN_CHUNK;
    LenChunk lens;
    lens.b0 = b0;
    for (int i = 0; i < n; ++i) lens.L[i] = L_host[b0 + i];
    verify_append_kernel<<<n * m, 256, 0, s>>>(
        max_len, m, nqv, lens, Lb_dev, Ls_tok, row_qb, inv, reinterpret_cast<uint4*>(k_cache),
        reinterpret_cast<uint4*>(v_cache), reinterpret_cast<uint4*>(kidx_cache), reinterpret_cast<const uint4*>(q_new),
        reinterpret_cast<const uint4*>(k_new), reinterpret_cast<const uint4*>(v_new),
        reinterpret_cast<const uint4*>(k_idx_new), reinterpret_cast<uint4*>(q_rot));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace qsa
