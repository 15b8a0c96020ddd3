// Seeded synthetic inputs for the QSA hot path (test and benchmark infrastructure).
//
// One counter-based generator, compiled twice from this one source: once for
// the host (OpenMP loops) and once as CUDA kernels.  Every value is a pure
// function of (seed, stream, element index), so any element of any tensor can
// be regenerated on the host to feed the CPU oracle, and the device fill gives
// bit-identical values.  Bit-identity holds because the arithmetic below uses
// only IEEE operations that are correctly rounded everywhere (+, -, *, /,
// sqrt), with contraction into FMA disabled on both sides (the build passes
// --fmad=false and -ffp-contract=off); the logarithm, cosine and exponential
// are short series written here from their Taylor / atanh expansions, not
// library calls.
//
// This file holds none of the attention method's arithmetic: only random
// numbers, a softmax of four of them (the head-weight distribution the
// workloads ask for), and the "planted block" construction of the workloads
// (keys = mean of a query block's indexer queries + 0.3 * noise).

#include <stdint.h>
#include <math.h>
#include <cuda_runtime.h>

#define GEN_HD __host__ __device__ __forceinline__

// ---------------------------------------------------------------- counters --
// SplitMix64 finaliser (Steele, Lea, Flood 2014).
GEN_HD uint64_t gen_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Counter-based draw: SplitMix64 state sequence key + (idx+1)*golden, where
// the key itself is a mix of (seed, stream).
GEN_HD uint64_t gen_u64(uint64_t seed, uint32_t stream, uint64_t idx) {
  uint64_t key = gen_mix64(seed * 0xD1B54A32D192ED03ull + (uint64_t)stream * 0x9E3779B97F4A7C15ull
                           + 0x632BE59BD9B4E019ull);
  return gen_mix64(key + (idx + 1ull) * 0x9E3779B97F4A7C15ull);
}

// (0, 1] with 53 random bits.
GEN_HD double gen_u01_open0(uint64_t r) { return (double)((r >> 11) + 1ull) * (1.0 / 9007199254740992.0); }
// [0, 1) with 53 random bits.
GEN_HD double gen_u01(uint64_t r) { return (double)(r >> 11) * (1.0 / 9007199254740992.0); }

// ------------------------------------------------------------ series math --
// ln(x) for x in (0, 1]: x = m * 2^e with m in [sqrt(1/2), sqrt(2)),
// ln m = 2 * atanh(s), s = (m-1)/(m+1), atanh by its odd power series.
GEN_HD double gen_ln(double x) {
  union { double d; uint64_t u; } b; b.d = x;
  int e = (int)((b.u >> 52) & 0x7FF) - 1023;
  b.u = (b.u & 0x000FFFFFFFFFFFFFull) | 0x3FF0000000000000ull;   // m in [1, 2)
  double m = b.d;
  if (m > 1.4142135623730951) { m = m * 0.5; e = e + 1; }
  double s = (m - 1.0) / (m + 1.0);
  double s2 = s * s;
  double p = 1.0 / 29.0;
  p = p * s2 + 1.0 / 27.0; p = p * s2 + 1.0 / 25.0; p = p * s2 + 1.0 / 23.0;
  p = p * s2 + 1.0 / 21.0; p = p * s2 + 1.0 / 19.0; p = p * s2 + 1.0 / 17.0;
  p = p * s2 + 1.0 / 15.0; p = p * s2 + 1.0 / 13.0; p = p * s2 + 1.0 / 11.0;
  p = p * s2 + 1.0 / 9.0;  p = p * s2 + 1.0 / 7.0;  p = p * s2 + 1.0 / 5.0;
  p = p * s2 + 1.0 / 3.0;  p = p * s2 + 1.0;
  return (double)e * 0.6931471805599453 + 2.0 * s * p;
}

// sin and cos of t in [0, pi/4] by Taylor series (error far below 1e-17).
GEN_HD void gen_sincos_small(double t, double* s_out, double* c_out) {
  double t2 = t * t;
  double s = 1.0 / 6227020800.0;            // 1/13!
  s = 1.0 / 39916800.0 - t2 * s;            // 1/11!
  s = 1.0 / 362880.0 - t2 * s;              // 1/9!
  s = 1.0 / 5040.0 - t2 * s;                // 1/7!
  s = 1.0 / 120.0 - t2 * s;                 // 1/5!
  s = 1.0 / 6.0 - t2 * s;                   // 1/3!
  s = 1.0 - t2 * s;
  double c = 1.0 / 87178291200.0;           // 1/14!
  c = 1.0 / 479001600.0 - t2 * c;           // 1/12!
  c = 1.0 / 3628800.0 - t2 * c;             // 1/10!
  c = 1.0 / 40320.0 - t2 * c;               // 1/8!
  c = 1.0 / 720.0 - t2 * c;                 // 1/6!
  c = 1.0 / 24.0 - t2 * c;                  // 1/4!
  c = 0.5 - t2 * c;                         // 1/2!
  c = 1.0 - t2 * c;
  *s_out = t * s;
  *c_out = c;
}

// cos(2*pi*u) for u in [0, 1): exact quadrant split, then octant reflection.
GEN_HD double gen_cos2pi(double u) {
  double a = u * 4.0;                       // exact
  double qd = floor(a);
  double f = a - qd;                        // exact, in [0, 1)
  int q = (int)qd;
  double s, c;
  if (f > 0.5) { gen_sincos_small((1.0 - f) * 1.5707963267948966, &c, &s); }
  else         { gen_sincos_small(f * 1.5707963267948966, &s, &c); }
  // cos(q*pi/2 + theta)
  if (q == 0) return c;
  if (q == 1) return -s;
  if (q == 2) return -c;
  return s;
}

// exp(y) for y in [-20, 0]: Taylor series of exp(y/16) in Horner form
// 1 + x(1 + x/2(1 + x/3(...(1 + x/20)))), then four squarings.
GEN_HD double gen_exp_nonpos(double y) {
  double x = y * 0.0625;
  double p = 1.0;
  for (int k = 20; k >= 1; --k) p = 1.0 + x * (1.0 / (double)k) * p;
  p = p * p; p = p * p; p = p * p; p = p * p;
  return p;
}

// ------------------------------------------------------------ conversions --
GEN_HD uint16_t gen_f32_to_bf16(float f) {
  union { float f; uint32_t u; } b; b.f = f;
  uint32_t u = b.u;
  u += 0x7FFFu + ((u >> 16) & 1u);          // round to nearest even (no NaN here)
  return (uint16_t)(u >> 16);
}
GEN_HD float gen_bf16_to_f32(uint16_t h) {
  union { float f; uint32_t u; } b; b.u = ((uint32_t)h) << 16;
  return b.f;
}
#ifdef __CUDA_ARCH__
#define GEN_D2F(x) __double2float_rn(x)
#else
#define GEN_D2F(x) ((float)(x))
#endif

// Standard normal by Box-Muller (cosine branch) from two counter draws.
GEN_HD double gen_normal(uint64_t seed, uint32_t stream, uint64_t idx) {
  double u1 = gen_u01_open0(gen_u64(seed, stream, 2ull * idx));
  double u2 = gen_u01(gen_u64(seed, stream, 2ull * idx + 1ull));
  double r = sqrt(-2.0 * gen_ln(u1));
  return r * gen_cos2pi(u2);
}

GEN_HD uint16_t gen_normal_bf16(uint64_t seed, uint32_t stream, uint64_t idx) {
  return gen_f32_to_bf16(GEN_D2F(gen_normal(seed, stream, idx)));
}

// Softmax over the 4 normals of token t (indices 4t .. 4t+3), rounded to bf16.
GEN_HD void gen_softmax4_bf16(uint64_t seed, uint32_t stream, uint64_t t, uint16_t* out4) {
  double n[4], mx;
  for (int h = 0; h < 4; ++h) n[h] = gen_normal(seed, stream, 4ull * t + (uint64_t)h);
  mx = n[0];
  for (int h = 1; h < 4; ++h) mx = n[h] > mx ? n[h] : mx;
  double e[4], s = 0.0;
  for (int h = 0; h < 4; ++h) { e[h] = gen_exp_nonpos(n[h] - mx); s = s + e[h]; }
  for (int h = 0; h < 4; ++h) out4[h] = gen_f32_to_bf16(GEN_D2F(e[h] / s));
}

// Planted key row value: mean vector element (fp64) + 0.3 * noise, to bf16.
GEN_HD uint16_t gen_planted(double mean, uint64_t seed, uint32_t stream, uint64_t idx) {
  double x = mean + 0.3 * gen_normal(seed, stream, idx);
  return gen_f32_to_bf16(GEN_D2F(x));
}

// Mean of n_vec consecutive 128-vectors starting at src (bf16), element c,
// summed in index order.
GEN_HD double gen_mean_elem(const uint16_t* src, int64_t n_vec, int c, int dim) {
  double acc = 0.0;
  for (int64_t v = 0; v < n_vec; ++v) acc = acc + (double)gen_bf16_to_f32(src[v * dim + c]);
  return acc / (double)n_vec;
}

// ------------------------------------------------------------ host entries --
extern "C" {

void qsagen_normal_bf16(uint64_t seed, uint32_t stream, uint64_t offset, uint64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = gen_normal_bf16(seed, stream, offset + (uint64_t)i);
}

void qsagen_normal_f64(uint64_t seed, uint32_t stream, uint64_t offset, uint64_t n, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = gen_normal(seed, stream, offset + (uint64_t)i);
}

void qsagen_uniform(uint64_t seed, uint32_t stream, uint64_t offset, uint64_t n, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = gen_u01(gen_u64(seed, stream, offset + (uint64_t)i));
}

void qsagen_softmax4_bf16(uint64_t seed, uint32_t stream, uint64_t tok0, uint64_t ntok, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)ntok; ++i) gen_softmax4_bf16(seed, stream, tok0 + (uint64_t)i, out + 4 * i);
}

// Planted blocks.  For block b = 0..nkb-1 with src_tok[b] >= 0: the mean of the
// n_src[b]*heads vectors q_src[src_tok[b]*heads ..) (each `dim` long) plus
// 0.3 * noise is written to key rows [b*r, min(b*r+r, n_keys)) of `keys`.
// keys[0] is absolute key row `row0`; the noise element index of key row j,
// element c, is (row0 + j) * dim + c.
void qsagen_plant(int64_t nkb, int r, int64_t n_keys, int64_t row0, int heads, int dim,
                  const int64_t* src_tok, const int64_t* n_src, const uint16_t* q_src,
                  uint16_t* keys, uint64_t seed, uint32_t stream) {
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t b = 0; b < nkb; ++b) {
    if (src_tok[b] < 0) continue;
    const uint16_t* src = q_src + src_tok[b] * (int64_t)heads * dim;
    int64_t nv = n_src[b] * heads;
    for (int c = 0; c < dim; ++c) {
      double mean = gen_mean_elem(src, nv, c, dim);
      for (int64_t j = b * r; j < b * r + r && j < n_keys; ++j)
        keys[j * dim + c] = gen_planted(mean, seed, stream, (uint64_t)((row0 + j) * dim + c));
    }
  }
}

// ---------------------------------------------------------- device entries --
__global__ void k_normal_bf16(uint64_t seed, uint32_t stream, uint64_t offset, uint64_t n, uint16_t* out) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n; i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = gen_normal_bf16(seed, stream, offset + i);
}
__global__ void k_softmax4_bf16(uint64_t seed, uint32_t stream, uint64_t tok0, uint64_t ntok, uint16_t* out) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < ntok; i += (uint64_t)gridDim.x * blockDim.x)
    gen_softmax4_bf16(seed, stream, tok0 + i, out + 4 * i);
}
__global__ void k_plant(int64_t nkb, int r, int64_t n_keys, int64_t row0, int heads, int dim,
                        const int64_t* src_tok, const int64_t* n_src, const uint16_t* q_src, uint16_t* keys,
                        uint64_t seed, uint32_t stream) {
  for (int64_t b = blockIdx.x; b < nkb; b += gridDim.x) {
    if (src_tok[b] < 0) continue;
    const uint16_t* src = q_src + src_tok[b] * (int64_t)heads * dim;
    int64_t nv = n_src[b] * heads;
    for (int c = threadIdx.x; c < dim; c += blockDim.x) {
      double mean = gen_mean_elem(src, nv, c, dim);
      for (int64_t j = b * r; j < b * r + r && j < n_keys; ++j)
        keys[j * dim + c] = gen_planted(mean, seed, stream, (uint64_t)((row0 + j) * dim + c));
    }
  }
}

int qsagen_normal_bf16_dev(uint64_t seed, uint32_t stream, uint64_t offset, uint64_t n, uint16_t* out, void* cs) {
  if (n == 0) return 0;
  uint64_t blocks = (n + 255) / 256;
  if (blocks > 148ull * 64ull) blocks = 148ull * 64ull;
  k_normal_bf16<<<(unsigned)blocks, 256, 0, (cudaStream_t)cs>>>(seed, stream, offset, n, out);
  return (int)cudaGetLastError();
}
int qsagen_softmax4_bf16_dev(uint64_t seed, uint32_t stream, uint64_t tok0, uint64_t ntok, uint16_t* out, void* cs) {
  if (ntok == 0) return 0;
  uint64_t blocks = (ntok + 255) / 256;
  if (blocks > 148ull * 64ull) blocks = 148ull * 64ull;
  k_softmax4_bf16<<<(unsigned)blocks, 256, 0, (cudaStream_t)cs>>>(seed, stream, tok0, ntok, out);
  return (int)cudaGetLastError();
}
int qsagen_plant_dev(int64_t nkb, int r, int64_t n_keys, int64_t row0, int heads, int dim,
                     const int64_t* src_tok, const int64_t* n_src, const uint16_t* q_src, uint16_t* keys,
                     uint64_t seed, uint32_t stream, void* cs) {
  if (nkb == 0) return 0;
  int64_t blocks = nkb < 148 * 32 ? nkb : 148 * 32;
  k_plant<<<(unsigned)blocks, 128, 0, (cudaStream_t)cs>>>(nkb, r, n_keys, row0, heads, dim, src_tok, n_src, q_src,
                                                           keys, seed, stream);
  return (int)cudaGetLastError();
}

}  // extern "C"
