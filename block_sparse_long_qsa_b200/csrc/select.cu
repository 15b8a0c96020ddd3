// Stage 2: per-query-block top-k block selection.
//
// Page "Qwen3.8-Flash-Next, 1/9의 학습 비용으로 Qwen3.7-Plus(397B-A17B) 수준에
// 도달한 125B-A6B 모델", section "QSA: 인덱서 자체의 비용을 줄이는 희소 어텐션":
// token budget K = 2048 with r = 4, i.e. 512 blocks per query; the tail
// tokens of the own (incomplete) block are always included.  This library's
// reading: block qb and qb-1 are forced; the other budget-2 slots go to the
// blocks of [0, qb-2] with the highest score, ties to the lower index, -0.0
// equal to +0.0; all blocks when qb+1 <= budget; output ascending.
//
// Scores are >= 0, so the IEEE bit pattern with the sign cleared orders them
// as unsigned integers.  One CTA per row:
//   1. rows with at most CAP candidates are loaded whole into shared memory;
//      longer rows draw a strided sample of 2048 scores whose order statistic
//      at a safely conservative rank, its low 16 bits cleared (two radix
//      passes), gives a threshold, and one coalesced
//      pass keeps the scores at or above it (ballot-compacted) -- a few
//      thousand candidates out of up to 262,143;
//   2. an exact MSB-first radix select (8-bit digits, shared histograms)
//      finds the k-th largest key among the candidates, starting at the
//      first digit where the smallest and largest candidate differ; ties at
//      the threshold are resolved by a second radix select on the block
//      indices;
//   3. if the sample's threshold left fewer than k or more than CAP
//      candidates (rare), the same radix select runs over the whole row in
//      global memory and an index-ordered pass collects the winners;
//   4. the winners plus the two forced blocks are bitonic-sorted ascending.
#include <climits>

#include "qsa_device.cuh"
#include "qsa_kernels.h"

namespace qsa {
namespace {

constexpr int THREADS = 512;
constexpr int NSAMPLE = 2048;

__host__ __device__ inline int cap_for(int budget) {
  int c = 3 * budget;
  if (c < 6144) c = 6144;
  if (c > 16384) c = 16384;
  return c;
}
__host__ __device__ inline int pow2_at_least(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

struct SelSmem {
  uint32_t* hist;   // [2][256]: the radix passes alternate between the two
  uint32_t* misc;   // [16]
  uint32_t* warp_tot;  // [32]
  uint32_t* sample; // [NSAMPLE]
  uint32_t* ckey;   // [cap]
  int32_t* cidx;    // [cap]
  int32_t* out;     // [pow2(budget)]
};

__device__ __forceinline__ uint32_t key_of(float x) { return __float_as_uint(x) & 0x7FFFFFFFu; }

// k-th largest (1-based k, 1 <= k <= n) of get(0..n-1) by MSB-first radix
// select.  Returns the key and the number of elements strictly greater.
// Every key may be known to share its bits above digit hi_shift with
// `common` (hi_shift < 24 skips those digits' passes; hi_shift < 0: all keys
// equal `common`); with lo_shift > 0 the select stops after that digit and
// returns the k-th largest key with its lower bits cleared (a lower bound).
template <class Get>
__device__ void radix_kth_largest(Get get, int64_t n, int64_t k, const SelSmem& sm, uint32_t& tau, int64_t& n_gt,
                                  uint32_t common = 0, int hi_shift = 24, int lo_shift = 0) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t mask = hi_shift >= 24 ? 0u : ~0u << (hi_shift + 8);
  uint32_t prefix = common & mask;
  int64_t kk = k;
  // Two histograms: pass p counts into hist[p % 2] while the other one is
  // cleared for pass p + 1, and the chosen digit goes to misc[2 (p % 2)], so
  // a pass needs two barriers (after the counts, after the scan).
  for (int i = tid; i < 256; i += blockDim.x) sm.hist[i] = 0;
  __syncthreads();
  int pass = 0;
  for (int shift = hi_shift; shift >= lo_shift; shift -= 8, ++pass) {
    uint32_t* hist = sm.hist + 256 * (pass & 1);
    uint32_t* next = sm.hist + 256 * ((pass + 1) & 1);
    for (int i = tid; i < 256; i += blockDim.x) next[i] = 0;
    for (int64_t i = tid; i < n; i += blockDim.x) {
      const uint32_t key = get(i);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    uint32_t* out2 = sm.misc + 2 * (pass & 1);
    if (warp == 0) {
      uint32_t c[8], s = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) { c[q] = hist[255 - 8 * lane - q]; s += c[q]; }
      uint32_t incl = s;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      const uint32_t excl = incl - s;
      if ((int64_t)excl < kk && kk <= (int64_t)incl) {
        uint32_t cum = excl;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (cum + c[q] >= kk) {
            out2[0] = (uint32_t)(255 - 8 * lane - q);
            out2[1] = (uint32_t)(kk - cum);
            break;
          }
          cum += c[q];
        }
      }
    }
    __syncthreads();
    const uint32_t bin = out2[0];
    kk = out2[1];
    prefix |= bin << shift;
    mask |= 0xFFu << shift;
  }
  __syncthreads();   // every thread has read the last digit before the caller reuses misc / hist
  tau = prefix;
  n_gt = k - kk;
}

// Block-wide exclusive prefix count of `flag` in thread order; returns the
// block total through *total.
__device__ __forceinline__ uint32_t block_excl_count(bool flag, const SelSmem& sm, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const uint32_t ball = __ballot_sync(0xffffffffu, flag);
  const uint32_t in_warp = __popc(ball & ((1u << lane) - 1u));
  if (lane == 0) sm.warp_tot[warp] = __popc(ball);
  __syncthreads();
  uint32_t before = 0, tot = 0;
  for (int w = 0; w < nwarps; ++w) {
    const uint32_t v = sm.warp_tot[w];
    if (w < warp) before += v;
    tot += v;
  }
  __syncthreads();
  *total = tot;
  return before + in_warp;
}

__global__ void __launch_bounds__(THREADS, 3)
select_kernel(const float* __restrict__ S, int64_t ld, const float* __restrict__ segmax, int64_t ld_seg,
              int64_t qb_begin, int64_t n_rows, const int64_t* __restrict__ row_qb, int budget,
              int32_t* __restrict__ sel, int32_t* __restrict__ cnt, uint32_t* err) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int cap = cap_for(budget);
  const int P = pow2_at_least(budget);
  SelSmem sm;
  sm.hist = reinterpret_cast<uint32_t*>(smem_raw);
  sm.misc = sm.hist + 512;
  sm.warp_tot = sm.misc + 16;
  sm.sample = sm.warp_tot + 32;
  sm.ckey = sm.sample + NSAMPLE;
  sm.cidx = reinterpret_cast<int32_t*>(sm.ckey + cap);
  sm.out = sm.cidx + cap;
  const int tid = threadIdx.x, lane = tid & 31;

  for (int64_t r = blockIdx.x; r < n_rows; r += gridDim.x) {
    const int64_t qb = row_qb ? row_qb[r] : qb_begin + r;
    const float* row = S + r * ld;
    int32_t* srow = sel + r * budget;
    if (qb + 1 <= budget) {
      for (int i = tid; i < budget; i += blockDim.x) srow[i] = i <= qb ? i : -1;
      if (tid == 0) cnt[r] = (int32_t)(qb + 1);
      continue;
    }
    const int64_t m = qb - 1;          // candidates 0 .. qb-2
    const int64_t k = budget - 2;
    if (tid == 0) { sm.misc[8] = 0; sm.misc[9] = 0; sm.misc[12] = 0xFFFFFFFFu; sm.misc[13] = 0u; }
    __syncthreads();
    // range of the candidates' keys (the exact select skips the digits they share)
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;

    bool global_path = false;
    int64_t nc = 0;
    if (k == 0) {
      // budget 2: only the forced blocks
    } else if (m <= cap) {
      for (int64_t i = tid; i < m; i += blockDim.x) {
        const uint32_t key = key_of(row[i]);
        sm.ckey[i] = key;
        sm.cidx[i] = (int32_t)i;
        kmin = min(kmin, key);
        kmax = max(kmax, key);
      }
      nc = m;
    } else if (segmax != nullptr) {
      // 1'. threshold from the segment maxima.  Segments 0 .. fs-1 (8 blocks
      //     each) hold candidate blocks only; blocks 8 fs .. qb-2 form the tail.
      //     If at least k segments reach tau0, at least k scores do, and every
      //     score >= tau0 lies in such a segment or in the tail.
      const int64_t fs = (qb - 1) >> 3;
      const float* mrow = segmax + r * ld_seg;
      // NSAMPLE / 4 evenly spaced 16-byte groups of 4 consecutive maxima (the
      // row is 16-byte aligned: ld_seg % 4 == 0; fs > cap / 8 >= 4 x groups)
      {
        const float4* mrow4 = reinterpret_cast<const float4*>(mrow);
        const int64_t fs4 = fs >> 2;
        for (int i = tid; i < NSAMPLE / 4; i += blockDim.x) {
          const float4 g = __ldcs(mrow4 + (int64_t)i * fs4 / (NSAMPLE / 4));
          reinterpret_cast<uint4*>(sm.sample)[i] = make_uint4(key_of(g.x), key_of(g.y), key_of(g.z), key_of(g.w));
        }
      }
      const float e = (float)NSAMPLE * (float)k / (float)fs;
      int64_t rs = (int64_t)ceilf(e + 4.f * sqrtf(e) + 8.f);
      if (rs > NSAMPLE) rs = NSAMPLE;
      __syncthreads();
      // tau0 = the rs-th largest sampled maximum with its low 16 bits cleared
      // (two radix passes; a slightly lower, still conservative threshold)
      uint32_t tau0;
      int64_t dummy;
      radix_kth_largest([&](int64_t i) { return sm.sample[i]; }, NSAMPLE, rs, sm, tau0, dummy, 0u, 24, 16);
      // 2'. the segments whose max reaches tau0 (listed in the sample buffer) ...
      if (tid == 0) sm.misc[11] = 0;
      __syncthreads();
      // SEG_UNROLL 16-byte loads (4 maxima each) per thread in flight before
      // any is tested: the scan is one row of up to 32K maxima per CTA, bound
      // by load latency otherwise; most groups have no maximum reaching tau0
      // and skip the compaction
      constexpr int SEG_UNROLL = 4;
      const float4* mrow4 = reinterpret_cast<const float4*>(mrow);
      const int64_t fs4 = (fs + 3) >> 2;     // rows are padded to a multiple of 4 (ld_seg)
      for (int64_t b0 = 0; b0 < fs4; b0 += (int64_t)blockDim.x * SEG_UNROLL) {
        float4 kv[SEG_UNROLL];
#pragma unroll
        for (int u = 0; u < SEG_UNROLL; ++u) {
          const int64_t g = b0 + (int64_t)u * blockDim.x + tid;
          kv[u] = g < fs4 ? __ldcs(mrow4 + g) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < SEG_UNROLL; ++u) {
          const int64_t g = b0 + (int64_t)u * blockDim.x + tid;
          const float vals[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
          bool any = false;
#pragma unroll
          for (int q = 0; q < 4; ++q) any |= (4 * g + q < fs) && key_of(vals[q]) >= tau0;
          if (!__any_sync(0xffffffffu, any)) continue;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int64_t sgi = 4 * g + q;
            const bool pass = sgi < fs && key_of(vals[q]) >= tau0;
            const uint32_t ball = __ballot_sync(0xffffffffu, pass);
            if (ball) {
              uint32_t base = 0;
              if (lane == 0) base = atomicAdd(&sm.misc[11], (uint32_t)__popc(ball));
              base = __shfl_sync(0xffffffffu, base, 0);
              const uint32_t pos = base + __popc(ball & ((1u << lane) - 1u));
              if (pass && pos < (uint32_t)NSAMPLE) sm.sample[pos] = (uint32_t)sgi;
            }
          }
        }
      }
      __syncthreads();
      const int64_t nsl = sm.misc[11];
      if (nsl > NSAMPLE) {
        global_path = true;
      } else {
        // ... and their scores >= tau0 (two 16-byte loads per segment), then the tail
        const float4* row4 = reinterpret_cast<const float4*>(row);
        constexpr int CAND_UNROLL = 4;
        for (int64_t b0 = 0; b0 < 2 * nsl; b0 += (int64_t)blockDim.x * CAND_UNROLL) {
          float4 v[CAND_UNROLL];
          int64_t i0[CAND_UNROLL];
#pragma unroll
          for (int u = 0; u < CAND_UNROLL; ++u) {
            const int64_t e2 = b0 + (int64_t)u * blockDim.x + tid;
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            i0[u] = 0;
            if (e2 < 2 * nsl) {
              i0[u] = 8 * (int64_t)sm.sample[e2 >> 1] + 4 * (e2 & 1);
              v[u] = __ldcs(row4 + (i0[u] >> 2));
            }
          }
#pragma unroll
          for (int u = 0; u < CAND_UNROLL; ++u) {
            const int64_t e2 = b0 + (int64_t)u * blockDim.x + tid;
            const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const bool pass = e2 < 2 * nsl && key_of(vals[q]) >= tau0;
              const uint32_t ball = __ballot_sync(0xffffffffu, pass);
              if (ball) {
                uint32_t base = 0;
                if (lane == 0) base = atomicAdd(&sm.misc[8], (uint32_t)__popc(ball));
                base = __shfl_sync(0xffffffffu, base, 0);
                const uint32_t pos = base + __popc(ball & ((1u << lane) - 1u));
                if (pass && pos < (uint32_t)cap) {
                  sm.ckey[pos] = key_of(vals[q]);
                  sm.cidx[pos] = (int32_t)(i0[u] + q);
                }
                if (pass) kmax = max(kmax, key_of(vals[q]));
              }
            }
          }
        }
        if (tid < 8) {
          const int64_t i = 8 * fs + tid;
          if (i < m && key_of(row[i]) >= tau0) {
            const uint32_t pos = atomicAdd(&sm.misc[8], 1u);
            if (pos < (uint32_t)cap) { sm.ckey[pos] = key_of(row[i]); sm.cidx[pos] = (int32_t)i; }
            kmax = max(kmax, key_of(row[i]));
          }
        }
        kmin = tau0;
        __syncthreads();
        nc = sm.misc[8];
        global_path = (nc < k || nc > cap);
      }
      __syncthreads();
    } else {
      // 1. threshold from a strided sample
      for (int i = tid; i < NSAMPLE; i += blockDim.x) sm.sample[i] = key_of(row[(int64_t)i * m / NSAMPLE]);
      const float e = (float)NSAMPLE * (float)k / (float)m;
      int64_t rs = (int64_t)ceilf(e + 4.f * sqrtf(e) + 8.f);
      if (rs > NSAMPLE) rs = NSAMPLE;
      __syncthreads();
      uint32_t tau0;
      int64_t dummy;
      radix_kth_largest([&](int64_t i) { return sm.sample[i]; }, NSAMPLE, rs, sm, tau0, dummy, 0u, 24, 16);
      // 2. filter pass: keep key >= tau0 (row start is 16-byte aligned: ld % 4 == 0)
      const float4* row4 = reinterpret_cast<const float4*>(row);
      const int64_t m4 = (m + 3) >> 2;
      // UNROLL independent 16-byte loads per thread per iteration keep enough
      // bytes in flight to stream the row at HBM speed
      constexpr int UNROLL = 4;
      const int64_t stride4 = (int64_t)blockDim.x * UNROLL;
      for (int64_t base4 = 0; base4 < m4; base4 += stride4) {
        float4 v[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          const int64_t i4 = base4 + (int64_t)u * blockDim.x + tid;
          v[u] = i4 < m4 ? __ldcs(row4 + i4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          const int64_t i4 = base4 + (int64_t)u * blockDim.x + tid;
          const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
          bool any = false;
#pragma unroll
          for (int q = 0; q < 4; ++q) any |= (4 * i4 + q < m) && key_of(vals[q]) >= tau0;
          if (!__any_sync(0xffffffffu, any)) continue;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int64_t idx = 4 * i4 + q;
            const bool pass = idx < m && key_of(vals[q]) >= tau0;
            const uint32_t ball = __ballot_sync(0xffffffffu, pass);
            if (ball) {
              uint32_t base = 0;
              if (lane == 0) base = atomicAdd(&sm.misc[8], (uint32_t)__popc(ball));
              base = __shfl_sync(0xffffffffu, base, 0);
              const uint32_t pos = base + __popc(ball & ((1u << lane) - 1u));
              if (pass && pos < (uint32_t)cap) { sm.ckey[pos] = key_of(vals[q]); sm.cidx[pos] = (int32_t)idx; }
              if (pass) kmax = max(kmax, key_of(vals[q]));
            }
          }
        }
      }
      kmin = tau0;
      __syncthreads();
      nc = sm.misc[8];
      global_path = (nc < k || nc > cap);
      __syncthreads();
    }

    if (k == 0) {
      if (tid == 0) sm.misc[8] = 0;
      __syncthreads();
    } else if (!global_path) {
      {
        const uint32_t wmin = __reduce_min_sync(0xffffffffu, kmin), wmax = __reduce_max_sync(0xffffffffu, kmax);
        if (lane == 0) { atomicMin(&sm.misc[12], wmin); atomicMax(&sm.misc[13], wmax); }
      }
      __syncthreads();
      const uint32_t lo = sm.misc[12], hi = sm.misc[13];
      // digits above the first bit where the smallest and largest candidate
      // keys differ are the same for every candidate
      const int same = lo == hi ? 32 : __clz(lo ^ hi);
      uint32_t tau;
      int64_t n_gt;
      radix_kth_largest([&](int64_t i) { return sm.ckey[i]; }, nc, k, sm, tau, n_gt, lo, 24 - 8 * (same >> 3));
      const int64_t need = k - n_gt;
      // count ties
      if (tid == 0) { sm.misc[8] = 0; sm.misc[10] = 0; }
      __syncthreads();
      for (int64_t i = tid; i < nc; i += blockDim.x)
        if (sm.ckey[i] == tau) atomicAdd(&sm.misc[10], 1u);
      __syncthreads();
      const int64_t n_eq = sm.misc[10];
      uint32_t idx_cut = 0xFFFFFFFFu;   // take ties with index <= idx_cut
      if (n_eq > need) {
        uint32_t ntau;
        int64_t d2;
        radix_kth_largest([&](int64_t i) { return sm.ckey[i] == tau ? ~(uint32_t)sm.cidx[i] : 0u; }, nc, need, sm,
                          ntau, d2);
        idx_cut = ~ntau;
      }
      for (int64_t b = 0; b < nc; b += blockDim.x) {
        const int64_t i = b + tid;
        bool take = false;
        int32_t ci = 0;
        if (i < nc) {
          const uint32_t key = sm.ckey[i];
          ci = sm.cidx[i];
          take = key > tau || (key == tau && (uint32_t)ci <= idx_cut);
        }
        const uint32_t ball = __ballot_sync(0xffffffffu, take);
        if (ball) {
          uint32_t base = 0;
          if (lane == 0) base = atomicAdd(&sm.misc[8], (uint32_t)__popc(ball));
          base = __shfl_sync(0xffffffffu, base, 0);
          const uint32_t pos = base + __popc(ball & ((1u << lane) - 1u));
          if (take && pos < (uint32_t)k) sm.out[pos] = ci;
        }
      }
      __syncthreads();
    } else {
      // 3. exact selection over the row in global memory
      uint32_t tau;
      int64_t n_gt;
      radix_kth_largest([&](int64_t i) { return key_of(row[i]); }, m, k, sm, tau, n_gt);
      const int64_t need = k - n_gt;
      if (tid == 0) sm.misc[8] = 0;
      __syncthreads();
      int64_t eq_taken = 0;
      for (int64_t base = 0; base < m; base += blockDim.x) {
        const int64_t i = base + tid;
        const uint32_t key = i < m ? key_of(row[i]) : 0u;
        const bool gt = i < m && key > tau;
        const bool eq = i < m && key == tau;
        uint32_t tot;
        const uint32_t rank = block_excl_count(eq, sm, &tot);
        if (gt || (eq && eq_taken + (int64_t)rank < need)) {
          const uint32_t pos = atomicAdd(&sm.misc[8], 1u);
          if (pos < (uint32_t)k) sm.out[pos] = (int32_t)i;
        }
        eq_taken += tot;
      }
      __syncthreads();
    }
    if (tid == 0 && sm.misc[8] != (uint32_t)k) report_error(err, QSA_ERR_DEVICE_BOUNDS);
    // 4. forced blocks, then ascending sort of the budget entries
    if (tid == 0) { sm.out[k] = (int32_t)(qb - 1); sm.out[k + 1] = (int32_t)qb; }
    for (int i = budget + tid; i < P; i += blockDim.x) sm.out[i] = INT_MAX;
    __syncthreads();
    if (P <= THREADS) {
      // one entry per thread: compare-exchange steps with a partner in the
      // same warp by shuffle, wider ones through two alternating shared
      // buffers (sm.out and the spent candidate keys), one barrier each
      int32_t v = tid < P ? sm.out[tid] : INT_MAX;
      int32_t* const buf0 = sm.out;
      int32_t* const buf1 = reinterpret_cast<int32_t*>(sm.ckey);
      int nb = 0;
      for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          int32_t o;
          if (stride >= 32) {
            nb ^= 1;
            int32_t* const b = nb ? buf1 : buf0;
            if (tid < P) b[tid] = v;
            __syncthreads();
            o = tid < P ? b[tid ^ stride] : v;
          } else {
            o = __shfl_xor_sync(0xffffffffu, v, stride);
          }
          // the lower slot of an ascending pair keeps the minimum
          const bool up = (tid & size) == 0, lower = (tid & stride) == 0;
          v = (lower == up) ? min(v, o) : max(v, o);
        }
      }
      if (tid < budget) srow[tid] = v;
      if (tid == 0) cnt[r] = budget;
      __syncthreads();
      continue;
    }
    for (int size = 2; size <= P; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < P / 2; i += blockDim.x) {
          const int lo = 2 * i - (i & (stride - 1));
          const int hi = lo + stride;
          const bool up = (lo & size) == 0;
          const int32_t a = sm.out[lo], b = sm.out[hi];
          if ((a > b) == up) { sm.out[lo] = b; sm.out[hi] = a; }
        }
        __syncthreads();
      }
    }
    for (int i = tid; i < budget; i += blockDim.x) srow[i] = sm.out[i];
    if (tid == 0) cnt[r] = budget;
    __syncthreads();
  }
}

}  // namespace

size_t select_smem_bytes(int budget) {
  const int cap = cap_for(budget);
  return (size_t)(512 + 16 + 32 + NSAMPLE) * 4 + (size_t)cap * 8 + (size_t)pow2_at_least(budget) * 4;
}

cudaError_t launch_select(const float* S, int64_t ld, const float* segmax, int64_t ld_seg, int64_t qb_begin,
                          int64_t n_rows, const int64_t* row_qb, int budget, int32_t* sel, int32_t* cnt, uint32_t* err,
                          cudaStream_t stream) {
  if (n_rows <= 0) return cudaSuccess;
  const size_t smem = select_smem_bytes(budget);
  static size_t attr_set[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && attr_set[dev] < smem) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = smem;
  }
  const int64_t grid = n_rows < 148 * 64 ? n_rows : 148 * 64;
  select_kernel<<<(unsigned)grid, THREADS, smem, stream>>>(S, ld, segmax, ld_seg, qb_begin, n_rows, row_qb, budget,
                                                          sel, cnt, err);
  return cudaGetLastError();
}

}  // namespace qsa
