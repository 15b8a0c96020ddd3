// Stage 3: sparse GQA attention over the selected micro-blocks ("sparse core
// attention", page "Qwen3.8-Flash-Next, 1/9의 학습 비용으로 Qwen3.7-Plus(397B-
// A17B) 수준에 도달한 125B-A6B 모델", section "QSA: 인덱서 자체의 비용을 줄이는
// 희소 어텐션"; 24 Q heads, 2 KV heads, head dim 256 from its spec table).
//
//   out[t][h] = sum_j softmax_j(q_rot[t][h] . k_rot[j][h/12] * scale) v[j][h/12]
//   over j in the selected blocks of block t/4 with j <= t.
//
// One CTA per query block (prefill: 4 tokens x 24 heads = 96 query rows, both
// KV heads) or per (sequence, key split) (decode: 24 rows).  The selected
// blocks are gathered 4 at a time (16 keys x 2 heads of K and V, 32 KB) with
// cp.async into 128-byte-swizzled shared memory through a multi-stage ring;
// QK^T and PV run on bf16 tensor-core MMAs with fp32 accumulation and an
// online softmax in base 2 (the running max is only raised when a tile's
// max exceeds it by more than 8, so the output rescale is rare).
#include <cfloat>

#include "qsa_device.cuh"
#include "qsa_kernels.h"

namespace qsa {
namespace {

constexpr int KEYS = 16;                         // keys per stage (4 blocks)
constexpr uint32_t ROW_BYTES = 512;              // 256 bf16
constexpr uint32_t KV_HEAD_BYTES = KEYS * ROW_BYTES;
constexpr uint32_t STAGE_BYTES = 2 * 2 * KV_HEAD_BYTES;   // K and V, 2 heads

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {
  return row * ROW_BYTES + ((chunk ^ (row & 7u)) << 4);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int NT>
struct Cfg {
  static constexpr int RG = NT * 12;                    // query rows per KV head
  static constexpr int WG = (RG + 15) / 16;             // warps per KV head
  static constexpr int RGP = 16 * WG;                   // padded rows per KV head
  static constexpr int WARPS = 2 * WG;
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int STAGES = NT == 4 ? 4 : 3;
  static constexpr uint32_t Q_BYTES = 2 * RGP * ROW_BYTES;
  static constexpr uint32_t SMEM_FIXED = Q_BYTES + STAGES * STAGE_BYTES;
};

struct AttnArgs {
  int64_t T;                 // prefill: tokens; decode: unused
  const uint16_t* q;         // prefill: q [T][24][256] (unrotated); decode: q_rot [B][24][256]
  const uint16_t* k;         // k_rot: prefill [T][2][256]; decode cache [B][max_len][2][256]
  const uint16_t* v;
  const float2* cs;          // prefill RoPE table [T][32]
  const int32_t* sel;        // [rows][budget]
  const int32_t* cnt;        // [rows]
  int budget;
  int64_t qb_begin;
  float scale_log2;
  uint16_t* out;             // prefill out [T][24][256]
  float* lse;                // prefill lse [T][24] (nullable)
  // decode
  int64_t max_len;
  const int64_t* Ls;
  int n_split;
  float* part_o;             // [B][n_split][24][256]
  float* part_lse;           // [B][n_split][24]
};

template <int NT>
__global__ void __launch_bounds__(Cfg<NT>::THREADS)
sparse_attn_kernel(AttnArgs a) {
  using C = Cfg<NT>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::Q_BYTES;
  int32_t* s_sel = reinterpret_cast<int32_t*>(smem + C::SMEM_FIXED);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = warp / C::WG;                   // KV head of this warp
  const int wi = warp % C::WG;                  // 16-row slice within the head group

  // ---- which rows / keys this CTA handles
  int64_t row_id, t_pos, qb;                    // row_id indexes sel/cnt
  int blk_begin = 0, blk_end;
  const uint16_t* kbase;
  const uint16_t* vbase;
  int64_t L = 0, b = 0;
  int split = 0;
  if (NT == 4) {
    qb = a.qb_begin + blockIdx.x;
    row_id = blockIdx.x;
    t_pos = 4 * qb;                             // first token of the block
    kbase = a.k;
    vbase = a.v;
  } else {
    b = blockIdx.x / a.n_split;
    split = (int)(blockIdx.x % a.n_split);
    L = a.Ls[b];
    qb = L >> 2;
    row_id = b;
    t_pos = L;
    kbase = a.k + b * a.max_len * 512;
    vbase = a.v + b * a.max_len * 512;
  }
  const int cnt = a.cnt[row_id];
  blk_end = cnt;
  if (NT == 1) {
    const int per = (cnt + a.n_split - 1) / a.n_split;
    blk_begin = split * per;
    blk_end = blk_begin + per < cnt ? blk_begin + per : cnt;
    if (blk_begin > blk_end) blk_begin = blk_end;
  }
  for (int i = tid; i < cnt; i += C::THREADS) s_sel[i] = a.sel[row_id * a.budget + i];

  // ---- Q tile: rows R = RGP*g + r, r = tok*12 + hh (r < RG), zero padding rows
  const uint32_t q_s = smem_u32(sQ);
  for (int e = tid; e < 2 * C::RGP * 28; e += C::THREADS) {
    const int R = e / 28, slot = e % 28;
    const int gg = R / C::RGP, r = R % C::RGP;
    const int tok = r / 12, hh = r % 12;
    const int64_t t = NT == 4 ? t_pos + tok : 0;
    const bool valid = r < C::RG && (NT == 1 || t < a.T);
    uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
    const int c_lo = slot < 4 ? slot : slot + 4;
    if (valid) {
      const uint4* src = NT == 4 ? reinterpret_cast<const uint4*>(a.q + (t * 24 + 12 * gg + hh) * 256)
                                 : reinterpret_cast<const uint4*>(a.q + (b * 24 + 12 * gg + hh) * 256);
      if (slot < 4) {
        lo = src[slot];
        hi = src[slot + 4];
        if (NT == 4) {   // RoPE pairs (i, i+32), i = 8*slot .. 8*slot+7
          const float2* cs = a.cs + t * 32 + 8 * slot;
          const uint32_t* x = reinterpret_cast<const uint32_t*>(&lo);
          const uint32_t* y = reinterpret_cast<const uint32_t*>(&hi);
          uint4 olo, ohi;
          uint32_t* ox = reinterpret_cast<uint32_t*>(&olo);
          uint32_t* oy = reinterpret_cast<uint32_t*>(&ohi);
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const float2 c0 = cs[2 * p], c1 = cs[2 * p + 1];
            const float x0 = bf16lo(x[p]), x1 = bf16hi(x[p]), y0 = bf16lo(y[p]), y1 = bf16hi(y[p]);
            ox[p] = pack_bf16x2(x0 * c0.x - y0 * c0.y, x1 * c1.x - y1 * c1.y);
            oy[p] = pack_bf16x2(y0 * c0.x + x0 * c0.y, y1 * c1.x + x1 * c1.y);
          }
          lo = olo;
          hi = ohi;
        }
      } else {
        lo = src[c_lo];
      }
    }
    *reinterpret_cast<uint4*>(sQ + swz(R, c_lo)) = lo;
    if (slot < 4) *reinterpret_cast<uint4*>(sQ + swz(R, slot + 4)) = hi;
  }
  __syncthreads();

  // ---- gather of one stage: blocks s_sel[blk0 .. blk0+3] -> K/V rows
  const int n_stages = (blk_end - blk_begin + 3) / 4;
  auto issue_stage = [&](int st) {
    const int buf = st % C::STAGES;
    const uint32_t base = smem_u32(sKV + buf * STAGE_BYTES);
    const int blk0 = blk_begin + 4 * st;
    // 16 keys x 2 heads x 32 chunks x {K, V}
    for (int e = tid; e < 2 * 2 * KEYS * 32; e += C::THREADS) {
      const int chunk = e & 31;
      const int key = (e >> 5) & 15;
      const int gg = (e >> 9) & 1;
      const int isv = e >> 10;
      const int bi = blk0 + (key >> 2);
      bool valid = bi < blk_end;
      int64_t j = 0;
      if (valid) {
        j = 4 * (int64_t)s_sel[bi] + (key & 3);
        valid = j <= (NT == 4 ? t_pos + 3 : t_pos) && (NT == 1 || j < a.T);
      }
      const uint16_t* src = (isv ? vbase : kbase) + (valid ? (j * 2 + gg) * 256 + chunk * 8 : 0);
      const uint32_t dst = base + isv * 2 * KV_HEAD_BYTES + gg * KV_HEAD_BYTES + swz(key, chunk);
      cp_async16(dst, src, valid);
    }
  };

  for (int st = 0; st < C::STAGES - 1; ++st) {
    if (st < n_stages) issue_stage(st);
    cp_async_commit();
  }

  // ---- per-warp state: 16 rows, this thread holds rows r0 = lane/4 and r0 + 8
  const int rbase = C::RGP * g + 16 * wi;      // first smem Q row of the warp
  float o[32][4];
#pragma unroll
  for (int n = 0; n < 32; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run[2] = {-FLT_MAX, -FLT_MAX}, l_run[2] = {0.f, 0.f};
  int64_t t_row[2];
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const int r = 16 * wi + (lane >> 2) + 8 * h2;          // row within the head group
    t_row[h2] = NT == 4 ? t_pos + (r < C::RG ? r / 12 : 0) : t_pos;
  }

  for (int st = 0; st < n_stages; ++st) {
    cp_async_wait<C::STAGES - 2>();
    __syncthreads();
    if (st + C::STAGES - 1 < n_stages) issue_stage(st + C::STAGES - 1);
    cp_async_commit();

    const int buf = st % C::STAGES;
    const uint32_t k_s = smem_u32(sKV + buf * STAGE_BYTES) + g * KV_HEAD_BYTES;
    const uint32_t v_s = smem_u32(sKV + buf * STAGE_BYTES) + 2 * KV_HEAD_BYTES + g * KV_HEAD_BYTES;

    // S = Q K^T for 16 rows x 16 keys
    float s[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 16; ++ks) {
      uint32_t af[4];
      ldsm_x4(q_s + swz(rbase + (lane & 15), 2 * ks + (lane >> 4)), af[0], af[1], af[2], af[3]);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(k_s + swz((lane & 7) + 8 * (lane >> 4), 2 * ks + ((lane >> 3) & 1)), b0, b1, b2, b3);
      mma_bf16_16816(s[0], af, b0, b1);
      mma_bf16_16816(s[1], af, b2, b3);
    }
    // mask, scale to log2 units
    const int blk0 = blk_begin + 4 * st;
    float mt[2] = {-FLT_MAX, -FLT_MAX};
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int key = 8 * n + 2 * (lane & 3) + (c & 1);
        const int h2 = c >> 1;
        const int bi = blk0 + (key >> 2);
        bool valid = bi < blk_end;
        if (valid) valid = 4 * (int64_t)s_sel[bi] + (key & 3) <= t_row[h2];
        const float x = valid ? s[n][c] * a.scale_log2 : -FLT_MAX;
        s[n][c] = x;
        mt[h2] = fmaxf(mt[h2], x);
      }
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      mt[h2] = fmaxf(mt[h2], __shfl_xor_sync(0xffffffffu, mt[h2], 1));
      mt[h2] = fmaxf(mt[h2], __shfl_xor_sync(0xffffffffu, mt[h2], 2));
    }
    const bool need = (mt[0] > m_run[0] + 8.f) || (mt[1] > m_run[1] + 8.f);
    if (__any_sync(0xffffffffu, need)) {
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const float m_new = fmaxf(m_run[h2], mt[h2]);
        const float corr = exp2f(m_run[h2] - m_new);
        l_run[h2] *= corr;
#pragma unroll
        for (int n = 0; n < 32; ++n) { o[n][2 * h2] *= corr; o[n][2 * h2 + 1] *= corr; }
        m_run[h2] = m_new;
      }
    }
    uint32_t pa[4];
    {
      float p[2][4];
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int h2 = c >> 1;
          const float e = s[n][c] == -FLT_MAX ? 0.f : exp2f(s[n][c] - m_run[h2]);
          p[n][c] = e;
          l_run[h2] += e;
        }
      pa[0] = pack_bf16x2(p[0][0], p[0][1]);
      pa[1] = pack_bf16x2(p[0][2], p[0][3]);
      pa[2] = pack_bf16x2(p[1][0], p[1][1]);
      pa[3] = pack_bf16x2(p[1][2], p[1][3]);
    }
    // O += P V
#pragma unroll
    for (int d = 0; d < 16; ++d) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(v_s + swz(lane & 15, 2 * d + (lane >> 4)), b0, b1, b2, b3);
      mma_bf16_16816(o[2 * d], pa, b0, b1);
      mma_bf16_16816(o[2 * d + 1], pa, b2, b3);
    }
  }
  cp_async_wait<0>();

  // ---- epilogue
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    l_run[h2] += __shfl_xor_sync(0xffffffffu, l_run[h2], 1);
    l_run[h2] += __shfl_xor_sync(0xffffffffu, l_run[h2], 2);
  }
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const int r = 16 * wi + (lane >> 2) + 8 * h2;
    if (r >= C::RG) continue;
    const int tok = r / 12, hh = r % 12, h = 12 * g + hh;
    const float inv = l_run[h2] > 0.f ? 1.f / l_run[h2] : 0.f;
    const float lse_v = l_run[h2] > 0.f ? (m_run[h2] + log2f(l_run[h2])) * 0.69314718055994531f : -FLT_MAX;
    if (NT == 4) {
      const int64_t t = t_pos + tok;
      if (t >= a.T) continue;
      uint16_t* orow = a.out + (t * 24 + h) * 256;
#pragma unroll
      for (int n = 0; n < 32; ++n) {
        const int dcol = 8 * n + 2 * (lane & 3);
        *reinterpret_cast<uint32_t*>(orow + dcol) = pack_bf16x2(o[n][2 * h2] * inv, o[n][2 * h2 + 1] * inv);
      }
      if (a.lse && (lane & 3) == 0) a.lse[t * 24 + h] = lse_v;
    } else {
      float* orow = a.part_o + ((b * a.n_split + split) * 24 + h) * 256;
#pragma unroll
      for (int n = 0; n < 32; ++n) {
        const int dcol = 8 * n + 2 * (lane & 3);
        *reinterpret_cast<float2*>(orow + dcol) = make_float2(o[n][2 * h2] * inv, o[n][2 * h2 + 1] * inv);
      }
      if ((lane & 3) == 0) a.part_lse[(b * a.n_split + split) * 24 + h] = lse_v;
    }
  }
}

// Merge of decode splits: out = sum_s w_s O_s / sum_s w_s, w_s = exp(lse_s - max).
__global__ void decode_combine_kernel(int n_split, const float* __restrict__ part_o,
                                      const float* __restrict__ part_lse, uint16_t* __restrict__ out,
                                      float* __restrict__ lse) {
  const int64_t b = blockIdx.x / 24;
  const int h = blockIdx.x % 24;
  const int d = threadIdx.x;                     // 256 threads, one per dim
  float mx = -FLT_MAX;
  for (int s = 0; s < n_split; ++s) mx = fmaxf(mx, part_lse[(b * n_split + s) * 24 + h]);
  float wsum = 0.f, acc = 0.f;
  for (int s = 0; s < n_split; ++s) {
    const float l = part_lse[(b * n_split + s) * 24 + h];
    if (l == -FLT_MAX) continue;
    const float w = __expf(l - mx);
    wsum += w;
    acc += w * part_o[((b * n_split + s) * 24 + h) * 256 + d];
  }
  out[(b * 24 + h) * 256 + d] = (uint16_t)f32_to_bf16_bits(wsum > 0.f ? acc / wsum : 0.f);
  if (lse && d == 0) lse[b * 24 + h] = mx + __logf(wsum);
}

template <int NT>
cudaError_t launch_attn(const AttnArgs& a, int64_t grid, cudaStream_t stream) {
  using C = Cfg<NT>;
  const size_t smem = C::SMEM_FIXED + (size_t)a.budget * 4;
  static size_t attr_set[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && attr_set[dev] < smem) {
    cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = smem;
  }
  sparse_attn_kernel<NT><<<(unsigned)grid, C::THREADS, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_attn_prefill(int64_t T, const uint16_t* q, const uint16_t* k_rot, const uint16_t* v,
                                       const float2* cs, const int32_t* sel, const int32_t* cnt, int budget,
                                       int64_t qb_begin, int64_t qb_end, float scale_log2, uint16_t* out, float* lse,
                                       cudaStream_t stream) {
  if (qb_end <= qb_begin) return cudaSuccess;
  AttnArgs a{};
  a.T = T; a.q = q; a.k = k_rot; a.v = v; a.cs = cs; a.sel = sel; a.cnt = cnt; a.budget = budget;
  a.qb_begin = qb_begin; a.scale_log2 = scale_log2; a.out = out; a.lse = lse;
  return launch_attn<4>(a, qb_end - qb_begin, stream);
}

cudaError_t launch_decode_attn(int B, int64_t max_len, const int64_t* L_dev, const uint16_t* q_rot,
                               const uint16_t* k_cache, const uint16_t* v_cache, const int32_t* sel,
                               const int32_t* cnt, int budget, int n_split, float scale_log2, float* part_o,
                               float* part_lse, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  AttnArgs a{};
  a.q = q_rot; a.k = k_cache; a.v = v_cache; a.sel = sel; a.cnt = cnt; a.budget = budget;
  a.scale_log2 = scale_log2; a.max_len = max_len; a.Ls = L_dev; a.n_split = n_split; a.part_o = part_o;
  a.part_lse = part_lse; a.T = INT64_MAX;
  return launch_attn<1>(a, (int64_t)B * n_split, s);
}

cudaError_t launch_decode_combine(int B, int n_split, const float* part_o, const float* part_lse, uint16_t* out,
                                  float* lse, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  decode_combine_kernel<<<(unsigned)(B * 24), 256, 0, s>>>(n_split, part_o, part_lse, out, lse);
  return cudaGetLastError();
}

}  // namespace qsa
