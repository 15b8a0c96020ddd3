// Stage 3 (prefill) on the 5th-generation tensor cores: sparse GQA attention
// over the selected micro-blocks ("sparse core attention", page "Qwen3.8-
// Flash-Next, 1/9의 학습 비용으로 Qwen3.7-Plus(397B-A17B) 수준에 도달한 125B-A6B
// 모델", section "QSA: 인덱서 자체의 비용을 줄이는 희소 어텐션"; shapes from its
// spec table).
//
//   out[t][h] = sum_j softmax_j(q_rot[t][h] . k_rot[j][g] / 16) v[j][g],
//   g = h / 12, j over the selected blocks of block t/4 with j <= t.
//
// Work item = (query block, KV head): 48 query rows (4 tokens x 12 heads)
// against up to budget x 4 keys.  Persistent CTAs (one per SM) walk the items.
//   * warps 0-7 (loaders): Q tile with RoPE applied on the fly, then the
//     selected K and V rows, 64 keys (16 blocks) per tile, gathered with
//     cp.async into the canonical 128-byte-swizzled K-major layout (8 KB per
//     64-dim chunk); a ring of three 32 KB K slots and one of three V slots.
//   * warp 10 (one thread): S = Q K^T with M = 128 (rows 48..127 are
//     padding whose results are never read), N = 64, K = 256 into one of
//     three TMEM S buffers; it frees the K slot.  Warp 11 (one thread):
//     O += P V with P taken from TMEM (A operand) and V as an MN-major
//     shared-memory operand, M = 128, N = 256, fp32 in TMEM; it frees the
//     V slot.
//   * warps 8-9 and 12-13 (softmax): two threads per query row (TMEM lanes
//     0..63), each with half of a tile's 64 columns: mask, running max in
//     base 2 (the two halves swap their tile maxima; the max is raised only
//     when a tile's max exceeds it by more than 8, so the O rescale is rare),
//     exp2, row sum, P packed to bf16 and stored back into the S buffer's
//     first 32 columns; at the end of an item each thread normalises and
//     writes its 128 of the row's 256 dims, bf16, with the row's lse.
//   * every mbarrier wait is bounded (timeout -> error word, clean exit): on
//     an abort every role leaves its loop, the loaders wait for their own
//     cp.async copies and each MMA issuer for its last commit (a wait that
//     ignores the abort) before TMEM is released.
#include <cfloat>

#include "qsa_device.cuh"
#include "qsa_kernels.h"

namespace qsa {
namespace {

constexpr int KT = 64;                              // keys per tile
// 8 loader warps issue a 64 KB tile in about half the time 4 take (the
// gathers are issue-bound between slot releases): 5 % faster at 1M tokens.
constexpr int LWARPS = 8;                            // loader warps (4 or 8)
constexpr int LOADERS = 32 * LWARPS;
constexpr int W_SOFT = LWARPS;                       // softmax warps W_SOFT, W_SOFT + 1 (columns 0..31)
constexpr int W_MMA = LWARPS + 2;
constexpr int W_SOFT2 = LWARPS + 4;                  // softmax warps W_SOFT2, W_SOFT2 + 1 (columns 32..63)
constexpr int THREADS = 32 * (LWARPS + 6);
constexpr uint32_t QROWS = 48;
constexpr uint32_t CHUNK_Q = QROWS * 128;           // 6 KB: 48 rows x 64 dims
constexpr uint32_t CHUNK_KV = KT * 128;             // 8 KB: 64 keys x 64 dims
constexpr uint32_t KV_BYTES = 4 * CHUNK_KV;         // 32 KB per K (or V) tile
constexpr uint32_t OFF_STAGE = 32768;               // Q region (24 KB) padded to 32 KB
constexpr uint32_t OFF_XCH = 4 * CHUNK_Q;           // softmax exchange (1 KB) in the Q region's padding
static_assert(OFF_XCH + 1024 <= OFF_STAGE, "exchange buffer");
// Separate K and V rings in the same 192 KB: a K slot is freed once S has
// read it, a V slot once P V has, so the next K tile lands while the
// softmax and P V of the current one run.  Three S / P buffers in TMEM let
// S run a tile further ahead of P V.  (2 K + 4 V slots, 4 K + 2 V slots or
// four S buffers were no faster; one ring of three K + V stages with two S
// buffers was 4 % slower at 1M tokens.)
constexpr int NK = 3, NV = 3;
constexpr int NSB = 3;                               // S / P buffers in TMEM
constexpr uint32_t OFF_V = OFF_STAGE + NK * KV_BYTES;
constexpr uint32_t OFF_BAR = OFF_V + NV * KV_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256;
static_assert(SMEM_BYTES <= 232448, "attention smem");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_S0 = 0, TM_O = 256;           // S buffers at columns 0, 64, 128; O at 256

__device__ __forceinline__ uint32_t swz128(uint32_t row, uint32_t c16) {
  return row * 128u + ((c16 ^ (row & 7u)) << 4);
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
// 32-byte global store (the address must be 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&x)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(x[0]), "r"(x[1]), "r"(x[2]),
               "r"(x[3]), "r"(x[4]), "r"(x[5]), "r"(x[6]), "r"(x[7])
               : "memory");
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// Two floats to packed bf16 (round to nearest even): lo in bits 0..15.
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// MN-major operand descriptor (128-byte swizzle): LBO = distance between
// 64-element atoms along N, SBO = distance between 8-row groups along K.
__device__ __forceinline__ uint64_t umma_desc_mn_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}
// O[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void umma_ts_bf16(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

struct TcArgs {
  int64_t T;                // keys are tokens [0, T)
  int64_t q_tok0;           // prefill: q, cs, out and lse start at token q_tok0
  const uint16_t* q;        // [T - q_tok0][24][256] unrotated
  const uint16_t* k_rot;    // [T][2][256]
  const uint16_t* v;        // [T][2][256]
  const float2* cs;         // [T][32] RoPE table
  const int32_t* sel;       // [rows][budget], rows relative to qb_begin
  const int32_t* cnt;       // [rows]
  int budget;
  int64_t qb_begin, n_qb;
  float scale_log2;
  uint16_t* out;            // [T][24][256]
  float* lse;               // [T][24] or null
  uint32_t* err;
  // decode: q = rotated new-token queries [B][24][256], k_rot / v = caches
  // [B][max_len][2][256], out / lse [B][24][...], one query token per sequence
  const int64_t* Ls;        // [rows] position of the row's query token
  int64_t rows_per_seq;     // decode rows per sequence (verify: the m new tokens), else 1
  int64_t max_len;
  // split-KV decode: each (sequence, KV head) is cut into n_split ranges of
  // whole tiles; with n_split > 1 every range writes its normalised O (fp32)
  // and its lse in base 2 to part_o [B][2][n_split][12][256] and
  // part_lse [B][2][n_split][12], merged afterwards by the combine kernel
  int n_split;
  float* part_o;
  float* part_lse;
  int inject;               // debug build: fault-injection code (QSA_INJECT_*), else 0
};

// One work item = (query block, KV head) for prefill, (sequence, KV head,
// split) for decode: the tiles [tile0, tile0 + n_tiles) of the row's selection
// (16 blocks per tile, nt_total tiles in all).  Items with no tile are skipped
// by every role alike.
template <bool DEC>
struct Item {
  int64_t row;              // selection row
  int g;                    // KV head
  int split;
  int cnt;                  // selected blocks of the row
  int nt_total, tile0, n_tiles;
  int64_t qb;               // query block
  int64_t t0;               // position of the item's first query token
  int64_t t_last;           // last key position any of its rows may read
  const uint16_t* kb;       // rotated keys of this sequence
  const uint16_t* vb;
  __device__ __forceinline__ Item(const TcArgs& a, int64_t w) {
    const int64_t rs = w >> 1;
    g = (int)(w & 1);
    row = DEC ? rs / a.n_split : rs;
    split = DEC ? (int)(rs % a.n_split) : 0;
    cnt = a.cnt[row];
    nt_total = (cnt + 15) / 16;
    const int per = DEC ? (nt_total + a.n_split - 1) / a.n_split : nt_total;
    tile0 = split * per;
    const int rest = nt_total - tile0;
    n_tiles = rest < 0 ? 0 : (rest < per ? rest : per);
    if (DEC) {
      const int64_t L = a.Ls[row];
      qb = L >> 2;
      t0 = L;
      t_last = L;
      kb = a.k_rot + (row / a.rows_per_seq) * a.max_len * 512;
      vb = a.v + (row / a.rows_per_seq) * a.max_len * 512;
    } else {
      qb = a.qb_begin + row;
      t0 = 4 * qb;
      t_last = 4 * qb + 3 < a.T - 1 ? 4 * qb + 3 : a.T - 1;
      kb = a.k_rot;
      vb = a.v;
    }
  }
};

template <bool DEC>
__global__ void __launch_bounds__(THREADS, 1) sparse_attn_tc_kernel(const TcArgs a) {
  constexpr int QR = DEC ? 12 : (int)QROWS;   // valid query rows per item
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;              // [NK]
  uint64_t* k_empty = k_full + NK;          // [NK]
  uint64_t* v_full = k_empty + NK;          // [NV]
  uint64_t* v_empty = v_full + NV;          // [NV]
  uint64_t* s_full = v_empty + NV;          // [NSB]
  uint64_t* p_full = s_full + NSB;          // [NSB]
  // [NSB]: P V number j completes pv_done[j % NSB]
  uint64_t* pv_done = p_full + NSB;
  uint64_t* o_full = pv_done + NSB;
  uint64_t* o_empty = o_full + 1;
  uint64_t* mma_done = o_empty + 1;          // [2]: the S and the P V issuer
  uint64_t* xbar = mma_done + 2;             // [2]: softmax row groups 0..31, 32..63
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xbar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((smem_u32(smem) & 1023u) != 0u) {
    if (tid == 0) report_error(a.err, QSA_ERR_DEVICE_BOUNDS);
    return;
  }
  if (tid == 0) {
    mbar_init(q_full, LOADERS);
    mbar_init(q_empty, 1);
    for (int s = 0; s < NK; ++s) { mbar_init(&k_full[s], LOADERS); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < NV; ++s) { mbar_init(&v_full[s], LOADERS); mbar_init(&v_empty[s], 1); }
    for (int b = 0; b < NSB; ++b) { mbar_init(&s_full[b], 1); mbar_init(&p_full[b], 4); mbar_init(&pv_done[b], 1); }
    mbar_init(&xbar[0], 64);
    mbar_init(&xbar[1], 64);
    mbar_init(o_full, 1);
    mbar_init(o_empty, 4);
    mbar_init(&mma_done[0], 1);
    mbar_init(&mma_done[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == W_MMA) { tmem_alloc(tmem_slot, TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t n_items = 2 * a.n_qb * (DEC ? a.n_split : 1);

  if (warp < LWARPS) {
    // ---------------------------------------------------------------- loaders
    int kst = 0, vst = 0;
    uint32_t keph = 1, veph = 1;
    uint32_t items_done = 0;
    bool ok = true;
    for (int64_t w = blockIdx.x; ok && w < n_items; w += gridDim.x) {
      const Item<DEC> it(a, w);
      if (it.n_tiles == 0) continue;
      const int g = it.g;
      const int32_t* sel = a.sel + it.row * a.budget + 16 * it.tile0;
      // Q tile, loaded after the item's first K / V tile is in flight (so
      // that tile's latency overlaps the wait for the previous item's last S
      // and the Q load).  Dims 64..255 (chunks 8..31) go by cp.async, zero-
      // filled past the sequence; prefill rotates dims 0..63 (pairs i, i+32,
      // chunks slot and slot + 4) in registers, decode queries arrive rotated.
      // The q_full arrival fires when this thread's copies have landed.
      auto load_q = [&]() -> bool {
        if (items_done > 0 && !mbar_wait(q_empty, (items_done - 1) & 1, abort_flag, a.err)) return false;
        for (int e = tid; e < QR * 24; e += LOADERS) {
          const int r = e / 24, q16 = 8 + e % 24;
          const int64_t t = it.t0 + r / 12;
          const int h = 12 * g + r % 12;
          const bool present = DEC || (t < a.T && t >= a.q_tok0);
          const uint16_t* src = present ? a.q + ((DEC ? it.row : t - a.q_tok0) * 24 + h) * 256 + 8 * q16 : a.q;
          cp_async16(smem_u32(smem + (q16 >> 3) * CHUNK_Q + swz128(r, q16 & 7)), src, present);
        }
        for (int e = tid; e < QR * 4; e += LOADERS) {
          const int r = e >> 2, slot = e & 3;
          const int64_t t = it.t0 + r / 12;
          const int h = 12 * g + r % 12;
          uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
          if (DEC || (t < a.T && t >= a.q_tok0)) {
            const uint4* src = reinterpret_cast<const uint4*>(a.q + ((DEC ? it.row : t - a.q_tok0) * 24 + h) * 256);
            lo = __ldg(src + slot);
            hi = __ldg(src + slot + 4);
            if (!DEC) {
              const float2* c8 = a.cs + (t - a.q_tok0) * 32 + 8 * slot;
              const uint32_t* x = reinterpret_cast<const uint32_t*>(&lo);
              const uint32_t* y = reinterpret_cast<const uint32_t*>(&hi);
              uint4 olo, ohi;
              uint32_t* ox = reinterpret_cast<uint32_t*>(&olo);
              uint32_t* oy = reinterpret_cast<uint32_t*>(&ohi);
#pragma unroll
              for (int p = 0; p < 4; ++p) {
                const float2 c0 = c8[2 * p], c1 = c8[2 * p + 1];
                const float x0 = bf16lo(x[p]), x1 = bf16hi(x[p]), y0 = bf16lo(y[p]), y1 = bf16hi(y[p]);
                ox[p] = pack_bf16x2(x0 * c0.x - y0 * c0.y, x1 * c1.x - y1 * c1.y);
                oy[p] = pack_bf16x2(y0 * c0.x + x0 * c0.y, y1 * c1.x + x1 * c1.y);
              }
              lo = olo;
              hi = ohi;
            }
          }
          *reinterpret_cast<uint4*>(smem + swz128(r, slot)) = lo;
          *reinterpret_cast<uint4*>(smem + swz128(r, slot + 4)) = hi;
        }
        fence_proxy_async();
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(q_full)) : "memory");
        return true;
      };
      // K / V tiles
      const int n_tiles = it.n_tiles;
      const int nsel = it.cnt - 16 * it.tile0;     // selected blocks from this item's first tile on
      const int64_t t_last = it.t_last;
      // Thread (warp w, lane c32) copies 16-byte chunk c32 of token w % 4 of
      // each of its KPT blocks of a tile (blocks k0 .. k0 + KPT - 1: warps
      // 0-3 the first 8 of the 16, warps 4-7 the last 8), for K and for V:
      // key slot n = 4k + w % 4.  The block indices of tiles i + 1 and i + 2
      // are loaded while tile i waits for its slots, so the index loads'
      // latency stays off the issue path.
      constexpr int KPT = 64 / LWARPS;
      const int w4 = (tid >> 5) & 3, c32 = tid & 31, k0 = KPT * (tid >> 7);
      // key positions fit in 32 bits (sequences are at most 2^24 tokens); a
      // key row holds both KV heads (512 elements), so the source of key j is
      // this lane's chunk of head g plus j * 512 elements, one wide multiply-add
      const int t_last32 = (int)t_last;
      const uint16_t* k_lane = it.kb + g * 256 + c32 * 8;
      const uint16_t* v_lane = it.vb + g * 256 + c32 * 8;
      int32_t kbv[KPT], kbn[KPT], kbm[KPT];
      auto load_idx = [&](int ti, int32_t (&dst)[KPT]) {
#pragma unroll
        for (int kk = 0; kk < KPT; ++kk) {
          const int k = 16 * ti + k0 + kk;
          dst[kk] = k < nsel ? __ldg(sel + k) : -1;
        }
      };
      load_idx(0, kbv);
      if (n_tiles > 1) load_idx(1, kbn);
      for (int i = 0; i < n_tiles; ++i) {
        if (i + 2 < n_tiles) load_idx(i + 2, kbm);
        if (!mbar_wait(&k_empty[kst], keph, abort_flag, a.err)) { ok = false; break; }
        size_t off[KPT];
        bool valid[KPT];
        {
          const uint32_t dst0 = smem_u32(smem + OFF_STAGE + kst * KV_BYTES) + (c32 >> 3) * CHUNK_KV;
#pragma unroll
          for (int kk = 0; kk < KPT; ++kk) {
            const int n = 4 * (k0 + kk) + w4;
#ifdef QSA_DEBUG_HOOKS
            // test hook: CTA 0's first tile names a block after the query
            // block (never read: the causal test below masks it too)
            if (a.inject == QSA_INJECT_ATTENTION_BAD_BLOCK && blockIdx.x == 0 && items_done == 0 && i == 0 &&
                k0 + kk == 0)
              kbv[kk] = (int)it.qb + 1;
#endif
            // a selected block is causal: -1 (padding) or 0 .. qb
            const bool in_range = kbv[kk] == -1 || QSA_BOUNDS_OK(kbv[kk] >= 0 && kbv[kk] <= it.qb, a.err);
            const int j = 4 * kbv[kk] + w4;
            valid[kk] = in_range && kbv[kk] >= 0 && j <= t_last32;
            off[kk] = valid[kk] ? (size_t)(uint32_t)j * 512u : 0;
            cp_async16(dst0 + swz128(n, c32 & 7), k_lane + off[kk], valid[kk]);
          }
        }
        // this thread's arrival fires when all its copies so far have landed:
        // no blocking wait, every slot in flight
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&k_full[kst]))
                     : "memory");
        if (!mbar_wait(&v_empty[vst], veph, abort_flag, a.err)) { ok = false; break; }
        {
          const uint32_t dst0 = smem_u32(smem + OFF_V + vst * KV_BYTES) + (c32 >> 3) * CHUNK_KV;
#pragma unroll
          for (int kk = 0; kk < KPT; ++kk) {
            const int n = 4 * (k0 + kk) + w4;
            cp_async16(dst0 + swz128(n, c32 & 7), v_lane + off[kk], valid[kk]);
          }
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&v_full[vst]))
                     : "memory");
        if (++kst == NK) { kst = 0; keph ^= 1; }
        if (++vst == NV) { vst = 0; veph ^= 1; }
#pragma unroll
        for (int kk = 0; kk < KPT; ++kk) { kbv[kk] = kbn[kk]; kbn[kk] = kbm[kk]; }
        if (i == 0 && !load_q()) { ok = false; break; }
      }
      ++items_done;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == W_MMA || warp == W_MMA + 1) {
    // -------------------------------------------------------------------- MMA
    // Two issuing threads: warp W_MMA issues every S, warp W_MMA + 1 every
    // P V, so a P V whose P is ready is not held behind the issue of the next
    // S (which waits for its K tile and for room in the tensor pipe); the
    // V slot a P V frees is refilled that much sooner.  S(i) overwrites the
    // TMEM buffer P(i - NSB) was read from, so it waits for P V(i - NSB).
    if (lane == 0) {
      const bool s_role = warp == W_MMA;
      constexpr uint32_t idesc_s = umma_idesc_bf16_f32(128, KT);
      constexpr uint32_t idesc_pv = umma_idesc_bf16_f32(128, 256) | (1u << 16);   // B (V) MN-major
      int stage = 0;                 // K slot (S issuer) or V slot (P V issuer)
      uint32_t fphase = 0;
      uint32_t items_done = 0, s_count = 0, p_count = 0;
      bool ok = true;
      const uint32_t q_base = smem_u32(smem);
      for (int64_t w = blockIdx.x; ok && w < n_items; w += gridDim.x) {
        const Item<DEC> it(a, w);
        const int n_tiles = it.n_tiles;
        if (n_tiles == 0) continue;
        if (s_role) {
          if (!mbar_wait(q_full, items_done & 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          for (int i = 0; i < n_tiles; ++i) {
            if (!mbar_wait(&k_full[stage], fphase, abort_flag, a.err)) { ok = false; break; }
            // P V number s_count - NSB read the buffer S(i) writes.  Its
            // barrier pv_done[(s_count - NSB) % NSB] is next completed by P V
            // s_count, which needs this S, and P V s_count - 2 NSB was waited
            // for before S(i - NSB), so the parity wait is exact
            if (s_count >= NSB) {
              const uint32_t g = s_count - NSB;
              if (!mbar_wait(&pv_done[g % NSB], (g / NSB) & 1, abort_flag, a.err)) { ok = false; break; }
            }
            fence_proxy_async();    // the slot was written by cp.async; the MMA reads it
            tc_fence_after();
            const uint32_t b = s_count % NSB;
            const uint32_t k_base = smem_u32(smem + OFF_STAGE + stage * KV_BYTES);
#pragma unroll
            for (int ks = 0; ks < 16; ++ks) {
              const uint32_t c = ks >> 2, koff = (ks & 3) * 32;
              const uint64_t ad = umma_desc_k_sw128(q_base + c * CHUNK_Q + koff);
              const uint64_t bd = umma_desc_k_sw128(k_base + c * CHUNK_KV + koff);
              umma_bf16(tmem + TM_S0 + 64 * b, ad, bd, idesc_s, ks > 0 ? 1u : 0u);
            }
#ifdef QSA_DEBUG_HOOKS
            // test hook: CTA 0 never signals its first S, so the softmax warps
            // time out and the CTA aborts
            if (!(a.inject == QSA_INJECT_ATTENTION_STALL && blockIdx.x == 0 && s_count == 0))
#endif
            tc_commit(&s_full[b]);
            tc_commit(&k_empty[stage]);
            if (i == n_tiles - 1) tc_commit(q_empty);
            ++s_count;
            if (++stage == NK) { stage = 0; fphase ^= 1; }
          }
        } else {
          for (int j = 0; j < n_tiles; ++j) {
            const uint32_t b = p_count % NSB;
            if (!mbar_wait(&p_full[b], (p_count / NSB) & 1, abort_flag, a.err)) { ok = false; break; }
            if (j == 0 && items_done > 0 && !mbar_wait(o_empty, (items_done - 1) & 1, abort_flag, a.err)) {
              ok = false;
              break;
            }
            if (!mbar_wait(&v_full[stage], fphase, abort_flag, a.err)) { ok = false; break; }
            fence_proxy_async();    // the slot was written by cp.async; the MMA reads it
            tc_fence_after();
            const uint32_t v_base = smem_u32(smem + OFF_V + stage * KV_BYTES);
#pragma unroll
            for (int ks = 0; ks < KT / 16; ++ks) {
              const uint64_t bd = umma_desc_mn_sw128(v_base + ks * 2048, CHUNK_KV, 1024);
              umma_ts_bf16(tmem + TM_O, tmem + TM_S0 + 64 * b + 8 * ks, bd, idesc_pv, (j > 0 || ks > 0) ? 1u : 0u);
            }
            tc_commit(&v_empty[stage]);
            tc_commit(&pv_done[p_count % NSB]);
            if (j == n_tiles - 1) tc_commit(o_full);
            ++p_count;
            if (++stage == NV) { stage = 0; fphase ^= 1; }
          }
        }
        ++items_done;
      }
      // every MMA this thread issued has retired before TMEM is released
      // (also after an abort: a wait that ignores the abort flag)
      uint64_t* done = &mma_done[s_role ? 0 : 1];
      tc_commit(done);
      mbar_wait_drain(done, 0, a.err);
    }
  } else if (warp == W_SOFT || warp == W_SOFT + 1 || warp == W_SOFT2 || warp == W_SOFT2 + 1) {
    // ---------------------------------------------------------------- softmax
    // Four warps: warps W_SOFT, W_SOFT + 1 take columns 0..31 of each tile's
    // S for query rows 0..31 and 32..63, warps W_SOFT2, W_SOFT2 + 1 columns
    // 32..63 of the same rows (a warp reaches TMEM lanes 32 (warp % 4) ..).
    // The two threads of a row swap their tile maxima (and at the end of an
    // item their row sums) through shared memory and a per-row-group
    // mbarrier, so both use the same running max; each rescales, normalises
    // and writes its own 128 of the row's 256 output dims.
    const int half = warp >= W_SOFT2 ? 1 : 0;
    const int quad = warp & 3;                      // 0 or 1: TMEM lanes 32 quad ..
    const int r = 32 * quad + lane;                 // query row = TMEM lane
    const bool row_ok = r < QR;
    const int tok = row_ok ? r / 12 : 0, hh = row_ok ? r % 12 : 0;
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    float* xch = reinterpret_cast<float*>(smem + OFF_XCH);   // [2 slots][2 halves][64 rows]
    uint64_t* xb = &xbar[quad];
    uint32_t xc = 0;                                // exchanges so far (slot and parity)
    // swap a value with the other thread of this row; false on abort / timeout
    auto exchange = [&](float mine, float& other) -> bool {
      const uint32_t slot = xc & 1;
      xch[(slot * 2 + half) * 64 + r] = mine;
      mbar_arrive(xb);                              // every lane: releases its own store
      const bool okx = __all_sync(0xffffffffu, mbar_wait(xb, xc & 1, abort_flag, a.err));
      other = xch[(slot * 2 + (half ^ 1)) * 64 + r];
      ++xc;
      return okx;
    };
    uint32_t items_done = 0, s_count = 0, pv_seq = 0;
    bool ok = true;
    for (int64_t w = blockIdx.x; ok && w < n_items; w += gridDim.x) {
      const Item<DEC> it(a, w);
      const int n_tiles = it.n_tiles;
      if (n_tiles == 0) continue;
      const int g = it.g;
      const int cnt = it.cnt;
      const int64_t t = it.t0 + tok;                  // this row's token position
      const int own_lim = (int)(t & 3);               // last visible token of the own block
      float m_run = -FLT_MAX, l_run = 0.f;
      for (int i = 0; i < n_tiles; ++i) {
        const uint32_t b = s_count % NSB;
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[b], (s_count / NSB) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[32];
        tmem_ld32(tmem + lane_off + TM_S0 + 64 * b + 32 * half, s);
        tmem_ld_wait(s);
        // Masking.  The selection is ascending and always ends with the own
        // block, so every key of a tile before the last one is visible to
        // every row; in the last tile, slots past cnt and the own block's
        // tokens after the row's token are masked.
        const int gi = it.tile0 + i;                  // tile index within the row's selection
        const bool last = gi == it.nt_total - 1;
        if (last) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int blk = 16 * gi + 8 * half + (c >> 2);
            const bool valid = blk < cnt && (blk < cnt - 1 || (c & 3) <= own_lim);
            s[c] = valid ? s[c] : -FLT_MAX;
          }
        }
        float mt = -FLT_MAX;
#pragma unroll
        for (int c = 0; c < 30; c += 3) mt = fmaxf(mt, max3f(s[c], s[c + 1], s[c + 2]));
        mt = fmaxf(mt, fmaxf(s[30], s[31]));
        mt = row_ok ? mt * a.scale_log2 : -FLT_MAX;   // raw max, then the (positive) scale
        // both threads of the row have read their S columns before either
        // writes P over them
        float mt_other;
        if (!exchange(mt, mt_other)) { ok = false; break; }
        mt = fmaxf(mt, mt_other);
#ifdef QSA_DEBUG_HOOKS
        // test hook: no lazy margin, every tile takes the new maximum and
        // rescales O (corr = 1 where the maximum did not grow)
        const bool need = a.inject == QSA_INJECT_ATTENTION_RESCALE_ALL || mt > m_run + 8.f;
#else
        const bool need = mt > m_run + 8.f;
#endif
        if (__any_sync(0xffffffffu, need)) {
          const float m_new = need ? fmaxf(m_run, mt) : m_run;
          const float corr = ex2(m_run - m_new);
          l_run *= corr;
          m_run = m_new;
          if (i >= 1) {
            // O may be rescaled only once P V(i - 1), number g = pv_seq + i - 1,
            // has accumulated into it.  S(i) has completed and was issued after
            // P V(i - NSB) completed, and P V(g + NSB) cannot have (it needs
            // P(i + 1) at least), so the parity of pv_done[g % NSB] is exact.
            // Only this rare path waits, so the softmax of tile i overlaps
            // P V(i - 1).
            const uint32_t g = pv_seq + (uint32_t)i - 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[g % NSB], (g / NSB) & 1, abort_flag, a.err))) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              float o[32];
              tmem_ld32(tmem + lane_off + TM_O + 128 * half + 32 * c, o);
              tmem_ld_wait(o);
              uint32_t u[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(o[e] * corr);
              tmem_st32(tmem + lane_off + TM_O + 128 * half + 32 * c, u);
            }
            tmem_st_wait();
          }
        }
        // p = 2^(s*scale - m); masked slots (-FLT_MAX) underflow to exactly 0
        uint32_t pk[16];
        float lsum0 = 0.f, lsum1 = 0.f;
        const float neg_m = -m_run;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2(fmaf(s[2 * e], a.scale_log2, neg_m));
          const float p1 = ex2(fmaf(s[2 * e + 1], a.scale_log2, neg_m));
          lsum0 += p0;
          lsum1 += p1;
          pk[e] = cvt_bf16x2(p0, p1);
        }
        l_run += lsum0 + lsum1;
        // keys 32 half .. +31 of the tile, packed two per column
        tmem_st16(tmem + lane_off + TM_S0 + 64 * b + 16 * half, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
        ++s_count;
      }
      if (!ok) break;
      // item end: O / l -> bf16
      if (!__all_sync(0xffffffffu, mbar_wait(o_full, items_done & 1, abort_flag, a.err))) { ok = false; break; }
      pv_seq += (uint32_t)n_tiles;   // every P V of the item has completed
      tc_fence_after();
      float l_other;
      if (!exchange(l_run, l_other)) { ok = false; break; }
      const float l_row = l_run + l_other;
      const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
      const bool write = row_ok && (DEC || (t < a.T && t >= a.q_tok0));
      const int64_t orow_idx = (DEC ? it.row : t - a.q_tok0) * 24 + 12 * g + hh;   // [token or sequence][head]
      uint16_t* orow = a.out + orow_idx * 256 + 128 * half;
      const bool partial = DEC && a.n_split > 1;
      const bool out32 = (reinterpret_cast<uintptr_t>(a.out) & 31) == 0;   // rows are 512 B apart
      const bool part32 = (reinterpret_cast<uintptr_t>(a.part_o) & 31) == 0;
      const int64_t prow = ((it.row * 2 + g) * (int64_t)a.n_split + it.split) * 12 + hh;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(tmem + lane_off + TM_O + 128 * half + 32 * c, o);
        tmem_ld_wait(o);
        // 32-byte stores where the output allows (full sectors, half the
        // store instructions of 16-byte ones)
        if (write && partial && part32) {
          float* dst = a.part_o + prow * 256 + 128 * half + 32 * c;   // rows are 1 KB apart
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = __float_as_uint(o[8 * q + e] * inv);
            st_global_v8(dst + 8 * q, x);
          }
        } else if (write && partial) {
          float4* dst = reinterpret_cast<float4*>(a.part_o + prow * 256 + 128 * half + 32 * c);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(o[4 * q] * inv, o[4 * q + 1] * inv, o[4 * q + 2] * inv, o[4 * q + 3] * inv);
        } else if (write && out32) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = cvt_bf16x2(o[16 * q + 2 * e] * inv, o[16 * q + 2 * e + 1] * inv);
            st_global_v8(orow + 32 * c + 16 * q, x);
          }
        } else if (write) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(cvt_bf16x2(o[8 * q] * inv, o[8 * q + 1] * inv),
                                cvt_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                                cvt_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                                cvt_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
        }
      }
      if (half == 0) {
        if (write && partial) a.part_lse[prow] = m_run + log2f(l_row);
        else if (write && a.lse) a.lse[orow_idx] = (m_run + log2f(l_row)) * 0.69314718055994531f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
      ++items_done;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

constexpr int MAX_SPLIT = 16;

// Split-KV merge, one CTA per (sequence, query head), one thread per dim:
// the ranges' normalised O weighted by 2^(lse_s - max) and renormalised, and
// lse = (max + log2 sum) ln 2.  Ranges without tiles are the ones the
// attention kernel skipped.
__global__ void __launch_bounds__(256) decode_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_lse,
                                                             const int32_t* __restrict__ cnt, int n_split,
                                                             uint16_t* __restrict__ out, float* __restrict__ lse) {
  const int bh = blockIdx.x;                    // sequence * 24 + head
  const int b = bh / 24, h = bh % 24, g = h / 12, hh = h % 12;
  const int d = threadIdx.x;
  const int nt = (cnt[b] + 15) / 16;
  const int per = (nt + n_split - 1) / n_split;
  const int ns = per > 0 ? (nt + per - 1) / per : 0;
  const int64_t row0 = ((int64_t)(b * 2 + g) * n_split) * 12 + hh;
  // all loads issued before any use (at most MAX_SPLIT ranges)
  float l2[MAX_SPLIT], ov[MAX_SPLIT];
#pragma unroll
  for (int sp = 0; sp < MAX_SPLIT; ++sp) {
    l2[sp] = sp < ns ? part_lse[row0 + 12 * sp] : -FLT_MAX;
    ov[sp] = sp < ns ? part_o[(row0 + 12 * sp) * 256 + d] : 0.f;
  }
  float mx = -FLT_MAX;
#pragma unroll
  for (int sp = 0; sp < MAX_SPLIT; ++sp) mx = fmaxf(mx, l2[sp]);
  float wsum = 0.f, acc = 0.f;
#pragma unroll
  for (int sp = 0; sp < MAX_SPLIT; ++sp) {
    if (sp < ns) {
      const float wgt = exp2f(l2[sp] - mx);
      wsum += wgt;
      acc = fmaf(wgt, ov[sp], acc);
    }
  }
  const float o = wsum > 0.f ? acc / wsum : 0.f;
  out[(int64_t)bh * 256 + d] = (uint16_t)f32_to_bf16_bits(o);
  if (lse && d == 0) lse[bh] = (mx + log2f(wsum)) * 0.69314718055994531f;
}

template <bool DEC>
cudaError_t launch_tc(const TcArgs& a, int64_t items, int num_sms, cudaStream_t stream) {
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(sparse_attn_tc_kernel<DEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const int grid = (int)(items < num_sms ? items : num_sms);
  sparse_attn_tc_kernel<DEC><<<grid, THREADS, SMEM_BYTES, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_attn_prefill_tc(int64_t T, const uint16_t* q, const uint16_t* k_rot, const uint16_t* v,
                                          const float2* cs, const int32_t* sel, const int32_t* cnt, int budget,
                                          int64_t qb_begin, int64_t qb_end, int64_t q_tok0, float scale_log2,
                                          uint16_t* out, float* lse, uint32_t* err, int num_sms, cudaStream_t stream) {
  if (qb_end <= qb_begin) return cudaSuccess;
  TcArgs a{};
  a.T = T; a.q_tok0 = q_tok0; a.q = q; a.k_rot = k_rot; a.v = v; a.cs = cs; a.sel = sel; a.cnt = cnt; a.budget = budget;
  a.qb_begin = qb_begin; a.n_qb = qb_end - qb_begin; a.scale_log2 = scale_log2; a.out = out; a.lse = lse;
  a.err = err; a.n_split = 1;
  a.inject = take_debug_injection(QSA_INJECT_ATTENTION_STALL);
  if (a.inject == 0) a.inject = take_debug_injection(QSA_INJECT_ATTENTION_BAD_BLOCK);
  if (a.inject == 0) a.inject = take_debug_injection(QSA_INJECT_ATTENTION_RESCALE_ALL);
  return launch_tc<false>(a, 2 * (qb_end - qb_begin), num_sms, stream);
}

cudaError_t launch_decode_attn_tc(int B, int64_t max_len, const int64_t* L_dev, const uint16_t* q_rot,
                                  const uint16_t* k_cache, const uint16_t* v_cache, const int32_t* sel,
                                  const int32_t* cnt, int budget, float scale_log2, int n_split, float* part_o,
                                  float* part_lse, uint16_t* out, float* lse, uint32_t* err, int num_sms,
                                  cudaStream_t stream, int rows_per_seq) {
  if (B <= 0) return cudaSuccess;
  if (n_split < 1 || rows_per_seq < 1) return cudaErrorInvalidValue;
  TcArgs a{};
  a.T = INT64_MAX; a.q = q_rot; a.k_rot = k_cache; a.v = v_cache; a.sel = sel; a.cnt = cnt; a.budget = budget;
  a.qb_begin = 0; a.n_qb = B; a.scale_log2 = scale_log2; a.out = out; a.lse = lse; a.err = err;
  a.Ls = L_dev; a.max_len = max_len; a.rows_per_seq = rows_per_seq;
  a.n_split = n_split; a.part_o = part_o; a.part_lse = part_lse;
  a.inject = take_debug_injection(QSA_INJECT_ATTENTION_RESCALE_ALL);
  return launch_tc<true>(a, 2 * (int64_t)B * n_split, num_sms, stream);
}

cudaError_t launch_decode_combine(int B, const float* part_o, const float* part_lse, const int32_t* cnt, int n_split,
                                  uint16_t* out, float* lse, cudaStream_t stream) {
  if (B <= 0) return cudaSuccess;
  if (n_split < 1 || n_split > MAX_SPLIT) return cudaErrorInvalidValue;
  decode_combine_kernel<<<B * 24, 256, 0, stream>>>(part_o, part_lse, cnt, n_split, out, lse);
  return cudaGetLastError();
}

}  // namespace qsa
