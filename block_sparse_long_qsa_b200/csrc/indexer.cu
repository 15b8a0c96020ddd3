// Stage 1, prefill: indexer block scores on the 5th-generation tensor cores.
//
//   s(t, j)   = sum_h w[t][h] * ReLU(q_idx[t][h] . k_idx[j]) / sqrt(128)
//   S(qb, kb) = max over t in block qb, j in block kb, j <= t, of s(t, j)
//
// ([PT] = page "Qwen3.8-Flash-Next, 1/9의 학습 비용으로 Qwen3.7-Plus(397B-A17B)
// 수준에 도달한 125B-A6B 모델", section "QSA: 인덱서 자체의 비용을 줄이는 희소
// 어텐션", eq. I_ib: ReLU of the per-head similarity, summed over the 4
// indexer heads; block-causal scoring of r = 4 token micro-blocks.)
//
// Design (one persistent CTA per SM, 576 threads):
//   * A = 128 keys x 128 dims (K-major, TMA, 128B swizzle), B = 64 query tokens
//     x 4 heads = 256 rows x 128 dims; D = A B^T is 128 x 256 fp32 in TMEM, so a
//     TMEM lane is one key and the 4 head values of one token sit in 4
//     consecutive columns of that lane.  The head-weighted ReLU sum and the max
//     over the 4 tokens of a query block happen in one thread's registers; the
//     max over the 4 keys of a key block is two warp shuffles.
//   * A query tile is 128 tokens (two N = 256 halves, two TMEM accumulators of
//     256 columns); each 32 KB key tile loaded from HBM feeds 2 x 8.4 MFLOP.
//   * Work unit = (query tile, key tile).  The causal triangle's units are
//     split evenly across CTAs in query-major order, so every CTA gets the
//     same number of MMAs whatever the chunk shape.
//   * warp 0: producer (3-stage TMA key ring, TMA Q tile, head weights); warp 1: TMEM
//     allocation and the single MMA-issuing thread; warps 2-17: epilogue,
//     8 warps per TMEM accumulator (tcgen05.ld -> ReLU, head weights, block
//     max -> fp32 scores), each 32-column load in flight behind the previous chunk.
//   * Every mbarrier wait is bounded; on timeout the CTA records
//     QSA_ERR_DEVICE_TIMEOUT and every role leaves its loop; before TMEM is
//     released the MMA thread waits for its last commit and the producer for
//     its last TMA loads (waits that ignore the abort), so nothing is in
//     flight when the CTA exits.
#include <type_traits>

#include "qsa_device.cuh"
#include "qsa_kernels.h"

namespace qsa {
namespace {

constexpr int QT = 128;                 // query tokens per tile
constexpr int KT = 128;                 // keys per tile
constexpr int STAGES = 3;
constexpr int THREADS = 576;
constexpr uint32_t Q_SUB_BYTES = 256 * 128;              // 256 rows x 64 bf16
constexpr uint32_t Q_BYTES = 4 * Q_SUB_BYTES;            // [half][k-chunk]
constexpr uint32_t K_SUB_BYTES = 128 * 128;              // 128 rows x 64 bf16
constexpr uint32_t K_STAGE_BYTES = 2 * K_SUB_BYTES;
constexpr uint32_t W_BYTES = QT * 4 * 4;                 // fp32 [128][4]
constexpr uint32_t OFF_K = Q_BYTES;
constexpr uint32_t OFF_W = OFF_K + STAGES * K_STAGE_BYTES;
constexpr uint32_t OFF_BAR = OFF_W + W_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 128;
static_assert(SMEM_BYTES <= 232448, "indexer smem");
constexpr uint32_t TMEM_COLS = 512;

// Key bands of BAND key tiles (32 MB of indexer keys): every band's units
// (query tile ascending, then key tile) are split evenly across the CTAs and
// the CTAs take the bands in order, so at any time they all read the same
// band of keys, which L2 serves to all of them, instead of sweeping the whole
// key range at unrelated offsets.  A query tile's Q operand is loaded once per
// (band, query tile) segment of a CTA.  Measured on B200 (1M tokens): DRAM
// reads of the indexer 37x lower than with one query-major split, and the 1M
// prefill 3-4 % faster (the power the reads drew goes to the clock); bands
// of 64 key tiles were slower (more Q reloads), 256 and 1024 alike.
constexpr int64_t BAND = 1024;

struct Sched {
  int64_t T0, Tend, n_tiles;
  int64_t qb_begin;
  int64_t R;                      // tokens per key-tile row: 1 (keys) or 4 (mean-pooled key blocks)
  int64_t A;                      // (T0 + QT - 1) / QT
  int64_t n_bands;
  __device__ __forceinline__ int64_t nkt(int64_t i) const {
    int64_t tl = T0 + QT * i + (QT - 1);
    if (tl > Tend - 1) tl = Tend - 1;
    return tl / (KT * R) + 1;
  }
  // sum over m < N of floor(m / R)
  __device__ __forceinline__ int64_t G(int64_t N) const {
    const int64_t q = N / R, r = N % R;
    return R * q * (q - 1) / 2 + r * q;
  }
  // units before tile i in query-major order (valid for i <= n_tiles - 1;
  // tiles before the last are full): sum over j < i of floor((A + j) / R) + 1
  __device__ __forceinline__ int64_t prefix(int64_t i) const { return i + G(A + i) - G(A); }
  __device__ __forceinline__ int64_t total() const { return prefix(n_tiles - 1) + nkt(n_tiles - 1); }
  // sum over j < i of nkt(j), 0 <= i <= n_tiles
  __device__ __forceinline__ int64_t sum_nkt(int64_t i) const { return i < n_tiles ? prefix(i) : total(); }
  // first tile j in [0, i) with nkt(j) >= x (nkt is non-decreasing), or i
  __device__ __forceinline__ int64_t first_reaching(int64_t i, int64_t x) const {
    int64_t lo = 0, hi = i;
    while (lo < hi) {
      const int64_t mid = (lo + hi) >> 1;
      if (nkt(mid) >= x) hi = mid; else lo = mid + 1;
    }
    return lo;
  }
  // sum over j < i of min(nkt(j), x): the units of tiles [0, i) with key tile < x
  __device__ __forceinline__ int64_t cmin(int64_t i, int64_t x) const {
    const int64_t f = first_reaching(i, x);
    return sum_nkt(f) + (i - f) * x;
  }
  // units before band b (key tiles < BAND b of every tile)
  __device__ __forceinline__ int64_t band_start(int64_t b) const { return cmin(n_tiles, BAND * b); }
  // units of band b in tiles [0, i)
  __device__ __forceinline__ int64_t in_band(int64_t b, int64_t i) const {
    return cmin(i, BAND * (b + 1)) - cmin(i, BAND * b);
  }
};

// A CTA's units: in every band, its even share (CTA c of G takes band
// positions [U_b c / G, U_b (c + 1) / G) of the band's U_b units), band after
// band, so all CTAs sweep the same band at the same time.
struct IterBand {
  const Sched* s;
  int64_t v, v_begin, v_end;   // position in the band's unit order; this CTA's range in the band
  int64_t tile, kt;
  int64_t left;                // units this CTA has left, this one included
  int band, seg_end;           // band; one past the last key tile of this (band, tile) segment
  int64_t cta, ncta;
  __device__ __forceinline__ void range(int b, int64_t& lo, int64_t& hi) const {
    const int64_t n = s->band_start(b + 1) - s->band_start(b);
    lo = n * cta / ncta;
    hi = n * (cta + 1) / ncta;
  }
  __device__ __forceinline__ void set_seg_end() {
    const int64_t n = s->nkt(tile), e = BAND * (band + 1);
    seg_end = (int)(n < e ? n : e);
  }
  // next band with units for this CTA, positioned at its first one
  __device__ __forceinline__ void advance_band() {
    for (++band; band < s->n_bands; ++band) {
      range(band, v_begin, v_end);
      if (v_end > v_begin) break;
    }
    if (band >= s->n_bands) return;
    v = v_begin;
    int64_t tl = 0, th = s->n_tiles - 1;         // largest tile whose in-band offset <= v
    while (tl < th) {
      const int64_t mid = (tl + th + 1) >> 1;
      if (s->in_band(band, mid) <= v) tl = mid; else th = mid - 1;
    }
    tile = tl;
    kt = BAND * band + (v - s->in_band(band, tile));
    set_seg_end();
  }
  // (u0, u1: the query-major split, unused by this schedule)
  __device__ __forceinline__ void begin(const Sched* sch, int64_t, int64_t) {
    s = sch; cta = blockIdx.x; ncta = gridDim.x;
    left = 0;
    for (int b = 0; b < s->n_bands; ++b) {
      int64_t lo, hi;
      range(b, lo, hi);
      left += hi - lo;
    }
    band = -1;
    if (left > 0) advance_band();
  }
  __device__ __forceinline__ bool valid() const { return left > 0; }
  // a new segment starts (a new query tile, or this CTA's first unit of a
  // band): the Q tile is (re)loaded
  __device__ __forceinline__ bool first_of_tile(int64_t) const { return kt == BAND * band || v == v_begin; }
  // the next unit of this CTA belongs to another segment
  __device__ __forceinline__ bool tile_ends_here() const {
    return (kt == seg_end - 1 || v + 1 == v_end) && left > 1;
  }
  __device__ __forceinline__ void next() {
    --left; ++v; ++kt;
    if (left <= 0) return;
    if (v == v_end) { advance_band(); return; }
    if (kt < seg_end) return;
    ++tile;                       // the next tile of the band (it reaches into the band too)
    kt = BAND * band;
    set_seg_end();
  }
};

// The units split evenly across CTAs in query-major order (the schedule of
// the mean-pooled indexer, whose compressed keys are a quarter of the size;
// its epilogue is at the register limit and the band bookkeeping spills).
struct IterQuery {
  const Sched* s;
  int64_t u, u_end, tile, kt, nkt;
  // units [u0, u1) of the query-major order
  __device__ __forceinline__ void begin(const Sched* sch, int64_t u0, int64_t u1) {
    s = sch; u = u0; u_end = u1;
    if (u < u_end) {
      int64_t lo = 0, hi = s->n_tiles - 1;
      while (lo < hi) {
        const int64_t mid = (lo + hi + 1) >> 1;
        if (s->prefix(mid) <= u) lo = mid; else hi = mid - 1;
      }
      tile = lo;
      kt = u - s->prefix(lo);
      nkt = s->nkt(tile);
    }
  }
  __device__ __forceinline__ bool valid() const { return u < u_end; }
  __device__ __forceinline__ bool first_of_tile(int64_t u0) const { return kt == 0 || u == u0; }
  __device__ __forceinline__ bool tile_ends_here() const { return kt == nkt - 1 && u + 1 < u_end; }
  __device__ __forceinline__ void next() {
    ++u; ++kt;
    if (kt == nkt) { ++tile; kt = 0; if (u < u_end) nkt = s->nkt(tile); }
  }
};

template <bool MEAN>
__global__ void __launch_bounds__(THREADS, 1)
indexer_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const uint16_t* __restrict__ w, float* __restrict__ S, int64_t ld,
                       float* __restrict__ segmax, int64_t ld_seg, int64_t T, int64_t q_tok0, int64_t qb_begin,
                       int64_t qb_end,
                       float scale, uint32_t* err, int inject) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sK = smem + OFF_K;
  const float* sW = reinterpret_cast<const float*>(smem + OFF_W);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* full = bars;               // [STAGES]
  uint64_t* empty = bars + STAGES;     // [STAGES]
  uint64_t* qfull = bars + 2 * STAGES;
  uint64_t* qempty = qfull + 1;
  uint64_t* accfull = qfull + 2;       // [2]
  uint64_t* accempty = qfull + 4;      // [2]
  uint64_t* done = qfull + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qfull + 7);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  using It = std::conditional_t<MEAN, IterQuery, IterBand>;

  if ((smem_u32(smem) & 1023u) != 0u) {  // the swizzled operand layout needs 1 KB alignment
    if (threadIdx.x == 0) report_error(err, QSA_ERR_DEVICE_BOUNDS);
    return;
  }

  Sched sch;
  sch.qb_begin = qb_begin;
  sch.T0 = qb_begin * 4;
  sch.Tend = qb_end * 4 < T ? qb_end * 4 : T;
  sch.n_tiles = (sch.Tend - sch.T0 + QT - 1) / QT;
  sch.R = MEAN ? 4 : 1;
  sch.A = (sch.T0 + QT - 1) / QT;
  sch.n_bands = MEAN ? 1 : (sch.nkt(sch.n_tiles - 1) + BAND - 1) / BAND;
  const int64_t W = sch.total();
  const int64_t u0 = W * (int64_t)blockIdx.x / gridDim.x;
  const int64_t u1 = W * (int64_t)(blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(qfull, 1);
    mbar_init(qempty, 1 + 16);
    for (int h = 0; h < 2; ++h) { mbar_init(&accfull[h], 1); mbar_init(&accempty[h], 8); }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp walks the units: at each new query tile all lanes load
    // the tile's head weights (bf16 -> fp32 into shared memory) and lane 0
    // issues the TMA loads; control flow stays warp-uniform so every exit is
    // taken by all lanes together.
    if (lane == 0) { tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); }
    float* sWf = reinterpret_cast<float*>(smem + OFF_W);
    It it; it.begin(&sch, u0, u1);
    int stage = 0; uint32_t ephase = 1; uint32_t qcount = 0;
    // for the drain at exit: bit s of `issued` / `par` = a load was issued into
    // stage s / the full-barrier phase parity of the last one; the same for
    // the Q tile (bit 31 of last_qpar: none issued)
    uint32_t issued = 0, par = 0;
    uint32_t last_qpar = 1u << 31;
    for (; it.valid(); it.next()) {
      if (it.first_of_tile(u0)) {
        bool ok = qcount == 0 || mbar_wait(qempty, (qcount - 1) & 1, abort_flag, err);
        if (!__all_sync(0xffffffffu, ok)) break;
        const int64_t t_first = sch.T0 + QT * it.tile;
        // lane l: tokens t_first + 4l .. +3
        float wv[16];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t t = t_first + 4 * lane + u;
          uint2 raw = make_uint2(0u, 0u);
          if (t < T) raw = __ldg(reinterpret_cast<const uint2*>(w + 4 * (t - q_tok0)));
          wv[4 * u + 0] = bf16lo(raw.x); wv[4 * u + 1] = bf16hi(raw.x);
          wv[4 * u + 2] = bf16lo(raw.y); wv[4 * u + 3] = bf16hi(raw.y);
        }
        // stored as token pairs: pair p holds {w(2p, h), w(2p+1, h)} for h = 0..3;
        // heads 2 and 3 are scaled by 2^64 to pair with relu_scaled() in the epilogue
        float4* dst = reinterpret_cast<float4*>(sWf + 16 * lane);
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
          const float* a0 = wv + 8 * pr;        // token 4*lane + 2*pr
          const float* a1 = a0 + 4;             // token 4*lane + 2*pr + 1
          dst[2 * pr] = make_float4(a0[0], a1[0], a0[1], a1[1]);
          dst[2 * pr + 1] = make_float4(a0[2] * kReluSatScale, a1[2] * kReluSatScale, a0[3] * kReluSatScale,
                                        a1[3] * kReluSatScale);
        }
        __syncwarp();
        if (lane == 0) {
          last_qpar = qcount & 1;
          mbar_arrive_expect_tx(qfull, Q_BYTES);
          for (int hf = 0; hf < 2; ++hf)
            for (int kc = 0; kc < 2; ++kc)
              tma_load_2d(sQ + (hf * 2 + kc) * Q_SUB_BYTES, &tm_q, kc * 64, (int32_t)(4 * (t_first - q_tok0) + 256 * hf),
                          qfull);
        }
        ++qcount;
      }
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(&empty[stage], ephase, abort_flag, err);
        if (ok) {
          // the load completes phase (wraps of this stage) of full[stage]
          issued |= 1u << stage;
          par = (par & ~(1u << stage)) | ((ephase ^ 1u) << stage);
          mbar_arrive_expect_tx(&full[stage], K_STAGE_BYTES);
          for (int kc = 0; kc < 2; ++kc)
            tma_load_2d(sK + stage * K_STAGE_BYTES + kc * K_SUB_BYTES, &tm_k, kc * 64, (int32_t)(KT * it.kt),
                        &full[stage]);
        }
      }
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
      if (++stage == STAGES) { stage = 0; ephase ^= 1; }
    }
    // Drain: every TMA load this warp issued has landed before the CTA exits
    // (after an abort some were never consumed).  A stage's full barrier
    // cannot move past its last issued load, so the parity test is exact.
    if (lane == 0) {
#pragma unroll
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u) mbar_wait_drain(&full[s], (par >> s) & 1u, err);
      if (last_qpar <= 1u) mbar_wait_drain(qfull, last_qpar, err);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(128, 256);
      It it; it.begin(&sch, u0, u1);
      int stage = 0; uint32_t fphase = 0; uint32_t qcount = 0;
      uint32_t acc_use[2] = {0, 0};
      bool ok = true;
      for (; ok && it.valid(); it.next()) {
        if (it.first_of_tile(u0)) {
          if (!mbar_wait(qfull, qcount & 1, abort_flag, err)) break;
          ++qcount;
        }
        if (!mbar_wait(&full[stage], fphase, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(sK + stage * K_STAGE_BYTES);
        for (int hf = 0; hf < 2; ++hf) {
          if (!mbar_wait(&accempty[hf], (acc_use[hf] & 1) ^ 1, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t b_base = smem_u32(sQ + hf * 2 * Q_SUB_BYTES);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t koff = (uint32_t)(k & 3) * 32;      // 16 bf16 = 32 bytes inside the swizzle atom
            const uint64_t ad = umma_desc_k_sw128(a_base + (k >> 2) * K_SUB_BYTES + koff);
            const uint64_t bd = umma_desc_k_sw128(b_base + (k >> 2) * Q_SUB_BYTES + koff);
            umma_bf16(tmem + hf * 256, ad, bd, idesc, k > 0 ? 1u : 0u);
          }
#ifdef QSA_DEBUG_HOOKS
          // test hook: CTA 0 never signals its first accumulator, so that
          // accumulator's epilogue warps time out and the CTA aborts
          if (!(inject == QSA_INJECT_INDEXER_STALL && blockIdx.x == 0 && acc_use[0] == 0 && hf == 0))
#endif
          tc_commit(&accfull[hf]);
          ++acc_use[hf];
        }
        if (!ok) break;
        tc_commit(&empty[stage]);
        if (it.tile_ends_here()) tc_commit(qempty);
        if (++stage == STAGES) { stage = 0; fphase ^= 1; }
      }
      // all issued MMAs retired before TMEM is released (also after an abort)
      tc_commit(done);
      mbar_wait_drain(done, 0, err);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    // Two groups of 8 warps, one per TMEM accumulator: group hf drains half hf
    // of every unit while the tensor core fills the other half.  Token, key and
    // block numbers fit in 32 bits (T <= 2^24), so the per-unit bookkeeping is
    // 32-bit; only the score addresses are formed in 64 bits, once per tile.
    const int e = warp - 2;                 // 0..15
    const int hf = e >> 3;                  // accumulator this warp drains
    const int quad = warp & 3;              // TMEM lanes 32*quad .. +31
    const int cgrp = (e >> 2) & 1;          // column group: tokens [32*cgrp, +32) of a half
    const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
    const float* wrow = sW + (64 * hf + 32 * cgrp) * 4;
    const bool la = (lane & 1) != 0, lb = (lane & 2) != 0, lc = (lane & 4) != 0;
    // query blocks (after the first of the warp's 8) this lane ends up holding:
    // qs, qs + 1 after the key-block butterfly, qs_seg after the segment step
    const int qs = (la ? 4 : 0) + (lb ? 2 : 0);
    const int qs_seg = qs + (lc ? 1 : 0);
    const int qb0 = (int)qb_begin, qe = (int)qb_end;
    It it; it.begin(&sch, u0, u1);
    uint32_t qcount = 0;
    uint32_t acc_use = 0;
    int t_first = 0;              // first token of this thread's columns (per tile)
    int qbf = 0;                  // first query block of those columns (per tile)
    float* s_rows = nullptr;      // score row of query block qbf (+ qs unless MEAN)
    float* g_row = nullptr;       // segment-maxima row of query block qbf + qs_seg
    for (; it.valid(); it.next()) {
      if (it.first_of_tile(u0)) {
        if (!__all_sync(0xffffffffu, mbar_wait(qfull, qcount & 1, abort_flag, err))) break;
        ++qcount;
        t_first = (int)(sch.T0 + QT * it.tile) + 64 * hf + 32 * cgrp;
        qbf = qb0 + (QT / 4) * (int)it.tile + 16 * hf + 8 * cgrp;
        s_rows = S + (int64_t)(qbf - qb0 + (MEAN ? 0 : qs)) * ld;
        if (segmax != nullptr) g_row = segmax + (int64_t)(qbf - qb0 + qs_seg) * ld_seg;
      }
      // this thread's TMEM lane: one key (token-pair max) or one key block (mean pool);
      // j is the first token it stands for, so "j <= t" is the causal test in both
      const int key0 = KT * (int)it.kt + 32 * quad;   // the warp's first TMEM row
      const int row = key0 + lane;
      const int j = MEAN ? 4 * row : row;
      const int kb = MEAN ? row : row >> 2;
      if (!__all_sync(0xffffffffu, mbar_wait(&accfull[hf], acc_use & 1, abort_flag, err))) break;
      ++acc_use;
      tc_fence_after();
      const int kt_last_key = MEAN ? 4 * (KT * (int)it.kt + KT - 1) : KT * (int)it.kt + KT - 1;
      // skip when every key block of this warp lies after every query block of its columns
      const int warp_first_key = MEAN ? 4 * key0 : key0;
      const bool live = warp_first_key <= t_first + 31 && qbf < qe;
      if (live) {
        // The causal test is needed only where the key tile reaches past the
        // first token of this thread's columns; the drain is compiled twice so
        // the common (unmasked) copy carries no per-score test.
        const bool masked = kt_last_key > t_first;
        auto drain = [&](auto mtag) {
          constexpr bool MASKED = decltype(mtag)::value;
          // key position relative to the first column token: where MASKED the
          // key tile ends after t_first and the warp's first key is at most
          // t_first + 31, so -512 < jd < 160
          const int jd = MASKED ? j - t_first : 0;
          float m[8];
          // 8 tokens (32 columns) of this key's row -> the maxima of query blocks 2c, 2c+1
          auto chunk = [&](const float (&v)[32], int c) {
  #pragma unroll
            for (int half_blk = 0; half_blk < 2; ++half_blk) {
              float sc[4];
  #pragma unroll
              for (int pr = 0; pr < 2; ++pr) {
                // tokens tl and tl+1 at once: packed f32x2 multiply-adds over the 4 heads.
                // The ReLU of heads 0, 1 runs on the ALU (max), that of heads 2, 3 on the
                // FMA pipe (saturating multiply by 2^-64, undone by the scaled weights).
                const int tl = 8 * c + 4 * half_blk + 2 * pr;   // token index within the 32 columns
                const float* x0 = &v[4 * (tl & 7)];
                const float* x1 = x0 + 4;
                const float4 wa = *reinterpret_cast<const float4*>(wrow + 4 * tl);       // heads 0, 1
                const float4 wb = *reinterpret_cast<const float4*>(wrow + 4 * tl + 4);   // heads 2, 3 (x 2^64)
                uint64_t acc = mul2(pk2(fmaxf(x0[0], 0.f), fmaxf(x1[0], 0.f)), pk2(wa.x, wa.y));
                acc = fma2(pk2(fmaxf(x0[1], 0.f), fmaxf(x1[1], 0.f)), pk2(wa.z, wa.w), acc);
                acc = fma2(pk2(relu_scaled(x0[2]), relu_scaled(x1[2])), pk2(wb.x, wb.y), acc);
                acc = fma2(pk2(relu_scaled(x0[3]), relu_scaled(x1[3])), pk2(wb.z, wb.w), acc);
                float s0, s1;
                upk2(acc, s0, s1);
                if constexpr (MASKED) {
                  s0 = (jd <= tl) ? s0 : 0.f;
                  s1 = (jd <= tl + 1) ? s1 : 0.f;
                }
                sc[2 * pr] = s0;
                sc[2 * pr + 1] = s1;
              }
              m[2 * c + half_blk] = fmaxf(max3f(sc[0], sc[1], sc[2]), sc[3]);
            }
          };
          // four 32-column loads, each in flight while the previous chunk is scored
          const uint32_t base = tmem + lane_addr + hf * 256 + 128 * cgrp;
          float va[32], vb[32];
          tmem_ld32(base, va);
          tmem_ld_wait(va);
          tmem_ld32(base + 32, vb);
          chunk(va, 0);
          tmem_ld_wait(vb);
          tmem_ld32(base + 64, va);
          chunk(vb, 1);
          tmem_ld_wait(va);
          tmem_ld32(base + 96, vb);
          chunk(va, 2);
          tmem_ld_wait(vb);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&accempty[hf]);
          chunk(vb, 3);
          if constexpr (MEAN) {
            // one key block per lane: the 8 block maxima are the scores
            // S(qbf + b, kb), stored by the 32 lanes as 32 consecutive floats
            float* srow = s_rows + kb;
            const int nb = qe - qbf < 8 ? qe - qbf : 8;
  #pragma unroll
            for (int b = 0; b < 8; ++b) {
              if (b < nb && kb <= qbf + b && QSA_BOUNDS_OK(kb < ld && qbf + b >= qb0, err)) srow[b * ld] = m[b] * scale;
            }
            if (segmax != nullptr) {
              // segment maxima over 8 key blocks = 8 lanes (bits 0..2): three
              // transposing steps leave lane (a, b, c) of each 8-lane group with
              // the maximum of query block qbf + 4 a + 2 b + c
              float n4[4], n2[2];
  #pragma unroll
              for (int i = 0; i < 4; ++i)
                n4[i] = fmaxf(la ? m[i + 4] : m[i], __shfl_xor_sync(0xffffffffu, la ? m[i] : m[i + 4], 1));
  #pragma unroll
              for (int i = 0; i < 2; ++i)
                n2[i] = fmaxf(lb ? n4[i + 2] : n4[i], __shfl_xor_sync(0xffffffffu, lb ? n4[i] : n4[i + 2], 2));
              const float sm = fmaxf(lc ? n2[1] : n2[0], __shfl_xor_sync(0xffffffffu, lc ? n2[0] : n2[1], 4));
              const int seg = (key0 + (lane & ~7)) >> 3;
              const int qb = qbf + qs_seg;
              // only segments starting at or before the row's own block: seg <= qb / 8 < ld_seg
              if (qb < qe && seg <= (qb >> 3) && QSA_BOUNDS_OK(seg < ld_seg && qb >= qb0, err)) g_row[seg] = sm * scale;
            }
          } else {
            // max over the 4 keys of the key block (lanes 4k .. 4k+3) as a transposing
            // butterfly: after the two steps lane (a = bit 0, b = bit 1) holds the
            // maxima of query blocks 4a + 2b and 4a + 2b + 1.
            float n4[4];
    #pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float send = la ? m[i] : m[i + 4];
              const float keep = la ? m[i + 4] : m[i];
              n4[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 1));
            }
            float val[2];
    #pragma unroll
            for (int i = 0; i < 2; ++i) {
              const float send = lb ? n4[i] : n4[i + 2];
              const float keep = lb ? n4[i + 2] : n4[i];
              val[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 2));
              const int qb = qbf + qs + i;
              if (qb < qe && kb <= qb && QSA_BOUNDS_OK(kb < ld && qb >= qb0, err)) s_rows[i * ld + kb] = val[i] * scale;
            }
            if (segmax != nullptr) {
              // segment maxima: max over the 8 key blocks of this warp's 32 keys
              // (lane bits 2..4).  A transposing step on bit 2 leaves each lane one
              // query block (4 a + 2 b + c0), then two plain steps; lanes 0..7 hold
              // the 8 query blocks.  Key blocks after a query block were scored as
              // 0 and scores are >= 0, so they do not raise a maximum.
              float sm = fmaxf(lc ? val[1] : val[0], __shfl_xor_sync(0xffffffffu, lc ? val[0] : val[1], 4));
              sm = fmaxf(sm, __shfl_xor_sync(0xffffffffu, sm, 8));
              sm = fmaxf(sm, __shfl_xor_sync(0xffffffffu, sm, 16));
              if (lane < 8) {
                const int seg = key0 >> 5;
                const int qb = qbf + qs_seg;
                // only segments starting at or before the row's own block: seg <= qb / 8 < ld_seg
                if (qb < qe && seg <= (qb >> 3) && QSA_BOUNDS_OK(seg < ld_seg && qb >= qb0, err))
                  g_row[seg] = sm * scale;
              }
            }
          }
        };
        if (masked) drain(std::true_type{});
        else drain(std::false_type{});
      } else {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[hf]);
      }
      if (it.tile_ends_here()) {
        __syncwarp();
        if (lane == 0) mbar_arrive(qempty);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_indexer_prefill(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const uint16_t* w,
                                   float* S, int64_t ld, float* segmax, int64_t ld_seg, int64_t T, int64_t q_tok0,
                                   int64_t qb_begin, int64_t qb_end, bool mean_pool, float scale, uint32_t* err,
                                   int num_sms, cudaStream_t stream) {
  if (qb_end <= qb_begin) return cudaSuccess;
  static bool attr_done[2][64] = {{false}, {false}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[mean_pool][dev]) {
    cudaError_t e = mean_pool ? cudaFuncSetAttribute(indexer_prefill_kernel<true>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES)
                              : cudaFuncSetAttribute(indexer_prefill_kernel<false>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done[mean_pool][dev] = true;
  }
  // units in this call; never more CTAs than units
  const int64_t T0 = qb_begin * 4;
  const int64_t Tend = qb_end * 4 < T ? qb_end * 4 : T;
  const int64_t n_tiles = (Tend - T0 + QT - 1) / QT;
  const int64_t key_tokens = mean_pool ? 4 * KT : KT;   // tokens covered by one key tile
  int64_t units = 0;
  for (int64_t i = 0; i < n_tiles && units < num_sms; ++i) {
    int64_t tl = T0 + QT * i + QT - 1;
    if (tl > Tend - 1) tl = Tend - 1;
    units += tl / key_tokens + 1;
  }
  const int grid = (int)(units < num_sms ? units : num_sms);
  const int inject = take_debug_injection(QSA_INJECT_INDEXER_STALL);
  if (mean_pool)
    indexer_prefill_kernel<true><<<grid, THREADS, SMEM_BYTES, stream>>>(tm_q, tm_k, w, S, ld, segmax, ld_seg, T,
                                                                        q_tok0, qb_begin, qb_end, scale, err, inject);
  else
    indexer_prefill_kernel<false><<<grid, THREADS, SMEM_BYTES, stream>>>(tm_q, tm_k, w, S, ld, segmax, ld_seg, T,
                                                                         q_tok0, qb_begin, qb_end, scale, err, inject);
  return cudaGetLastError();
}

// Mean-pooled indexer keys: kbar[b][c] = bf16 of the mean of k_idx rows
// 4b .. min(4b + 4, T) - 1 (exact fp64 sum, one fp64 division, round to
// nearest even), one thread per (block, dim).
namespace {
__global__ void kbar_kernel(const uint16_t* __restrict__ k_idx, int64_t T, int64_t nkb, uint16_t* __restrict__ kbar) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nkb * 128) return;
  const int64_t b = i >> 7, c = i & 127;
  const int64_t t0 = 4 * b;
  const int n = (int)(T - t0 < 4 ? T - t0 : 4);
  double sum = 0.0;
  for (int r = 0; r < n; ++r) sum += (double)__uint_as_float((uint32_t)k_idx[(t0 + r) * 128 + c] << 16);
  kbar[i] = f64_to_bf16_rne(sum / (double)n);
}
}  // namespace

cudaError_t launch_kbar(const uint16_t* k_idx, int64_t T, uint16_t* kbar, cudaStream_t stream) {
  const int64_t nkb = (T + 3) / 4;
  if (nkb <= 0) return cudaSuccess;
  const int64_t n = nkb * 128;
  kbar_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(k_idx, T, nkb, kbar);
  return cudaGetLastError();
}

}  // namespace qsa
