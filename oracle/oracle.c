/*
 * oracle.c -- plain, slow fp64 CPU oracle of the QSA hot path.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code with
 * the CUDA path: no kernels, headers, tables or helpers.
 *
 * Every function is the plain definition written out in fp64 (inputs are bf16
 * values, converted exactly), with no blocking, fusion or reordering beyond
 * what the definition states.  Where a step needs a library primitive it is
 * plain libm (pow, cos, sin, exp, log) or qsort.
 *
 * Cited pages:
 *   [PT] "Qwen3.8-Flash-Next, 1/9의 학습 비용으로 Qwen3.7-Plus(397B-A17B) 수준에
 *        도달한 125B-A6B 모델" (discuss.pytorch.kr): spec table; section
 *        "QSA: 인덱서 자체의 비용을 줄이는 희소 어텐션" with equation I_ib;
 *        section "100만 토큰까지 늘리기" (rope_parameters listing).
 *   [LF] "Qwen 팀, 새 구조를 적용한 Qwen3.8-Flash-Next 공개 가중치로 출시"
 *        (llmfeed.kr): spec list.
 *
 * Readings where the pages are silent (the choices this oracle implements):
 *   - block score = max over causal token pairs (j <= t) of the token score
 *     s(t,j) = sum_h w_h(t) * ReLU(q_idx_h(t) . k_idx(j)) / sqrt(d_idx);
 *     with block size 1 and w_h = sqrt(d_idx) this is [PT] eq. I_ib with the
 *     block key equal to the token key;
 *   - selection per query block: blocks qb and qb-1 forced, the rest the top
 *     (budget-2) of [0, qb-2] by (score descending, index ascending); all
 *     qb+1 blocks when qb+1 <= budget; returned ascending;
 *   - RoPE: rotate-half pairs (i, i + rope_dim/2), inv_freq_i =
 *     theta^(-2i/rope_dim), on Q and K dims [0, rope_dim) only;
 *   - attention scale 1/sqrt(head_dim) unless given; Q head h reads KV head
 *     h / (n_q_heads / n_kv_heads).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int32_t n_q_heads;   /* 24  [PT spec table, "Qwen Sparse Attention" row] */
  int32_t n_kv_heads;  /* 2 */
  int32_t head_dim;    /* 256 */
  int32_t rope_dim;    /* 64 */
  double rope_theta;   /* 1e7 [PT "100만 토큰까지 늘리기", rope_theta] */
  int32_t idx_heads;   /* 4   [PT spec table, "QSA 인덱서" row] */
  int32_t idx_dim;     /* 128 */
  int32_t block;       /* r = 4 [PT §QSA, "r = 4"] */
  int32_t budget;      /* 512 blocks = 2048 tokens [PT spec table, "QSA 예산"] */
  double softmax_scale;/* 0 => 1/sqrt(head_dim) */
  int32_t aggregation; /* 0: max over causal token pairs (the stated block score);
                          1: mean-pooled block keys [PT §QSA, I_ib over k-bar_b] */
  /* YaRN [PT "100만 토큰까지 늘리기": rope_type yarn, factor 4.0,
   * original_max_position_embeddings 262144]; factor <= 1 means plain RoPE */
  double yarn_factor;
  double yarn_original_max;
  double yarn_beta_fast;  /* 32 (not on the pages: the method's usual value) */
  double yarn_beta_slow;  /* 1 */
  /* Mean-pooled indexer only ([PT] §QSA: the block's keys are compressed
   * before the positional step and the compressed key gets one block-start
   * position).  idx_rope = 1: the indexer queries are rotated at their token
   * positions and the compressed key of block b at its start position
   * 4b, with the layer's RoPE (dims [0, rope_dim), as for Q and K); token t
   * sits at position idx_pos0 + t.  idx_exact = 1: the compressed and rotated
   * indexer operands are kept in fp64 instead of being rounded to bf16 (a
   * diagnostic reading; the default rounds them, as the model's tensors are
   * bf16). */
  int32_t idx_rope;
  int32_t idx_exact;
  int64_t idx_pos0;
} oracle_params;

static double bf16_to_f64(uint16_t h) {
  union { float f; uint32_t u; } b;
  b.u = ((uint32_t)h) << 16;
  return (double)b.f;
}

/* ------------------------------------------------------------------ RoPE --
 * Rotary position embedding on dims [0, rope_dim) of one head vector
 * ([PT] spec table "RoPE 차원 64"; rope_theta and partial_rotary_factor 0.25
 * in [PT] "100만 토큰까지 늘리기").  y may not alias x. */
/* Frequency of rotary pair i.  Plain: theta^(-2i/rope_dim).  YaRN (static,
 * factor s > 1): "NTK-by-parts" -- a pair whose wavelength 2 pi / f_i fits
 * more than beta_fast times into the original context keeps f_i, one fitting
 * fewer than beta_slow times gets f_i / s, and in between the two are mixed
 * linearly in the pair index i, from the index where the rotation count
 * crosses beta_fast (rounded down) to where it crosses beta_slow (rounded
 * up); the rotation count r(i) = L_orig f_i / (2 pi) crosses n at
 * i(n) = rope_dim ln(L_orig / (2 pi n)) / (2 ln theta). */
static double rope_freq(const oracle_params* p, int i) {
  const double d = (double)p->rope_dim;
  const double f = pow(p->rope_theta, -2.0 * (double)i / d);
  const double s = p->yarn_factor;
  if (!(s > 1.0)) return f;
  const double two_pi = 2.0 * acos(-1.0);
  const double i_fast = d * log(p->yarn_original_max / (two_pi * p->yarn_beta_fast)) / (2.0 * log(p->rope_theta));
  const double i_slow = d * log(p->yarn_original_max / (two_pi * p->yarn_beta_slow)) / (2.0 * log(p->rope_theta));
  double lo = floor(i_fast), hi = ceil(i_slow);
  if (lo < 0.0) lo = 0.0;
  if (hi > d - 1.0) hi = d - 1.0;
  if (hi == lo) hi += 0.001;
  double ramp = ((double)i - lo) / (hi - lo);   /* 0: keep f, 1: f / s */
  if (ramp < 0.0) ramp = 0.0;
  if (ramp > 1.0) ramp = 1.0;
  return f / s * ramp + f * (1.0 - ramp);
}

/* YaRN's attention factor 0.1 ln s + 1 on the rotated dims (1 for plain RoPE). */
static double rope_scale(const oracle_params* p) {
  return p->yarn_factor > 1.0 ? 0.1 * log(p->yarn_factor) + 1.0 : 1.0;
}

void oracle_rope(const oracle_params* p, const double* x, int64_t pos, double* y) {
  int half = p->rope_dim / 2;
  const double m = rope_scale(p);
  for (int c = 0; c < p->head_dim; ++c) y[c] = x[c];
  for (int i = 0; i < half; ++i) {
    double inv_freq = rope_freq(p, i);
    double a = (double)pos * inv_freq;
    double ca = cos(a), sa = sin(a);
    y[i] = m * (x[i] * ca - x[i + half] * sa);
    y[i + half] = m * (x[i + half] * ca + x[i] * sa);
  }
}

/* ----------------------------------------------------------- token score --
 * s(t, j) = sum_h w_h(t) * ReLU(q_idx_h(t) . k_idx(j)) / sqrt(idx_dim)
 * ([PT] §QSA eq. I_ib: ReLU of per-head query/key similarity summed over the
 * indexer heads; head weights and the 1/sqrt(d) are the stated reading). */
double oracle_token_score(const oracle_params* p, const uint16_t* q_t, const uint16_t* w_t,
                          const uint16_t* k_j) {
  double s = 0.0;
  for (int h = 0; h < p->idx_heads; ++h) {
    double dot = 0.0;
    for (int c = 0; c < p->idx_dim; ++c) dot += bf16_to_f64(q_t[h * p->idx_dim + c]) * bf16_to_f64(k_j[c]);
    double relu = dot > 0.0 ? dot : 0.0;
    s += bf16_to_f64(w_t[h]) * relu;
  }
  return s / sqrt((double)p->idx_dim);
}

/* fp64 -> bf16 bit pattern, rounded to the nearest bf16 value, ties to the
 * one with an even last bit (IEEE round-to-nearest-even), subnormals
 * included.  The bf16 values next to |x| are the multiples of the spacing
 * u = 2^(e - 8) around it (|x| in [2^(e-1), 2^e); u = 2^-133 below the
 * normal range): lo = floor(|x| / u) u and lo + u.  Both divisions by u and
 * the products are exact in fp64 (powers of two). */
static uint16_t bf16_round_nearest_even(double x) {
  const double a = fabs(x);
  const uint16_t sign = signbit(x) ? 0x8000u : 0u;
  if (a == 0.0) return sign;
  int e;
  (void)frexp(a, &e);
  const double u = ldexp(1.0, e - 8 > -133 ? e - 8 : -133);
  const double n_lo = floor(a / u);                 /* lo = n_lo u, exact */
  const double below = a - n_lo * u, above = (n_lo + 1.0) * u - a;
  double n = n_lo;
  if (above < below || (above == below && fmod(n_lo, 2.0) != 0.0)) n = n_lo + 1.0;
  union { float f; uint32_t u32; } c;
  c.f = (float)(n * u);                             /* exact: a bf16 value */
  return (uint16_t)(sign | (c.u32 >> 16));
}

/* RoPE of the first rope_dim dims of an n-dim vector at position pos (the
 * same rotation as oracle_rope, for the indexer's 128-dim vectors). */
static void rope_vec(const oracle_params* p, const double* x, int n, int64_t pos, double* y) {
  const int half = p->rope_dim / 2;
  const double m = rope_scale(p);
  for (int c = 0; c < n; ++c) y[c] = x[c];
  for (int i = 0; i < half; ++i) {
    const double a = (double)pos * rope_freq(p, i);
    const double ca = cos(a), sa = sin(a);
    y[i] = m * (x[i] * ca - x[i + half] * sa);
    y[i + half] = m * (x[i + half] * ca + x[i] * sa);
  }
}

/* The value an indexer operand takes: rounded to bf16 unless idx_exact. */
static double idx_operand(const oracle_params* p, double v) {
  return p->idx_exact ? v : bf16_to_f64(bf16_round_nearest_even(v));
}

/* Compressed key of block kb ([PT] §QSA: the keys of a micro-block are
 * mean-pooled into k-bar_b before the positional step).  Mean over the
 * block's n present keys: exact fp64 sum, one fp64 division by n, one
 * rounding to bf16 (the model's tensors are bf16; not with idx_exact).  With
 * idx_rope the compressed key then gets the block's start position
 * idx_pos0 + kb r (rotated, then rounded to bf16 unless idx_exact). */
static void mean_key(const oracle_params* p, const uint16_t* k_idx, int64_t kb, int n, double* kbar) {
  double mean[512];
  for (int c = 0; c < p->idx_dim; ++c) {
    double sum = 0.0;
    for (int i = 0; i < n; ++i) sum += bf16_to_f64(k_idx[(kb * p->block + i) * p->idx_dim + c]);
    mean[c] = idx_operand(p, sum / (double)n);
  }
  if (p->idx_rope) {
    rope_vec(p, mean, p->idx_dim, p->idx_pos0 + kb * p->block, kbar);
    for (int c = 0; c < p->idx_dim; ++c) kbar[c] = idx_operand(p, kbar[c]);
  } else {
    for (int c = 0; c < p->idx_dim; ++c) kbar[c] = mean[c];
  }
}

/* ----------------------------------------------------------- block score --
 * S(qb, kb) for kb = 0..qb: max over present tokens t of block qb and keys
 * j of block kb with j <= t of s(t, j) ([PT] §QSA: micro-blocks of r tokens,
 * only fully observed earlier blocks plus the own block's causal part).
 * q_blk / w_blk hold the n_present tokens qb*r .. qb*r+n_present-1;
 * k_idx holds keys from token 0. */
void oracle_block_scores(const oracle_params* p, int64_t qb, int n_present, const uint16_t* q_blk,
                         const uint16_t* w_blk, const uint16_t* k_idx, double* S) {
  int r = p->block;
  if (p->aggregation == 1) {
    /* mean pooling: S(qb, kb) = max over present t of block qb of
     *   sum_h w_h(t) ReLU(q_idx_h(t) . k-bar_kb) / sqrt(idx_dim);
     * k-bar of the own block averages its present keys (the own block is
     * always selected, so this entry never decides a selection) */
    double kbar[512];
    /* the indexer queries of the block's present tokens, rotated at their
     * positions with idx_rope (rounded to bf16 unless idx_exact) */
    double* qv = (double*)malloc(sizeof(double) * (size_t)n_present * p->idx_heads * p->idx_dim);
    double x[512];
    for (int i = 0; i < n_present; ++i)
      for (int h = 0; h < p->idx_heads; ++h) {
        const uint16_t* q_th = q_blk + ((int64_t)i * p->idx_heads + h) * p->idx_dim;
        double* dst = qv + ((int64_t)i * p->idx_heads + h) * p->idx_dim;
        for (int c = 0; c < p->idx_dim; ++c) x[c] = bf16_to_f64(q_th[c]);
        if (p->idx_rope) {
          rope_vec(p, x, p->idx_dim, p->idx_pos0 + qb * r + i, dst);
          for (int c = 0; c < p->idx_dim; ++c) dst[c] = idx_operand(p, dst[c]);
        } else {
          for (int c = 0; c < p->idx_dim; ++c) dst[c] = x[c];
        }
      }
    for (int64_t kb = 0; kb <= qb; ++kb) {
      mean_key(p, k_idx, kb, kb == qb ? n_present : r, kbar);
      double best = -INFINITY;
      for (int i = 0; i < n_present; ++i) {
        const double* q_t = qv + (int64_t)i * p->idx_heads * p->idx_dim;
        double s = 0.0;
        for (int h = 0; h < p->idx_heads; ++h) {
          double dot = 0.0;
          for (int c = 0; c < p->idx_dim; ++c) dot += q_t[h * p->idx_dim + c] * kbar[c];
          s += bf16_to_f64(w_blk[(int64_t)i * p->idx_heads + h]) * (dot > 0.0 ? dot : 0.0);
        }
        s /= sqrt((double)p->idx_dim);
        if (s > best) best = s;
      }
      S[kb] = best;
    }
    free(qv);
    return;
  }
  for (int64_t kb = 0; kb <= qb; ++kb) {
    double best = -INFINITY;
    for (int i = 0; i < n_present; ++i) {
      int64_t t = qb * r + i;
      for (int64_t j = kb * r; j < kb * r + r; ++j) {
        if (j > t) continue;
        double s = oracle_token_score(p, q_blk + (int64_t)i * p->idx_heads * p->idx_dim,
                                      w_blk + (int64_t)i * p->idx_heads, k_idx + j * p->idx_dim);
        if (s > best) best = s;
      }
    }
    S[kb] = best;
  }
}

/* ------------------------------------------------------------- selection --
 * [PT] §QSA: budget K = 2048 tokens = 512 blocks of r = 4; the tail of the
 * own (incomplete) block is always included.  Reading: blocks qb and qb-1
 * forced, the remaining budget-2 slots go to the highest-scoring blocks of
 * [0, qb-2], ties to the lower index; all blocks when qb+1 <= budget. */
typedef struct { double s; int64_t idx; } scored;

static int cmp_desc_score_asc_idx(const void* a, const void* b) {
  const scored* x = (const scored*)a;
  const scored* y = (const scored*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->idx > y->idx) - (x->idx < y->idx);
}

static int cmp_i32(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

void oracle_select(const oracle_params* p, int64_t qb, const double* S, int32_t* sel, int32_t* cnt) {
  int budget = p->budget;
  for (int i = 0; i < budget; ++i) sel[i] = -1;
  if (qb + 1 <= budget) {
    for (int64_t kb = 0; kb <= qb; ++kb) sel[kb] = (int32_t)kb;
    *cnt = (int32_t)(qb + 1);
    return;
  }
  int64_t m = qb - 1; /* candidates 0 .. qb-2 */
  scored* c = (scored*)malloc(sizeof(scored) * (size_t)m);
  for (int64_t kb = 0; kb < m; ++kb) { c[kb].s = S[kb]; c[kb].idx = kb; }
  qsort(c, (size_t)m, sizeof(scored), cmp_desc_score_asc_idx);
  int n = 0;
  for (int i = 0; i < budget - 2; ++i) sel[n++] = (int32_t)c[i].idx;
  sel[n++] = (int32_t)(qb - 1);
  sel[n++] = (int32_t)qb;
  free(c);
  qsort(sel, (size_t)n, sizeof(int32_t), cmp_i32);
  *cnt = n;
}

/* ------------------------------------------------------------- attention --
 * Softmax attention of one token's n_q_heads rotated queries over n keys
 * (already rotated) -- "sparse core attention" over the selected blocks,
 * GQA with n_q_heads / n_kv_heads query heads per KV head ([PT] §QSA;
 * spec table "Q 헤드 24개, KV 헤드 2개, 헤드 차원 256").
 * q_rot [H][d], k_rot/v [n][G][d] -> out [H][d], lse [H]. */
void oracle_attend(const oracle_params* p, const double* q_rot, int64_t n, const double* k_rot,
                   const double* v, double* out, double* lse) {
  int H = p->n_q_heads, G = p->n_kv_heads, d = p->head_dim;
  double scale = p->softmax_scale > 0.0 ? p->softmax_scale : 1.0 / sqrt((double)d);
  double* l = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  for (int h = 0; h < H; ++h) {
    int g = h / (H / G);
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
      double dot = 0.0;
      for (int c = 0; c < d; ++c) dot += q_rot[h * d + c] * k_rot[(j * G + g) * d + c];
      l[j] = dot * scale;
      if (l[j] > m) m = l[j];
    }
    double z = 0.0;
    for (int c = 0; c < d; ++c) out[h * d + c] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
      double e = exp(l[j] - m);
      z += e;
      for (int c = 0; c < d; ++c) out[h * d + c] += e * v[(j * G + g) * d + c];
    }
    for (int c = 0; c < d; ++c) out[h * d + c] /= z;
    lse[h] = m + log(z);
  }
  free(l);
}

/* Keys token t may read: every j in the selected blocks with j <= t. */
static int64_t gather_keys(const oracle_params* p, const int32_t* sel, int32_t cnt, int64_t t, int64_t* js) {
  int64_t n = 0;
  for (int i = 0; i < cnt; ++i) {
    if (sel[i] < 0) continue;
    for (int64_t j = (int64_t)sel[i] * p->block; j < (int64_t)sel[i] * p->block + p->block; ++j)
      if (j <= t) js[n++] = j;
  }
  return n;
}

/* Attention of one query token over an explicit list of candidate keys
 * (the same definition as oracle_attend_blocks, for callers that hold only
 * the rows a token can read): token at position pos_t with unrotated q_t
 * [H][d]; n keys at positions pos_j[n] with unrotated k_rows, v_rows
 * [n][G][d].  Keys with pos_j > pos_t are skipped (causality); the rest are
 * rotated at their positions and attended as by oracle_attend.
 * out [H][d], lse [H]. */
void oracle_attend_gathered(const oracle_params* p, int64_t pos_t, const uint16_t* q_t, int64_t n,
                            const int64_t* pos_j, const uint16_t* k_rows, const uint16_t* v_rows, double* out,
                            double* lse) {
  int H = p->n_q_heads, G = p->n_kv_heads, d = p->head_dim;
  double* kr = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * G * d);
  double* vv = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * G * d);
  double* x = (double*)malloc(sizeof(double) * (size_t)d);
  double* qr = (double*)malloc(sizeof(double) * (size_t)H * d);
  int64_t m = 0;
  for (int64_t e = 0; e < n; ++e) {
    if (pos_j[e] > pos_t) continue;
    for (int g = 0; g < G; ++g) {
      for (int c = 0; c < d; ++c) x[c] = bf16_to_f64(k_rows[(e * G + g) * d + c]);
      oracle_rope(p, x, pos_j[e], kr + (m * G + g) * d);
      for (int c = 0; c < d; ++c) vv[(m * G + g) * d + c] = bf16_to_f64(v_rows[(e * G + g) * d + c]);
    }
    ++m;
  }
  for (int h = 0; h < H; ++h) {
    for (int c = 0; c < d; ++c) x[c] = bf16_to_f64(q_t[h * d + c]);
    oracle_rope(p, x, pos_t, qr + h * d);
  }
  oracle_attend(p, qr, m, kr, vv, out, lse);
  free(kr); free(vv); free(x); free(qr);
}

/* ---------------------------------------------------------------- prefill --
 * Scores for query blocks [qb_begin, qb_end) into S[(qb-qb_begin)*ld + kb],
 * kb <= qb (other entries untouched).  T tokens in total. */
void oracle_index_scores(const oracle_params* p, int64_t T, const uint16_t* q_idx, const uint16_t* w,
                         const uint16_t* k_idx, int64_t qb_begin, int64_t qb_end, double* S, int64_t ld) {
  int r = p->block;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t qb = qb_begin; qb < qb_end; ++qb) {
    int64_t t0 = qb * r;
    int n_present = (int)((T - t0) < r ? (T - t0) : r);
    oracle_block_scores(p, qb, n_present, q_idx + t0 * p->idx_heads * p->idx_dim, w + t0 * p->idx_heads,
                        k_idx, S + (qb - qb_begin) * ld);
  }
}

/* Selection for rows [qb_begin, qb_end) of a score matrix laid out as above. */
void oracle_select_rows(const oracle_params* p, const double* S, int64_t ld, int64_t qb_begin, int64_t qb_end,
                        int32_t* sel, int32_t* cnt) {
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t qb = qb_begin; qb < qb_end; ++qb)
    oracle_select(p, qb, S + (qb - qb_begin) * ld, sel + (qb - qb_begin) * p->budget, cnt + (qb - qb_begin));
}

/* Attention for the present tokens of the listed query blocks, on a given
 * selection sel[i][budget] / cnt[i] (the oracle's own or another one's).
 * q [T][H][d], k/v [T][G][d] unrotated bf16; token t sits at position pos0+t.
 * out [n_blocks*r][H][d], lse [n_blocks*r][H] (rows of absent tokens zeroed). */
void oracle_attend_blocks(const oracle_params* p, int64_t T, int64_t pos0, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, int64_t n_blocks, const int64_t* qb_list, const int32_t* sel,
                          const int32_t* cnt, double* out, double* lse) {
  int H = p->n_q_heads, G = p->n_kv_heads, d = p->head_dim, r = p->block;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t b = 0; b < n_blocks; ++b) {
    int64_t qb = qb_list[b];
    const int32_t* s = sel + b * p->budget;
    int64_t* js = (int64_t*)malloc(sizeof(int64_t) * (size_t)p->budget * r);
    double* kr = (double*)malloc(sizeof(double) * (size_t)p->budget * r * G * d);
    double* vv = (double*)malloc(sizeof(double) * (size_t)p->budget * r * G * d);
    double* x = (double*)malloc(sizeof(double) * (size_t)d);
    double* qr = (double*)malloc(sizeof(double) * (size_t)H * d);
    for (int i = 0; i < r; ++i) {
      int64_t t = qb * r + i;
      double* o = out + (b * r + i) * H * d;
      double* ls = lse + (b * r + i) * H;
      if (t >= T) {
        memset(o, 0, sizeof(double) * (size_t)H * d);
        memset(ls, 0, sizeof(double) * (size_t)H);
        continue;
      }
      int64_t n = gather_keys(p, s, cnt[b], t, js);
      for (int64_t e = 0; e < n; ++e)
        for (int g = 0; g < G; ++g) {
          for (int c = 0; c < d; ++c) x[c] = bf16_to_f64(k[(js[e] * G + g) * d + c]);
          oracle_rope(p, x, pos0 + js[e], kr + (e * G + g) * d);
          for (int c = 0; c < d; ++c) vv[(e * G + g) * d + c] = bf16_to_f64(v[(js[e] * G + g) * d + c]);
        }
      for (int h = 0; h < H; ++h) {
        for (int c = 0; c < d; ++c) x[c] = bf16_to_f64(q[(t * H + h) * d + c]);
        oracle_rope(p, x, pos0 + t, qr + h * d);
      }
      oracle_attend(p, qr, n, kr, vv, o, ls);
    }
    free(js); free(kr); free(vv); free(x); free(qr);
  }
}

/* Block scores and selection for the listed query blocks (stages 1 and 2).
 * sel_out [n][budget], cnt_out [n]. */
void oracle_select_blocks_list(const oracle_params* p, int64_t T, const uint16_t* q_idx, const uint16_t* w,
                               const uint16_t* k_idx, int64_t n_blocks, const int64_t* qb_list, int32_t* sel_out,
                               int32_t* cnt_out) {
  int r = p->block;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t b = 0; b < n_blocks; ++b) {
    int64_t qb = qb_list[b];
    int64_t t0 = qb * r;
    int n_present = (int)((T - t0) < r ? (T - t0) : r);
    double* S = (double*)malloc(sizeof(double) * (size_t)(qb + 1));
    oracle_block_scores(p, qb, n_present, q_idx + t0 * p->idx_heads * p->idx_dim, w + t0 * p->idx_heads, k_idx, S);
    oracle_select(p, qb, S, sel_out + b * p->budget, cnt_out + b);
    free(S);
  }
}

/* Whole prefill for the listed query blocks: scores, selection, attention.
 * sel_out [n][budget], cnt_out [n]; out / lse as oracle_attend_blocks. */
void oracle_prefill_blocks(const oracle_params* p, int64_t T, int64_t pos0, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, const uint16_t* q_idx, const uint16_t* w, const uint16_t* k_idx,
                           int64_t n_blocks, const int64_t* qb_list, int32_t* sel_out, int32_t* cnt_out,
                           double* out, double* lse) {
  oracle_select_blocks_list(p, T, q_idx, w, k_idx, n_blocks, qb_list, sel_out, cnt_out);
  oracle_attend_blocks(p, T, pos0, q, k, v, n_blocks, qb_list, sel_out, cnt_out, out, lse);
}

/* ----------------------------------------------------------------- decode --
 * One decode token at position L of a sequence whose L earlier tokens sit in
 * caches (k_cache already rotated, bf16).  The new token is appended (its key
 * rotated at L in fp64, not re-rounded; the full KV is kept -- sparse
 * attention selects, it does not evict).  Its query block qb = L / r holds
 * the present block-mates qb*r .. L, whose indexer queries are ring_q_idx /
 * ring_w for tokens qb*r .. L-1 followed by the new token's.  The result is by
 * definition that of a prefill's token L over the same keys.
 * If sel_in is non-NULL it replaces the oracle's own selection.
 * k_cache, v_cache [L][G][d]; kidx_cache [L][idx_dim]; ring_q_idx
 * [n_ring][idx_heads][idx_dim] and ring_w [n_ring][idx_heads] hold the block-mates
 * qb*r .. L-1 in order (n_ring must equal L - qb*r); q_new [H][d];
 * k_new, v_new [G][d]; q_idx_new [idx_heads][idx_dim]; k_idx_new [idx_dim];
 * w_new [idx_heads]  ->  out [H][d], lse [H], sel_out [budget], cnt_out.
 * Returns 0, or -1 (nothing computed) when n_ring is not the number of
 * block-mates before the new token. */
int32_t oracle_decode(const oracle_params* p, int64_t L, const uint16_t* k_cache, const uint16_t* v_cache,
                      const uint16_t* kidx_cache, const uint16_t* ring_q_idx, const uint16_t* ring_w, int32_t n_ring,
                      const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new, const uint16_t* q_idx_new,
                      const uint16_t* k_idx_new, const uint16_t* w_new, const int32_t* sel_in, int32_t cnt_in,
                      int32_t* sel_out, int32_t* cnt_out, double* out, double* lse) {
  int H = p->n_q_heads, G = p->n_kv_heads, d = p->head_dim, r = p->block;
  int IH = p->idx_heads, ID = p->idx_dim;
  int64_t qb = L / r;
  int n_prev = (int)(L - qb * r);            /* block-mates before the new token */
  if (n_ring != n_prev) return -1;
  int n_present = n_prev + 1;
  uint16_t* qblk = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)n_present * IH * ID);
  uint16_t* wblk = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)n_present * IH);
  uint16_t* keys = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(L + 1) * ID);
  if (n_prev > 0) {
    memcpy(qblk, ring_q_idx, sizeof(uint16_t) * (size_t)n_prev * IH * ID);
    memcpy(wblk, ring_w, sizeof(uint16_t) * (size_t)n_prev * IH);
  }
  memcpy(qblk + (size_t)n_prev * IH * ID, q_idx_new, sizeof(uint16_t) * (size_t)IH * ID);
  memcpy(wblk + (size_t)n_prev * IH, w_new, sizeof(uint16_t) * (size_t)IH);
  if (L > 0) memcpy(keys, kidx_cache, sizeof(uint16_t) * (size_t)L * ID);
  memcpy(keys + L * ID, k_idx_new, sizeof(uint16_t) * (size_t)ID);

  /* a given selection may hold more than budget blocks (a reused one) */
  int32_t cap = sel_in && cnt_in > p->budget ? cnt_in : p->budget;
  int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
  int32_t cnt;
  if (sel_in) {
    for (int32_t i = 0; i < cap; ++i) sel[i] = i < cnt_in ? sel_in[i] : -1;
    cnt = cnt_in;
  } else {
    double* S = (double*)malloc(sizeof(double) * (size_t)(qb + 1));
    oracle_block_scores(p, qb, n_present, qblk, wblk, keys, S);
    oracle_select(p, qb, S, sel, &cnt);
    free(S);
  }
  if (sel_out) memcpy(sel_out, sel, sizeof(int32_t) * (size_t)p->budget);
  if (cnt_out) *cnt_out = cnt;

  int64_t* js = (int64_t*)malloc(sizeof(int64_t) * (size_t)cap * r);
  int64_t n = gather_keys(p, sel, cnt, L, js);
  double* kr = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * G * d);
  double* vv = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * G * d);
  double* x = (double*)malloc(sizeof(double) * (size_t)d);
  double* qr = (double*)malloc(sizeof(double) * (size_t)H * d);
  for (int64_t e = 0; e < n; ++e) {
    int64_t j = js[e];
    for (int g = 0; g < G; ++g) {
      if (j < L) {
        for (int c = 0; c < d; ++c) kr[(e * G + g) * d + c] = bf16_to_f64(k_cache[(j * G + g) * d + c]);
        for (int c = 0; c < d; ++c) vv[(e * G + g) * d + c] = bf16_to_f64(v_cache[(j * G + g) * d + c]);
      } else {
        for (int c = 0; c < d; ++c) x[c] = bf16_to_f64(k_new[g * d + c]);
        oracle_rope(p, x, L, kr + (e * G + g) * d);
        for (int c = 0; c < d; ++c) vv[(e * G + g) * d + c] = bf16_to_f64(v_new[g * d + c]);
      }
    }
  }
  for (int h = 0; h < H; ++h) {
    for (int c = 0; c < d; ++c) x[c] = bf16_to_f64(q_new[h * d + c]);
    oracle_rope(p, x, L, qr + h * d);
  }
  oracle_attend(p, qr, n, kr, vv, out, lse);
  free(qblk); free(wblk); free(keys); free(sel); free(js); free(kr); free(vv); free(x); free(qr);
  return 0;
}

/* ---------------------------------------------------------- top-k reuse --
 * [PT] section "추측 디코딩을 위한 MTP와 그 밖에 유지된 설계": the MTP draft
 * layer reuses the top-k indices between the steps of one speculative round
 * (as GLM-5 does).  A later draft token at query block qb attends the reused
 * set together with the blocks that stage 2 forces for every query block, its
 * own block qb and qb - 1:
 *   attended = sorted( {sel_in[i] : i < cnt_in}  U  {qb - 1, qb} ),
 * qb - 1 only when qb >= 1.  Entries of sel_in must be causal (0 .. qb);
 * returns -1 when one is not.  out holds at least cnt_in + 2 entries; returns
 * the number written. */
int32_t oracle_reuse_selection(int64_t qb, const int32_t* sel_in, int32_t cnt_in, int32_t* out) {
  int64_t n_blocks = qb + 1;
  unsigned char* in_set = (unsigned char*)calloc((size_t)n_blocks, 1);
  for (int32_t i = 0; i < cnt_in; ++i) {
    if (sel_in[i] < 0 || sel_in[i] > qb) { free(in_set); return -1; }
    in_set[sel_in[i]] = 1;
  }
  in_set[qb] = 1;
  if (qb >= 1) in_set[qb - 1] = 1;
  int32_t n = 0;
  for (int64_t b = 0; b < n_blocks; ++b)
    if (in_set[b]) out[n++] = (int32_t)b;
  free(in_set);
  return n;
}
