// C ABI of the QSA hot path: argument validation, workspace planning, tensor
// map encoding and kernel launches on the caller's stream.  Every entry point
// validates on the host before launching anything and returns a qsa_status.
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "qsa.h"
#include "qsa_kernels.h"
#include "qsa_debug.h"

namespace {

constexpr size_t HEADER_BYTES = 256;            // device error word + padding
constexpr size_t ALIGN = 256;
constexpr int MAX_DEV = 64;

// Last failure of this thread, for qsa_last_error().
thread_local char g_last_error[256] = "";

qsa_status fail(qsa_status st, const char* what, const char* detail = "") {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s%s%s", what, detail[0] ? ": " : "", detail);
  return st;
}

size_t align_up(size_t x, size_t a = ALIGN) { return (x + a - 1) / a * a; }
int64_t round4(int64_t x) { return (x + 3) / 4 * 4; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qsa_status check_params(const qsa_params* p) {
  if (!p) return QSA_ERR_INVALID_ARG;
  if (p->n_q_heads != 24 || p->n_kv_heads != 2 || p->head_dim != 256 || p->rope_dim != 64 || p->idx_heads != 4 ||
      p->idx_dim != 128 || p->block_size != 4)
    return QSA_ERR_UNSUPPORTED;
  if (!(p->rope_theta > 1.0) || !std::isfinite(p->rope_theta)) return QSA_ERR_INVALID_ARG;
  if (p->budget_blocks < 2 || p->budget_blocks > 4096) return QSA_ERR_UNSUPPORTED;
  if (!(p->softmax_scale >= 0.f) || !std::isfinite(p->softmax_scale)) return QSA_ERR_INVALID_ARG;
  if (p->aggregation != QSA_AGG_TOKEN_MAX && p->aggregation != QSA_AGG_MEAN_POOL) return QSA_ERR_INVALID_ARG;
  if (!std::isfinite(p->yarn_factor) || p->yarn_factor < 0.0) return QSA_ERR_INVALID_ARG;
  if (p->yarn_factor > 1.0 && !(p->yarn_original_max >= 1.0 && std::isfinite(p->yarn_original_max) &&
                                p->yarn_beta_slow > 0.0 && p->yarn_beta_fast > p->yarn_beta_slow &&
                                std::isfinite(p->yarn_beta_fast)))
    return QSA_ERR_INVALID_ARG;
  if (p->idx_rope != 0 && p->idx_rope != 1) return QSA_ERR_INVALID_ARG;
  if (p->idx_rope && p->aggregation != QSA_AGG_MEAN_POOL) return QSA_ERR_INVALID_ARG;
  return QSA_OK;
}

bool mean_pool(const qsa_params* p) { return p->aggregation == QSA_AGG_MEAN_POOL; }
// the mean-pooled indexer with its block-start positions
bool idx_rope(const qsa_params* p) { return p->idx_rope == 1; }
// bytes of the mean-pooled keys of T tokens ([ceil(T/4)][128] bf16)
size_t kbar_bytes(int64_t T) { return (size_t)((T + 3) / 4) * 256; }

float softmax_scale(const qsa_params* p) {
  return p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt((float)p->head_dim);
}

// Rotary frequencies of the 32 pairs, with static YaRN when yarn_factor > 1:
// the pair index where the number of rotations over the original context,
// L f_i / (2 pi), equals n is d ln(L / (2 pi n)) / (2 ln theta); pairs before
// the beta_fast index (rounded down) keep f_i, pairs after the beta_slow index
// (rounded up) take f_i / s, linear in the index in between.
void inv_freq(const qsa_params* p, double* f) {
  const int half = p->rope_dim / 2;
  const double d = (double)p->rope_dim, s = p->yarn_factor;
  double lo = 0.0, hi = 1.0;
  if (s > 1.0) {
    const double two_pi = 6.283185307179586476925286766559;
    const double ln_theta = std::log(p->rope_theta);
    lo = std::floor(d * std::log(p->yarn_original_max / (two_pi * p->yarn_beta_fast)) / (2.0 * ln_theta));
    hi = std::ceil(d * std::log(p->yarn_original_max / (two_pi * p->yarn_beta_slow)) / (2.0 * ln_theta));
    lo = std::max(lo, 0.0);
    hi = std::min(hi, d - 1.0);
    if (hi == lo) hi += 0.001;
  }
  for (int i = 0; i < half; ++i) {
    const double base = std::pow(p->rope_theta, -2.0 * (double)i / d);
    if (!(s > 1.0)) {
      f[i] = base;
      continue;
    }
    const double t = std::min(std::max(((double)i - lo) / (hi - lo), 0.0), 1.0);   // share of f / s
    f[i] = base / s * t + base * (1.0 - t);
  }
}

// YaRN's attention factor on the rotated dims (1 without YaRN).
double rope_attn_factor(const qsa_params* p) {
  return p->yarn_factor > 1.0 ? 0.1 * std::log(p->yarn_factor) + 1.0 : 1.0;
}

// --------------------------------------------------------------- device info
struct DevInfo {
  bool known = false;
  bool sm100 = false;
  int num_sms = 0;
};
DevInfo g_dev[MAX_DEV];
std::mutex g_dev_mu;

qsa_status device_info(DevInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaGetDevice");
  if (dev < 0 || dev >= MAX_DEV) return fail(QSA_ERR_CUDA, "device ordinal out of range");
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.known) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return fail(QSA_ERR_CUDA, "cudaDeviceGetAttribute");
    d.sm100 = (major == 10 && minor == 0);
    d.num_sms = sms;
    d.known = true;
  }
  *out = d;
  return d.sm100 ? QSA_OK : fail(QSA_ERR_ARCH, "device is not sm_100");
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D bf16 tensor [rows][cols] (row-major), box [box_rows][box_cols], 128B swizzle.
qsa_status make_map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                       uint32_t box_cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(QSA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char d[64];
    std::snprintf(d, sizeof(d), "CUresult %d", (int)r);
    return fail(QSA_ERR_CUDA, "cuTensorMapEncodeTiled", d);
  }
  return QSA_OK;
}

// ----------------------------------------------------------------- tracing
// Every kernel launch of the library is wrapped in an NVTX range named
// "qsa.<kernel>" (free when no tool is attached; lets ncu --nvtx filter one
// stage of a step).  When tracing is enabled, each launch is also bracketed
// by two CUDA events recorded on the launching stream.
const char* nvtx_name(int32_t id) {
  switch (id) {
    case QSA_KERNEL_ROPE_TABLE: return "qsa.rope_table";
    case QSA_KERNEL_ROPE_K: return "qsa.rope_k";
    case QSA_KERNEL_INDEXER: return "qsa.indexer";
    case QSA_KERNEL_SELECT: return "qsa.select";
    case QSA_KERNEL_ATTENTION: return "qsa.attention";
    case QSA_KERNEL_DECODE_APPEND: return "qsa.decode_append";
    case QSA_KERNEL_DECODE_INDEXER: return "qsa.decode_indexer";
    case QSA_KERNEL_DECODE_ATTENTION: return "qsa.decode_attention";
    case QSA_KERNEL_DECODE_COMBINE: return "qsa.decode_combine";
    case QSA_KERNEL_KBAR: return "qsa.kbar";
    case QSA_KERNEL_VERIFY_EXPAND: return "qsa.verify_expand";
    case QSA_KERNEL_IDX_ROPE: return "qsa.idx_rope";
    default: return "qsa.other";
  }
}

struct TraceState {
  std::mutex mu;
  bool on = false;
  int cap = 0, n = 0;
  std::vector<cudaEvent_t> ev;
  std::vector<int32_t> ids;
};
TraceState g_trace;

template <class F>
cudaError_t traced(int32_t id, cudaStream_t s, F&& f) {
  int slot = -1;
  {
    std::lock_guard<std::mutex> lk(g_trace.mu);
    if (g_trace.on && g_trace.n < g_trace.cap) slot = g_trace.n++;
  }
  if (slot >= 0) cudaEventRecord(g_trace.ev[2 * slot], s);
  nvtxRangePushA(nvtx_name(id));
  cudaError_t e = f();
  nvtxRangePop();
  if (slot >= 0) {
    cudaEventRecord(g_trace.ev[2 * slot + 1], s);
    g_trace.ids[slot] = id;
  }
  return e;
}

qsa_status from_cuda(cudaError_t e, const char* where = "kernel launch") {
  if (e == cudaSuccess) return QSA_OK;
  return fail(QSA_ERR_CUDA, where, cudaGetErrorString(e));
}

// Indexer launch for query blocks [qb0, qb1) into S (ld), maps built here.
// Keys: tokens [0, T) of k_idx; q_idx / w hold tokens [q_tok0, T).  With kbar
// (mean pooling) the compressed keys [ceil(T/4)][128], already computed, are
// scored instead.
qsa_status run_indexer(int64_t T, int64_t q_tok0, const uint16_t* q_idx, const uint16_t* w, const uint16_t* k_idx,
                       const uint16_t* kbar, int64_t qb0, int64_t qb1, float* S, int64_t ld, float* segmax,
                       int64_t ld_seg, uint32_t* err, int num_sms, cudaStream_t st) {
  if (qb1 <= qb0) return QSA_OK;
  CUtensorMap tq, tk;
  qsa_status rs;
  if ((rs = make_map_2d(&tq, q_idx, (uint64_t)(T - q_tok0) * 4, 128, 256, 64)) != QSA_OK) return rs;
  if (kbar) {
    if ((rs = make_map_2d(&tk, kbar, (uint64_t)((T + 3) / 4), 128, 128, 64)) != QSA_OK) return rs;
  } else if ((rs = make_map_2d(&tk, k_idx, (uint64_t)T, 128, 128, 64)) != QSA_OK) {
    return rs;
  }
  const float scale = 1.0f / std::sqrt(128.0f);
  return from_cuda(traced(QSA_KERNEL_INDEXER, st, [&] {
    return qsa::launch_indexer_prefill(tq, tk, w, S, ld, segmax, ld_seg, T, q_tok0, qb0, qb1, kbar != nullptr, scale,
                                       err, num_sms, st);
  }), "indexer launch");
}

// Compressed keys of tokens [0, T) into kbar (mean pooling only).
// With block-start positions (p->idx_rope) each compressed key is also
// rotated at the position of its block's first token, pos0 + 4b.
qsa_status run_kbar(const qsa_params* p, const uint16_t* k_idx, int64_t T, int64_t pos0, uint16_t* kbar,
                    cudaStream_t st) {
  if (idx_rope(p)) {
    double f[32];
    inv_freq(p, f);
    return from_cuda(traced(QSA_KERNEL_KBAR, st, [&] {
      return qsa::launch_kbar_rope(k_idx, T, pos0, f, rope_attn_factor(p), kbar, st);
    }), "mean-pool launch");
  }
  return from_cuda(traced(QSA_KERNEL_KBAR, st, [&] { return qsa::launch_kbar(k_idx, T, kbar, st); }),
                   "mean-pool launch");
}
// Indexer queries rotated at positions pos0 + t (block-start positions only).
qsa_status run_idx_rope_q(const qsa_params* p, int64_t T, int64_t pos0, const uint16_t* q_idx, uint16_t* out,
                          cudaStream_t st) {
  double f[32];
  inv_freq(p, f);
  return from_cuda(traced(QSA_KERNEL_IDX_ROPE, st, [&] {
    return qsa::launch_idx_rope_q(T, pos0, f, rope_attn_factor(p), q_idx, out, st);
  }), "indexer RoPE launch");
}
// bytes of the rotated indexer queries of T tokens ([T][4][128] bf16)
size_t qrot_bytes(int64_t T) { return (size_t)T * 1024; }

// ------------------------------------------------------------ prefill layout
struct PrefillLayout {
  size_t cs, k_rot, sel, cnt, kbar, qrot, slab, total_fixed;
};
PrefillLayout prefill_layout(int64_t T, int budget, bool need_krot, bool need_sel, bool need_cnt, bool mean,
                             bool rope_idx = false) {
  const int64_t nqb = (T + 3) / 4;
  PrefillLayout L;
  size_t off = HEADER_BYTES;
  L.cs = off; off = align_up(off + (size_t)T * 32 * sizeof(float2));
  L.k_rot = off; off = align_up(off + (need_krot ? (size_t)T * 1024 : 0));
  L.sel = off; off = align_up(off + (need_sel ? (size_t)nqb * budget * 4 : 0));
  L.cnt = off; off = align_up(off + (need_cnt ? (size_t)nqb * 4 : 0));
  L.kbar = off; off = align_up(off + (mean ? kbar_bytes(T) : 0));
  L.qrot = off; off = align_up(off + (rope_idx ? qrot_bytes(T) : 0));
  L.slab = off;
  L.total_fixed = off;
  return L;
}
// Slab bytes of one row of a chunk ending at query block qb1: the scores
// (round4(qb1) floats) and the segment maxima (round4(ceil(qb1 / 8)) floats).
size_t slab_row_bytes(int64_t qb1) { return ((size_t)round4(qb1) + (size_t)round4((qb1 + 7) / 8)) * 4; }
// largest qb1 in (qb0, nqb] whose slab (qb1-qb0) x slab_row_bytes(qb1) fits
int64_t chunk_end(int64_t qb0, int64_t nqb, size_t slab_bytes) {
  int64_t lo = qb0 + 1, hi = nqb;
  if (slab_row_bytes(lo) > slab_bytes) return qb0;  // not even one row
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) / 2;
    if ((size_t)(mid - qb0) * slab_row_bytes(mid) <= slab_bytes) lo = mid; else hi = mid - 1;
  }
  return lo;
}
constexpr int64_t MIN_ROWS = 64;
constexpr size_t PREF_CAP = (size_t)16 << 30;

}  // namespace

extern "C" {

void qsa_default_params(qsa_params* p) {
  if (!p) return;
  p->n_q_heads = 24;
  p->n_kv_heads = 2;
  p->head_dim = 256;
  p->rope_dim = 64;
  p->rope_theta = 1e7;
  p->idx_heads = 4;
  p->idx_dim = 128;
  p->block_size = 4;
  p->budget_blocks = 512;
  p->softmax_scale = 0.f;
  p->aggregation = QSA_AGG_TOKEN_MAX;
  p->yarn_factor = 0.0;
  p->yarn_original_max = 262144.0;
  p->yarn_beta_fast = 32.0;
  p->yarn_beta_slow = 1.0;
  p->idx_rope = 0;
}

const char* qsa_last_error(void) { return g_last_error; }

const char* qsa_status_string(qsa_status s) {
  switch (s) {
    case QSA_OK: return "ok";
    case QSA_ERR_INVALID_ARG: return "invalid argument";
    case QSA_ERR_UNSUPPORTED: return "unsupported shape";
    case QSA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case QSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case QSA_ERR_CUDA: return "CUDA error";
    case QSA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case QSA_ERR_DEVICE_BOUNDS: return "device-side check failed";
    case QSA_ERR_ARCH: return "device is not sm_100";
  }
  return "unknown status";
}

qsa_status qsa_index_scores(const qsa_params* p, int64_t T, const uint16_t* q_idx, const uint16_t* w,
                            const uint16_t* k_idx, int64_t qb_begin, int64_t qb_end, float* scores, int64_t ld,
                            void* ws, size_t ws_bytes, void* stream) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (T <= 0 || T > ((int64_t)1 << 24)) return T <= 0 ? QSA_ERR_INVALID_ARG : QSA_ERR_UNSUPPORTED;
  const int64_t nqb = (T + 3) / 4;
  if (qb_begin < 0 || qb_end < qb_begin || qb_end > nqb || ld < qb_end || ld % 4 != 0) return QSA_ERR_INVALID_ARG;
  if (!q_idx || !w || !k_idx || !scores) return QSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(w) || !aligned16(k_idx) || !aligned16(scores)) return QSA_ERR_MISALIGNED;
  const bool mp = mean_pool(p), rope = idx_rope(p);
  if (mp && !ws) return QSA_ERR_INVALID_ARG;
  const size_t kbar_off = HEADER_BYTES, qrot_off = align_up(kbar_off + (mp ? kbar_bytes(T) : 0));
  if (ws && ws_bytes < qrot_off + (rope ? qrot_bytes(T) : 0)) return QSA_ERR_WORKSPACE_TOO_SMALL;
  if (ws && !aligned16(ws)) return QSA_ERR_MISALIGNED;
  DevInfo di;
  if ((st = device_info(&di)) != QSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(ws);
  if (err && cudaMemsetAsync(err, 0, 4, s) != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaMemsetAsync");
  uint16_t* kbar = mp ? reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + kbar_off) : nullptr;
  if (kbar && (st = run_kbar(p, k_idx, T, 0, kbar, s)) != QSA_OK) return st;
  const uint16_t* qi = q_idx;
  if (rope) {   // token t at position t
    uint16_t* qr = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + qrot_off);
    if ((st = run_idx_rope_q(p, T, 0, q_idx, qr, s)) != QSA_OK) return st;
    qi = qr;
  }
  return run_indexer(T, 0, qi, w, k_idx, kbar, qb_begin, qb_end, scores, ld, nullptr, 0, err, di.num_sms, s);
}

qsa_status qsa_index_workspace_size(const qsa_params* p, int64_t T, size_t* bytes) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (T <= 0 || !bytes) return QSA_ERR_INVALID_ARG;
  if (T > ((int64_t)1 << 24)) return QSA_ERR_UNSUPPORTED;
  *bytes = align_up(HEADER_BYTES + (mean_pool(p) ? kbar_bytes(T) : 0)) + (idx_rope(p) ? qrot_bytes(T) : 0);
  return QSA_OK;
}

qsa_status qsa_select_workspace_size(const qsa_params* p, size_t* bytes) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (!bytes) return QSA_ERR_INVALID_ARG;
  *bytes = HEADER_BYTES;
  return QSA_OK;
}

qsa_status qsa_select_blocks(const qsa_params* p, const float* scores, int64_t ld, int64_t qb_begin, int64_t qb_end,
                             int32_t* sel, int32_t* cnt, void* ws, size_t ws_bytes, void* stream) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (qb_begin < 0 || qb_end < qb_begin || ld < qb_end || ld % 4 != 0) return QSA_ERR_INVALID_ARG;
  if (!scores || !sel || !cnt || !ws) return QSA_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(sel) || !aligned16(cnt) || !aligned16(ws)) return QSA_ERR_MISALIGNED;
  if (ws_bytes < HEADER_BYTES) return QSA_ERR_WORKSPACE_TOO_SMALL;
  DevInfo di;
  if ((st = device_info(&di)) != QSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(ws);
  if (cudaMemsetAsync(err, 0, 4, s) != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaMemsetAsync");
  return from_cuda(traced(QSA_KERNEL_SELECT, s, [&] {
    return qsa::launch_select(scores, ld, nullptr, 0, qb_begin, qb_end - qb_begin, nullptr, p->budget_blocks, sel, cnt,
                              err, s);
  }));
}

qsa_status qsa_prefill_workspace_size(const qsa_params* p, int64_t T, size_t* min_bytes, size_t* pref_bytes) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (T <= 0) return QSA_ERR_INVALID_ARG;
  if (T > ((int64_t)1 << 24)) return QSA_ERR_UNSUPPORTED;
  const int64_t nqb = (T + 3) / 4;
  // worst case: the library keeps k_rot, sel and cnt itself
  PrefillLayout L = prefill_layout(T, p->budget_blocks, true, true, true, mean_pool(p), idx_rope(p));
  const int64_t min_rows = nqb < MIN_ROWS ? nqb : MIN_ROWS;
  const size_t row_bytes = slab_row_bytes(nqb);
  if (min_bytes) *min_bytes = L.total_fixed + (size_t)min_rows * row_bytes;
  if (pref_bytes) {
    // whole triangle in one pass is nqb rows of round4(nqb); cap it
    size_t full = (size_t)nqb * row_bytes;
    size_t cap = PREF_CAP > (size_t)min_rows * row_bytes ? PREF_CAP : (size_t)min_rows * row_bytes;
    *pref_bytes = L.total_fixed + (full < cap ? full : cap);
  }
  return QSA_OK;
}

qsa_status qsa_prefill(const qsa_params* p, int64_t T, int64_t pos0, const uint16_t* q, const uint16_t* k,
                       const uint16_t* v, const uint16_t* q_idx, const uint16_t* w, const uint16_t* k_idx,
                       uint16_t* out, float* lse, int32_t* sel_out, int32_t* cnt_out, uint16_t* k_rot_out, void* ws,
                       size_t ws_bytes, void* stream) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (T <= 0 || pos0 < 0) return QSA_ERR_INVALID_ARG;
  if (T > ((int64_t)1 << 24) || pos0 + T > ((int64_t)1 << 40)) return QSA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !q_idx || !w || !k_idx || !out || !ws) return QSA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, q_idx, w, k_idx, out, lse, sel_out, cnt_out, k_rot_out, ws};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return QSA_ERR_MISALIGNED;
  const int budget = p->budget_blocks;
  const int64_t nqb = (T + 3) / 4;
  PrefillLayout L = prefill_layout(T, budget, k_rot_out == nullptr, sel_out == nullptr, cnt_out == nullptr,
                                   mean_pool(p), idx_rope(p));
  if (ws_bytes < L.total_fixed) return QSA_ERR_WORKSPACE_TOO_SMALL;
  const size_t slab_bytes = ws_bytes - L.total_fixed;
  const int64_t min_rows = nqb < MIN_ROWS ? nqb : MIN_ROWS;
  if (slab_bytes < (size_t)min_rows * slab_row_bytes(nqb)) return QSA_ERR_WORKSPACE_TOO_SMALL;
  DevInfo di;
  if ((st = device_info(&di)) != QSA_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* err = reinterpret_cast<uint32_t*>(base);
  float2* cs = reinterpret_cast<float2*>(base + L.cs);
  uint16_t* k_rot = k_rot_out ? k_rot_out : reinterpret_cast<uint16_t*>(base + L.k_rot);
  int32_t* sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(base + L.sel);
  int32_t* cnt = cnt_out ? cnt_out : reinterpret_cast<int32_t*>(base + L.cnt);
  float* slab = reinterpret_cast<float*>(base + L.slab);

  if (cudaMemsetAsync(err, 0, 4, s) != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaMemsetAsync");
  double f[32];
  inv_freq(p, f);
  if ((st = from_cuda(traced(QSA_KERNEL_ROPE_TABLE, s, [&] {
         return qsa::launch_rope_table(T, pos0, f, rope_attn_factor(p), cs, s);
       }))) != QSA_OK)
    return st;
  if ((st = from_cuda(traced(QSA_KERNEL_ROPE_K, s, [&] { return qsa::launch_rope_k(T, k, cs, k_rot, s); }))) != QSA_OK)
    return st;
  uint16_t* kbar = mean_pool(p) ? reinterpret_cast<uint16_t*>(base + L.kbar) : nullptr;
  if (kbar && (st = run_kbar(p, k_idx, T, pos0, kbar, s)) != QSA_OK) return st;
  const uint16_t* qi = q_idx;
  if (idx_rope(p)) {   // the indexer queries rotated at their positions pos0 + t
    uint16_t* qr = reinterpret_cast<uint16_t*>(base + L.qrot);
    if ((st = run_idx_rope_q(p, T, pos0, q_idx, qr, s)) != QSA_OK) return st;
    qi = qr;
  }
  const float scale_log2 = softmax_scale(p) * 1.4426950408889634f;
  for (int64_t qb0 = 0; qb0 < nqb;) {
    const int64_t qb1 = chunk_end(qb0, nqb, slab_bytes);
    if (qb1 <= qb0) return QSA_ERR_WORKSPACE_TOO_SMALL;
    const int64_t ld = round4(qb1);
    const int64_t ld_seg = round4((qb1 + 7) / 8);
    float* segmax = slab + (size_t)(qb1 - qb0) * ld;
    if ((st = run_indexer(T, 0, qi, w, k_idx, kbar, qb0, qb1, slab, ld, segmax, ld_seg, err, di.num_sms, s)) !=
        QSA_OK)
      return st;
    if ((st = from_cuda(traced(QSA_KERNEL_SELECT, s, [&] {
           return qsa::launch_select(slab, ld, segmax, ld_seg, qb0, qb1 - qb0, nullptr, budget, sel + qb0 * budget,
                                     cnt + qb0, err, s);
         }))) != QSA_OK)
      return st;
    if ((st = from_cuda(traced(QSA_KERNEL_ATTENTION, s, [&] {
           return qsa::launch_sparse_attn_prefill_tc(T, q, k_rot, v, cs, sel + qb0 * budget, cnt + qb0, budget, qb0,
                                                     qb1, 0, scale_log2, out, lse, err, di.num_sms, s);
         }))) != QSA_OK)
      return st;
    qb0 = qb1;
  }
  return QSA_OK;
}

// --------------------------------------------------------- cached prefill
namespace {
struct CachedLayout {
  size_t cs, qst, wst, sel, cnt, kbar, slab, total_fixed;
};
// r = L_old % 4 tokens of the partial block before the new ones are staged
// in front of the new tokens' q_idx / w (nothing is staged when r == 0).
CachedLayout cached_layout(int64_t L_old, int64_t T_new, int budget, bool need_sel, bool need_cnt, bool mean) {
  const int64_t r = L_old % 4;
  const int64_t nq = (L_old + T_new - 1) / 4 - L_old / 4 + 1;
  CachedLayout L;
  size_t off = HEADER_BYTES;
  L.cs = off; off = align_up(off + (size_t)T_new * 32 * sizeof(float2));
  L.qst = off; off = align_up(off + (r ? (size_t)(r + T_new) * 4 * 128 * 2 : 0));
  L.wst = off; off = align_up(off + (r ? (size_t)(r + T_new) * 4 * 2 : 0));
  L.sel = off; off = align_up(off + (need_sel ? (size_t)nq * budget * 4 : 0));
  L.cnt = off; off = align_up(off + (need_cnt ? (size_t)nq * 4 : 0));
  L.kbar = off; off = align_up(off + (mean ? kbar_bytes(L_old + T_new) : 0));
  L.slab = off;
  L.total_fixed = off;
  return L;
}
}  // namespace

qsa_status qsa_prefill_cached_workspace_size(const qsa_params* p, int64_t L_old, int64_t T_new, size_t* min_bytes,
                                             size_t* pref_bytes) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (idx_rope(p)) return QSA_ERR_UNSUPPORTED;   // block-start positions: prefill and decode only
  if (L_old < 0 || T_new <= 0) return QSA_ERR_INVALID_ARG;
  if (L_old + T_new > ((int64_t)1 << 24)) return QSA_ERR_UNSUPPORTED;
  const int64_t nkb = (L_old + T_new + 3) / 4, qbA = L_old / 4, nq = nkb - qbA;
  CachedLayout L = cached_layout(L_old, T_new, p->budget_blocks, true, true, mean_pool(p));
  const int64_t min_rows = nq < MIN_ROWS ? nq : MIN_ROWS;
  const size_t row_bytes = slab_row_bytes(nkb);
  if (min_bytes) *min_bytes = L.total_fixed + (size_t)min_rows * row_bytes;
  if (pref_bytes) {
    const size_t full = (size_t)nq * row_bytes;
    const size_t cap = PREF_CAP > (size_t)min_rows * row_bytes ? PREF_CAP : (size_t)min_rows * row_bytes;
    *pref_bytes = L.total_fixed + (full < cap ? full : cap);
  }
  return QSA_OK;
}

qsa_status qsa_prefill_cached(const qsa_params* p, int64_t L_old, int64_t T_new, uint16_t* k_cache, uint16_t* v_cache,
                              uint16_t* kidx_cache, const uint16_t* qidx_prev, const uint16_t* w_prev,
                              const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* q_idx,
                              const uint16_t* w, const uint16_t* k_idx, uint16_t* out, float* lse, int32_t* sel_out,
                              int32_t* cnt_out, void* ws, size_t ws_bytes, void* stream) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (idx_rope(p)) return QSA_ERR_UNSUPPORTED;   // block-start positions: prefill and decode only
  if (L_old < 0 || T_new <= 0) return QSA_ERR_INVALID_ARG;
  if (L_old + T_new > ((int64_t)1 << 24)) return QSA_ERR_UNSUPPORTED;
  const int64_t r = L_old % 4;
  if (!k_cache || !v_cache || !kidx_cache || !q || !k || !v || !q_idx || !w || !k_idx || !out || !ws)
    return QSA_ERR_INVALID_ARG;
  if (r && (!qidx_prev || !w_prev)) return QSA_ERR_INVALID_ARG;
  const void* ptrs[] = {k_cache, v_cache, kidx_cache, qidx_prev, w_prev, q, k, v, q_idx, w, k_idx, out, lse,
                        sel_out, cnt_out, ws};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return QSA_ERR_MISALIGNED;
  const int budget = p->budget_blocks;
  const int64_t T = L_old + T_new;               // keys: tokens [0, T)
  const int64_t nkb = (T + 3) / 4, qbA = L_old / 4, nq = nkb - qbA;
  CachedLayout L = cached_layout(L_old, T_new, budget, sel_out == nullptr, cnt_out == nullptr, mean_pool(p));
  if (ws_bytes < L.total_fixed) return QSA_ERR_WORKSPACE_TOO_SMALL;
  const size_t slab_bytes = ws_bytes - L.total_fixed;
  const int64_t min_rows = nq < MIN_ROWS ? nq : MIN_ROWS;
  if (slab_bytes < (size_t)min_rows * slab_row_bytes(nkb)) return QSA_ERR_WORKSPACE_TOO_SMALL;
  DevInfo di;
  if ((st = device_info(&di)) != QSA_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* err = reinterpret_cast<uint32_t*>(base);
  float2* cs = reinterpret_cast<float2*>(base + L.cs);
  int32_t* sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(base + L.sel);
  int32_t* cnt = cnt_out ? cnt_out : reinterpret_cast<int32_t*>(base + L.cnt);
  float* slab = reinterpret_cast<float*>(base + L.slab);

  if (cudaMemsetAsync(err, 0, 4, s) != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaMemsetAsync");
  // new tokens into the caches: rotated keys at positions L_old .., values, indexer keys
  double f[32];
  inv_freq(p, f);
  if ((st = from_cuda(traced(QSA_KERNEL_ROPE_TABLE, s, [&] {
         return qsa::launch_rope_table(T_new, L_old, f, rope_attn_factor(p), cs, s);
       }))) != QSA_OK)
    return st;
  if ((st = from_cuda(traced(QSA_KERNEL_ROPE_K, s, [&] {
         return qsa::launch_rope_k(T_new, k, cs, k_cache + L_old * 512, s);
       }))) != QSA_OK)
    return st;
  if (cudaMemcpyAsync(v_cache + L_old * 512, v, (size_t)T_new * 1024, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(kidx_cache + L_old * 128, k_idx, (size_t)T_new * 256, cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess)
    return fail(QSA_ERR_CUDA, "cudaMemcpyAsync (cache append)");
  // indexer queries from the first new query block's first token on
  const uint16_t* qi = q_idx;
  const uint16_t* wi = w;
  if (r) {
    uint16_t* qst = reinterpret_cast<uint16_t*>(base + L.qst);
    uint16_t* wst = reinterpret_cast<uint16_t*>(base + L.wst);
    if (cudaMemcpyAsync(qst, qidx_prev, (size_t)r * 1024, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(qst + r * 512, q_idx, (size_t)T_new * 1024, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(wst, w_prev, (size_t)r * 8, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(wst + r * 4, w, (size_t)T_new * 8, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return fail(QSA_ERR_CUDA, "cudaMemcpyAsync (indexer query staging)");
    qi = qst;
    wi = wst;
  }
  // compressed keys of all cached and new tokens (mean pooling; the caches
  // now hold the new rows)
  uint16_t* kbar = mean_pool(p) ? reinterpret_cast<uint16_t*>(base + L.kbar) : nullptr;
  if (kbar && (st = run_kbar(p, kidx_cache, T, 0, kbar, s)) != QSA_OK) return st;
  const float scale_log2 = softmax_scale(p) * 1.4426950408889634f;
  for (int64_t qb0 = qbA; qb0 < nkb;) {
    const int64_t qb1 = chunk_end(qb0, nkb, slab_bytes);
    if (qb1 <= qb0) return QSA_ERR_WORKSPACE_TOO_SMALL;
    const int64_t ld = round4(qb1);
    const int64_t ld_seg = round4((qb1 + 7) / 8);
    float* segmax = slab + (size_t)(qb1 - qb0) * ld;
    int32_t* sel_c = sel + (qb0 - qbA) * budget;
    int32_t* cnt_c = cnt + (qb0 - qbA);
    if ((st = run_indexer(T, 4 * qbA, qi, wi, kidx_cache, kbar, qb0, qb1, slab, ld, segmax, ld_seg, err, di.num_sms,
                          s)) != QSA_OK)
      return st;
    if ((st = from_cuda(traced(QSA_KERNEL_SELECT, s, [&] {
           return qsa::launch_select(slab, ld, segmax, ld_seg, qb0, qb1 - qb0, nullptr, budget, sel_c, cnt_c, err, s);
         }))) != QSA_OK)
      return st;
    if ((st = from_cuda(traced(QSA_KERNEL_ATTENTION, s, [&] {
           return qsa::launch_sparse_attn_prefill_tc(T, q, k_cache, v_cache, cs, sel_c, cnt_c, budget, qb0, qb1, L_old,
                                                     scale_log2, out, lse, err, di.num_sms, s);
         }))) != QSA_OK)
      return st;
    qb0 = qb1;
  }
  return QSA_OK;
}

// ------------------------------------------------------------------ decode
namespace {
struct DecodeLayout {
  size_t Ls, qbs, S, sel, sel_r, cnt, q_rot, part_o, part_lse, ring_rot, total;
  int64_t ld;
  int sel_r_ld;   // row stride of the merged reused selections
};
// Split-KV ranges per (sequence, KV head): at most this many.
constexpr int DECODE_MAX_SPLIT = 16;
DecodeLayout decode_layout(int B, int64_t max_len, int budget) {
  DecodeLayout L;
  L.ld = round4(max_len / 4 + 1);
  size_t off = HEADER_BYTES;
  L.Ls = off; off = align_up(off + (size_t)B * 8);
  L.qbs = off; off = align_up(off + (size_t)B * 8);
  L.S = off; off = align_up(off + (size_t)B * L.ld * 4);
  L.sel = off; off = align_up(off + (size_t)B * budget * 4);
  L.sel_r_ld = budget + 4;
  L.sel_r = off; off = align_up(off + (size_t)B * L.sel_r_ld * 4);
  L.cnt = off; off = align_up(off + (size_t)B * 4);
  L.q_rot = off; off = align_up(off + (size_t)B * 24 * 256 * 2);
  L.part_o = off; off = align_up(off + (size_t)B * 2 * DECODE_MAX_SPLIT * 12 * 256 * 4);
  L.part_lse = off; off = align_up(off + (size_t)B * 2 * DECODE_MAX_SPLIT * 12 * 4);
  L.ring_rot = off; off = align_up(off + (size_t)B * 4 * 4 * 128 * 2);
  L.total = off;
  return L;
}
// Number of split-KV ranges: the one that minimises the most work any SM
// does, in tiles: (items it runs) x (tiles per item + 1.5 for the per-item
// overhead), plus 1 for the combine when there is more than one range, given
// the largest selection of the batch (measured on B200: at 64 sequences x 32
// tiles one range per (sequence, KV head) is best).  qsa_set_decode_splits
// (1 .. 16) overrides the choice for the whole process.
std::atomic<int> g_forced_splits{0};
int decode_splits(int B, int64_t max_L, int budget, int num_sms) {
  const int forced = g_forced_splits.load(std::memory_order_relaxed);
  if (forced >= 1 && forced <= DECODE_MAX_SPLIT) return forced;
  int64_t cnt = max_L / 4 + 1;
  if (cnt > budget) cnt = budget;
  const int nt = (int)((cnt + 15) / 16);
  int best = 1;
  double best_cost = 1e300;
  for (int sp = 1; sp <= DECODE_MAX_SPLIT && sp <= nt; ++sp) {
    const int64_t items = 2 * (int64_t)B * sp;
    const double waves = (double)((items + num_sms - 1) / num_sms);
    const double cost = waves * ((nt + sp - 1) / sp + 1.5) + (sp > 1 ? 1.0 : 0.0);
    if (cost < best_cost - 1e-9) { best_cost = cost; best = sp; }
  }
  return best;
}
}  // namespace

qsa_status qsa_set_decode_splits(int32_t n) {
  if (n < 0 || n > DECODE_MAX_SPLIT) return QSA_ERR_INVALID_ARG;
  g_forced_splits.store(n, std::memory_order_relaxed);
  return QSA_OK;
}

qsa_status qsa_decode_workspace_size(const qsa_params* p, int32_t B, int64_t max_len, size_t* bytes) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (B <= 0 || max_len <= 0 || !bytes) return QSA_ERR_INVALID_ARG;
  if (B > 4096 || max_len > ((int64_t)1 << 24)) return QSA_ERR_UNSUPPORTED;
  *bytes = decode_layout(B, max_len, p->budget_blocks).total;
  return QSA_OK;
}

namespace {
// One decode step; kbar_cache non-null only for the mean-pooled indexer;
// sel_in / cnt_in non-null: stages 1 and 2 are skipped, the append kernel
// merges each given selection with the token's forced blocks into the sel_r
// region and the attention reads that.
qsa_status decode_impl(const qsa_params* p, int32_t B, int64_t max_len, const int64_t* cache_len, uint16_t* k_cache,
                       uint16_t* v_cache, uint16_t* kidx_cache, uint16_t* kbar_cache, uint16_t* qidx_ring,
                       uint16_t* w_ring, const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new,
                       const uint16_t* q_idx_new, const uint16_t* k_idx_new, const uint16_t* w_new, uint16_t* out,
                       int32_t* sel_out, float* lse_out, void* ws, size_t ws_bytes, void* stream,
                       const int32_t* sel_in = nullptr, const int32_t* cnt_in = nullptr) {
  qsa_status st;
  if (B <= 0 || max_len <= 0 || !cache_len) return QSA_ERR_INVALID_ARG;
  if (B > 4096 || max_len > ((int64_t)1 << 24)) return QSA_ERR_UNSUPPORTED;
  const void* ptrs[] = {k_cache, v_cache, kidx_cache, qidx_ring, w_ring, q_new, k_new, v_new,
                        q_idx_new, k_idx_new, w_new, out, ws};
  for (const void* ptr : ptrs) {
    if (!ptr) return QSA_ERR_INVALID_ARG;
    if (!aligned16(ptr)) return QSA_ERR_MISALIGNED;
  }
  if ((sel_out && !aligned16(sel_out)) || (lse_out && !aligned16(lse_out)) || (kbar_cache && !aligned16(kbar_cache)))
    return QSA_ERR_MISALIGNED;
  const int64_t kbar_len = (max_len + 3) / 4;
  int64_t max_L = 0;
  for (int b = 0; b < B; ++b) {
    if (cache_len[b] < 0 || cache_len[b] >= max_len) return QSA_ERR_INVALID_ARG;
    if (cache_len[b] > max_L) max_L = cache_len[b];
  }
  const int budget = p->budget_blocks;
  DecodeLayout L = decode_layout(B, max_len, budget);
  if (ws_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
  DevInfo di;
  if ((st = device_info(&di)) != QSA_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* err = reinterpret_cast<uint32_t*>(base);
  int64_t* Ls = reinterpret_cast<int64_t*>(base + L.Ls);
  int64_t* qbs = reinterpret_cast<int64_t*>(base + L.qbs);
  float* S = reinterpret_cast<float*>(base + L.S);
  const bool reuse = sel_in != nullptr;
  int32_t* sel_r = reinterpret_cast<int32_t*>(base + L.sel_r);
  int32_t* sel = reuse ? sel_r : (sel_out ? sel_out : reinterpret_cast<int32_t*>(base + L.sel));
  const int sel_ld = reuse ? L.sel_r_ld : budget;
  int32_t* cnt = reinterpret_cast<int32_t*>(base + L.cnt);
  uint16_t* q_rot = reinterpret_cast<uint16_t*>(base + L.q_rot);
  // block-start positions: the append kernel writes the block-mates' indexer
  // queries rotated at their positions here, and the decode indexer reads them
  uint16_t* ring_rot = idx_rope(p) ? reinterpret_cast<uint16_t*>(base + L.ring_rot) : nullptr;

  if (cudaMemsetAsync(err, 0, 4, s) != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaMemsetAsync");
  double f[32];
  inv_freq(p, f);
  // the append kernel receives the lengths as launch parameters and stores
  // them (and L/4) in the workspace for the later kernels
  if ((st = from_cuda(traced(QSA_KERNEL_DECODE_APPEND, s, [&] {
         return qsa::launch_decode_append(B, max_len, cache_len, Ls, qbs, f, rope_attn_factor(p), k_cache, v_cache,
                                          kidx_cache, qidx_ring, w_ring, q_new, k_new, v_new, q_idx_new, k_idx_new,
                                          w_new, q_rot, kbar_cache, kbar_len, sel_in, cnt_in, budget, sel_r, L.sel_r_ld,
                                          cnt, err, s, idx_rope(p), ring_rot);
       }))) != QSA_OK)
    return st;
  const float scale = 1.0f / std::sqrt(128.0f);
  if (!reuse) {
    if ((st = from_cuda(traced(QSA_KERNEL_DECODE_INDEXER, s, [&] {
           return qsa::launch_decode_indexer(B, max_len, max_L, Ls, kidx_cache, kbar_cache, kbar_len,
                                             ring_rot ? ring_rot : qidx_ring, w_ring, S, L.ld, scale, s);
         }))) != QSA_OK)
      return st;
    if ((st = from_cuda(traced(QSA_KERNEL_SELECT, s, [&] {
           return qsa::launch_select(S, L.ld, nullptr, 0, 0, B, qbs, budget, sel, cnt, err, s);
         }))) != QSA_OK)
      return st;
  }
  const float scale_log2 = softmax_scale(p) * 1.4426950408889634f;
  // a merged reused selection holds at most budget + 2 blocks
  const int n_split = decode_splits(B, max_L, reuse ? budget + 2 : budget, di.num_sms);
  float* part_o = reinterpret_cast<float*>(base + L.part_o);
  float* part_lse = reinterpret_cast<float*>(base + L.part_lse);
  if ((st = from_cuda(traced(QSA_KERNEL_DECODE_ATTENTION, s, [&] {
         return qsa::launch_decode_attn_tc(B, max_len, Ls, q_rot, k_cache, v_cache, sel, cnt, sel_ld, scale_log2,
                                           n_split, part_o, part_lse, out, lse_out, err, di.num_sms, s);
       }))) != QSA_OK)
    return st;
  if (n_split == 1) return QSA_OK;
  return from_cuda(traced(QSA_KERNEL_DECODE_COMBINE, s, [&] {
    return qsa::launch_decode_combine(B, part_o, part_lse, cnt, n_split, out, lse_out, s);
  }));
}
}  // namespace

qsa_status qsa_decode(const qsa_params* p, int32_t B, int64_t max_len, const int64_t* cache_len, uint16_t* k_cache,
                      uint16_t* v_cache, uint16_t* kidx_cache, uint16_t* qidx_ring, uint16_t* w_ring,
                      const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new, const uint16_t* q_idx_new,
                      const uint16_t* k_idx_new, const uint16_t* w_new, uint16_t* out, int32_t* sel_out,
                      float* lse_out, void* ws, size_t ws_bytes, void* stream) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (mean_pool(p)) return QSA_ERR_UNSUPPORTED;   // needs the compressed-key cache: qsa_decode_mean_pool
  return decode_impl(p, B, max_len, cache_len, k_cache, v_cache, kidx_cache, nullptr, qidx_ring, w_ring, q_new, k_new,
                     v_new, q_idx_new, k_idx_new, w_new, out, sel_out, lse_out, ws, ws_bytes, stream);
}

qsa_status qsa_decode_mean_pool(const qsa_params* p, int32_t B, int64_t max_len, const int64_t* cache_len,
                                uint16_t* k_cache, uint16_t* v_cache, uint16_t* kidx_cache, uint16_t* kbar_cache,
                                uint16_t* qidx_ring, uint16_t* w_ring, const uint16_t* q_new, const uint16_t* k_new,
                                const uint16_t* v_new, const uint16_t* q_idx_new, const uint16_t* k_idx_new,
                                const uint16_t* w_new, uint16_t* out, int32_t* sel_out, float* lse_out, void* ws,
                                size_t ws_bytes, void* stream) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (!mean_pool(p)) return QSA_ERR_INVALID_ARG;
  if (!kbar_cache) return QSA_ERR_INVALID_ARG;
  return decode_impl(p, B, max_len, cache_len, k_cache, v_cache, kidx_cache, kbar_cache, qidx_ring, w_ring, q_new,
                     k_new, v_new, q_idx_new, k_idx_new, w_new, out, sel_out, lse_out, ws, ws_bytes, stream);
}

qsa_status qsa_decode_reuse(const qsa_params* p, int32_t B, int64_t max_len, const int64_t* cache_len,
                            uint16_t* k_cache, uint16_t* v_cache, uint16_t* kidx_cache, uint16_t* kbar_cache,
                            uint16_t* qidx_ring, uint16_t* w_ring, const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new,
                            const uint16_t* q_idx_new, const uint16_t* k_idx_new, const uint16_t* w_new,
                            const int32_t* sel_in, const int32_t* cnt_in, uint16_t* out, float* lse_out, void* ws,
                            size_t ws_bytes, void* stream) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (!sel_in) return QSA_ERR_INVALID_ARG;
  if (!aligned16(sel_in) || (cnt_in && !aligned16(cnt_in))) return QSA_ERR_MISALIGNED;
  if (mean_pool(p) != (kbar_cache != nullptr)) return QSA_ERR_INVALID_ARG;   // the cache is kept for that mode only
  return decode_impl(p, B, max_len, cache_len, k_cache, v_cache, kidx_cache, kbar_cache, qidx_ring, w_ring, q_new, k_new,
                     v_new, q_idx_new, k_idx_new, w_new, out, nullptr, lse_out, ws, ws_bytes, stream, sel_in, cnt_in);
}

qsa_status qsa_mean_pool_keys(const qsa_params* p, int64_t T, const uint16_t* k_idx, uint16_t* kbar, void* stream) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (T <= 0 || !k_idx || !kbar) return QSA_ERR_INVALID_ARG;
  if (T > ((int64_t)1 << 24)) return QSA_ERR_UNSUPPORTED;
  if (!aligned16(k_idx) || !aligned16(kbar)) return QSA_ERR_MISALIGNED;
  DevInfo di;
  if ((st = device_info(&di)) != QSA_OK) return st;
  return run_kbar(p, k_idx, T, 0, kbar, static_cast<cudaStream_t>(stream));
}

qsa_status qsa_check_device_error(void* ws, void* stream) {
  if (!ws) return QSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t h = 0;
  if (cudaMemcpyAsync(&h, ws, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return QSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return QSA_ERR_CUDA;
  if (h != 0 && cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) return QSA_ERR_CUDA;
  if (h == 0) return QSA_OK;
  return (h == QSA_ERR_DEVICE_TIMEOUT || h == QSA_ERR_DEVICE_BOUNDS) ? static_cast<qsa_status>(h) : QSA_ERR_CUDA;
}

qsa_status qsa_trace_begin(int32_t capacity) {
  if (capacity <= 0 || capacity > (1 << 20)) return QSA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_trace.mu);
  if (g_trace.on) return QSA_ERR_INVALID_ARG;
  g_trace.ev.assign((size_t)2 * capacity, nullptr);
  for (auto& e : g_trace.ev)
    if (cudaEventCreate(&e) != cudaSuccess) return QSA_ERR_CUDA;
  g_trace.ids.assign((size_t)capacity, 0);
  g_trace.cap = capacity;
  g_trace.n = 0;
  g_trace.on = true;
  return QSA_OK;
}

qsa_status qsa_trace_end(int32_t* kernel_ids, float* ms, int32_t capacity, int32_t* n_out) {
  std::lock_guard<std::mutex> lk(g_trace.mu);
  if (!g_trace.on) return QSA_ERR_INVALID_ARG;
  qsa_status st = QSA_OK;
  const int n = g_trace.n;
  if (n > 0 && cudaEventSynchronize(g_trace.ev[2 * n - 1]) != cudaSuccess) st = QSA_ERR_CUDA;
  int written = 0;
  for (int i = 0; i < n && st == QSA_OK; ++i) {
    if (i >= capacity || !kernel_ids || !ms) break;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, g_trace.ev[2 * i], g_trace.ev[2 * i + 1]) != cudaSuccess) { st = QSA_ERR_CUDA; break; }
    kernel_ids[i] = g_trace.ids[i];
    ms[i] = t;
    ++written;
  }
  for (auto e : g_trace.ev)
    if (e) cudaEventDestroy(e);
  g_trace.ev.clear();
  g_trace.ids.clear();
  g_trace.on = false;
  g_trace.n = g_trace.cap = 0;
  if (n_out) *n_out = written;
  return st;
}

}  // extern "C"

// Test hooks of the debug build (include/qsa_debug.h).
#ifdef QSA_DEBUG_HOOKS
namespace qsa {
namespace {
std::atomic<int> g_debug_inject{0};
}  // namespace
int take_debug_injection(int code) {
  int expected = code;
  return g_debug_inject.compare_exchange_strong(expected, 0) ? code : 0;
}
}  // namespace qsa

extern "C" qsa_status qsa_debug_inject(int32_t code) {
  if (code < QSA_INJECT_NONE || code > QSA_INJECT_ATTENTION_RESCALE_ALL) return QSA_ERR_INVALID_ARG;
  qsa::g_debug_inject.store(code);
  return QSA_OK;
}
#endif


// ------------------------------------------------------------------ verify
namespace {
constexpr int VERIFY_MAX_M = 16;
struct VerifyLayout {
  size_t Lb, Ls, rqb, S, selb, cntb, selt, cntt, q_rot, part_o, part_lse, total;
  int64_t ld;
  int nqv, max_split;
};
// Query blocks that m consecutive tokens can touch: (m + 2) / 4 + 1.
VerifyLayout verify_layout(int B, int m, int64_t max_len, int budget) {
  VerifyLayout L;
  const int64_t rows = (int64_t)B * m;
  L.nqv = (m + 2) / 4 + 1;
  L.ld = round4(max_len / 4 + 1);
  // split-KV ranges are worth having only while the token rows leave SMs
  // idle: at most enough to give 296 (two per SM) items
  int ms = (int)((296 + 2 * rows - 1) / (2 * rows));
  L.max_split = ms < 1 ? 1 : (ms > DECODE_MAX_SPLIT ? DECODE_MAX_SPLIT : ms);
  const int64_t nrow = (int64_t)B * L.nqv;
  size_t off = HEADER_BYTES;
  L.Lb = off; off = align_up(off + (size_t)B * 8);
  L.Ls = off; off = align_up(off + (size_t)rows * 8);
  L.rqb = off; off = align_up(off + (size_t)nrow * 8);
  L.S = off; off = align_up(off + (size_t)nrow * L.ld * 4);
  L.selb = off; off = align_up(off + (size_t)nrow * budget * 4);
  L.cntb = off; off = align_up(off + (size_t)nrow * 4);
  L.selt = off; off = align_up(off + (size_t)rows * budget * 4);
  L.cntt = off; off = align_up(off + (size_t)rows * 4);
  L.q_rot = off; off = align_up(off + (size_t)rows * 24 * 256 * 2);
  L.part_o = off; off = align_up(off + (L.max_split > 1 ? (size_t)rows * 2 * L.max_split * 12 * 256 * 4 : 0));
  L.part_lse = off; off = align_up(off + (L.max_split > 1 ? (size_t)rows * 2 * L.max_split * 12 * 4 : 0));
  L.total = off;
  return L;
}
}  // namespace

qsa_status qsa_verify_workspace_size(const qsa_params* p, int32_t B, int32_t m, int64_t max_len, size_t* bytes) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (idx_rope(p)) return QSA_ERR_UNSUPPORTED;   // block-start positions: prefill and decode only
  if (B <= 0 || m <= 0 || max_len <= 0 || !bytes) return QSA_ERR_INVALID_ARG;
  if (B > 4096 || m > VERIFY_MAX_M || max_len > ((int64_t)1 << 24)) return QSA_ERR_UNSUPPORTED;
  *bytes = verify_layout(B, m, max_len, p->budget_blocks).total;
  return QSA_OK;
}

qsa_status qsa_verify(const qsa_params* p, int32_t B, int32_t m, int64_t max_len, const int64_t* cache_len,
                      uint16_t* k_cache, uint16_t* v_cache, uint16_t* kidx_cache, uint16_t* kbar_cache,
                      const uint16_t* qidx_prev,
                      const uint16_t* w_prev, const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new,
                      const uint16_t* q_idx_new, const uint16_t* k_idx_new, const uint16_t* w_new, uint16_t* out,
                      int32_t* sel_out, float* lse_out, void* ws, size_t ws_bytes, void* stream) {
  qsa_status st = check_params(p);
  if (st != QSA_OK) return st;
  if (idx_rope(p)) return QSA_ERR_UNSUPPORTED;   // block-start positions: prefill and decode only
  if (B <= 0 || m <= 0 || max_len <= 0 || !cache_len) return QSA_ERR_INVALID_ARG;
  if (mean_pool(p) != (kbar_cache != nullptr)) return QSA_ERR_INVALID_ARG;   // the compressed keys go with mean pool
  if (kbar_cache && !aligned16(kbar_cache)) return QSA_ERR_MISALIGNED;
  if (B > 4096 || m > VERIFY_MAX_M || max_len > ((int64_t)1 << 24)) return QSA_ERR_UNSUPPORTED;
  const void* ptrs[] = {k_cache, v_cache, kidx_cache, q_new, k_new, v_new, q_idx_new, k_idx_new, w_new, out, ws};
  for (const void* ptr : ptrs) {
    if (!ptr) return QSA_ERR_INVALID_ARG;
    if (!aligned16(ptr)) return QSA_ERR_MISALIGNED;
  }
  if ((qidx_prev && !aligned16(qidx_prev)) || (w_prev && !aligned16(w_prev)) || (lse_out && !aligned16(lse_out)) ||
      (sel_out && !aligned16(sel_out)))
    return QSA_ERR_MISALIGNED;
  int64_t max_L = 0;
  bool any_partial = false;
  for (int b = 0; b < B; ++b) {
    if (cache_len[b] < 0 || cache_len[b] + m > max_len) return QSA_ERR_INVALID_ARG;
    if (cache_len[b] > max_L) max_L = cache_len[b];
    any_partial |= (cache_len[b] & 3) != 0;
  }
  // block-mates before the new tokens come from qidx_prev / w_prev
  if (any_partial && (!qidx_prev || !w_prev)) return QSA_ERR_INVALID_ARG;
  const int budget = p->budget_blocks;
  VerifyLayout L = verify_layout(B, m, max_len, budget);
  if (ws_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
  DevInfo di;
  if ((st = device_info(&di)) != QSA_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* err = reinterpret_cast<uint32_t*>(base);
  int64_t* Lb = reinterpret_cast<int64_t*>(base + L.Lb);
  int64_t* Ls = reinterpret_cast<int64_t*>(base + L.Ls);
  int64_t* rqb = reinterpret_cast<int64_t*>(base + L.rqb);
  float* S = reinterpret_cast<float*>(base + L.S);
  int32_t* selb = reinterpret_cast<int32_t*>(base + L.selb);
  int32_t* cntb = reinterpret_cast<int32_t*>(base + L.cntb);
  int32_t* selt = sel_out ? sel_out : reinterpret_cast<int32_t*>(base + L.selt);
  int32_t* cntt = reinterpret_cast<int32_t*>(base + L.cntt);
  uint16_t* q_rot = reinterpret_cast<uint16_t*>(base + L.q_rot);
  float* part_o = reinterpret_cast<float*>(base + L.part_o);
  float* part_lse = reinterpret_cast<float*>(base + L.part_lse);

  if (cudaMemsetAsync(err, 0, 4, s) != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaMemsetAsync");
  double f[32];
  inv_freq(p, f);
  if ((st = from_cuda(traced(QSA_KERNEL_DECODE_APPEND, s, [&] {
         return qsa::launch_verify_append(B, m, L.nqv, max_len, cache_len, Lb, Ls, rqb, f, rope_attn_factor(p),
                                          k_cache, v_cache, kidx_cache, q_new, k_new, v_new, k_idx_new, q_rot, s);
       }))) != QSA_OK)
    return st;
  const int64_t kbar_len = (max_len + 3) / 4;
  if (kbar_cache && (st = from_cuda(traced(QSA_KERNEL_KBAR, s, [&] {
                       return qsa::launch_verify_kbar(B, m, L.nqv, max_len, kbar_len, Lb, rqb, kidx_cache,
                                                      kbar_cache, s);
                     }))) != QSA_OK)
    return st;
  const float scale = 1.0f / std::sqrt(128.0f);
  if ((st = from_cuda(traced(QSA_KERNEL_DECODE_INDEXER, s, [&] {
         return qsa::launch_verify_indexer(B, L.nqv, m, max_len, max_L, Lb, rqb, kidx_cache, kbar_cache, kbar_len,
                                           qidx_prev, w_prev, q_idx_new, w_new, S, L.ld, scale, s);
       }))) != QSA_OK)
    return st;
  if ((st = from_cuda(traced(QSA_KERNEL_SELECT, s, [&] {
         return qsa::launch_select(S, L.ld, nullptr, 0, 0, (int64_t)B * L.nqv, rqb, budget, selb, cntb, err, s);
       }))) != QSA_OK)
    return st;
  if ((st = from_cuda(traced(QSA_KERNEL_VERIFY_EXPAND, s, [&] {
         return qsa::launch_verify_expand(B, m, L.nqv, budget, Ls, selb, cntb, selt, cntt, s);
       }))) != QSA_OK)
    return st;
  const int rows = B * m;
  int n_split = decode_splits(rows, max_L + m - 1, budget, di.num_sms);
  if (n_split > L.max_split) n_split = L.max_split;
  const float scale_log2 = softmax_scale(p) * 1.4426950408889634f;
  if ((st = from_cuda(traced(QSA_KERNEL_DECODE_ATTENTION, s, [&] {
         return qsa::launch_decode_attn_tc(rows, max_len, Ls, q_rot, k_cache, v_cache, selt, cntt, budget, scale_log2,
                                           n_split, part_o, part_lse, out, lse_out, err, di.num_sms, s, m);
       }))) != QSA_OK)
    return st;
  if (n_split == 1) return QSA_OK;
  return from_cuda(traced(QSA_KERNEL_DECODE_COMBINE, s, [&] {
    return qsa::launch_decode_combine(rows, part_o, part_lse, cntt, n_split, out, lse_out, s);
  }));
}
