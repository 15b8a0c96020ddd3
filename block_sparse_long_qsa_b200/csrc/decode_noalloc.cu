// qsa_decode_noalloc: the decode step with its scratch memory in a fixed,
// library-owned device array instead of a caller-provided workspace.
//
// Who needs this: callers that cannot allocate device memory at the point
// where they run a decode step -- for example code whose device memory is
// owned and fully budgeted by another runtime (an inference server's pool, a
// plugin inside a host framework) and which may not call cudaMalloc on the
// request path, where it would synchronise the device and can fail under
// memory pressure.  Such callers still pass their own inputs, outputs and KV
// caches; only the decode scratch (score rows, selections, split partials,
// error word) lives here.
//
// The array below is reserved on every GPU on which this file's device code
// is loaded (with CUDA's default lazy module loading: at the first call of
// this entry point on that GPU) and stays reserved until the process exits.
#include "qsa.h"
#include "qsa_kernels.h"

namespace {

// Largest decode scratch this entry point serves (64 MiB: e.g. 64 sequences
// at 256K context need about 41 MiB).
constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)64 << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of g_decode_scratch on the current device.  In host code
// the symbol name is only a host-side handle; kernels must be given the
// address cudaGetSymbolAddress returns.  It is looked up on every call (a
// host-side lookup once the module is loaded), so a context that was torn
// down and created again never gets a stale address.
qsa_status scratch_for_current_device(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return QSA_ERR_CUDA;
  *out = p;
  return QSA_OK;
}

}  // namespace

extern "C" qsa_status qsa_decode_noalloc(const qsa_params* p, int32_t B, int64_t max_len, const int64_t* cache_len,
                                         uint16_t* k_cache, uint16_t* v_cache, uint16_t* kidx_cache,
                                         uint16_t* qidx_ring, uint16_t* w_ring, const uint16_t* q_new,
                                         const uint16_t* k_new, const uint16_t* v_new, const uint16_t* q_idx_new,
                                         const uint16_t* k_idx_new, const uint16_t* w_new, uint16_t* out,
                                         int32_t* sel_out, float* lse_out, void* stream) {
  size_t need = 0;
  qsa_status st = qsa_decode_workspace_size(p, B, max_len, &need);
  if (st != QSA_OK) return st;
  if (need > NOALLOC_SCRATCH_BYTES) return QSA_ERR_WORKSPACE_TOO_SMALL;   // beyond the fixed scratch size
  void* scratch = nullptr;
  if ((st = scratch_for_current_device(&scratch)) != QSA_OK) return st;
  // The regular decode step on the fixed scratch.  It clears the error word
  // at its start and writes everything else before reading it, so nothing of
  // an earlier call's contents is used.
  return qsa_decode(p, B, max_len, cache_len, k_cache, v_cache, kidx_cache, qidx_ring, w_ring, q_new, k_new, v_new,
                    q_idx_new, k_idx_new, w_new, out, sel_out, lse_out, scratch, NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" qsa_status qsa_decode_noalloc_check_error(void* stream) {
  void* scratch = nullptr;
  qsa_status st = scratch_for_current_device(&scratch);
  if (st != QSA_OK) return st;
  return qsa_check_device_error(scratch, stream);
}
