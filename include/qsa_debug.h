/*
 * qsa_debug.h -- test hooks of the debug build of the QSA library
 * (libqsa_debug.so, built from the same sources with QSA_DEBUG_BOUNDS,
 * QSA_DEBUG_HOOKS and a 20 ms device wait limit).  The pages have no
 * counterpart: these exist to test the library's own failure handling.  The
 * release library (libqsa.so) does not export them.
 *
 * In the debug build:
 *   - every bounded device wait gives up after 20 ms instead of 2 s;
 *   - the attention kernels check that every selected block index is -1
 *     (padding) or a causal block 0 .. qb of the query block, and the
 *     indexer checks every score and segment-maximum store against the
 *     output's row range and leading dimension; a failed check records
 *     QSA_ERR_DEVICE_BOUNDS (read with qsa_check_device_error) and the access
 *     is skipped;
 *   - qsa_debug_inject arms one fault (or, for QSA_INJECT_ATTENTION_RESCALE_ALL,
 *     one change of schedule that leaves the result within rounding of the
 *     normal one) for the next launch of the kernel it names.  The faults make no out-of-range access and leave no wait
 *     unbounded: a stall withholds one completion signal, so a waiting role
 *     times out, records QSA_ERR_DEVICE_TIMEOUT and the CTA drains what it
 *     issued and exits; a bad block names a block after the query block,
 *     which the bounds check reports (and the causal test masks).
 */
#ifndef QSA_DEBUG_H_
#define QSA_DEBUG_H_

#include <stdint.h>

#include "qsa.h"

#ifdef __cplusplus
extern "C" {
#endif

enum {
  QSA_INJECT_NONE = 0,
  QSA_INJECT_INDEXER_STALL = 1,        /* next indexer launch: CTA 0 never signals its first accumulator */
  QSA_INJECT_ATTENTION_STALL = 2,      /* next prefill attention launch: CTA 0 never signals its first S tile */
  QSA_INJECT_ATTENTION_BAD_BLOCK = 3,  /* next prefill attention launch: CTA 0's first gathered block is qb + 1 */
  QSA_INJECT_ATTENTION_RESCALE_ALL = 4 /* next attention launch (prefill or decode): the online softmax takes a
                                          new running maximum, and rescales the accumulated output, on every tile
                                          (no lazy margin), so that path runs on ordinary inputs */
};

/* Arms `code` for the next launch of the kernel it names (one launch; a new
 * call replaces an armed code).  QSA_ERR_INVALID_ARG for an unknown code. */
qsa_status qsa_debug_inject(int32_t code);

#ifdef __cplusplus
}
#endif
#endif /* QSA_DEBUG_H_ */
