/*
 * vdit_attn_testing.h -- test-only entry point of libvdit_attn.so.
 *
 * Not part of the compute path.  It exists so that the failure detection of
 * the forward kernel can be exercised on a GPU without faulting it: every
 * wait of the kernel on one of its own pipeline barriers is bounded in time,
 * and when one runs out the kernel abandons its work, releases its tensor
 * memory, records VDIT_ERR_TIMEOUT in the device status word and returns, so
 * the CUDA context stays usable.  The pages have no counterpart; this covers
 * the failure-detection layer of the library itself.
 */
#ifndef VDIT_ATTN_TESTING_H
#define VDIT_ATTN_TESTING_H

#include "vdit_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Faults the test entry point can inject, all on the host side of the
 * pipeline: nothing is made to fault, trap or hang. */
#define VDIT_TESTING_NO_FAULT 0
/* The TMA producer never loads K/V, so the MMA issuer's wait for the first K
 * tile runs out; no MMA is ever issued. */
#define VDIT_TESTING_WITHHOLD_KV 1

/*
 * vdit_testing_attn_fwd -- vdit_attn_fwd with an injected fault and a
 * per-wait time limit of wait_timeout_ns nanoseconds (1e6 .. 1e10; product
 * calls use 2e9).  Same argument rules and return codes as vdit_attn_fwd;
 * VDIT_ERR_INVALID_ARG for an unknown fault or an out-of-range limit.  The
 * timeout itself is reported by vdit_get_device_status as VDIT_ERR_TIMEOUT.
 * The outputs of a faulted call are unspecified.
 */
vdit_status vdit_testing_attn_fwd(const void* q, const void* k, const void* v,
                                  void* o, float* lse, int B, int H, int Sq,
                                  int Skv, int D, float scale, int mask_kind,
                                  int chunk_tokens, int fault,
                                  unsigned long long wait_timeout_ns,
                                  void* stream);

/*
 * vdit_testing_cross_cta_spans -- the cross-attention call (mask CROSS; same
 * arguments, rules and outputs as vdit_attn_fwd) that also records, for each
 * CTA of its persistent grid, the SM it ran on and when its TMA producer
 * started and finished (%globaltimer, ns).  It exists so a test can see how
 * many of the kernel's CTAs an SM holds at once, which the occupancy query
 * does not report correctly for this kernel.
 *   spans     : device uint64 [max_ctas][3] = {smid, start ns, end ns},
 *               8-byte aligned; must hold one row per CTA of the grid
 *   grid_ctas : out, the number of CTAs launched (rows written)
 * VDIT_ERR_INVALID_ARG if spans or grid_ctas is NULL or max_ctas is smaller
 * than the grid.  Asynchronous on `stream`.
 */
vdit_status vdit_testing_cross_cta_spans(const void* q, const void* k,
                                         const void* v, void* o, float* lse,
                                         int B, int H, int Sq, int Skv, int D,
                                         float scale, unsigned long long* spans,
                                         int max_ctas, int* grid_ctas,
                                         void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VDIT_ATTN_TESTING_H */
