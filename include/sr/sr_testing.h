/*
 * sr_testing.h -- test-support entry points of libsr.so.
 *
 * These expose single internal kernels of the replay group so that each can
 * be checked against the fp64 oracle in isolation.  They are not part of the
 * replay API (include/sr/sr.h) and follow its conventions: device pointers,
 * caller-owned buffers, a caller workspace whose first 256 bytes hold the
 * device status word, asynchronous on `stream`, sr_status return values.
 */
#ifndef SR_SR_TESTING_H
#define SR_SR_TESTING_H

#include "sr/sr.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Dense projection on the tcgen05 tensor cores, the GEMM every projection of
 * the replay group uses (in_proj, out_proj, SwiGLU gate/up, down):
 *   epi 0:  c = a b0^T
 *   epi 1:  c = r + a b0^T
 *   epi 2:  c = SiLU(a b0^T) * (a b1^T)
 * a [m, k], b0 / b1 [n, k], c and r [m, n]; all bf16 row-major; k % 64 == 0,
 * n % 32 == 0.  workspace >= 256 bytes.  form: 0 the library's default, 1 one
 * CTA per 128 x 256 output tile, 2 a cluster of two CTAs (two SMs) per
 * 256 x 256 tile sharing cta_group::2 products; both give bit-identical c. */
SR_API sr_status sr_test_gemm(const void *a, const void *b0, const void *b1, void *c, const void *r,
                              int32_t m, int32_t n, int32_t k, int32_t epi, int32_t form, void *workspace,
                              size_t workspace_bytes, void *stream);

/* A bounded on-chip wait made to run out.  The paper has no counterpart: this
 * checks the library's own failure detection.  Every tcgen05 / TMA kernel
 * waits on mbarriers with a time limit (half a second), after which it sets
 * SR_DEV_TIMEOUT in the status word, frees its tensor memory and returns.
 * This call launches one CTA that allocates 128 tensor-memory columns, waits
 * on an mbarrier through the same wait with the given limit_ns (0 < limit_ns
 * <= the kernels' own limit, else SR_ERR_INVALID_ARG), then frees the tensor
 * memory and exits.  With arrive == 0 nothing arrives at the barrier, so the
 * wait runs out and SR_DEV_TIMEOUT is set; with arrive != 0 the CTA's first
 * thread arrives before waiting, so the wait completes and no flag is set.
 * The workspace (>= 256 bytes, 256-byte aligned) receives the status word at
 * offset 0 and the wait's duration in nanoseconds (uint64) at offset 8. */
SR_API sr_status sr_test_wait_timeout(uint64_t limit_ns, int32_t arrive, void *workspace, size_t workspace_bytes,
                                      void *stream);

#ifdef __cplusplus
}
#endif
#endif /* SR_SR_TESTING_H */
