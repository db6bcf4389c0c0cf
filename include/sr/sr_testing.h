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
 * n % 32 == 0.  workspace >= 256 bytes. */
SR_API sr_status sr_test_gemm(const void *a, const void *b0, const void *b1, void *c, const void *r,
                              int32_t m, int32_t n, int32_t k, int32_t epi, void *workspace,
                              size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* SR_SR_TESTING_H */
