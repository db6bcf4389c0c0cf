// Shared device/host helpers of libsr (internal; not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sr/sr.h"

namespace sr {

// Workspace header: the first kWsHeader bytes of every workspace hold the
// device status word (uint32 at offset 0).  Scratch regions follow.
constexpr size_t kWsHeader = 256;
constexpr size_t kWsAlign = 256;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Thread-local last-error plumbing (api.cu).
sr_status set_error(sr_status s, const char *fmt, ...);
sr_status cuda_error(cudaError_t e, const char *where);

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Bounds checks of the checked build.  Compiled with -DSR_CHECKED (the
// library libsr_checked.so), SR_IN_BOUNDS(i, n, status) tests 0 <= i < n for a
// global-memory index about to be used; on failure it ORs SR_DEV_BAD_ACCESS
// into the status word and returns false, and the caller skips the access.
// In the ordinary build it is the constant true and costs nothing.  A check
// never traps: it is a stand-in for a memory checker that can run on any GPU.
__device__ __forceinline__ bool in_bounds_checked(long long i, long long n, uint32_t *status) {
    const bool ok = i >= 0 && i < n;
    if (!ok && status) atomicOr(status, SR_DEV_BAD_ACCESS);
    return ok;
}
#ifdef SR_CHECKED
#define SR_IN_BOUNDS(i, n, status) ::sr::in_bounds_checked((long long)(i), (long long)(n), (status))
#else
#define SR_IN_BOUNDS(i, n, status) true
#endif

// Reads and checks the bounds of sequence n.  On a bad entry ORs a flag into
// the status word and returns false; the caller then skips the sequence.
__device__ __forceinline__ bool seq_bounds(const int32_t *cu, int n, int total, int max_len,
                                           uint32_t *status, int &bos, int &eos) {
    bos = cu[n];
    eos = cu[n + 1];
    bool ok = (bos >= 0) && (bos <= eos) && (eos <= total) && (n != 0 || bos == 0);
    if (!ok) {
        if (status) atomicOr(status, SR_DEV_BAD_CU_SEQLENS);
        return false;
    }
    if (eos - bos > max_len) {
        if (status) atomicOr(status, SR_DEV_SEQ_TOO_LONG);
        return false;
    }
    return true;
}

// Longest-first dispatch.  A grid row r of a per-sequence kernel takes the
// sequence of rank r in the order of decreasing length (ties: lower index
// first), so the longest replays start in the first wave instead of trailing
// the last one.  With more than kLongestFirstMax sequences the row keeps its
// own index.  `scratch` is shared memory for n + 1 ints; every thread of the
// block calls this, and it ends with a block barrier.
constexpr int kLongestFirstMax = 256;
__device__ __forceinline__ int longest_first(const int32_t *cu, int n, int r, int *scratch) {
    if (n > kLongestFirstMax) return r;
    for (int m = threadIdx.x; m < n; m += blockDim.x) scratch[m] = cu[m + 1] - cu[m];
    __syncthreads();
    for (int m = threadIdx.x; m < n; m += blockDim.x) {
        const int lm = scratch[m];
        int rank = 0;
        for (int j = 0; j < n; ++j) {
            const int lj = scratch[j];
            rank += (lj > lm) || (lj == lm && j < m);
        }
        if (rank == r) scratch[n] = m;
    }
    __syncthreads();
    const int seq = scratch[n];
    __syncthreads();  // the scratch may be reused right after
    return seq;
}

}  // namespace sr
