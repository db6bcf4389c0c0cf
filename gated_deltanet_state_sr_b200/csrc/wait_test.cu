// sr_test_wait_timeout: makes one bounded mbarrier wait run out on purpose.
//
// Every tcgen05 / TMA kernel of the library waits on mbarriers through
// tc::mbar_wait, which gives up after a time limit; the kernel then records
// SR_DEV_TIMEOUT, frees its tensor memory and returns instead of hanging.
// A healthy replay never reaches that path, so this entry point runs it
// directly: one CTA allocates tensor memory, waits on an mbarrier that nothing
// arrives at (or, as the control case, that its own thread 0 arrives at) with a
// short caller-given limit, reports, frees the tensor memory and exits.
#include "common.cuh"
#include "sr/sr_testing.h"
#include "tc.cuh"

namespace sr {
namespace {

constexpr uint32_t kTestTmemCols = 128;

__global__ void __launch_bounds__(128) wait_timeout_kernel(uint64_t limit_ns, int arrive, uint32_t *status,
                                                           unsigned long long *elapsed_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tmem_slot;
    const int warp = threadIdx.x / 32;
    if (warp == 0) {
        tc::tmem_alloc(&tmem_slot, kTestTmemCols);
        tc::tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (arrive && threadIdx.x == 0) tc::mbar_arrive(&bar);

    const uint64_t t0 = tc::globaltimer_ns();
    const bool ok = tc::mbar_wait(&bar, 0, limit_ns);
    const uint64_t t1 = tc::globaltimer_ns();
    const bool all_ok = __syncthreads_and(ok) != 0;
    if (threadIdx.x == 0) {
        if (!all_ok) atomicOr(status, SR_DEV_TIMEOUT);
        *elapsed_ns = static_cast<unsigned long long>(t1 - t0);
    }
    // the exit path every timed-out kernel takes: tensor memory back, then return
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem_slot, kTestTmemCols);
}

}  // namespace
}  // namespace sr

using namespace sr;

extern "C" sr_status sr_test_wait_timeout(uint64_t limit_ns, int32_t arrive, void *workspace,
                                          size_t workspace_bytes, void *stream) {
    if (limit_ns == 0 || limit_ns > tc::kWaitLimitNs)
        return set_error(SR_ERR_INVALID_ARG, "sr_test_wait_timeout: limit_ns must be in (0, %llu]",
                         static_cast<unsigned long long>(tc::kWaitLimitNs));
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kWsAlign) != 0 || workspace_bytes < kWsHeader)
        return set_error(SR_ERR_WORKSPACE, "sr_test_wait_timeout: need a 256-byte aligned workspace of >= %zu bytes",
                         kWsHeader);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, kWsHeader, st);
    if (e != cudaSuccess) return cuda_error(e, "sr_test_wait_timeout: clearing the status word");
    auto *status = static_cast<uint32_t *>(workspace);
    auto *elapsed = reinterpret_cast<unsigned long long *>(static_cast<char *>(workspace) + 8);
    wait_timeout_kernel<<<1, 128, 0, st>>>(limit_ns, arrive ? 1 : 0, status, elapsed);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_error(e, "sr_test_wait_timeout: launch");
    return SR_OK;
}
