// Chunked gated-delta replay on tensor cores (placeholder until the kernel lands).
#include "common.cuh"
#include "kernels.h"

namespace sr {

bool gdn_chunked_supported(const sr_gdn_args &) { return false; }
size_t gdn_scratch_bytes(const sr_gdn_args &) { return 0; }
cudaError_t gdn_chunked(const sr_gdn_args &a, float scale, uint32_t *status, void *, cudaStream_t st) {
    return gdn_sequential(a, scale, status, st);
}

size_t mamba2_scratch_bytes(const sr_mamba2_args &) { return 0; }
cudaError_t mamba2_replay(const sr_mamba2_args &a, uint32_t *status, void *, cudaStream_t st) {
    return mamba2_sequential(a, status, st);
}

}  // namespace sr
