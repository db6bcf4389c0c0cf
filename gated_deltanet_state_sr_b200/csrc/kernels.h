// Internal launchers of libsr (not part of the C ABI).  Each returns the
// cudaError_t of its launches; shapes were validated by api.cu.
#pragma once

#include <cuda_runtime.h>

#include "sr/sr.h"

namespace sr {

// Raw gated-delta replay.
cudaError_t gdn_sequential(const sr_gdn_args &a, float scale, uint32_t *status, cudaStream_t st);
bool gdn_chunked_supported(const sr_gdn_args &a);
size_t gdn_scratch_bytes(const sr_gdn_args &a);
cudaError_t gdn_chunked(const sr_gdn_args &a, float scale, uint32_t *status, void *scratch,
                        cudaStream_t st);

// Mamba2 replay.
cudaError_t mamba2_sequential(const sr_mamba2_args &a, uint32_t *status, cudaStream_t st);
size_t mamba2_scratch_bytes(const sr_mamba2_args &a);
cudaError_t mamba2_replay(const sr_mamba2_args &a, uint32_t *status, void *scratch, cudaStream_t st);

}  // namespace sr
