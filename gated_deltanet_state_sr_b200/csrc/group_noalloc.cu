// sr_group_replay_noalloc: the group replay for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain a workspace: a plug-in that a host
// framework hands only its input and output buffers, a serving engine that
// has already given all spare HBM to its KV-cache pool and forbids further
// cudaMalloc, or a latency-critical path where the implicit synchronisation of
// cudaMalloc / cudaFree is not acceptable.  For them the scratch of a group
// replay lives in one file-scope device array of fixed size that every GPU
// loading this library holds until the process exits.  Replays whose scratch
// does not fit are rejected, and the caller has to use sr_group_replay with a
// workspace of its own instead.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace sr {
namespace {

// Scratch of sr_group_replay_noalloc.  In host code this name is only a
// host-side stand-in: the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SR_GROUP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device.  Outside a stream
// capture it is looked up on every call, so a module that was reloaded (after
// cudaDeviceReset, say) is found at its new address; inside a capture, where
// a lookup might have to load the module, the address of the last call on this
// device outside a capture is used.
sr_status scratch_on_current_device(cudaStream_t stream, void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_error(e, "sr_group_replay_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return set_error(SR_ERR_UNSUPPORTED, "device index %d too large", dev);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return cuda_error(e, "sr_group_replay_noalloc: cudaStreamIsCapturing");
    std::lock_guard<std::mutex> lock(g_mu);
    if (cap == cudaStreamCaptureStatusNone) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_error(e, "sr_group_replay_noalloc: cudaGetSymbolAddress");
        g_scratch_ptr[dev] = p;
    } else if (!g_scratch_ptr[dev]) {
        return set_error(SR_ERR_INVALID_ARG,
                         "sr_group_replay_noalloc: the first call on a device must come before any stream "
                         "capture (it looks up the scratch array's device address)");
    }
    *out = g_scratch_ptr[dev];
    return SR_OK;
}

}  // namespace
}  // namespace sr

using namespace sr;

extern "C" sr_status sr_group_replay_noalloc(const sr_group_args *a, void *stream, const void **status_scratch) {
    const size_t need = sr_group_replay_workspace(a);
    if (need == 0) return sr_group_replay(a, nullptr, 0, stream);  // reports the validation error
    if (need > SR_GROUP_NOALLOC_SCRATCH_BYTES)
        return set_error(SR_ERR_WORKSPACE,
                         "sr_group_replay_noalloc: this replay needs %zu bytes of scratch but the built-in array "
                         "holds %zu; call sr_group_replay with a caller workspace instead",
                         need, size_t(SR_GROUP_NOALLOC_SCRATCH_BYTES));
    void *scratch = nullptr;
    if (sr_status s = scratch_on_current_device(static_cast<cudaStream_t>(stream), &scratch)) return s;
    if (status_scratch) *status_scratch = scratch;
    // sr_group_replay clears the status word at the start of the array; every
    // other scratch byte is written before it is read within the call.
    return sr_group_replay(a, scratch, SR_GROUP_NOALLOC_SCRATCH_BYTES, stream);
}
