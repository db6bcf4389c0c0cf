// Replay of whole linear-attention groups (placeholder until its kernels land).
#include "common.cuh"
#include "kernels.h"

using namespace sr;

extern "C" {
size_t sr_group_replay_workspace(const sr_group_args *) { return 0; }
sr_status sr_group_replay(const sr_group_args *a, void *, size_t, void *) {
    if (!a) return set_error(SR_ERR_INVALID_ARG, "args is NULL");
    return set_error(SR_ERR_UNSUPPORTED, "sr_group_replay: not built yet");
}
}
