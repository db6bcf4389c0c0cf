// Anchor sidecar plumbing around the replay ("SuffixReplay: Prefix Caching
// via Suffix Replay for Hybrid LLMs", Algorithm Design 2 and System Design).
//
//   sr_anchor_capture      writes selected hidden rows into the anchor pool
//                          through a destination table prepared on the host
//                          (System Design, Anchor Sidecar: indexed copies
//                          inside captured CUDA graphs, no host sync).
//   sr_sparse_anchor_plan  host: which prefix positions carry token-wise
//                          sparse anchors (a fixed number per 64-token page,
//                          at the page's end or spread evenly) and which of
//                          them a replay of k = min(ratio * n, k_max) anchors
//                          reads (Algorithm Design 2 and 3), as rows of a
//                          page-major pool.
#include <math.h>

#include "common.cuh"

namespace sr {
namespace {

// One warp per captured row: 16-byte vector copies (hidden % 8 == 0).
__global__ void __launch_bounds__(256) capture_kernel(const __nv_bfloat16 *__restrict__ hidden,
                                                      __nv_bfloat16 *__restrict__ pool,
                                                      const int32_t *__restrict__ src_rows,
                                                      const int32_t *__restrict__ dst_rows, int n, int H,
                                                      int src_total, int pool_rows, uint32_t *status) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * 8 + warp;
    if (i >= n) return;
    const int s = src_rows[i], d = dst_rows[i];
    if (s < 0 || s >= src_total || d < 0 || d >= pool_rows) {
        if (lane == 0) atomicOr(status, SR_DEV_BAD_INDEX);
        return;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(hidden + size_t(s) * H);
    uint4 *dst = reinterpret_cast<uint4 *>(pool + size_t(d) * H);
    for (int c = lane; c < H / 8; c += 32) dst[c] = src[c];
}

}  // namespace
}  // namespace sr

using namespace sr;

extern "C" sr_status sr_anchor_capture(const sr_capture_args *a, void *ws, size_t ws_bytes, void *stream) {
    if (!a) return set_error(SR_ERR_INVALID_ARG, "args is NULL");
    if (a->n < 0 || a->hidden <= 0 || a->src_rows_total < 0 || a->pool_rows < 0)
        return set_error(SR_ERR_INVALID_ARG, "bad n / hidden / src_rows_total / pool_rows");
    if (a->hidden % 8) return set_error(SR_ERR_UNSUPPORTED, "hidden must be a multiple of 8 (got %d)", a->hidden);
    if (a->n > 0 && (!a->hidden_states || !a->pool || !a->src_rows || !a->dst_rows))
        return set_error(SR_ERR_INVALID_ARG, "hidden_states, pool, src_rows and dst_rows are required");
    if ((reinterpret_cast<uintptr_t>(a->hidden_states) | reinterpret_cast<uintptr_t>(a->pool)) % 16)
        return set_error(SR_ERR_INVALID_ARG, "hidden_states and pool must be 16-byte aligned");
    if (!ws) return set_error(SR_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", kWsHeader);
    if (reinterpret_cast<uintptr_t>(ws) % kWsAlign) return set_error(SR_ERR_WORKSPACE, "workspace not 256-byte aligned");
    if (ws_bytes < kWsHeader) return set_error(SR_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, kWsHeader);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t *status = static_cast<uint32_t *>(ws);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return cuda_error(e, "sr_anchor_capture: clearing the status word");
    if (a->n == 0) return SR_OK;
    capture_kernel<<<(a->n + 7) / 8, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(a->hidden_states),
                                                   static_cast<__nv_bfloat16 *>(a->pool), a->src_rows, a->dst_rows,
                                                   a->n, a->hidden, a->src_rows_total, a->pool_rows, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_error(e, "sr_anchor_capture: launch");
    return SR_OK;
}

extern "C" sr_status sr_sparse_anchor_plan(const sr_anchor_plan_args *a, int64_t *positions, int32_t *pool_rows,
                                           int64_t capacity, int64_t *count) {
    if (!a || !count) return set_error(SR_ERR_INVALID_ARG, "args and count are required");
    *count = 0;
    const int64_t n = a->n_prefix;
    const int P = a->page_size, m = a->anchors_per_page;
    if (n < 0 || P <= 0 || m <= 0 || m > P || a->k_max < 0 || !(a->ratio >= 0.0) || a->ratio > 1.0)
        return set_error(SR_ERR_INVALID_ARG, "bad n_prefix / page_size / anchors_per_page / k_max / ratio");
    if (a->layout != SR_ANCHORS_PAGE_TAIL && a->layout != SR_ANCHORS_UNIFORM)
        return set_error(SR_ERR_INVALID_ARG, "bad layout %d", a->layout);
    if (a->layout == SR_ANCHORS_UNIFORM && P % m)
        return set_error(SR_ERR_INVALID_ARG, "uniform layout needs page_size %% anchors_per_page == 0");
    // offset of slot i inside its page
    auto slot_offset = [&](int i) -> int64_t {
        return a->layout == SR_ANCHORS_PAGE_TAIL ? int64_t(P - m + i) : int64_t(i + 1) * (P / m) - 1;
    };
    // anchors that exist: every slot position below n
    const int64_t full_pages = n / P;
    int64_t available = full_pages * m;
    for (int i = 0; i < m; ++i)
        if (full_pages * P + slot_offset(i) < n) ++available;
    // replay budget in anchors: k = min(ceil(ratio * n), k_max)
    int64_t k = int64_t(ceil(a->ratio * double(n) - 1e-9));
    if (k < 0) k = 0;
    if (k > a->k_max) k = a->k_max;
    if (k > available) k = available;
    *count = k;
    if (k > capacity)
        return set_error(SR_ERR_INVALID_ARG, "capacity %lld < %lld anchors", (long long)capacity, (long long)k);
    // the last k anchors, oldest first: anchor j (0-based, in position order) is slot j % m of page j / m
    const int64_t first = available - k;
    for (int64_t j = 0; j < k; ++j) {
        const int64_t ord = first + j, page = ord / m;
        const int slot = int(ord % m);
        if (positions) positions[j] = page * P + slot_offset(slot);
        if (pool_rows) {
            const int64_t block = a->block_table ? a->block_table[page] : page;
            if (block < 0) return set_error(SR_ERR_INVALID_ARG, "block_table[%lld] < 0", (long long)page);
            const int64_t row = block * m + slot;
            if (row > INT32_MAX) return set_error(SR_ERR_UNSUPPORTED, "pool row beyond int32");
            pool_rows[j] = int32_t(row);
        }
    }
    return SR_OK;
}
