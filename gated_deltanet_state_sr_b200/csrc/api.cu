// C ABI of libsr: host-side validation, workspace sizing and dispatch.
// Declarations and the contract of every entry point are in include/sr/sr.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include "common.cuh"
#include "kernels.h"

namespace sr {

namespace {
thread_local char g_err[512] = "";
}

sr_status set_error(sr_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

sr_status cuda_error(cudaError_t e, const char *where) {
    return set_error(SR_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

static bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static sr_status check_workspace(void *ws, size_t bytes, size_t need) {
    if (!ws) return set_error(SR_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
    if (!aligned(ws, kWsAlign)) return set_error(SR_ERR_WORKSPACE, "workspace not 256-byte aligned");
    if (bytes < need)
        return set_error(SR_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", bytes, need);
    return SR_OK;
}

static sr_status check_varlen(int n_seqs, int total, int max_len, const int32_t *cu) {
    if (!cu) return set_error(SR_ERR_INVALID_ARG, "cu_seqlens is NULL");
    if (n_seqs < 0 || total < 0 || max_len < 0)
        return set_error(SR_ERR_INVALID_ARG, "negative n_seqs / total_tokens / max_seqlen");
    if (n_seqs > 65535) return set_error(SR_ERR_UNSUPPORTED, "n_seqs > 65535");
    if (max_len > total) return set_error(SR_ERR_INVALID_ARG, "max_seqlen > total_tokens");
    return SR_OK;
}

sr_status validate_gdn(const sr_gdn_args *a) {
    if (!a) return set_error(SR_ERR_INVALID_ARG, "args is NULL");
    if (sr_status s = check_varlen(a->n_seqs, a->total_tokens, a->max_seqlen, a->cu_seqlens)) return s;
    if (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->s_out)
        return set_error(SR_ERR_INVALID_ARG, "q, k, v, g, beta and s_out are required");
    if (a->h_k <= 0 || a->h_v <= 0 || a->h_v % a->h_k != 0)
        return set_error(SR_ERR_INVALID_ARG, "need h_k > 0, h_v > 0 and h_v %% h_k == 0 (h_k=%d h_v=%d)",
                         a->h_k, a->h_v);
    if (a->h_v > 65535) return set_error(SR_ERR_UNSUPPORTED, "h_v > 65535");
    if (a->d_k != a->d_v || (a->d_k != 64 && a->d_k != 128))
        return set_error(SR_ERR_UNSUPPORTED, "head dims must satisfy d_k == d_v in {64,128} (got %d,%d)",
                         a->d_k, a->d_v);
    if (a->dtype != SR_BF16 && a->dtype != SR_FP32) return set_error(SR_ERR_INVALID_ARG, "bad dtype");
    if (a->algo < SR_GDN_AUTO || a->algo > SR_GDN_TCGEN05_FUSED) return set_error(SR_ERR_INVALID_ARG, "bad algo");
    const bool tc = a->algo == SR_GDN_TCGEN05 || a->algo == SR_GDN_TCGEN05_FUSED;
    if ((a->algo == SR_GDN_CHUNKED || tc) && a->dtype != SR_BF16)
        return set_error(SR_ERR_UNSUPPORTED, "the chunked kernels take bf16 q/k/v only");
    if (tc && !gdn_tc_supported(a->d_k))
        return set_error(SR_ERR_UNSUPPORTED, "the tcgen05 kernels take d_k = d_v = 128 only");
    if (!aligned(a->s_out, 16) || (a->h0 && !aligned(a->h0, 16)))
        return set_error(SR_ERR_INVALID_ARG, "s_out and h0 must be 16-byte aligned");
    const size_t esz = a->dtype == SR_BF16 ? 2 : 4;
    if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->v, 16) || (a->o && !aligned(a->o, 16)))
        return set_error(SR_ERR_INVALID_ARG, "q, k, v and o must be 16-byte aligned");
    (void)esz;
    if (!isfinite(a->scale)) return set_error(SR_ERR_INVALID_ARG, "scale is not finite");
    return SR_OK;
}

}  // namespace sr

using namespace sr;

extern "C" {

const char *sr_last_error(void) { return g_err; }

int32_t sr_version(void) { return 0x000100; }

// The tcgen05 form a call runs: 0 none, 1 two-phase, 2 fused.
static int gdn_tc_form(const sr_gdn_args *a) {
    if (a->algo == SR_GDN_TCGEN05_FUSED) return 2;
    if (a->algo == SR_GDN_TCGEN05) return 1;
    return a->algo == SR_GDN_AUTO && a->dtype == SR_BF16 && gdn_tc_supported(a->d_k) ? 1 : 0;
}

static size_t gdn_need(const sr_gdn_args *a) {
    const int form = gdn_tc_form(a);
    if (form == 1) return kWsHeader + gdn_tc_image_bytes(a->total_tokens, a->n_seqs, a->h_v, 1);
    return kWsHeader + (form == 0 ? gdn_scratch_bytes(*a) : 0);
}

size_t sr_gdn_replay_workspace(const sr_gdn_args *a) {
    if (validate_gdn(a) != SR_OK) return 0;
    return gdn_need(a);
}

sr_status sr_gdn_replay(const sr_gdn_args *a, void *ws, size_t ws_bytes, void *stream) {
    if (sr_status s = validate_gdn(a)) return s;
    const size_t need = gdn_need(a);
    if (sr_status s = check_workspace(ws, ws_bytes, need)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t *status = static_cast<uint32_t *>(ws);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return cuda_error(e, "sr_gdn_replay: clearing the status word");
    const float scale = a->scale != 0.f ? a->scale : 1.0f / sqrtf(float(a->d_k));
    const bool chunked = a->algo == SR_GDN_CHUNKED || (a->algo == SR_GDN_AUTO && a->dtype == SR_BF16 &&
                                                        gdn_chunked_supported(*a));
    void *scratch = static_cast<char *>(ws) + kWsHeader;
    const int form = gdn_tc_form(a);
    if (form)
        e = gdn_tc(*a, scale, status, form == 1 ? scratch : nullptr, st);
    else
        e = chunked ? gdn_chunked(*a, scale, status, scratch, st) : gdn_sequential(*a, scale, status, st);
    if (e != cudaSuccess) return cuda_error(e, "sr_gdn_replay: kernel launch");
    return SR_OK;
}

static sr_status validate_mamba2(const sr_mamba2_args *a) {
    if (!a) return set_error(SR_ERR_INVALID_ARG, "args is NULL");
    if (sr_status s = check_varlen(a->n_seqs, a->total_tokens, a->max_seqlen, a->cu_seqlens)) return s;
    if (!a->x || !a->B || !a->C || !a->dt || !a->A || !a->s_out)
        return set_error(SR_ERR_INVALID_ARG, "x, B, C, dt, A and s_out are required");
    if (a->n_heads <= 0 || a->n_groups <= 0 || a->n_heads % a->n_groups != 0)
        return set_error(SR_ERR_INVALID_ARG, "need n_heads %% n_groups == 0");
    if (a->head_dim != 64 || a->d_state != 128)
        return set_error(SR_ERR_UNSUPPORTED, "supported: head_dim 64, d_state 128 (got %d, %d)",
                         a->head_dim, a->d_state);
    if (a->n_heads > 65535) return set_error(SR_ERR_UNSUPPORTED, "n_heads > 65535");
    if (a->algo < SR_MAMBA2_AUTO || a->algo > SR_MAMBA2_TCGEN05) return set_error(SR_ERR_INVALID_ARG, "bad algo");
    if ((a->algo == SR_MAMBA2_CHUNKED || a->algo == SR_MAMBA2_TCGEN05) && (a->n_groups != 1 || a->n_heads % 2))
        return set_error(SR_ERR_UNSUPPORTED, "the chunk kernels need one B/C group and an even head count");
    if (!aligned(a->s_out, 16) || (a->h0 && !aligned(a->h0, 16)) || !aligned(a->x, 16) ||
        !aligned(a->B, 16) || !aligned(a->C, 16) || (a->y && !aligned(a->y, 16)))
        return set_error(SR_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    return SR_OK;
}

size_t sr_mamba2_replay_workspace(const sr_mamba2_args *a) {
    if (validate_mamba2(a) != SR_OK) return 0;
    return kWsHeader + mamba2_scratch_bytes(*a);
}

sr_status sr_mamba2_replay(const sr_mamba2_args *a, void *ws, size_t ws_bytes, void *stream) {
    if (sr_status s = validate_mamba2(a)) return s;
    const size_t need = kWsHeader + mamba2_scratch_bytes(*a);
    if (sr_status s = check_workspace(ws, ws_bytes, need)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t *status = static_cast<uint32_t *>(ws);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return cuda_error(e, "sr_mamba2_replay: clearing the status word");
    e = mamba2_replay(*a, status, static_cast<char *>(ws) + kWsHeader, st);
    if (e != cudaSuccess) return cuda_error(e, "sr_mamba2_replay: kernel launch");
    return SR_OK;
}

sr_status sr_prepare_lo8_weights(const void *w, void *w_lo8, int64_t n, void *stream) {
    if (n < 0) return set_error(SR_ERR_INVALID_ARG, "n must be >= 0");
    if (n > 0 && (!w || !w_lo8)) return set_error(SR_ERR_INVALID_ARG, "w and w_lo8 are required");
    if (n == 0) return SR_OK;
    cudaError_t e = prepare_lo8(w, w_lo8, n, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_error(e, "sr_prepare_lo8_weights");
    return SR_OK;
}

sr_status sr_device_status(const void *ws, void *stream, uint32_t *flags) {
    if (!ws || !flags) return set_error(SR_ERR_INVALID_ARG, "workspace and flags are required");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_error(e, "sr_device_status");
    *flags = v;
    if (v) return set_error(SR_ERR_DEVICE, "device status flags 0x%x", v);
    return SR_OK;
}

}  // extern "C"

#include "sr/sr_testing.h"

extern "C" sr_status sr_test_gemm(const void *a, const void *b0, const void *b1, void *c, const void *r,
                                  int32_t m, int32_t n, int32_t k, int32_t epi, int32_t form, void *ws,
                                  size_t ws_bytes, void *stream) {
    if (!a || !b0 || !c || (epi == EPI_SWIGLU && !b1) || (epi == EPI_RESIDUAL && !r))
        return set_error(SR_ERR_INVALID_ARG, "sr_test_gemm: missing operand");
    if (epi < 0 || epi > 2) return set_error(SR_ERR_INVALID_ARG, "sr_test_gemm: bad epilogue");
    if (form < 0 || form > 2) return set_error(SR_ERR_INVALID_ARG, "sr_test_gemm: bad form");
    if (m <= 0 || n <= 0 || k <= 0 || k % 64 || n % 32)
        return set_error(SR_ERR_UNSUPPORTED, "sr_test_gemm: need m, n, k > 0, k %% 64 == 0, n %% 32 == 0");
    if (sr_status s = check_workspace(ws, ws_bytes, kWsHeader)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t *status = static_cast<uint32_t *>(ws);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), st);
    GemmProblemDesc d{a, nullptr, b0, b1, c, r, nullptr, nullptr};
    GemmOptions opt;
    opt.form = form;
    if (e == cudaSuccess) e = gemm_tc(&d, 1, m, n, k, n, epi, 1, 0, status, st, opt);
    if (e != cudaSuccess) return cuda_error(e, "sr_test_gemm");
    return SR_OK;
}
