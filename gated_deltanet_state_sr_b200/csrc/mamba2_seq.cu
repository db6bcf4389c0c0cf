// Token-by-token Mamba2 replay in fp32 (FFMA).
//
//     S_t = exp(dt_t A_h) S_{t-1} + dt_t x_t B_t^T,   y_t = S_t C_t
// ("SuffixReplay: Prefix Caching via Suffix Replay for Hybrid LLMs", Eq. 4,
// the per-head-decay instance with no erase term).  One thread per row p of
// the P x N_s state; B_t and C_t are staged in shared memory per batch of
// tokens and read by broadcast.  Accuracy reference for the chunked kernel.
#include "common.cuh"

namespace sr {

namespace {

constexpr int kTokBatch = 16;

template <int P, int NS>
__global__ void __launch_bounds__(P)
mamba2_seq_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ B,
                  const __nv_bfloat16 *__restrict__ C, const float *__restrict__ dt,
                  const float *__restrict__ A, const int32_t *__restrict__ cu,
                  const float *__restrict__ h0, __nv_bfloat16 *__restrict__ y,
                  float *__restrict__ s_out, int total, int max_len, int H, int G,
                  uint32_t *status) {
    const int n = blockIdx.y, h = blockIdx.x, p = threadIdx.x;
    const int gi = h / (H / G);
    int bos, eos;
    if (!seq_bounds(cu, n, total, max_len, status, bos, eos)) return;

    __shared__ __align__(16) float s_B[kTokBatch][NS];
    __shared__ __align__(16) float s_C[kTokBatch][NS];
    __shared__ float s_a[kTokBatch], s_d[kTokBatch];

    float S[NS];
    const size_t srow = ((size_t(n) * H + h) * P + p) * NS;
#pragma unroll
    for (int j = 0; j < NS; ++j) S[j] = h0 ? h0[srow + j] : 0.f;
    const float Ah = A[h];

    for (int t0 = bos; t0 < eos; t0 += kTokBatch) {
        const int nt = min(kTokBatch, eos - t0);
        __syncthreads();
        for (int e = threadIdx.x; e < nt * NS; e += P) {
            const int tt = e / NS, j = e % NS;
            const size_t off = (size_t(t0 + tt) * G + gi) * NS + j;
            s_B[tt][j] = __bfloat162float(B[off]);
            s_C[tt][j] = __bfloat162float(C[off]);
        }
        if (threadIdx.x < nt) {
            const float d = dt[size_t(t0 + threadIdx.x) * H + h];
            s_d[threadIdx.x] = d;
            s_a[threadIdx.x] = expf(d * Ah);
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const size_t tok = size_t(t0 + tt) * H + h;
            const float w = s_d[tt] * __bfloat162float(x[tok * P + p]);
            const float a = s_a[tt];
            float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
#pragma unroll
            for (int j = 0; j < NS; j += 4) {
                const float4 bb = *reinterpret_cast<const float4 *>(&s_B[tt][j]);
                const float4 cc = *reinterpret_cast<const float4 *>(&s_C[tt][j]);
                S[j] = fmaf(w, bb.x, a * S[j]);
                S[j + 1] = fmaf(w, bb.y, a * S[j + 1]);
                S[j + 2] = fmaf(w, bb.z, a * S[j + 2]);
                S[j + 3] = fmaf(w, bb.w, a * S[j + 3]);
                r0 = fmaf(S[j], cc.x, r0);
                r1 = fmaf(S[j + 1], cc.y, r1);
                r2 = fmaf(S[j + 2], cc.z, r2);
                r3 = fmaf(S[j + 3], cc.w, r3);
            }
            if (y) y[tok * P + p] = __float2bfloat16_rn((r0 + r1) + (r2 + r3));
        }
    }
#pragma unroll
    for (int j = 0; j < NS; j += 4)
        *reinterpret_cast<float4 *>(s_out + srow + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
}

}  // namespace

cudaError_t mamba2_sequential(const sr_mamba2_args &a, uint32_t *status, cudaStream_t st) {
    if (a.n_seqs == 0) return cudaSuccess;
    dim3 grid(a.n_heads, a.n_seqs);
    mamba2_seq_kernel<64, 128><<<grid, 64, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(a.x), static_cast<const __nv_bfloat16 *>(a.B),
        static_cast<const __nv_bfloat16 *>(a.C), a.dt, a.A, a.cu_seqlens, a.h0,
        static_cast<__nv_bfloat16 *>(a.y), a.s_out, a.total_tokens, a.max_seqlen, a.n_heads,
        a.n_groups, status);
    return cudaGetLastError();
}

}  // namespace sr
