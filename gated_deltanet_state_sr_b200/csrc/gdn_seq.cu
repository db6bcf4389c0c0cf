// Token-by-token Gated DeltaNet replay in fp32 (FFMA).
//
// The exact-order form of the recurrence
//     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
// ("Tail-Replay: Escaping the Curse of Linear Attention in Prefix Caching for
// Hybrid LLMs", Sec. 2; "SuffixReplay", Eq. 4), evaluated as
//     u = beta (v - alpha S k),  S <- alpha S + u k^T,  o = scale S q.
// Rows of S evolve independently (row i only reads v_i), so the d_v rows are
// split across threads and CTAs: each thread keeps one full row of S (d_k
// fp32 values) in registers; k_t and q_t are staged in shared memory in
// batches of kTokBatch tokens and read by broadcast.  This kernel serves the
// fp32-input mode and is the accuracy reference for the chunked kernel.
#include "common.cuh"

namespace sr {

namespace {

constexpr int kRows = 64;      // rows of S per CTA (one per thread)
constexpr int kTokBatch = 16;  // tokens staged per shared-memory batch

template <int DK, typename Tin>
__global__ void __launch_bounds__(kRows)
gdn_token_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                 const float *__restrict__ g, const float *__restrict__ beta,
                 const int32_t *__restrict__ cu, const float *__restrict__ h0,
                 Tin *__restrict__ o, float *__restrict__ s_out, int total, int max_len,
                 int h_k, int h_v, int d_v, float scale, uint32_t *status) {
    const int n = blockIdx.z, h = blockIdx.y;
    const int row = blockIdx.x * kRows + threadIdx.x;
    const int hk = h / (h_v / h_k);
    int bos, eos;
    if (!seq_bounds(cu, n, total, max_len, status, bos, eos)) return;

    __shared__ __align__(16) float s_k[kTokBatch][DK];
    __shared__ __align__(16) float s_q[kTokBatch][DK];
    __shared__ float s_a[kTokBatch], s_b[kTokBatch];

    float S[DK];
    const size_t srow = ((size_t(n) * h_v + h) * d_v + row) * DK;
    if (h0) {
#pragma unroll
        for (int j = 0; j < DK; j += 4) {
            float4 t = *reinterpret_cast<const float4 *>(h0 + srow + j);
            S[j] = t.x; S[j + 1] = t.y; S[j + 2] = t.z; S[j + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < DK; ++j) S[j] = 0.f;
    }

    for (int t0 = bos; t0 < eos; t0 += kTokBatch) {
        const int nt = min(kTokBatch, eos - t0);
        __syncthreads();
        for (int e = threadIdx.x; e < nt * DK; e += kRows) {
            const int tt = e / DK, j = e % DK;
            const size_t off = (size_t(t0 + tt) * h_k + hk) * DK + j;
            s_k[tt][j] = to_f32(k[off]);
            s_q[tt][j] = to_f32(q[off]);
        }
        if (threadIdx.x < nt) {
            const size_t off = size_t(t0 + threadIdx.x) * h_v + h;
            s_a[threadIdx.x] = expf(g[off]);
            s_b[threadIdx.x] = beta[off];
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const size_t tok = size_t(t0 + tt) * h_v + h;
            const float vi = to_f32(v[tok * d_v + row]);
            const float a = s_a[tt], b = s_b[tt];
            float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
            for (int j = 0; j < DK; j += 4) {
                const float4 kk = *reinterpret_cast<const float4 *>(&s_k[tt][j]);
                p0 = fmaf(S[j], kk.x, p0);
                p1 = fmaf(S[j + 1], kk.y, p1);
                p2 = fmaf(S[j + 2], kk.z, p2);
                p3 = fmaf(S[j + 3], kk.w, p3);
            }
            const float u = b * (vi - a * ((p0 + p1) + (p2 + p3)));
#pragma unroll
            for (int j = 0; j < DK; j += 4) {
                const float4 kk = *reinterpret_cast<const float4 *>(&s_k[tt][j]);
                S[j] = fmaf(u, kk.x, a * S[j]);
                S[j + 1] = fmaf(u, kk.y, a * S[j + 1]);
                S[j + 2] = fmaf(u, kk.z, a * S[j + 2]);
                S[j + 3] = fmaf(u, kk.w, a * S[j + 3]);
            }
            if (o) {
                float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
#pragma unroll
                for (int j = 0; j < DK; j += 4) {
                    const float4 qq = *reinterpret_cast<const float4 *>(&s_q[tt][j]);
                    r0 = fmaf(S[j], qq.x, r0);
                    r1 = fmaf(S[j + 1], qq.y, r1);
                    r2 = fmaf(S[j + 2], qq.z, r2);
                    r3 = fmaf(S[j + 3], qq.w, r3);
                }
                o[tok * d_v + row] = from_f32<Tin>(scale * ((r0 + r1) + (r2 + r3)));
            }
        }
    }
#pragma unroll
    for (int j = 0; j < DK; j += 4)
        *reinterpret_cast<float4 *>(s_out + srow + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
}

template <int DK, typename Tin>
cudaError_t launch(const sr_gdn_args &a, float scale, uint32_t *status, cudaStream_t st) {
    dim3 grid(a.d_v / kRows, a.h_v, a.n_seqs);
    gdn_token_kernel<DK, Tin><<<grid, kRows, 0, st>>>(
        static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k), static_cast<const Tin *>(a.v),
        a.g, a.beta, a.cu_seqlens, a.h0, static_cast<Tin *>(a.o), a.s_out, a.total_tokens,
        a.max_seqlen, a.h_k, a.h_v, a.d_v, scale, status);
    return cudaGetLastError();
}

}  // namespace

// Host launcher: shapes were validated by the caller (d_k = d_v in {64,128}).
cudaError_t gdn_sequential(const sr_gdn_args &a, float scale, uint32_t *status, cudaStream_t st) {
    if (a.n_seqs == 0) return cudaSuccess;
    if (a.dtype == SR_FP32)
        return a.d_k == 64 ? launch<64, float>(a, scale, status, st)
                           : launch<128, float>(a, scale, status, st);
    return a.d_k == 64 ? launch<64, __nv_bfloat16>(a, scale, status, st)
                       : launch<128, __nv_bfloat16>(a, scale, status, st);
}

}  // namespace sr
