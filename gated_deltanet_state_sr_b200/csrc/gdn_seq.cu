// Token-by-token Gated DeltaNet replay in fp32 (FFMA).
//
// The exact-order form of the recurrence
//     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
// ("Tail-Replay: Escaping the Curse of Linear Attention in Prefix Caching for
// Hybrid LLMs", Sec. 2; "SuffixReplay", Eq. 4), evaluated as
//     u = beta (v - alpha S k),  S <- alpha S + u k^T,  o = scale S q.
// Rows of S evolve independently (row i only reads v_i), so the d_v rows are
// split across CTAs, and each row across kSplit threads: thread (row, part)
// keeps the row's columns 16 i + 4 part .. + 3 (i = 0 .. d_k / 16 - 1) of S in
// registers, so that the row's kSplit threads read one contiguous 64-byte run
// of k_t or q_t per step (a broadcast, free of bank conflicts); the two dot
// products per token close with two shuffles.  k_t, q_t, v_t and the gates are
// staged in shared memory in batches of kTokBatch tokens.  This kernel serves
// the fp32-input mode and is the accuracy reference for the chunked kernel.
#include "common.cuh"

namespace sr {

namespace {

constexpr int kRows = 64;      // rows of S per CTA
constexpr int kSplit = 4;      // threads per row
constexpr int kThreadsTok = kRows * kSplit;
constexpr int kTokBatch = 16;  // tokens staged per shared-memory batch

// four consecutive inputs as fp32
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

template <int DK, typename Tin>
__global__ void __launch_bounds__(kThreadsTok, 3)
gdn_token_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                 const float *__restrict__ g, const float *__restrict__ beta,
                 const int32_t *__restrict__ cu, const float *__restrict__ h0,
                 Tin *__restrict__ o, float *__restrict__ s_out, int total, int max_len,
                 int h_k, int h_v, int d_v, float scale, uint32_t *status) {
    constexpr int NJ = DK / 16;  // float4 groups of a thread's columns
    __shared__ int s_rank[kLongestFirstMax + 1];
    // z-slices are dispatched in order: the longest sequences start first
    const int n = longest_first(cu, gridDim.z, blockIdx.z, s_rank), h = blockIdx.y;
    const int rl = threadIdx.x / kSplit, part = threadIdx.x % kSplit;
    const int row0 = blockIdx.x * kRows, row = row0 + rl;
    const int hk = h / (h_v / h_k);
    int bos, eos;
    if (!seq_bounds(cu, n, total, max_len, status, bos, eos)) return;

    __shared__ __align__(16) float s_k[kTokBatch][DK];
    __shared__ __align__(16) float s_q[kTokBatch][DK];
    __shared__ __align__(16) float s_v[kTokBatch][kRows];
    __shared__ float s_a[kTokBatch], s_b[kTokBatch];

    float S[4 * NJ];  // S[4 i + e] = S[row][16 i + 4 part + e]
    const size_t srow = ((size_t(n) * h_v + h) * d_v + row) * DK;
#pragma unroll
    for (int i = 0; i < NJ; ++i) {
        const float4 t = h0 ? *reinterpret_cast<const float4 *>(h0 + srow + 16 * i + 4 * part)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        S[4 * i] = t.x; S[4 * i + 1] = t.y; S[4 * i + 2] = t.z; S[4 * i + 3] = t.w;
    }

    // The next batch's k, q, v and gates are loaded into registers while the
    // current batch runs, then staged between two block barriers.
    constexpr int KQ = (kTokBatch * DK / 4 + kThreadsTok - 1) / kThreadsTok;  // float4 of k (and of q) per thread
    constexpr int VV = (kTokBatch * kRows / 4 + kThreadsTok - 1) / kThreadsTok;
    float4 rk[KQ], rq[KQ], rv[VV];
    float ra = 0.f, rb = 0.f;
    auto fetch = [&](int t0) {
        const int nt = min(kTokBatch, eos - t0);
#pragma unroll
        for (int m = 0; m < KQ; ++m) {
            const int e = threadIdx.x + m * kThreadsTok;
            if (e < nt * DK / 4) {
                const int tt = (4 * e) / DK, j = (4 * e) % DK;
                const size_t off = (size_t(t0 + tt) * h_k + hk) * DK + j;
                rk[m] = load4(k + off);
                rq[m] = load4(q + off);
            }
        }
#pragma unroll
        for (int m = 0; m < VV; ++m) {
            const int e = threadIdx.x + m * kThreadsTok;
            if (e < nt * kRows / 4) {
                const int tt = (4 * e) / kRows, r = (4 * e) % kRows;
                rv[m] = load4(v + (size_t(t0 + tt) * h_v + h) * d_v + row0 + r);
            }
        }
        if (threadIdx.x < nt) {
            const size_t off = size_t(t0 + threadIdx.x) * h_v + h;
            ra = g[off];
            rb = beta[off];
        }
    };
    auto stage = [&](int t0) {
        const int nt = min(kTokBatch, eos - t0);
#pragma unroll
        for (int m = 0; m < KQ; ++m) {
            const int e = threadIdx.x + m * kThreadsTok;
            if (e < nt * DK / 4) {
                const int tt = (4 * e) / DK, j = (4 * e) % DK;
                *reinterpret_cast<float4 *>(&s_k[tt][j]) = rk[m];
                *reinterpret_cast<float4 *>(&s_q[tt][j]) = rq[m];
            }
        }
#pragma unroll
        for (int m = 0; m < VV; ++m) {
            const int e = threadIdx.x + m * kThreadsTok;
            if (e < nt * kRows / 4) {
                const int tt = (4 * e) / kRows, r = (4 * e) % kRows;
                *reinterpret_cast<float4 *>(&s_v[tt][r]) = rv[m];
            }
        }
        if (threadIdx.x < nt) {
            s_a[threadIdx.x] = expf(ra);
            s_b[threadIdx.x] = rb;
        }
    };
    if (bos < eos) fetch(bos);
    for (int t0 = bos; t0 < eos; t0 += kTokBatch) {
        const int nt = min(kTokBatch, eos - t0);
        __syncthreads();  // the previous batch's tokens are done with the staging buffers
        stage(t0);
        __syncthreads();
        if (t0 + kTokBatch < eos) fetch(t0 + kTokBatch);
        for (int tt = 0; tt < nt; ++tt) {
            const float a = s_a[tt], b = s_b[tt], vi = s_v[tt][rl];
            float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
            for (int i = 0; i < NJ; ++i) {
                const float4 kk = *reinterpret_cast<const float4 *>(&s_k[tt][16 * i + 4 * part]);
                p0 = fmaf(S[4 * i], kk.x, p0);
                p1 = fmaf(S[4 * i + 1], kk.y, p1);
                p2 = fmaf(S[4 * i + 2], kk.z, p2);
                p3 = fmaf(S[4 * i + 3], kk.w, p3);
            }
            float pk = (p0 + p1) + (p2 + p3);
            pk += __shfl_xor_sync(0xffffffffu, pk, 1);
            pk += __shfl_xor_sync(0xffffffffu, pk, 2);
            const float u = b * (vi - a * pk);
#pragma unroll
            for (int i = 0; i < NJ; ++i) {
                const float4 kk = *reinterpret_cast<const float4 *>(&s_k[tt][16 * i + 4 * part]);
                S[4 * i] = fmaf(u, kk.x, a * S[4 * i]);
                S[4 * i + 1] = fmaf(u, kk.y, a * S[4 * i + 1]);
                S[4 * i + 2] = fmaf(u, kk.z, a * S[4 * i + 2]);
                S[4 * i + 3] = fmaf(u, kk.w, a * S[4 * i + 3]);
            }
            if (o) {
                float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
#pragma unroll
                for (int i = 0; i < NJ; ++i) {
                    const float4 qq = *reinterpret_cast<const float4 *>(&s_q[tt][16 * i + 4 * part]);
                    r0 = fmaf(S[4 * i], qq.x, r0);
                    r1 = fmaf(S[4 * i + 1], qq.y, r1);
                    r2 = fmaf(S[4 * i + 2], qq.z, r2);
                    r3 = fmaf(S[4 * i + 3], qq.w, r3);
                }
                float pq = (r0 + r1) + (r2 + r3);
                pq += __shfl_xor_sync(0xffffffffu, pq, 1);
                pq += __shfl_xor_sync(0xffffffffu, pq, 2);
                if (part == 0) o[(size_t(t0 + tt) * h_v + h) * d_v + row] = from_f32<Tin>(scale * pq);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NJ; ++i)
        *reinterpret_cast<float4 *>(s_out + srow + 16 * i + 4 * part) =
            make_float4(S[4 * i], S[4 * i + 1], S[4 * i + 2], S[4 * i + 3]);
}

template <int DK, typename Tin>
cudaError_t launch(const sr_gdn_args &a, float scale, uint32_t *status, cudaStream_t st) {
    dim3 grid(a.d_v / kRows, a.h_v, a.n_seqs);
    gdn_token_kernel<DK, Tin><<<grid, kThreadsTok, 0, st>>>(
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
