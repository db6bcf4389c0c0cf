// Chunked Mamba2 replay on tensor cores (bf16 operands, fp32 state).
//
// Recurrence ("SuffixReplay: Prefix Caching via Suffix Replay for Hybrid
// LLMs", Eq. 4, the per-head-decay instance with no erase term):
//     S_t = exp(dt_t A_h) S_{t-1} + dt_t x_t B_t^T,   y_t = S_t C_t.
// Inside a chunk of C tokens with gamma_t = sum_{r<=t} dt_r A_h (chunk
// relative) and entry state S_0:
//     y_t = sum_{s<=t} e^{gamma_t-gamma_s} dt_s (C_t . B_s) x_s + e^{gamma_t} S_0 C_t
//     S_C = e^{gamma_C} S_0 + sum_s dt_s e^{gamma_C-gamma_s} x_s B_s^T.
// With one B/C group (G = 1) the token-token product G = C B^T is shared by
// every head: a CTA takes one sequence and two heads, computes G once per
// chunk and applies each head's decay mask to it.  The written operand
// X diag(dt e^{gamma_C-gamma}) of the state update is an exact hi + lo bf16
// pair (x and B are exact bf16 inputs, so the state tracks fp32 arithmetic).
// Exponentials only ever see differences gamma_t - gamma_s with s <= t.
#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace sr {

namespace {

using namespace ms;

constexpr int C = 64;          // tokens per chunk
constexpr int P = 64;          // head dim
constexpr int NS = 128;        // state dim
constexpr int ROWN = NS + 8;   // bf16 row pitch of [*, 128] tiles (272 B)
constexpr int ROWX = P + 8;    // bf16 row pitch of [*, 64] tiles (144 B)
constexpr int ROWG = C + 4;    // fp32 row pitch of G (272 B)
constexpr int kThreads = 256;  // two heads x four warps

struct M2Smem {
    __nv_bfloat16 cm[2][C * ROWN];     // C of the chunk, double-buffered
    __nv_bfloat16 bm[2][C * ROWN];     // B of the chunk
    __nv_bfloat16 x[2][2][C * ROWX];   // [buffer][head] x of the chunk
    float g[C * ROWG];                 // G = C B^T
    __nv_bfloat16 gh[2][C * ROWX];     // [head] masked, decayed, dt-scaled G
    __nv_bfloat16 xwh[2][C * ROWX];    // [head] x diag(w), hi part
    __nv_bfloat16 xwl[2][C * ROWX];    // [head] lo part
    __nv_bfloat16 sb[2][P * ROWN];     // [head] bf16 state entering the chunk
    float gam[2][C];
    float dt[2][C];
};

__device__ __forceinline__ void bar_group(int id) {  // 128-thread named barrier of one head
    asm volatile("bar.sync %0, 128;\n" ::"r"(id) : "memory");
}

__global__ void __launch_bounds__(kThreads)
mamba2_chunk_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ Bg,
                    const __nv_bfloat16 *__restrict__ Cg, const float *__restrict__ dt,
                    const float *__restrict__ A, const int32_t *__restrict__ cu,
                    const float *__restrict__ h0, __nv_bfloat16 *__restrict__ y,
                    float *__restrict__ s_out, int total, int max_len, int H, uint32_t *status) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    M2Smem &sm = *reinterpret_cast<M2Smem *>(smem_raw);
    const int n = longest_first(cu, gridDim.y, blockIdx.y, reinterpret_cast<int *>(sm.g));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hh = warp >> 2, wq = warp & 3;  // head of the pair, warp within the head
    const int tid_h = tid & 127;
    const int h = 2 * blockIdx.x + hh;
    const int grp = lane >> 2, qd = lane & 3;
    int bos, eos;
    if (!seq_bounds(cu, n, total, max_len, status, bos, eos)) return;
    const int len = eos - bos;
    const int nchunks = (len + C - 1) / C;
    const float Ah = A[h];

    auto stage = [&](int c, int b) {
        // B, C: 64 rows x 256 B; x: 2 heads x 64 rows x 128 B
        for (int e = tid; e < C * 16; e += kThreads) {
            const int r = e >> 4, sg = e & 15;
            const int t = c * C + r;
            const bool ok = t < len;
            const size_t tt = size_t(bos) + (ok ? size_t(t) : 0);
            cp_async16(smem_u32(&sm.cm[b][r * ROWN + sg * 8]), Cg + tt * NS + sg * 8, ok);
            cp_async16(smem_u32(&sm.bm[b][r * ROWN + sg * 8]), Bg + tt * NS + sg * 8, ok);
        }
        for (int e = tid; e < 2 * C * 8; e += kThreads) {
            const int hd = e >> 9, r = (e >> 3) & 63, sg = e & 7;
            const int t = c * C + r;
            const bool ok = t < len;
            const size_t tt = size_t(bos) + (ok ? size_t(t) : 0);
            cp_async16(smem_u32(&sm.x[b][hd][r * ROWX + sg * 8]),
                       x + (tt * H + 2 * blockIdx.x + hd) * P + sg * 8, ok);
        }
        cp_async_commit();
    };

    // ---- state rows of this warp: p = 16 wq .. 16 wq + 15 of head h, all NS columns
    float S[NS / 8][4];
    const size_t sbase = (size_t(n) * H + h) * P * NS;
    {
        const int r0 = wq * 16 + grp;
#pragma unroll
        for (int j = 0; j < NS / 8; ++j) {
            const int c0 = j * 8 + 2 * qd;
            if (h0) {
                const float2 a = *reinterpret_cast<const float2 *>(h0 + sbase + size_t(r0) * NS + c0);
                const float2 b = *reinterpret_cast<const float2 *>(h0 + sbase + size_t(r0 + 8) * NS + c0);
                S[j][0] = a.x; S[j][1] = a.y; S[j][2] = b.x; S[j][3] = b.y;
            } else {
                S[j][0] = S[j][1] = S[j][2] = S[j][3] = 0.f;
            }
            *reinterpret_cast<uint32_t *>(&sm.sb[hh][r0 * ROWN + c0]) = pack_bf16(S[j][0], S[j][1]);
            *reinterpret_cast<uint32_t *>(&sm.sb[hh][(r0 + 8) * ROWN + c0]) = pack_bf16(S[j][2], S[j][3]);
        }
    }
    // dt of the next chunk: thread tid < 128 holds token (tid & 63) of head (tid >> 6)
    const int dh = (tid >> 6) & 1, dtok = tid & 63;
    float dt_next = 0.f;
    if (nchunks > 0) {
        stage(0, 0);
        if (tid < 128 && dtok < len) dt_next = dt[(size_t(bos) + dtok) * H + 2 * blockIdx.x + dh];
    }

    for (int c = 0; c < nchunks; ++c) {
        const int cur = c & 1;
        const int clen = min(C, len - c * C);
        if (tid < 128) sm.dt[dh][dtok] = dt_next;
        cp_async_wait_all();
        __syncthreads();
        if (wq == 0) {  // one warp per head: gamma = inclusive prefix sum of dt A
            const float a0 = sm.dt[hh][2 * lane] * Ah, a1 = sm.dt[hh][2 * lane + 1] * Ah;
            float incl = a0 + a1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            const float excl = incl - (a0 + a1);
            sm.gam[hh][2 * lane] = excl + a0;
            sm.gam[hh][2 * lane + 1] = excl + a0 + a1;
        }
        if (c + 1 < nchunks) {
            stage(c + 1, cur ^ 1);
            const int t = (c + 1) * C + dtok;
            dt_next = (tid < 128 && t < len) ? dt[(size_t(bos) + t) * H + 2 * blockIdx.x + dh] : 0.f;
        }
        __syncthreads();
        const float *gam = sm.gam[hh];
        const float gC = gam[C - 1];

        // ---- G = C B^T (shared by both heads): warp -> rows 16 (w & 3), columns 32 (w >> 2)
        {
            const int mb = warp & 3, n0 = (warp >> 2) * 32;
            float acc[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < NS / 16; ++kk) {
                uint32_t a[4];
                ldsm_x4(a, smem_u32(&sm.cm[cur][(mb * 16 + (lane & 15)) * ROWN + kk * 16 + (lane >> 4) * 8]));
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    uint32_t b[4];
                    const int brow = n0 + np * 16 + (lane & 7) + 8 * (lane >> 4);
                    ldsm_x4(b, smem_u32(&sm.bm[cur][brow * ROWN + kk * 16 + 8 * ((lane >> 3) & 1)]));
                    mma16816(acc[2 * np], a, b[0], b[1]);
                    mma16816(acc[2 * np + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = mb * 16 + grp, s = n0 + j * 8 + 2 * qd;
                *reinterpret_cast<float2 *>(&sm.g[t * ROWG + s]) = make_float2(acc[j][0], acc[j][1]);
                *reinterpret_cast<float2 *>(&sm.g[(t + 8) * ROWG + s]) = make_float2(acc[j][2], acc[j][3]);
            }
        }
        // ---- x diag(dt_s e^{gamma_C - gamma_s}) as hi + lo (per head; 32 values per thread)
        {
            const int s = tid_h >> 1, p0 = (tid_h & 1) * 32;
            const float w = sm.dt[hh][s] * __expf(gC - gam[s]);
            const __nv_bfloat16 *xr = &sm.x[cur][hh][s * ROWX + p0];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const uint4 u = *reinterpret_cast<const uint4 *>(xr + v * 8);
                const __nv_bfloat162 *x2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(x2[e]);
                    split_bf16(f.x * w, f.y * w, hi[e], lo[e]);
                }
                *reinterpret_cast<uint4 *>(&sm.xwh[hh][s * ROWX + p0 + v * 8]) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(&sm.xwl[hh][s * ROWX + p0 + v * 8]) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        }
        __syncthreads();

        // ---- G~_ts = G_ts e^{gamma_t - gamma_s} dt_s for s <= t (per head, 32 values per thread)
        {
            const int t = tid_h >> 1, s0 = (tid_h & 1) * 32;
            const float gt = gam[t];
#pragma unroll
            for (int v = 0; v < 32; v += 2) {
                const int s = s0 + v;
                const float2 gg = *reinterpret_cast<const float2 *>(&sm.g[t * ROWG + s]);
                const float e0 = __expf(s <= t ? gt - gam[s] : -INFINITY) * sm.dt[hh][s];
                const float e1 = __expf(s + 1 <= t ? gt - gam[s + 1] : -INFINITY) * sm.dt[hh][s + 1];
                *reinterpret_cast<uint32_t *>(&sm.gh[hh][t * ROWX + s]) = pack_bf16(gg.x * e0, gg.y * e1);
            }
        }
        bar_group(1 + hh);

        // ---- y = G~ x + e^{gamma_t} C S_0^T   (warp wq: tokens 16 wq .. 16 wq + 15, all 64 p)
        if (y) {
            float acc[P / 8][4], acc2[P / 8][4];
#pragma unroll
            for (int j = 0; j < P / 8; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[j][e] = acc2[j][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                uint32_t a[4];
                ldsm_x4(a, smem_u32(&sm.gh[hh][(wq * 16 + (lane & 15)) * ROWX + kk * 16 + (lane >> 4) * 8]));
#pragma unroll
                for (int np = 0; np < P / 16; ++np) {
                    uint32_t b[4];
                    const int brow = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                    ldsm_x4_t(b, smem_u32(&sm.x[cur][hh][brow * ROWX + np * 16 + 8 * (lane >> 4)]));
                    mma16816(acc[2 * np], a, b[0], b[1]);
                    mma16816(acc[2 * np + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int kk = 0; kk < NS / 16; ++kk) {
                uint32_t a[4];
                ldsm_x4(a, smem_u32(&sm.cm[cur][(wq * 16 + (lane & 15)) * ROWN + kk * 16 + (lane >> 4) * 8]));
#pragma unroll
                for (int np = 0; np < P / 16; ++np) {
                    uint32_t b[4];
                    const int brow = np * 16 + (lane & 7) + 8 * (lane >> 4);
                    ldsm_x4(b, smem_u32(&sm.sb[hh][brow * ROWN + kk * 16 + 8 * ((lane >> 3) & 1)]));
                    mma16816(acc2[2 * np], a, b[0], b[1]);
                    mma16816(acc2[2 * np + 1], a, b[2], b[3]);
                }
            }
            const int t = wq * 16 + grp;
            const float f0 = __expf(gam[t]), f1 = __expf(gam[t + 8]);
            const size_t tok = size_t(bos) + size_t(c) * C;
#pragma unroll
            for (int j = 0; j < P / 8; ++j) {
                const int p = j * 8 + 2 * qd;
                if (t < clen)
                    *reinterpret_cast<uint32_t *>(y + ((tok + t) * H + h) * P + p) =
                        pack_bf16(acc[j][0] + f0 * acc2[j][0], acc[j][1] + f0 * acc2[j][1]);
                if (t + 8 < clen)
                    *reinterpret_cast<uint32_t *>(y + ((tok + t + 8) * H + h) * P + p) =
                        pack_bf16(acc[j][2] + f1 * acc2[j][2], acc[j][3] + f1 * acc2[j][3]);
            }
        }
        bar_group(1 + hh);  // sb of this head is no longer read

        // ---- S_C = e^{gamma_C} S_0 + (x diag(w))^T B   (warp wq: state rows p = 16 wq .. 16 wq + 15)
        {
            const float fC = __expf(gC);
#pragma unroll
            for (int j = 0; j < NS / 8; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) S[j][e] *= fC;
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                uint32_t ah[4], al[4];
                const int arow = kk * 16 + (lane & 7) + 8 * (lane >> 4);
                const int acol = wq * 16 + 8 * ((lane >> 3) & 1);
                ldsm_x4_t(ah, smem_u32(&sm.xwh[hh][arow * ROWX + acol]));
                ldsm_x4_t(al, smem_u32(&sm.xwl[hh][arow * ROWX + acol]));
#pragma unroll
                for (int np = 0; np < NS / 16; ++np) {
                    uint32_t b[4];
                    const int brow = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                    ldsm_x4_t(b, smem_u32(&sm.bm[cur][brow * ROWN + np * 16 + 8 * (lane >> 4)]));
                    mma16816(S[2 * np], ah, b[0], b[1]);
                    mma16816(S[2 * np + 1], ah, b[2], b[3]);
                    mma16816(S[2 * np], al, b[0], b[1]);
                    mma16816(S[2 * np + 1], al, b[2], b[3]);
                }
            }
            const int r0 = wq * 16 + grp;
#pragma unroll
            for (int j = 0; j < NS / 8; ++j) {
                const int c0 = j * 8 + 2 * qd;
                *reinterpret_cast<uint32_t *>(&sm.sb[hh][r0 * ROWN + c0]) = pack_bf16(S[j][0], S[j][1]);
                *reinterpret_cast<uint32_t *>(&sm.sb[hh][(r0 + 8) * ROWN + c0]) = pack_bf16(S[j][2], S[j][3]);
            }
        }
        __syncthreads();
    }

    {
        const int r0 = wq * 16 + grp;
#pragma unroll
        for (int j = 0; j < NS / 8; ++j) {
            const int c0 = j * 8 + 2 * qd;
            *reinterpret_cast<float2 *>(s_out + sbase + size_t(r0) * NS + c0) = make_float2(S[j][0], S[j][1]);
            *reinterpret_cast<float2 *>(s_out + sbase + size_t(r0 + 8) * NS + c0) = make_float2(S[j][2], S[j][3]);
        }
    }
}

}  // namespace

size_t mamba2_scratch_bytes(const sr_mamba2_args &) { return 0; }

// The tcgen05 chunk kernel (or, on request, this mma.sync one) for one B/C
// group and an even head count; the fp32 token-by-token kernel otherwise.
cudaError_t mamba2_replay(const sr_mamba2_args &a, uint32_t *status, void *, cudaStream_t st) {
    if (a.n_seqs == 0) return cudaSuccess;
    const bool chunk_ok = a.n_groups == 1 && a.n_heads % 2 == 0;
    int algo = a.algo;
    if (algo == SR_MAMBA2_AUTO) algo = chunk_ok ? SR_MAMBA2_TCGEN05 : SR_MAMBA2_SEQUENTIAL;
    if (algo == SR_MAMBA2_SEQUENTIAL || a.total_tokens == 0) return mamba2_sequential(a, status, st);
    if (!chunk_ok) return cudaErrorInvalidValue;
    if (algo == SR_MAMBA2_TCGEN05) return mamba2_tc(a, status, st);
    const int smem = int(sizeof(M2Smem));
    cudaError_t e = cudaFuncSetAttribute(mamba2_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.n_heads / 2, a.n_seqs);
    mamba2_chunk_kernel<<<grid, kThreads, smem, st>>>(
        static_cast<const __nv_bfloat16 *>(a.x), static_cast<const __nv_bfloat16 *>(a.B),
        static_cast<const __nv_bfloat16 *>(a.C), a.dt, a.A, a.cu_seqlens, a.h0, static_cast<__nv_bfloat16 *>(a.y),
        a.s_out, a.total_tokens, a.max_seqlen, a.n_heads, status);
    return cudaGetLastError();
}

}  // namespace sr
