// Chunked gated-delta replay on tensor cores (bf16 operands, fp32 state).
//
// Recurrence ("Tail-Replay: Escaping the Curse of Linear Attention in Prefix
// Caching for Hybrid LLMs", Sec. 2; "SuffixReplay", Eq. 4):
//     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = scale S_t q_t.
// Write S_t = alpha_t S_{t-1} + u_t k_t^T with u_t = beta_t (v_t - alpha_t S_{t-1} k_t).
// Inside a chunk of C tokens with log-decay prefix gamma_t = sum_{r<=t} g_r
// (relative to the chunk start) and entry state S_0, unrolling gives the
// lower-triangular system
//     (I + A) U = diag(beta) V - diag(beta e^gamma) K S_0^T,
//     A_ts = beta_t e^{gamma_t - gamma_s} (k_t . k_s)   for s < t,
// so with T = (I + A)^{-1}, W = T diag(beta e^gamma) K and Ut = T diag(beta) V:
//     U   = Ut - W S_0^T
//     O   = scale (diag(e^gamma) Q S_0^T + M U),  M_ts = e^{gamma_t-gamma_s} q_t.k_s, s <= t
//     S_C = e^{gamma_C} S_0 + U^T diag(e^{gamma_C - gamma}) K.
// Only differences gamma_t - gamma_s with s <= t are ever exponentiated (the
// exp argument is masked to -inf before the call), so strong decay underflows
// to zero instead of overflowing.
//
// One CTA per (group, sequence, V head) keeps the whole d_v x d_k fp32 state
// in mma.sync accumulator registers (warp w owns rows 16w..16w+15) and walks
// the sequence chunk by chunk.  q/k/v of the next chunk are prefetched with
// cp.async as soon as the current chunk's last reader of each buffer is done.
// (I + A)^{-1} is formed in fp32 on the CUDA cores: 16x16 diagonal blocks by
// forward substitution, then the off-diagonal blocks by block substitution.
//
// Precision: T diag(beta) and U enter the products that feed the state as
// exact hi + lo bf16 pairs (a CPU emulation of these rounding points puts the
// state error near 1e-4 of max|S|, against 3e-3 with plain bf16 operands).  With SPLIT, k and v also arrive as hi + lo pairs (the layer
// computes them in fp32) and every product that reaches the state uses the
// three-term expansion hi*hi + lo*hi + hi*lo.
#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace sr {

namespace {

using namespace ms;

constexpr int C = 64;        // tokens per chunk
constexpr int ROWP = C + 8;  // bf16 row pitch of C x C tiles (144 B)
constexpr int ROWA = C + 4;  // fp32 row pitch of C x C tiles (272 B)

// exp(gt - gs) for s <= t, else 0 (masked before the exponential).
__device__ __forceinline__ float decay(float gt, float gs, bool keep) {
    return __expf(keep ? gt - gs : -INFINITY);
}

template <int D, bool SPLIT>
struct Smem {
    static constexpr int ROW = D + 8;  // bf16 row pitch of C x D and D x D tiles
    __nv_bfloat16 k[C * ROW];
    __nv_bfloat16 q[C * ROW];
    __nv_bfloat16 v[C * ROW];
    __nv_bfloat16 kl[SPLIT ? C * ROW : 8];  // low parts of k, v (SPLIT)
    __nv_bfloat16 vl[SPLIT ? C * ROW : 8];
    __nv_bfloat16 sb[D * ROW];   // bf16 copy of the state entering the chunk
    __nv_bfloat16 p[C * ROWP];   // masked, decayed, scaled Q K^T
    // R1: A (fp32) during the solve, then -W (bf16)
    union { float a[C * ROWA]; __nv_bfloat16 w[C * ROW]; } r1;
    // R2: T (fp32) during the solve, then U (bf16)
    union { float t[C * ROWA]; __nv_bfloat16 u[C * ROW]; } r2;
    // R3: T diag(beta e^gamma) (bf16; it only meets the state through W, where
    // one rounding stays far inside the tolerance) and T diag(beta) as a hi + lo
    // bf16 pair, then U diag(e^{gamma_C-gamma}) as a hi + lo bf16 pair.
    union {
        struct { __nv_bfloat16 t1[C * ROWP], t2[C * ROWP], t2l[C * ROWP]; } s;
        struct { __nv_bfloat16 ud[C * ROW], udl[C * ROW]; } d;
    } r3;
    float gam[C];   // gamma_t, chunk-relative
    float beta[C];
};

template <int D, bool SPLIT>
__global__ void __launch_bounds__(D * 2)
gdn_chunk_kernel(const __grid_constant__ GdnBatch p) {
    constexpr int NW = D / 16;         // warps; warp w owns state rows 16w..16w+15
    constexpr int NT = NW * 32;
    constexpr int ROW = Smem<D, SPLIT>::ROW;
    constexpr int WPM = NW / 4;        // warps per 16-token block of the chunk
    constexpr int NCOL = D / WPM;      // output columns per warp in the C x D products
    constexpr int NPW = 32 / NW;       // n8 tiles per warp in the C x C products
    constexpr int SEG = D / 8;         // 16-byte segments per row

    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem<D, SPLIT> &sm = *reinterpret_cast<Smem<D, SPLIT> *>(smem_raw);

    const int h = blockIdx.x, n = blockIdx.y, grp_i = blockIdx.z;
    const int h_k = p.h_k, h_v = p.h_v;
    const int hk = h / (h_v / h_k);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = lane >> 2, qd = lane & 3;
    int bos, eos;
    if (!seq_bounds(p.cu, n, p.total, p.max_len, p.status, bos, eos)) return;
    const int len = eos - bos;
    const int nchunks = (len + C - 1) / C;
    const float scale = p.scale;

    const size_t qk_stride = size_t(h_k) * D;  // elements between consecutive tokens
    const size_t v_stride = size_t(h_v) * D;
    const size_t qk_off = size_t(bos) * qk_stride + size_t(hk) * D;
    const size_t v_off = size_t(bos) * v_stride + size_t(h) * D;
    const __nv_bfloat16 *qh = p.q[grp_i] + qk_off;
    const __nv_bfloat16 *kh = p.k[grp_i] + qk_off;
    const __nv_bfloat16 *vh = p.v[grp_i] + v_off;
    const __nv_bfloat16 *klh = SPLIT ? p.k_lo[grp_i] + qk_off : nullptr;
    const __nv_bfloat16 *vlh = SPLIT ? p.v_lo[grp_i] + v_off : nullptr;
    __nv_bfloat16 *o = p.o[grp_i];
    const float *h0 = p.h0[grp_i];

    // Stage rows of chunk c from `src` (token pitch `stride`) into `dst`; rows
    // past the sequence end are zero-filled.
    auto stage = [&](__nv_bfloat16 *dst, const __nv_bfloat16 *src, size_t stride, int c) {
        for (int e = tid; e < C * SEG; e += NT) {
            const int r = e / SEG, sgm = e % SEG;
            const int t = c * C + r;
            const bool ok = t < len;
            cp_async16(smem_u32(&dst[r * ROW + sgm * 8]), src + (ok ? size_t(t) : 0) * stride + sgm * 8, ok);
        }
    };

    // ---- state: warp w owns rows 16w..16w+15, all D columns (D/8 n-tiles)
    float S[D / 8][4];
    const size_t sbase = (size_t(n) * h_v + h) * D * D;
    {
        const int r0 = warp * 16 + grp;
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
            const int c0 = j * 8 + 2 * qd;
            if (h0) {
                const float2 a = *reinterpret_cast<const float2 *>(h0 + sbase + size_t(r0) * D + c0);
                const float2 b = *reinterpret_cast<const float2 *>(h0 + sbase + size_t(r0 + 8) * D + c0);
                S[j][0] = a.x; S[j][1] = a.y; S[j][2] = b.x; S[j][3] = b.y;
            } else {
                S[j][0] = S[j][1] = S[j][2] = S[j][3] = 0.f;
            }
            *reinterpret_cast<uint32_t *>(&sm.sb[r0 * ROW + c0]) = pack_bf16(S[j][0], S[j][1]);
            *reinterpret_cast<uint32_t *>(&sm.sb[(r0 + 8) * ROW + c0]) = pack_bf16(S[j][2], S[j][3]);
        }
    }

    const float *gh = p.g[grp_i] + size_t(bos) * h_v + h;
    const float *bh = p.beta[grp_i] + size_t(bos) * h_v + h;
    float g_next = 0.f, b_next = 0.f;
    if (nchunks > 0) {
        stage(sm.k, kh, qk_stride, 0);
        stage(sm.q, qh, qk_stride, 0);
        stage(sm.v, vh, v_stride, 0);
        if (SPLIT) {
            stage(sm.kl, klh, qk_stride, 0);
            stage(sm.vl, vlh, v_stride, 0);
        }
        cp_async_commit();
        if (tid < C && tid < len) {
            g_next = gh[size_t(tid) * h_v];
            b_next = bh[size_t(tid) * h_v];
        }
    }

    for (int c = 0; c < nchunks; ++c) {
        const int clen = min(C, len - c * C);
        const bool more = c + 1 < nchunks;
        // ---- gates of this chunk: gamma = inclusive prefix sum of g (padding has g = beta = 0)
        if (tid < C) {
            sm.gam[tid] = g_next;
            sm.beta[tid] = b_next;
        }
        cp_async_wait_all();
        __syncthreads();
        if (warp == 0) {
            float a0 = sm.gam[2 * lane], a1 = sm.gam[2 * lane + 1];
            float pair = a0 + a1;
            float incl = pair;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            const float excl = incl - pair;
            sm.gam[2 * lane] = excl + a0;
            sm.gam[2 * lane + 1] = excl + a0 + a1;
        }
        if (more) {
            const int t = (c + 1) * C + tid;
            g_next = (tid < C && t < len) ? gh[size_t(t) * h_v] : 0.f;
            b_next = (tid < C && t < len) ? bh[size_t(t) * h_v] : 0.f;
        }
        __syncthreads();

        const float gC = sm.gam[C - 1];

        // ---- (1)(2): A = strict-lower(beta_t e^{g_t-g_s} K K^T), P = lower(scale e^{g_t-g_s} Q K^T)
        {
            const int mb = warp / WPM;
            const int nt0 = (warp % WPM) * NPW;
            float akk[NPW][4], aqk[NPW][4];
#pragma unroll
            for (int j = 0; j < NPW; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) akk[j][e] = aqk[j][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t ak[4], aq[4], akl[4];
                const int arow = mb * 16 + (lane & 15), acol = kk * 16 + (lane >> 4) * 8;
                ldsm_x4(ak, smem_u32(&sm.k[arow * ROW + acol]));
                ldsm_x4(aq, smem_u32(&sm.q[arow * ROW + acol]));
                if (SPLIT) ldsm_x4(akl, smem_u32(&sm.kl[arow * ROW + acol]));
#pragma unroll
                for (int np = 0; np < NPW / 2; ++np) {
                    uint32_t b[4], bl[4];
                    const int brow = (nt0 + 2 * np) * 8 + (lane & 7) + 8 * (lane >> 4);
                    const int bcol = kk * 16 + 8 * ((lane >> 3) & 1);
                    ldsm_x4(b, smem_u32(&sm.k[brow * ROW + bcol]));
                    mma16816(akk[2 * np], ak, b[0], b[1]);
                    mma16816(akk[2 * np + 1], ak, b[2], b[3]);
                    mma16816(aqk[2 * np], aq, b[0], b[1]);
                    mma16816(aqk[2 * np + 1], aq, b[2], b[3]);
                    if (SPLIT) {
                        ldsm_x4(bl, smem_u32(&sm.kl[brow * ROW + bcol]));
                        mma16816(akk[2 * np], ak, bl[0], bl[1]);
                        mma16816(akk[2 * np + 1], ak, bl[2], bl[3]);
                        mma16816(akk[2 * np], akl, b[0], b[1]);
                        mma16816(akk[2 * np + 1], akl, b[2], b[3]);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < NPW; ++j) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int t = mb * 16 + grp + 8 * hh;
                    const int s = (nt0 + j) * 8 + 2 * qd;
                    const float gt = sm.gam[t], bt = sm.beta[t];
                    const float d0 = decay(gt, sm.gam[s], s <= t), d1 = decay(gt, sm.gam[s + 1], s + 1 <= t);
                    sm.r1.a[t * ROWA + s] = (s < t) ? bt * d0 * akk[j][2 * hh] : 0.f;
                    sm.r1.a[t * ROWA + s + 1] = (s + 1 < t) ? bt * d1 * akk[j][2 * hh + 1] : 0.f;
                    *reinterpret_cast<uint32_t *>(&sm.p[t * ROWP + s]) =
                        pack_bf16(scale * d0 * aqk[j][2 * hh], scale * d1 * aqk[j][2 * hh + 1]);
                }
            }
        }
        __syncthreads();

        // ---- (3) T = (I + A)^{-1}: diagonal 16x16 blocks by forward substitution
        // (thread = one column of one block; each row of A is read as 4 float4
        // before it is used, so the loads pipeline ahead of the FMA chain)
        float *Af = sm.r1.a;
        float *Tf = sm.r2.t;
        if (tid < C) {
            const int b = tid >> 4, cc = tid & 15;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const float4 *ar = reinterpret_cast<const float4 *>(&Af[(16 * b + r) * ROWA + 16 * b]);
                float a[16];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const float4 f = ar[v];
                    a[4 * v] = f.x; a[4 * v + 1] = f.y; a[4 * v + 2] = f.z; a[4 * v + 3] = f.w;
                }
                float acc = (r == cc) ? 1.f : 0.f;
#pragma unroll
                for (int s2 = 0; s2 < r; ++s2) acc = fmaf(-a[s2], x[s2], acc);
                x[r] = (r < cc) ? 0.f : acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) Tf[(16 * b + r) * ROWA + 16 * b + cc] = x[r];
        }
        __syncthreads();
        // Off-diagonal blocks, level by level: T_ij = -T_ii X_ij with
        // X_ij = sum_{k=j}^{i-1} A_ik T_kj.  X_ij is kept in the (free) strictly
        // upper block (j, i).  One work item = one row segment of 4 columns.
        auto blk = [](int bi, int bj, int r, int cc) { return (16 * bi + r) * ROWA + 16 * bj + cc; };
        for (int level = 1; level <= 3; ++level) {
            const int items = (4 - level) * 64;
            for (int it = tid; it < items; it += NT) {
                const int j = it >> 6, i = j + level, r = (it >> 2) & 15, c4 = (it & 3) * 4;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int kb = j; kb < i; ++kb) {
                    const float4 *ar = reinterpret_cast<const float4 *>(&Af[blk(i, kb, r, 0)]);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const float4 a = ar[v];
                        const float am[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float4 t = *reinterpret_cast<const float4 *>(&Tf[blk(kb, j, 4 * v + e, c4)]);
                            acc.x = fmaf(am[e], t.x, acc.x);
                            acc.y = fmaf(am[e], t.y, acc.y);
                            acc.z = fmaf(am[e], t.z, acc.z);
                            acc.w = fmaf(am[e], t.w, acc.w);
                        }
                    }
                }
                *reinterpret_cast<float4 *>(&Tf[blk(j, i, r, c4)]) = acc;
            }
            __syncthreads();
            for (int it = tid; it < items; it += NT) {
                const int j = it >> 6, i = j + level, r = (it >> 2) & 15, c4 = (it & 3) * 4;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                const float4 *dr = reinterpret_cast<const float4 *>(&Tf[blk(i, i, r, 0)]);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const float4 d = dr[v];
                    const float dm[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float4 xx = *reinterpret_cast<const float4 *>(&Tf[blk(j, i, 4 * v + e, c4)]);
                        acc.x = fmaf(dm[e], xx.x, acc.x);
                        acc.y = fmaf(dm[e], xx.y, acc.y);
                        acc.z = fmaf(dm[e], xx.z, acc.z);
                        acc.w = fmaf(dm[e], xx.w, acc.w);
                    }
                }
                *reinterpret_cast<float4 *>(&Tf[blk(i, j, r, c4)]) = make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
            }
            __syncthreads();
        }
        // T1 = T diag(beta e^gamma), T2 = T diag(beta) as hi + lo bf16 (lower triangle incl. diagonal)
        for (int e = tid; e < C * C / 2; e += NT) {
            const int t = e / (C / 2), s = (e % (C / 2)) * 2;
            const float t0 = (s <= t) ? Tf[t * ROWA + s] : 0.f;
            const float t1 = (s + 1 <= t) ? Tf[t * ROWA + s + 1] : 0.f;
            const float b0 = sm.beta[s], b1 = sm.beta[s + 1];
            const float e0 = __expf(sm.gam[s]), e1 = __expf(sm.gam[s + 1]);
            uint32_t hi, lo;
            *reinterpret_cast<uint32_t *>(&sm.r3.s.t1[t * ROWP + s]) = pack_bf16(t0 * b0 * e0, t1 * b1 * e1);
            split_bf16(t0 * b0, t1 * b1, hi, lo);
            *reinterpret_cast<uint32_t *>(&sm.r3.s.t2[t * ROWP + s]) = hi;
            *reinterpret_cast<uint32_t *>(&sm.r3.s.t2l[t * ROWP + s]) = lo;
        }
        __syncthreads();

        // ---- (4) -W = -T1 K -> smem;  Ut = T2 V -> registers (this warp's U tile)
        const int mb = warp / WPM;
        const int n0 = (warp % WPM) * NCOL;
        const int arow4 = mb * 16 + (lane & 15);
        float acc_u[NCOL / 8][4];
        {
            float acc_w[NCOL / 8][4];
#pragma unroll
            for (int j = 0; j < NCOL / 8; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc_w[j][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                uint32_t ah[4];
                const int acol = kk * 16 + (lane >> 4) * 8;
                ldsm_x4(ah, smem_u32(&sm.r3.s.t1[arow4 * ROWP + acol]));
#pragma unroll
                for (int np = 0; np < NCOL / 16; ++np) {
                    uint32_t bk[4], bkl[4];
                    const int brow = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                    const int bcol = n0 + np * 16 + 8 * (lane >> 4);
                    ldsm_x4_t(bk, smem_u32(&sm.k[brow * ROW + bcol]));
                    mma16816(acc_w[2 * np], ah, bk[0], bk[1]);
                    mma16816(acc_w[2 * np + 1], ah, bk[2], bk[3]);
                    if (SPLIT) {
                        ldsm_x4_t(bkl, smem_u32(&sm.kl[brow * ROW + bcol]));
                        mma16816(acc_w[2 * np], ah, bkl[0], bkl[1]);
                        mma16816(acc_w[2 * np + 1], ah, bkl[2], bkl[3]);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < NCOL / 8; ++j) {
                const int t = mb * 16 + grp, col = n0 + j * 8 + 2 * qd;
                *reinterpret_cast<uint32_t *>(&sm.r1.w[t * ROW + col]) = pack_bf16(-acc_w[j][0], -acc_w[j][1]);
                *reinterpret_cast<uint32_t *>(&sm.r1.w[(t + 8) * ROW + col]) = pack_bf16(-acc_w[j][2], -acc_w[j][3]);
            }
        }
#pragma unroll
        for (int j = 0; j < NCOL / 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc_u[j][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) {
            uint32_t ah[4], al[4];
            const int acol = kk * 16 + (lane >> 4) * 8;
            ldsm_x4(ah, smem_u32(&sm.r3.s.t2[arow4 * ROWP + acol]));
            ldsm_x4(al, smem_u32(&sm.r3.s.t2l[arow4 * ROWP + acol]));
#pragma unroll
            for (int np = 0; np < NCOL / 16; ++np) {
                uint32_t bv[4], bvl[4];
                const int brow = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                const int bcol = n0 + np * 16 + 8 * (lane >> 4);
                ldsm_x4_t(bv, smem_u32(&sm.v[brow * ROW + bcol]));
                mma16816(acc_u[2 * np], ah, bv[0], bv[1]);
                mma16816(acc_u[2 * np + 1], ah, bv[2], bv[3]);
                mma16816(acc_u[2 * np], al, bv[0], bv[1]);
                mma16816(acc_u[2 * np + 1], al, bv[2], bv[3]);
                if (SPLIT) {
                    ldsm_x4_t(bvl, smem_u32(&sm.vl[brow * ROW + bcol]));
                    mma16816(acc_u[2 * np], ah, bvl[0], bvl[1]);
                    mma16816(acc_u[2 * np + 1], ah, bvl[2], bvl[3]);
                }
            }
        }
        __syncthreads();
        // v (and its low part) are no longer read in this chunk: prefetch the next chunk's
        if (more) {
            stage(sm.v, vh, v_stride, c + 1);
            if (SPLIT) stage(sm.vl, vlh, v_stride, c + 1);
            cp_async_commit();
        }

        // ---- (5) U = Ut - W S_0^T ; store U and U diag(e^{gamma_C - gamma}) (hi + lo)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t a[4];
            ldsm_x4(a, smem_u32(&sm.r1.w[(mb * 16 + (lane & 15)) * ROW + kk * 16 + (lane >> 4) * 8]));
#pragma unroll
            for (int np = 0; np < NCOL / 16; ++np) {
                uint32_t b[4];
                const int brow = n0 + np * 16 + (lane & 7) + 8 * (lane >> 4);
                const int bcol = kk * 16 + 8 * ((lane >> 3) & 1);
                ldsm_x4(b, smem_u32(&sm.sb[brow * ROW + bcol]));
                mma16816(acc_u[2 * np], a, b[0], b[1]);
                mma16816(acc_u[2 * np + 1], a, b[2], b[3]);
            }
        }
        {
            const int t = mb * 16 + grp;
            const float f0 = __expf(gC - sm.gam[t]), f1 = __expf(gC - sm.gam[t + 8]);
#pragma unroll
            for (int j = 0; j < NCOL / 8; ++j) {
                const int col = n0 + j * 8 + 2 * qd;
                *reinterpret_cast<uint32_t *>(&sm.r2.u[t * ROW + col]) = pack_bf16(acc_u[j][0], acc_u[j][1]);
                *reinterpret_cast<uint32_t *>(&sm.r2.u[(t + 8) * ROW + col]) = pack_bf16(acc_u[j][2], acc_u[j][3]);
                uint32_t hi, lo;
                split_bf16(f0 * acc_u[j][0], f0 * acc_u[j][1], hi, lo);
                *reinterpret_cast<uint32_t *>(&sm.r3.d.ud[t * ROW + col]) = hi;
                *reinterpret_cast<uint32_t *>(&sm.r3.d.udl[t * ROW + col]) = lo;
                split_bf16(f1 * acc_u[j][2], f1 * acc_u[j][3], hi, lo);
                *reinterpret_cast<uint32_t *>(&sm.r3.d.ud[(t + 8) * ROW + col]) = hi;
                *reinterpret_cast<uint32_t *>(&sm.r3.d.udl[(t + 8) * ROW + col]) = lo;
            }
        }
        __syncthreads();

        // ---- (6) O = scale e^gamma (Q S_0^T) + P U
        if (o) {
            float acc_o[NCOL / 8][4];
#pragma unroll
            for (int j = 0; j < NCOL / 8; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc_o[j][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t a[4];
                ldsm_x4(a, smem_u32(&sm.q[(mb * 16 + (lane & 15)) * ROW + kk * 16 + (lane >> 4) * 8]));
#pragma unroll
                for (int np = 0; np < NCOL / 16; ++np) {
                    uint32_t b[4];
                    const int brow = n0 + np * 16 + (lane & 7) + 8 * (lane >> 4);
                    const int bcol = kk * 16 + 8 * ((lane >> 3) & 1);
                    ldsm_x4(b, smem_u32(&sm.sb[brow * ROW + bcol]));
                    mma16816(acc_o[2 * np], a, b[0], b[1]);
                    mma16816(acc_o[2 * np + 1], a, b[2], b[3]);
                }
            }
            const int t = mb * 16 + grp;
            const float f0 = scale * __expf(sm.gam[t]), f1 = scale * __expf(sm.gam[t + 8]);
#pragma unroll
            for (int j = 0; j < NCOL / 8; ++j) {
                acc_o[j][0] *= f0; acc_o[j][1] *= f0; acc_o[j][2] *= f1; acc_o[j][3] *= f1;
            }
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                uint32_t a[4];
                ldsm_x4(a, smem_u32(&sm.p[(mb * 16 + (lane & 15)) * ROWP + kk * 16 + (lane >> 4) * 8]));
#pragma unroll
                for (int np = 0; np < NCOL / 16; ++np) {
                    uint32_t b[4];
                    const int brow = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                    const int bcol = n0 + np * 16 + 8 * (lane >> 4);
                    ldsm_x4_t(b, smem_u32(&sm.r2.u[brow * ROW + bcol]));
                    mma16816(acc_o[2 * np], a, b[0], b[1]);
                    mma16816(acc_o[2 * np + 1], a, b[2], b[3]);
                }
            }
            const size_t tok0 = size_t(bos) + size_t(c) * C;
#pragma unroll
            for (int j = 0; j < NCOL / 8; ++j) {
                const int col = n0 + j * 8 + 2 * qd;
                if (t < clen)
                    *reinterpret_cast<uint32_t *>(o + (tok0 + t) * v_stride + size_t(h) * D + col) =
                        pack_bf16(acc_o[j][0], acc_o[j][1]);
                if (t + 8 < clen)
                    *reinterpret_cast<uint32_t *>(o + (tok0 + t + 8) * v_stride + size_t(h) * D + col) =
                        pack_bf16(acc_o[j][2], acc_o[j][3]);
            }
        }
        __syncthreads();  // every warp is done reading sb and q
        if (more) {
            stage(sm.q, qh, qk_stride, c + 1);
            cp_async_commit();
        }

        // ---- (7) S_C = e^{gamma_C} S_0 + (U diag(e^{gamma_C-gamma}))^T K
        {
            const float fC = __expf(gC);
#pragma unroll
            for (int j = 0; j < D / 8; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) S[j][e] *= fC;
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                uint32_t ah[4], al[4];
                const int arow = kk * 16 + (lane & 7) + 8 * (lane >> 4);
                const int acol = warp * 16 + 8 * ((lane >> 3) & 1);
                ldsm_x4_t(ah, smem_u32(&sm.r3.d.ud[arow * ROW + acol]));
                ldsm_x4_t(al, smem_u32(&sm.r3.d.udl[arow * ROW + acol]));
#pragma unroll
                for (int np = 0; np < D / 16; ++np) {
                    uint32_t b[4], bl[4];
                    const int brow = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                    const int bcol = np * 16 + 8 * (lane >> 4);
                    ldsm_x4_t(b, smem_u32(&sm.k[brow * ROW + bcol]));
                    mma16816(S[2 * np], ah, b[0], b[1]);
                    mma16816(S[2 * np + 1], ah, b[2], b[3]);
                    mma16816(S[2 * np], al, b[0], b[1]);
                    mma16816(S[2 * np + 1], al, b[2], b[3]);
                    if (SPLIT) {
                        ldsm_x4_t(bl, smem_u32(&sm.kl[brow * ROW + bcol]));
                        mma16816(S[2 * np], ah, bl[0], bl[1]);
                        mma16816(S[2 * np + 1], ah, bl[2], bl[3]);
                    }
                }
            }
            const int r0 = warp * 16 + grp;
#pragma unroll
            for (int j = 0; j < D / 8; ++j) {
                const int c0 = j * 8 + 2 * qd;
                *reinterpret_cast<uint32_t *>(&sm.sb[r0 * ROW + c0]) = pack_bf16(S[j][0], S[j][1]);
                *reinterpret_cast<uint32_t *>(&sm.sb[(r0 + 8) * ROW + c0]) = pack_bf16(S[j][2], S[j][3]);
            }
        }
        __syncthreads();  // k (and its low part) are free
        if (more) {
            stage(sm.k, kh, qk_stride, c + 1);
            if (SPLIT) stage(sm.kl, klh, qk_stride, c + 1);
            cp_async_commit();
        }
    }

    // ---- final state
    {
        float *s_out = p.s_out[grp_i];
        const int r0 = warp * 16 + grp;
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
            const int c0 = j * 8 + 2 * qd;
            *reinterpret_cast<float2 *>(s_out + sbase + size_t(r0) * D + c0) = make_float2(S[j][0], S[j][1]);
            *reinterpret_cast<float2 *>(s_out + sbase + size_t(r0 + 8) * D + c0) = make_float2(S[j][2], S[j][3]);
        }
    }
}

template <int D, bool SPLIT>
cudaError_t launch_chunked(const GdnBatch &b, int n_groups, int n_seqs, cudaStream_t st) {
    const size_t smem = sizeof(Smem<D, SPLIT>);
    cudaError_t e = cudaFuncSetAttribute(gdn_chunk_kernel<D, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(b.h_v, n_seqs, n_groups);
    gdn_chunk_kernel<D, SPLIT><<<grid, D * 2, smem, st>>>(b);
    return cudaGetLastError();
}

}  // namespace

bool gdn_chunked_supported(const sr_gdn_args &a) {
    return a.dtype == SR_BF16 && a.d_k == a.d_v && (a.d_k == 64 || a.d_k == 128);
}

size_t gdn_scratch_bytes(const sr_gdn_args &) { return 0; }

cudaError_t gdn_chunked_batch(const GdnBatch &b, int n_groups, int n_seqs, int d, bool split, cudaStream_t st) {
    if (n_seqs == 0 || b.h_v == 0 || n_groups == 0) return cudaSuccess;
    if (d == 64) return split ? launch_chunked<64, true>(b, n_groups, n_seqs, st)
                              : launch_chunked<64, false>(b, n_groups, n_seqs, st);
    return split ? launch_chunked<128, true>(b, n_groups, n_seqs, st)
                 : launch_chunked<128, false>(b, n_groups, n_seqs, st);
}

cudaError_t gdn_chunked(const sr_gdn_args &a, float scale, uint32_t *status, void *, cudaStream_t st) {
    GdnBatch b{};
    b.q[0] = static_cast<const __nv_bfloat16 *>(a.q);
    b.k[0] = static_cast<const __nv_bfloat16 *>(a.k);
    b.v[0] = static_cast<const __nv_bfloat16 *>(a.v);
    b.g[0] = a.g;
    b.beta[0] = a.beta;
    b.h0[0] = a.h0;
    b.o[0] = static_cast<__nv_bfloat16 *>(a.o);
    b.s_out[0] = a.s_out;
    b.cu = a.cu_seqlens;
    b.total = a.total_tokens;
    b.max_len = a.max_seqlen;
    b.h_k = a.h_k;
    b.h_v = a.h_v;
    b.scale = scale;
    b.status = status;
    return gdn_chunked_batch(b, 1, a.n_seqs, a.d_k, false, st);
}


}  // namespace sr
