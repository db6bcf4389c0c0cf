// Chunked gated-delta replay on the 5th-generation tensor cores (d = 128).
//
// Same chunk algebra as gdn_chunk.cu ("Tail-Replay", Sec. 2; "SuffixReplay",
// Eq. 4): per chunk of C = 64 tokens with chunk-relative log-decay gamma,
//     A   = strict-lower(beta_t e^{gamma_t-gamma_s} k_t.k_s),  T = (I + A)^{-1}
//     W   = T diag(beta e^gamma) K,   Ut = T diag(beta) V,    U = Ut - W S^T
//     O   = scale (diag(e^gamma) Q S^T + M U),  M = lower(e^{gamma_t-gamma_s} q_t.k_s)
//     S  <- e^{gamma_C} S + U^T diag(e^{gamma_C-gamma}) K
// Here every product is a tcgen05.mma with M = 128 issued by one thread, the
// fp32 state S (d_v x d_k) lives in tensor memory for the whole sequence, and
// the token dimension is put on N so that M is a head dimension:
//     [K;Q] K^T  (K and Q rows stacked: one M = 128 product gives K K^T and Q K^T)
//     W^T = K^T T1^T,  Ut^T = V^T T2^T,  U^T += S (-W)^T,  O^T = S Qg^T + U^T P^T,
//     S  += (U diag(e^{gamma_C-gamma}))^T K.
// q, k, v tiles arrive by TMA (128-byte swizzle); T1, T2, P, -W^T, the bf16
// copies of S and U and the scaled Qg are written by the threads in the same
// swizzled layouts.  Eight warps do the masking, the fp32 (I + A)^{-1} solve
// and the conversions; T diag(beta) and U diag(...) enter the products that
// feed the state as exact hi + lo bf16 pairs, and with split inputs k and v do
// too (three-term products), exactly as in the mma.sync kernel.
// Every mbarrier wait is bounded; a timeout records SR_DEV_TIMEOUT, drains the
// MMAs, frees tensor memory and ends the CTA.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"
#include "tc.cuh"

namespace sr {

namespace {

using namespace tc;

constexpr int C = 64, D = 128;
constexpr int kThreads = 256;
constexpr int ROWA = C + 4;  // fp32 row pitch of A and T in the solve

// shared-memory layout (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;           // [K_j0][Q_j0][K_j1][Q_j1], 8 KB each
constexpr uint32_t OFF_V = 32768;        // [V_i0][V_i1]
constexpr uint32_t OFF_KL = 49152;       // [Kl_j0][Kl_j1]    (split)
constexpr uint32_t OFF_VL = 65536;       // [Vl_i0][Vl_i1]    (split)
constexpr uint32_t kIn[2] = {49152, 81920};  // end of the inputs (plain, split)
constexpr uint32_t SZ_P = 8192;          // P   [t][s]
constexpr uint32_t SZ_TR = 24576;        // T1, T2h, T2l [t][s]; later -W^T [j][t] (16 KB)
constexpr uint32_t SZ_SB = 32768;        // S bf16 [i][j], two 64-column halves
constexpr uint32_t SZ_QG = 16384;        // Qg [t][j], two halves
constexpr uint32_t SZ_XR = 49152;        // A, T fp32 (2 x 17408); later Udh, Udl, Ub [i][t]
constexpr uint32_t SZ_MISC = 2048;       // gamma, beta, column factors, barriers, TMEM address, flags

constexpr uint32_t smem_bytes(bool split) {
    return kIn[split] + SZ_P + SZ_TR + SZ_SB + SZ_QG + SZ_XR + SZ_MISC + 1024 /* alignment */;
}

struct GdnTcParams {
    CUtensorMap q[kMaxGroups], k[kMaxGroups], v[kMaxGroups], kl[kMaxGroups], vl[kMaxGroups];
    CUtensorMap om[kMaxGroups];  // o, for the tile store of full chunks
    const float *g[kMaxGroups];
    const float *beta[kMaxGroups];
    const float *h0[kMaxGroups];
    __nv_bfloat16 *o[kMaxGroups];
    float *s_out[kMaxGroups];
    const int32_t *cu;
    int total, max_len, h_k, h_v;
    float scale;
    uint32_t *status;
};

// One warp: acc (16 x 16 fp32 in the m16n8k16 accumulator layout, two 8-column
// halves) += X Y for 16 x 16 fp32 blocks X, Y in shared memory (row pitch ROWA).
// Each operand is split into exact bf16 pairs hi + lo and the product is taken
// as Xh Yh + Xh Yl + Xl Yh, which leaves out only Xl Yl (2^-16 relative).
__device__ __forceinline__ void blk_mma(float (&acc)[2][4], const float *X, const float *Y, int lane) {
    const int g = lane >> 2, q = lane & 3;
    uint32_t ah[4], al[4];
    const float2 x0 = *reinterpret_cast<const float2 *>(X + g * ROWA + 2 * q);
    const float2 x1 = *reinterpret_cast<const float2 *>(X + (g + 8) * ROWA + 2 * q);
    const float2 x2 = *reinterpret_cast<const float2 *>(X + g * ROWA + 2 * q + 8);
    const float2 x3 = *reinterpret_cast<const float2 *>(X + (g + 8) * ROWA + 2 * q + 8);
    ms::split_bf16(x0.x, x0.y, ah[0], al[0]);
    ms::split_bf16(x1.x, x1.y, ah[1], al[1]);
    ms::split_bf16(x2.x, x2.y, ah[2], al[2]);
    ms::split_bf16(x3.x, x3.y, ah[3], al[3]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int n = 8 * nt + g;
        uint32_t bh0, bl0, bh1, bl1;
        ms::split_bf16(Y[(2 * q) * ROWA + n], Y[(2 * q + 1) * ROWA + n], bh0, bl0);
        ms::split_bf16(Y[(2 * q + 8) * ROWA + n], Y[(2 * q + 9) * ROWA + n], bh1, bl1);
        ms::mma16816(acc[nt], ah, bh0, bh1);
        ms::mma16816(acc[nt], ah, bl0, bl1);
        ms::mma16816(acc[nt], al, bh0, bh1);
    }
}

// Loads a 16 x 16 fp32 block into the accumulator layout of blk_mma.
__device__ __forceinline__ void blk_load(float (&acc)[2][4], const float *Z, int lane) {
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const float2 a = *reinterpret_cast<const float2 *>(Z + g * ROWA + 8 * nt + 2 * q);
        const float2 b = *reinterpret_cast<const float2 *>(Z + (g + 8) * ROWA + 8 * nt + 2 * q);
        acc[nt][0] = a.x; acc[nt][1] = a.y; acc[nt][2] = b.x; acc[nt][3] = b.y;
    }
}

// Stores sign * acc (accumulator layout of blk_mma) as a 16 x 16 fp32 block.
__device__ __forceinline__ void blk_store(float *Z, const float (&acc)[2][4], int lane, float sign) {
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        *reinterpret_cast<float2 *>(Z + g * ROWA + 8 * nt + 2 * q) = make_float2(sign * acc[nt][0], sign * acc[nt][1]);
        *reinterpret_cast<float2 *>(Z + (g + 8) * ROWA + 8 * nt + 2 * q) =
            make_float2(sign * acc[nt][2], sign * acc[nt][3]);
    }
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 f = __bfloat1622float2(h);
    __nv_bfloat162 l = __floats2bfloat162_rn(a - f.x, b - f.y);
    hi = *reinterpret_cast<uint32_t *>(&h);
    lo = *reinterpret_cast<uint32_t *>(&l);
}

template <bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1) gdn_tc_kernel(const __grid_constant__ GdnTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t base = smem_u32(sm);
    const uint32_t oP = kIn[SPLIT], oTR = oP + SZ_P, oSB = oTR + SZ_TR, oQG = oSB + SZ_SB, oXR = oQG + SZ_QG;
    const uint32_t oMISC = oXR + SZ_XR;
    float *gam = reinterpret_cast<float *>(sm + oMISC);          // [64]
    float *bet = gam + C;                                         // [64]
    float *fb = gam + 2 * C;                                      // [64] beta_s e^{gamma_s}
    float *fu = gam + 3 * C;                                      // [64] e^{gamma_C - gamma_t}
    float *eg = reinterpret_cast<float *>(sm + oMISC + 1536);     // [64] e^{gamma_t}
    float *ei = eg + C;                                           // [64] e^{-gamma_t}
    uint64_t *bar_k = reinterpret_cast<uint64_t *>(sm + oMISC + 1024);  // K (+ k low part) landed
    uint64_t *bar_q = bar_k + 1;                                          // Q landed
    uint64_t *bar_v = bar_k + 2;                                          // V (+ v low part) landed
    uint64_t *bar_mma = bar_k + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_mma + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *Af = reinterpret_cast<float *>(sm + oXR);
    float *Tf = reinterpret_cast<float *>(sm + oXR + C * ROWA * 4);

    const int h = blockIdx.x, gi = blockIdx.z;
    const int n = longest_first(p.cu, gridDim.y, blockIdx.y, reinterpret_cast<int *>(sm + oXR));
    const int h_k = p.h_k, h_v = p.h_v;
    const int hk = h / (h_v / h_k);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;  // TMEM lane this thread reads
    int bos, eos;
    if (!seq_bounds(p.cu, n, p.total, p.max_len, p.status, bos, eos)) return;
    const int len = eos - bos;
    const int nchunks = (len + C - 1) / C;
    const size_t sbase = (size_t(n) * h_v + h) * D * D;
    const float *h0 = p.h0[gi];
    float *s_out = p.s_out[gi];

    if (nchunks == 0) {  // empty sequence: the state is h0 (or zero)
        for (int e = tid; e < D * D / 4; e += kThreads) {
            const float4 v = h0 ? reinterpret_cast<const float4 *>(h0 + sbase)[e] : make_float4(0.f, 0.f, 0.f, 0.f);
            reinterpret_cast<float4 *>(s_out + sbase)[e] = v;
        }
        return;
    }

    if (tid == 0) {
        mbar_init(bar_k, 1);
        mbar_init(bar_q, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t R0 = tmem, R1 = tmem + 64, R2 = tmem + 128, R3 = tmem + 256;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;

    // ---- initial state into TMEM: thread -> row i = `row`, columns [64 half, 64 half + 64)
    {
        uint32_t r[32];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const int j0 = 64 * half + 32 * part;
#pragma unroll
            for (int e = 0; e < 32; ++e)
                r[e] = __float_as_uint(h0 ? h0[sbase + size_t(row) * D + j0 + e] : 0.f);
            tmem_st_32x32b_x32(R2 + lane_off + j0, r);
        }
        tmem_st_wait();
    }

    const CUtensorMap *mq = &p.q[gi], *mk = &p.k[gi], *mv = &p.v[gi], *mkl = &p.kl[gi], *mvl = &p.vl[gi];
    const CUtensorMap *mo = &p.om[gi];
    // Each input is refilled as soon as the last product reading it has completed.
    auto issue_k = [&](int c) {
        const int y = bos + c * C;
        mbar_arrive_expect_tx(bar_k, SPLIT ? 32768u : 16384u);
        tma_load_2d(sm + OFF_KQ, mk, bar_k, hk * D, y);
        tma_load_2d(sm + OFF_KQ + 16384, mk, bar_k, hk * D + 64, y);
        if (SPLIT) {
            tma_load_2d(sm + OFF_KL, mkl, bar_k, hk * D, y);
            tma_load_2d(sm + OFF_KL + 8192, mkl, bar_k, hk * D + 64, y);
        }
    };
    auto issue_q = [&](int c) {
        const int y = bos + c * C;
        mbar_arrive_expect_tx(bar_q, 16384u);
        tma_load_2d(sm + OFF_KQ + 8192, mq, bar_q, hk * D, y);
        tma_load_2d(sm + OFF_KQ + 24576, mq, bar_q, hk * D + 64, y);
    };
    auto issue_v = [&](int c) {
        const int y = bos + c * C;
        mbar_arrive_expect_tx(bar_v, SPLIT ? 32768u : 16384u);
        tma_load_2d(sm + OFF_V, mv, bar_v, h * D, y);
        tma_load_2d(sm + OFF_V + 8192, mv, bar_v, h * D + 64, y);
        if (SPLIT) {
            tma_load_2d(sm + OFF_VL, mvl, bar_v, h * D, y);
            tma_load_2d(sm + OFF_VL + 8192, mvl, bar_v, h * D + 64, y);
        }
    };
    if (tid == 0) {
        prefetch_tmap(mq); prefetch_tmap(mk); prefetch_tmap(mv);
        if (p.o[gi]) prefetch_tmap(mo);
        if (SPLIT) { prefetch_tmap(mkl); prefetch_tmap(mvl); }
        issue_k(0);
        issue_q(0);
        issue_v(0);
    }

    const float *gh = p.g[gi] + size_t(bos) * h_v + h;
    const float *bh = p.beta[gi] + size_t(bos) * h_v + h;
    __nv_bfloat16 *o = p.o[gi];
    const size_t v_stride = size_t(h_v) * D;
    const float scale = p.scale;
    uint32_t kq_phase = 0, v_phase = 0, mma_phase = 0;
    float g_next = 0.f, b_next = 0.f;  // gates of the next chunk (threads tid < C)
    if (tid < C && tid < len) {
        g_next = gh[size_t(tid) * h_v];
        b_next = bh[size_t(tid) * h_v];
    }
    bool ok = true;

    // wait for the next completion of the MMA barrier (all threads), then order TMEM reads
    auto wait_mma = [&]() -> bool {
        const bool w = mbar_wait(bar_mma, mma_phase);
        mma_phase ^= 1;
        tc_fence_after();
        return w;
    };
    auto check = [&](bool w) -> bool {  // collective barrier: true when any thread's wait failed
        const bool stop = __syncthreads_or(!w) != 0;
        if (stop && tid == 0) *abort_flag = 1;
        return stop;
    };

    constexpr uint32_t ID_KK = idesc_bf16_f32_major(128, 64, 0, 0);   // K-major A and B
    constexpr uint32_t ID_MN_K = idesc_bf16_f32_major(128, 64, 1, 0); // MN-major A, K-major B
    constexpr uint32_t ID_K_MN = idesc_bf16_f32_major(128, 64, 0, 1); // K-major A, MN-major B
    constexpr uint32_t ID_S = idesc_bf16_f32_major(128, 128, 0, 1);   // state update (N = 128)

    for (int c = 0; c < nchunks; ++c) {
        const int clen = min(C, len - c * C);
        // ---- gates of the chunk: gamma = inclusive prefix sum of g; padding has g = beta = 0
        if (tid < C) {
            gam[tid] = g_next;
            bet[tid] = b_next;
            const int t = (c + 1) * C + tid;
            g_next = t < len ? gh[size_t(t) * h_v] : 0.f;
            b_next = t < len ? bh[size_t(t) * h_v] : 0.f;
        }
        const bool tma_ok = mbar_wait(bar_k, kq_phase) && mbar_wait(bar_q, kq_phase);
        kq_phase ^= 1;
        if (tid == 0) bulk_wait_read();  // the previous chunk's o tile has left the Qg region
        __syncthreads();
        if (warp == 0) {
            const float a0 = gam[2 * lane], a1 = gam[2 * lane + 1];
            float incl = a0 + a1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            const float excl = incl - (a0 + a1);
            gam[2 * lane] = excl + a0;
            gam[2 * lane + 1] = excl + a0 + a1;
        }
        if (check(tma_ok)) break;
        const float gC = gam[C - 1];
        if (tid < C) {  // per-column factors, read after later barriers
            const float e = __expf(gam[tid]);
            fb[tid] = bet[tid] * e;
            fu[tid] = __expf(gC - gam[tid]);
            eg[tid] = e;
            ei[tid] = __expf(-gam[tid]);
        }
        // e^{gamma_t - gamma_s} = e^{gamma_t} e^{-gamma_s} while e^{-gamma_C} stays far from
        // the fp32 range (gamma_C > -80); stronger decay takes the exponential of each
        // masked difference
        const bool fact = gC > -80.f;

        // ---- MMA 1: [K;Q] K^T -> R0 (rows 0-63: K K^T, rows 64-127: Q K^T)
        if (tid == 0) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t a = base + OFF_KQ + (k >> 2) * 16384 + (k & 3) * 32;
                mma_bf16_ss(R0, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), ID_KK, k > 0);
            }
            if (SPLIT) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {  // [K;Q] Kl^T, and Kl K^T into R1 (rows 0-63)
                    const uint32_t a = base + OFF_KQ + (k >> 2) * 16384 + (k & 3) * 32;
                    const uint32_t bl = base + OFF_KL + (k >> 2) * 8192 + (k & 3) * 32;
                    mma_bf16_ss(R0, sdesc_sw128(a, 16, 1024), sdesc_sw128(bl, 16, 1024), ID_KK, 1);
                    mma_bf16_ss(R1, sdesc_sw128(bl, 16, 1024), sdesc_sw128(a, 16, 1024), ID_KK, k > 0);
                }
            }
            mma_commit(bar_mma);
        }
        // ---- meanwhile: bf16 copy of S (entering the chunk) and S <- e^{gamma_C} S in TMEM
        {
            const float fC = __expf(gC);
            uint32_t r[32];
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                tmem_ld_32x32b_x32(R2 + lane_off + 64 * half + 32 * part, r);
                tmem_ld_wait();
                uint8_t *sb = sm + oSB + half * 16384;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 w;
                    w.x = pack2(__uint_as_float(r[8 * q4 + 0]), __uint_as_float(r[8 * q4 + 1]));
                    w.y = pack2(__uint_as_float(r[8 * q4 + 2]), __uint_as_float(r[8 * q4 + 3]));
                    w.z = pack2(__uint_as_float(r[8 * q4 + 4]), __uint_as_float(r[8 * q4 + 5]));
                    w.w = pack2(__uint_as_float(r[8 * q4 + 6]), __uint_as_float(r[8 * q4 + 7]));
                    *reinterpret_cast<uint4 *>(sb + sw128(row, 4 * part + q4)) = w;
                }
#pragma unroll
                for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * fC);
                tmem_st_32x32b_x32(R2 + lane_off + 64 * half + 32 * part, r);
            }
            tmem_st_wait();
        }
        // ---- Qg = scale e^{gamma_t} Q (same swizzled geometry as the Q tiles)
        for (int e = tid; e < 1024; e += kThreads) {
            const int sub = e >> 9, t = (e >> 3) & 63, ch = e & 7;
            const uint32_t off = sw128(t, ch);
            const uint4 u = *reinterpret_cast<const uint4 *>(sm + OFF_KQ + 8192 + sub * 16384 + off);
            const float f = scale * __expf(gam[t]);
            const __nv_bfloat162 *x2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
            uint4 w;
            uint32_t *wp = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
                const float2 xf = __bfloat1622float2(x2[q2]);
                wp[q2] = pack2(xf.x * f, xf.y * f);
            }
            *reinterpret_cast<uint4 *>(sm + oQG + sub * 8192 + off) = w;
        }
        fence_async_smem();
        tc_fence_before();
        if (check(true)) break;
        // ---- O^T = S Qg^T -> R3 (issued now, completes with the next commit)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t a = base + oSB + (k >> 2) * 16384 + (k & 3) * 32;
                const uint32_t b = base + oQG + (k >> 2) * 8192 + (k & 3) * 32;
                mma_bf16_ss(R3, sdesc_sw128(a, 16, 1024), sdesc_sw128(b, 16, 1024), ID_KK, k > 0);
            }
        }
        const bool m1 = wait_mma();  // MMA 1 done (the O^T product may still run)

        // ---- A (fp32, for the solve) from K K^T and P (bf16 tile) from Q K^T
        {
            uint32_t r[32], r2[32];
            tmem_ld_32x32b_x32(R0 + lane_off + 32 * half, r);
            if (SPLIT && quad < 2) tmem_ld_32x32b_x32(R1 + lane_off + 32 * half, r2);
            tmem_ld_wait();
            if (quad < 2) {
                const int t = row;
                const float gt = gam[t], bt = bet[t], ft = fb[t];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    float a4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int s = 32 * half + e + u;
                        float kk = __uint_as_float(r[e + u]);
                        if (SPLIT) kk += __uint_as_float(r2[e + u]);
                        const float d = fact ? ft * ei[s] : bt * __expf(gt - gam[s]);
                        a4[u] = (s < t) ? d * kk : 0.f;
                    }
                    *reinterpret_cast<float4 *>(&Af[t * ROWA + 32 * half + e]) = make_float4(a4[0], a4[1], a4[2], a4[3]);
                }
            } else {
                const int t = row - 64;
                const float gt = gam[t], st = scale * eg[t];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int s = 32 * half + 8 * q4 + 2 * u;
                        float d0, d1;
                        if (fact) {
                            d0 = s <= t ? st * ei[s] : 0.f;
                            d1 = s + 1 <= t ? st * ei[s + 1] : 0.f;
                        } else {
                            d0 = scale * __expf(s <= t ? gt - gam[s] : -INFINITY);
                            d1 = scale * __expf(s + 1 <= t ? gt - gam[s + 1] : -INFINITY);
                        }
                        w[u] = pack2(d0 * __uint_as_float(r[8 * q4 + 2 * u]), d1 * __uint_as_float(r[8 * q4 + 2 * u + 1]));
                    }
                    *reinterpret_cast<uint4 *>(sm + oP + sw128(t, 4 * half + q4)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
        tc_fence_before();
        if (check(m1)) break;
        if (tid == 0 && c + 1 < nchunks) issue_q(c + 1);  // Q read by MMA 1 and the Qg copy only

        // ---- T = (I + A)^{-1} by 16x16 blocks (A strictly lower):
        //   T_ii  = (I + A_ii)^{-1}, fp32 forward substitution, one column per thread
        //   B_ik  = T_ii A_ik (k < i), kept in the unused upper blocks of T
        //   T_ij  = -sum_{k=j}^{i-1} B_ik T_kj, in three rounds of independent products
        // The block products run on mma.sync with split bf16 operands (blk_mma).
        // T_ii by 8 x 8 halves: D = (I + N)^{-1} of each half by forward substitution,
        // then the lower-left half -D2 (N21 D1) (its temporary N21 D1 sits in the
        // unused upper-right half of the diagonal block of A)
        if (tid < C) {
            const int r0 = 8 * (tid >> 3), cc = tid & 7;
            float x[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float4 *ar = reinterpret_cast<const float4 *>(&Af[(r0 + r) * ROWA + r0]);
                const float4 f0 = ar[0], f1 = ar[1];
                const float a[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
                float acc = (r == cc) ? 1.f : 0.f;
#pragma unroll
                for (int s2 = 0; s2 < r; ++s2) acc = fmaf(-a[s2], x[s2], acc);
                x[r] = (r < cc) ? 0.f : acc;
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) Tf[(r0 + r) * ROWA + r0 + cc] = x[r];
        }
        __syncthreads();
        {
            const int b = tid >> 6, r = (tid >> 3) & 7, cc = tid & 7, d0 = 16 * b;
            float y = 0.f;  // (N21 D1)[r][cc]
#pragma unroll
            for (int m = 0; m < 8; ++m) y = fmaf(Af[(d0 + 8 + r) * ROWA + d0 + m], Tf[(d0 + m) * ROWA + d0 + cc], y);
            Af[(d0 + r) * ROWA + d0 + 8 + cc] = y;
            Tf[(d0 + r) * ROWA + d0 + 8 + cc] = 0.f;  // upper-right half of T_ii
        }
        __syncthreads();
        {
            const int b = tid >> 6, r = (tid >> 3) & 7, cc = tid & 7, d0 = 16 * b;
            float x = 0.f;
#pragma unroll
            for (int m = 0; m < 8; ++m) x = fmaf(Tf[(d0 + 8 + r) * ROWA + d0 + 8 + m], Af[(d0 + m) * ROWA + d0 + 8 + cc], x);
            Tf[(d0 + 8 + r) * ROWA + d0 + cc] = -x;
        }
        __syncthreads();
        auto blk = [](int bi, int bj) { return 16 * bi * ROWA + 16 * bj; };
        {
            // B_ik for (i, k) = (1,0) (2,0) (2,1) (3,0) (3,1) (3,2): warp w takes pair w
            if (warp < 6) {
                const int i = warp < 1 ? 1 : (warp < 3 ? 2 : 3), k = warp - i * (i - 1) / 2;
                float acc[2][4] = {};
                blk_mma(acc, Tf + blk(i, i), Af + blk(i, k), lane);
                blk_store(Tf + blk(k, i), acc, lane, 1.f);  // kept in the upper block (k, i)
            }
        }
        __syncthreads();
        // T_ij = -sum_{k=j}^{i-1} B_ik T_kj in three rounds of independent products;
        // the partial sums of T_20, T_31 and T_30 wait in their own blocks:
        //   1: T_10, T_21, T_32 and the partials B_20 T_00, B_31 T_11, B_30 T_00
        //   2: T_20, T_31 (partial + last term) and B_31 T_10 added to T_30's partial
        //   3: T_30
        // (B_ik is kept in the upper block (k, i))
        if (warp < 6) {
            // warps 0-2: (i, j) = (1,0) (2,1) (3,2); warps 3-5: (2,0) (3,1) (3,0)
            const int i = warp < 3 ? warp + 1 : (warp == 3 ? 2 : 3);
            const int j = warp < 3 ? warp : (warp == 4 ? 1 : 0);
            float acc[2][4] = {};
            blk_mma(acc, Tf + blk(j, i), Tf + blk(j, j), lane);  // B_ij T_jj
            blk_store(Tf + blk(i, j), acc, lane, warp < 3 ? -1.f : 1.f);
        }
        __syncthreads();
        if (warp < 3) {
            // warp 0: T_20 = -(P_20 + B_21 T_10); warp 1: T_31 = -(P_31 + B_32 T_21);
            // warp 2: P_30 += B_31 T_10
            const int i = warp == 0 ? 2 : 3, j = warp == 1 ? 1 : 0, k = warp == 1 ? 2 : 1;
            float acc[2][4];
            blk_load(acc, Tf + blk(i, j), lane);
            blk_mma(acc, Tf + blk(k, i), Tf + blk(k, j), lane);
            blk_store(Tf + blk(i, j), acc, lane, warp < 2 ? -1.f : 1.f);
        }
        __syncthreads();
        if (warp == 0) {  // T_30 = -(P_30 + B_32 T_20)
            float acc[2][4];
            blk_load(acc, Tf + blk(3, 0), lane);
            blk_mma(acc, Tf + blk(2, 3), Tf + blk(2, 0), lane);
            blk_store(Tf + blk(3, 0), acc, lane, -1.f);
        }
        __syncthreads();
        // T1 = T diag(beta e^gamma) (bf16), T2 = T diag(beta) (hi + lo): K-major tiles [t][s].
        // A thread always covers the same 8 columns, so their factors stay in registers.
        {
            const int ch = tid & 7;
            float cb[8], cbe[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                cb[u] = bet[8 * ch + u];
                cbe[u] = fb[8 * ch + u];
            }
            for (int t = tid >> 3; t < C; t += kThreads / 8) {
                const float4 *tr = reinterpret_cast<const float4 *>(&Tf[t * ROWA + 8 * ch]);
                const float4 ta = tr[0], tb = tr[1];
                float tv[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
                uint32_t w1[4], wh[4], wl[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int s0 = 8 * ch + 2 * u;
                    const float t0 = (s0 <= t) ? tv[2 * u] : 0.f;
                    const float t1 = (s0 + 1 <= t) ? tv[2 * u + 1] : 0.f;
                    w1[u] = pack2(t0 * cbe[2 * u], t1 * cbe[2 * u + 1]);
                    split2(t0 * cb[2 * u], t1 * cb[2 * u + 1], wh[u], wl[u]);
                }
                const uint32_t off = sw128(t, ch);
                *reinterpret_cast<uint4 *>(sm + oTR + off) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
                *reinterpret_cast<uint4 *>(sm + oTR + 8192 + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
                *reinterpret_cast<uint4 *>(sm + oTR + 16384 + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (check(true)) break;

        // ---- MMA 2: W^T = K^T T1^T -> R1 ; Ut^T = V^T T2^T -> R0
        if (tid == 0) {
            if (!mbar_wait(bar_v, v_phase)) *abort_flag = 1;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t kmn = base + OFF_KQ + k * 2048;  // K as MN-major A (j blocks 16 KB apart)
                const uint32_t t1 = base + oTR + k * 32;
                mma_bf16_ss(R1, sdesc_sw128(kmn, 16384, 1024), sdesc_sw128(t1, 16, 1024), ID_MN_K, k > 0);
                if (SPLIT)
                    mma_bf16_ss(R1, sdesc_sw128(base + OFF_KL + k * 2048, 8192, 1024), sdesc_sw128(t1, 16, 1024),
                                ID_MN_K, 1);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t vmn = base + OFF_V + k * 2048;   // V as MN-major A (i blocks 8 KB apart)
                const uint32_t t2h = base + oTR + 8192 + k * 32, t2l = base + oTR + 16384 + k * 32;
                mma_bf16_ss(R0, sdesc_sw128(vmn, 8192, 1024), sdesc_sw128(t2h, 16, 1024), ID_MN_K, k > 0);
                mma_bf16_ss(R0, sdesc_sw128(vmn, 8192, 1024), sdesc_sw128(t2l, 16, 1024), ID_MN_K, 1);
                if (SPLIT)
                    mma_bf16_ss(R0, sdesc_sw128(base + OFF_VL + k * 2048, 8192, 1024), sdesc_sw128(t2h, 16, 1024),
                                ID_MN_K, 1);
            }
            mma_commit(bar_mma);
        }
        v_phase ^= 1;
        const bool m2 = wait_mma() && *abort_flag == 0;

        // ---- -W^T (bf16) as the MN-major B tile [j][t] of the next product
        {
            uint32_t r[32];
            tmem_ld_32x32b_x32(R1 + lane_off + 32 * half, r);
            tmem_ld_wait();
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint4 w;
                w.x = pack2(-__uint_as_float(r[8 * q4 + 0]), -__uint_as_float(r[8 * q4 + 1]));
                w.y = pack2(-__uint_as_float(r[8 * q4 + 2]), -__uint_as_float(r[8 * q4 + 3]));
                w.z = pack2(-__uint_as_float(r[8 * q4 + 4]), -__uint_as_float(r[8 * q4 + 5]));
                w.w = pack2(-__uint_as_float(r[8 * q4 + 6]), -__uint_as_float(r[8 * q4 + 7]));
                *reinterpret_cast<uint4 *>(sm + oTR + sw128(row, 4 * half + q4)) = w;
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (check(m2)) break;
        if (tid == 0 && c + 1 < nchunks) issue_v(c + 1);  // V read by MMA 2 only

        // ---- MMA 3: U^T = Ut^T + S (-W)^T -> R0
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t a = base + oSB + (k >> 2) * 16384 + (k & 3) * 32;
                const uint32_t b = base + oTR + k * 2048;
                mma_bf16_ss(R0, sdesc_sw128(a, 16, 1024), sdesc_sw128(b, 8192, 1024), ID_K_MN, 1);
            }
            mma_commit(bar_mma);
        }
        const bool m3 = wait_mma();

        // ---- U diag(e^{gamma_C - gamma}) (hi + lo) and U (bf16): K-major tiles [i][t]
        {
            uint32_t r[32];
            tmem_ld_32x32b_x32(R0 + lane_off + 32 * half, r);
            tmem_ld_wait();
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint32_t wh[4], wl[4], wb[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int t = 32 * half + 8 * q4 + 2 * u;
                    const float u0 = __uint_as_float(r[8 * q4 + 2 * u]), u1 = __uint_as_float(r[8 * q4 + 2 * u + 1]);
                    split2(u0 * fu[t], u1 * fu[t + 1], wh[u], wl[u]);
                    wb[u] = pack2(u0, u1);
                }
                const uint32_t off = sw128(row, 4 * half + q4);
                *reinterpret_cast<uint4 *>(sm + oXR + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
                *reinterpret_cast<uint4 *>(sm + oXR + 16384 + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
                *reinterpret_cast<uint4 *>(sm + oXR + 32768 + off) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (check(m3)) break;

        // ---- MMA 4: S += (U diag)^T K -> R2 ; O^T += U^T P^T -> R3
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t kmn = base + OFF_KQ + k * 2048;  // K as MN-major B (j blocks 16 KB apart)
                const uint32_t uh = base + oXR + k * 32, ul = base + oXR + 16384 + k * 32;
                mma_bf16_ss(R2, sdesc_sw128(uh, 16, 1024), sdesc_sw128(kmn, 16384, 1024), ID_S, 1);
                mma_bf16_ss(R2, sdesc_sw128(ul, 16, 1024), sdesc_sw128(kmn, 16384, 1024), ID_S, 1);
                if (SPLIT)
                    mma_bf16_ss(R2, sdesc_sw128(uh, 16, 1024), sdesc_sw128(base + OFF_KL + k * 2048, 8192, 1024),
                                ID_S, 1);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t ub = base + oXR + 32768 + k * 32, pb = base + oP + k * 32;
                mma_bf16_ss(R3, sdesc_sw128(ub, 16, 1024), sdesc_sw128(pb, 16, 1024), ID_KK, 1);
            }
            mma_commit(bar_mma);
        }
        const bool m4 = wait_mma();
        if (check(m4)) break;
        // K is free now: fetch the next chunk's while O is written out
        if (tid == 0 && c + 1 < nchunks) issue_k(c + 1);

        // ---- o_t (bf16): thread = value channel i, 32 tokens.  A full chunk goes
        // through the (now free) Qg region as a [t][i] tile and one TMA store; the
        // ragged last chunk is stored element by element, so that no row of the
        // next sequence is touched.
        const bool tile_store = o != nullptr && clen == C;
        if (o) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(R3 + lane_off + 32 * half, r);
            tmem_ld_wait();
            if (tile_store) {
                uint8_t *ot = sm + oQG + (row >> 6) * 8192;
                const uint32_t cofs = uint32_t(row & 7) * 2;
                const uint32_t chunk = uint32_t(row & 63) >> 3;
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    *reinterpret_cast<__nv_bfloat16 *>(ot + sw128(32 * half + e, chunk) + cofs) =
                        __float2bfloat16_rn(__uint_as_float(r[e]));
                fence_async_smem();
            } else {
                const size_t tok0 = size_t(bos) + size_t(c) * C;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int t = 32 * half + e;
                    if (t < clen)
                        o[(tok0 + t) * v_stride + size_t(h) * D + row] = __float2bfloat16_rn(__uint_as_float(r[e]));
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0 && tile_store) {
            tma_store_2d(mo, sm + oQG, h * D, bos + c * C);
            tma_store_2d(mo, sm + oQG + 8192, h * D + 64, bos + c * C);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait_all();

    __syncthreads();
    ok = *abort_flag == 0;
    if (ok) {
        // ---- final state: TMEM -> s_out
        uint32_t r[32];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const int j0 = 64 * half + 32 * part;
            tmem_ld_32x32b_x32(R2 + lane_off + j0, r);
            tmem_ld_wait();
            float4 *dst = reinterpret_cast<float4 *>(s_out + sbase + size_t(row) * D + j0);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                dst[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                     __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
        }
    } else if (tid == 0) {
        atomicOr(p.status, SR_DEV_TIMEOUT);
        // let in-flight MMAs and TMA copies finish before tensor memory and shared memory are released
        mma_commit(bar_mma);
        mbar_wait(bar_mma, mma_phase);
        for (int i = 0; i < 64; ++i) __nanosleep(1000);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// 2-D bf16 map over [rows, cols] (row pitch `cols`), 64 x 64 boxes, 128-byte swizzle.
bool map_64x64(CUtensorMap *m, const void *base, int rows, int cols) {
    return make_map_bf16(m, base, rows, cols, cols, 64, 64);
}

template <bool SPLIT>
cudaError_t launch(const GdnTcParams &p, int n_groups, int n_seqs, cudaStream_t st) {
    const int smem = int(smem_bytes(SPLIT));
    cudaError_t e = cudaFuncSetAttribute(gdn_tc_kernel<SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.h_v, n_seqs, n_groups);
    gdn_tc_kernel<SPLIT><<<grid, kThreads, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool gdn_tc_supported(int d) { return d == 128; }

cudaError_t gdn_tc_batch(const GdnBatch &b, int n_groups, int n_seqs, bool split, cudaStream_t st) {
    if (n_seqs == 0 || n_groups == 0 || b.total == 0) return gdn_chunked_batch(b, n_groups, n_seqs, 128, split, st);
    GdnTcParams p{};
    const int T = b.total, qkw = b.h_k * D, vw = b.h_v * D;
    for (int g = 0; g < n_groups; ++g) {
        if (!map_64x64(&p.q[g], b.q[g], T, qkw) || !map_64x64(&p.k[g], b.k[g], T, qkw) ||
            !map_64x64(&p.v[g], b.v[g], T, vw))
            return cudaErrorInvalidValue;
        if (split && (!map_64x64(&p.kl[g], b.k_lo[g], T, qkw) || !map_64x64(&p.vl[g], b.v_lo[g], T, vw)))
            return cudaErrorInvalidValue;
        if (b.o[g] && !map_64x64(&p.om[g], b.o[g], T, vw)) return cudaErrorInvalidValue;
        p.g[g] = b.g[g];
        p.beta[g] = b.beta[g];
        p.h0[g] = b.h0[g];
        p.o[g] = b.o[g];
        p.s_out[g] = b.s_out[g];
    }
    p.cu = b.cu;
    p.total = b.total;
    p.max_len = b.max_len;
    p.h_k = b.h_k;
    p.h_v = b.h_v;
    p.scale = b.scale;
    p.status = b.status;
    return split ? launch<true>(p, n_groups, n_seqs, st) : launch<false>(p, n_groups, n_seqs, st);
}

cudaError_t gdn_tc(const sr_gdn_args &a, float scale, uint32_t *status, cudaStream_t st) {
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
    return gdn_tc_batch(b, 1, a.n_seqs, false, st);
}

}  // namespace sr
