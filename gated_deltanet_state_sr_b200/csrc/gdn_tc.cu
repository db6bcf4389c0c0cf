// Chunked gated-delta replay on the 5th-generation tensor cores (d = 128).
//
// Same chunk algebra as gdn_chunk.cu ("Tail-Replay", Sec. 2; "SuffixReplay",
// Eq. 4): per chunk of C = 64 tokens with chunk-relative log-decay gamma,
//     A   = strict-lower(beta_t e^{gamma_t-gamma_s} k_t.k_s),  T = (I + A)^{-1}
//     W   = T diag(beta e^gamma) K,   Ut = T diag(beta) V,    U = Ut - W S^T
//     O   = scale (diag(e^gamma) Q S^T + M U),  M = lower(e^{gamma_t-gamma_s} q_t.k_s)
//     S  <- e^{gamma_C} S + U^T diag(e^{gamma_C-gamma}) K
// Every product is a tcgen05.mma with M = 128 issued by one thread, the fp32
// state S (d_v x d_k) lives in tensor memory for the whole sequence, and the
// token dimension is put on N so that M is a head dimension:
//     [K;Q] K^T  (K and Q rows stacked: one M = 128 product gives K K^T and Q K^T)
//     W^T = K^T T1^T,  Ut^T = V^T T2^T,  U^T += S (-W)^T,  O^T = S Qg^T + U^T P^T,
//     S  += (U diag(e^{gamma_C-gamma}))^T K.
// q, k, v tiles arrive by TMA (128-byte swizzle); T1, T2, P, -W^T, the bf16
// copies of S and U and the scaled Qg are written by the threads in the same
// swizzled layouts.  Eight warps do the masking, the fp32 (I + A)^{-1} solve
// and the conversions; T diag(beta) and U diag(...) enter the products that
// feed the state as exact hi + lo bf16 pairs, and with split inputs k and v do
// too (three-term products), exactly as in the mma.sync kernel.
//
// Two forms share these steps:
//  * fused (gdn_tc_kernel): one CTA per (group, sequence, V head) runs every
//    step of every chunk in order.  No scratch memory.
//  * two-phase (gdn_prep_kernel, then gdn_seq_kernel): the gates, P, A, the
//    solve, T2, W and Qg of a chunk depend only on that chunk's q, k, g and
//    beta, not on the state.  The prep kernel computes them for every (chunk,
//    V head) at once (two CTAs per SM) and stores a 56.5 KB image per unit,
//    [P | Qg, -W stacked | T2 hi | T2 lo | decay factors], in the operand
//    layouts of the products that read it.  The sequential kernel then walks
//    each sequence with only the state-dependent chain left per chunk:
//        S -> bf16;  [O^T | U^T] = S [Qg ; -W]^T + [0 | V^T T2^T];
//        U -> hi, lo, bf16;  S += (U diag)^T K;  O^T += U^T P^T;  o out,
//    with the bf16 copy of S and U's tiles kept in tensor memory as the A
//    operands of the products, while the next chunk's tiles and image stream
//    in behind a whole chunk.
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

constexpr int C = 64;  // chunk length; every tile is 128 wide in the head dims (the state is 128 x 128 in TMEM)
constexpr int kThreads = 256;
constexpr int ROWA = C + 4;               // fp32 row pitch of A and T in the solve
constexpr uint32_t SZ_AT = C * ROWA * 4;  // one fp32 64 x 64 matrix with padded rows

// input tiles (bytes from a 1024-aligned base) of the fused and the sequential kernels
constexpr uint32_t OFF_KQ = 0;           // [K_j0][Q_j0][K_j1][Q_j1], 8 KB each
constexpr uint32_t OFF_V = 32768;        // [V_i0][V_i1]
constexpr uint32_t OFF_KL = 49152;       // [Kl_j0][Kl_j1]    (split)
constexpr uint32_t OFF_VL = 65536;       // [Vl_i0][Vl_i1]    (split)
constexpr uint32_t kIn[2] = {49152, 81920};  // end of the inputs (plain, split)

constexpr uint32_t SZ_P = 8192;          // P   [t][s]
constexpr uint32_t SZ_TR = 24576;        // T1, T2h, T2l [t][s]; later -W^T [j][t] (16 KB)
constexpr uint32_t SZ_SB = 32768;        // S bf16 [i][j], two 64-column halves
constexpr uint32_t SZ_QG = 16384;        // Qg [t][j], two halves
constexpr uint32_t SZ_XR = 49152;        // fused: A, T fp32, later Udh, Udl, Ub [i][t]; sequential: U tiles
constexpr uint32_t SZ_MISC = 2048;       // gates, column factors, barriers, TMEM address, flags

constexpr uint32_t smem_fused(bool split) {
    return kIn[split] + SZ_P + SZ_TR + SZ_SB + SZ_QG + SZ_XR + SZ_MISC + 1024 /* alignment */;
}

// Chunk image of the two-phase form, per (group, chunk slot, V head): bf16
// tiles in the 128-byte swizzled layouts of the products that read them, and
// the chunk's decay factors.  [Qg ; -W] is laid out as the sequential kernel's
// stacked N = 128 operand, so one bulk copy brings it in.
constexpr uint32_t IMG_P = 0;        // P, K-major [t][s]
constexpr uint32_t IMG_QGW = 8192;   // [Qg_j0 | -W_j0 | Qg_j1 | -W_j1], K-major [t][j], 8 KB each
constexpr uint32_t IMG_T2H = 40960;  // T diag(beta), hi, K-major [t][s]
constexpr uint32_t IMG_T2L = 49152;  // T diag(beta), lo
constexpr uint32_t IMG_GATE = 57344; // fp32 e^{gamma_C - gamma_t} for t < 64, then e^{gamma_C} (512 B)
constexpr uint32_t kImg = 57856;

// prep kernel: K/Q tiles at 0 (32 KB), then two fp32 64 x 64 slots (A and T),
// then the gates.  P and T2 hi reuse the Q tiles once the first product has
// read them, T1 and T2 lo the A matrix after the solve, -W^T the T matrix once
// T1 and T2 are formed.  With split k the low part of K arrives at 32 KB and the
// first product reads it there; T then takes that slot (A the next), and the
// low part is loaded again for W^T once T1 and T2 are formed.  Both forms take
// 69 KB, three CTAs per SM.
constexpr uint32_t OFF_KL_PREP = 32768;
constexpr uint32_t smem_prep() { return 32768 + 2 * SZ_AT + SZ_MISC + 1024; }

static_assert(3 * (smem_prep() + 1024) <= 233472, "three prep CTAs must fit one SM");

// Chunk c of the sequence n starting at token bos has the image slot
// floor(bos / C) + n + c: distinct chunks get distinct slots, all below
// floor(total / C) + n_seqs.
__host__ __device__ inline int chunk_slot(int bos, int n, int c) { return bos / C + n + c; }

constexpr uint32_t ID_KK = idesc_bf16_f32_major(128, 64, 0, 0);    // K-major A and B
constexpr uint32_t ID_MN_K = idesc_bf16_f32_major(128, 64, 1, 0);  // MN-major A, K-major B
constexpr uint32_t ID_K_MN = idesc_bf16_f32_major(128, 64, 0, 1);  // K-major A, MN-major B
constexpr uint32_t ID_S = idesc_bf16_f32_major(128, 128, 0, 1);    // state update (N = 128)
constexpr uint32_t ID_KK128 = idesc_bf16_f32_major(128, 128, 0, 0);  // K-major A and B, N = 128

struct GdnTcParams {
    CUtensorMap q[kMaxGroups], k[kMaxGroups], v[kMaxGroups], kl[kMaxGroups], vl[kMaxGroups];
    CUtensorMap om[kMaxGroups];  // o, for the tile store of full chunks
    const float *g[kMaxGroups];
    const float *beta[kMaxGroups];
    const float *h0[kMaxGroups];
    __nv_bfloat16 *o[kMaxGroups];
    float *s_out[kMaxGroups];
    const int32_t *cu;
    uint8_t *img;  // two-phase: chunk images [group][slot][V head][kImg]
    int total, max_len, h_k, h_v, n_seqs, slots;
    int d;  // head dim d_k = d_v: 128, or 64 (the upper half of every 128-wide tile stays zero)
    int want_o;  // 0: no group writes o, so the two-phase form neither forms nor moves P and Qg
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

// ---------------------------------------------------------------- chunk steps
// (every thread of the CTA calls each step; `row` = quad * 32 + lane is the
// TMEM lane a thread reads, `half` = warp / 4 the column half it covers)

// Warp 0: gam[0..63] <- its inclusive prefix sum.
__device__ __forceinline__ void gate_prefix(float *gam, int lane) {
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

// Descriptor of (addr + bytes) from the descriptor of addr.  The start-address
// field holds addr >> 4, below 2^14 for every shared-memory address, so a byte
// offset adds without a carry out of the field; the products below form each
// operand's descriptor once and step it by constants.
__device__ __forceinline__ uint64_t dadd(uint64_t d, uint32_t bytes) { return d + uint64_t(bytes >> 4); }
// The shared-memory base, re-read where a product group is issued so that its
// descriptors live only there (kept out of the registers of the chunk loop).
__device__ __forceinline__ uint32_t fresh(uint32_t base) {
    uint32_t b;
    asm volatile("mov.b32 %0, %1;" : "=r"(b) : "r"(base));
    return b;
}

// [K;Q] K^T -> R0 (rows 0-63: K K^T, rows 64-127: Q K^T); with split k also
// [K;Q] Kl^T into R0 and Kl K^T into R1 (rows 0-63).  One thread issues.
template <bool SPLIT>
__device__ __forceinline__ void mma_kqk(uint32_t base, uint32_t R0, uint32_t R1, uint32_t kl_off = OFF_KL) {
    base = fresh(base);
    const uint64_t dk = sdesc_sw128(base + OFF_KQ, 16, 1024);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint64_t a = dadd(dk, (k >> 2) * 16384 + (k & 3) * 32);
        mma_bf16_ss(R0, a, a, ID_KK, k > 0);
    }
    if (SPLIT) {
        const uint64_t dl = sdesc_sw128(base + kl_off, 16, 1024);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint64_t a = dadd(dk, (k >> 2) * 16384 + (k & 3) * 32);
            const uint64_t bl = dadd(dl, (k >> 2) * 8192 + (k & 3) * 32);
            mma_bf16_ss(R0, a, bl, ID_KK, 1);
            mma_bf16_ss(R1, bl, a, ID_KK, k > 0);
        }
    }
}

// A (fp32 [t][s] with row pitch ROWA) from K K^T and P (bf16 K-major tile [t][s]
// at p_off) from Q K^T.  e^{gamma_t - gamma_s} = e^{gamma_t} e^{-gamma_s} while
// e^{-gamma_C} stays far from the fp32 range (`fact`: gamma_C > -80); stronger
// decay takes the exponential of each masked difference.
template <bool SPLIT>
__device__ __forceinline__ void build_a_p(uint8_t *sm, uint32_t p_off, float *Af, uint32_t R0, uint32_t R1,
                                          uint32_t lane_off, int quad, int half, int row, const float *gam,
                                          const float *bet, const float *fb, const float *eg, const float *ei,
                                          bool fact, float scale, bool want_p = true) {
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
    } else if (want_p) {
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
            *reinterpret_cast<uint4 *>(sm + p_off + sw128(t, 4 * half + q4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// T = (I + A)^{-1} by 16x16 blocks (A strictly lower), into Tf:
//   T_ii  = (I + A_ii)^{-1}, fp32 forward substitution by 8 x 8 halves
//   B_ik  = T_ii A_ik (k < i), kept in the unused upper blocks of T
//   T_ij  = -sum_{k=j}^{i-1} B_ik T_kj, in three rounds of independent products
// The block products run on mma.sync with split bf16 operands (blk_mma).  Ends
// with a block barrier.
__device__ __forceinline__ void t_solve(float *Af, float *Tf, int tid, int warp, int lane) {
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
}

// T1 = T diag(beta e^gamma) (bf16) and T2 = T diag(beta) (hi + lo) as K-major
// tiles [t][s] at o1, o2h, o2l.  A thread always covers the same 8 columns, so
// their factors stay in registers.
__device__ __forceinline__ void write_t12(uint8_t *sm, const float *Tf, const float *bet, const float *fb,
                                          uint32_t o1, uint32_t o2h, uint32_t o2l, int tid) {
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
        *reinterpret_cast<uint4 *>(sm + o1 + off) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
        *reinterpret_cast<uint4 *>(sm + o2h + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        *reinterpret_cast<uint4 *>(sm + o2l + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
    }
}

// W^T = K^T T1^T -> RW (split: + Kl^T T1^T, the low part of K at kl_off).  One thread issues.
template <bool SPLIT>
__device__ __forceinline__ void mma_w(uint32_t base, uint32_t o1, uint32_t RW, uint32_t kl_off = OFF_KL) {
    base = fresh(base);
    const uint64_t dk = sdesc_sw128(base + OFF_KQ, 16384, 1024);  // K as MN-major A (j blocks 16 KB apart)
    const uint64_t dl = sdesc_sw128(base + kl_off, 8192, 1024);
    const uint64_t dt = sdesc_sw128(base + o1, 16, 1024);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        mma_bf16_ss(RW, dadd(dk, k * 2048), dadd(dt, k * 32), ID_MN_K, k > 0);
        if (SPLIT) mma_bf16_ss(RW, dadd(dl, k * 2048), dadd(dt, k * 32), ID_MN_K, 1);
    }
}

// Ut^T = V^T T2^T -> RU from the hi and lo tiles of T2 (split: + Vl^T T2h^T);
// with acc0 the first product adds to what RU holds.
template <bool SPLIT>
__device__ __forceinline__ void mma_ut(uint32_t base, uint32_t o2h, uint32_t o2l, uint32_t RU, bool acc0) {
    base = fresh(base);
    const uint64_t dv = sdesc_sw128(base + OFF_V, 8192, 1024);  // V as MN-major A (i blocks 8 KB apart)
    const uint64_t dvl = sdesc_sw128(base + OFF_VL, 8192, 1024);
    const uint64_t dh = sdesc_sw128(base + o2h, 16, 1024), dl = sdesc_sw128(base + o2l, 16, 1024);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        mma_bf16_ss(RU, dadd(dv, k * 2048), dadd(dh, k * 32), ID_MN_K, k > 0 || acc0);
        mma_bf16_ss(RU, dadd(dv, k * 2048), dadd(dl, k * 32), ID_MN_K, 1);
        if (SPLIT) mma_bf16_ss(RU, dadd(dvl, k * 2048), dadd(dh, k * 32), ID_MN_K, 1);
    }
}

// U^T += S (-W)^T -> RU, S bf16 at sb_off, -W^T (MN-major [j][t]) at w_off.
__device__ __forceinline__ void mma_sw(uint32_t base, uint32_t sb_off, uint32_t w_off, uint32_t RU) {
    base = fresh(base);
    const uint64_t da = sdesc_sw128(base + sb_off, 16, 1024), db = sdesc_sw128(base + w_off, 8192, 1024);
#pragma unroll
    for (int k = 0; k < 8; ++k)
        mma_bf16_ss(RU, dadd(da, (k >> 2) * 16384 + (k & 3) * 32), dadd(db, k * 2048), ID_K_MN, 1);
}

// O^T = S Qg^T -> RO (the first product of the chunk's output).
__device__ __forceinline__ void mma_sq(uint32_t base, uint32_t sb_off, uint32_t qg_off, uint32_t RO) {
    base = fresh(base);
    const uint64_t da = sdesc_sw128(base + sb_off, 16, 1024), db = sdesc_sw128(base + qg_off, 16, 1024);
#pragma unroll
    for (int k = 0; k < 8; ++k)
        mma_bf16_ss(RO, dadd(da, (k >> 2) * 16384 + (k & 3) * 32), dadd(db, (k >> 2) * 8192 + (k & 3) * 32),
                    ID_KK, k > 0);
}

// [O^T | S (-W)^T] = S [Qg ; -W]^T -> RD (128 columns) in one product group:
// S bf16 at sb_off, the stacked K-major tiles [Qg_j0 | -W_j0 | Qg_j1 | -W_j1]
// (64 rows each) at qgw_off.
__device__ __forceinline__ void mma_sqw(uint32_t base, uint32_t sb_off, uint32_t qgw_off, uint32_t RD) {
    base = fresh(base);
    const uint64_t da = sdesc_sw128(base + sb_off, 16, 1024), db = sdesc_sw128(base + qgw_off, 16, 1024);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
        mma_bf16_ss(RD, dadd(da, off), dadd(db, off), ID_KK128, k > 0);
    }
}

// S += (U diag)^T K -> RS and O^T += U^T P^T -> RO, from the U tiles (Udh, Udl,
// Ub) at xr_off and P at p_off.
template <bool SPLIT>
__device__ __forceinline__ void mma_update(uint32_t base, uint32_t xr_off, uint32_t p_off, uint32_t RS,
                                           uint32_t RO) {
    base = fresh(base);
    const uint64_t dk = sdesc_sw128(base + OFF_KQ, 16384, 1024);  // K as MN-major B (j blocks 16 KB apart)
    const uint64_t dkl = sdesc_sw128(base + OFF_KL, 8192, 1024);
    const uint64_t du = sdesc_sw128(base + xr_off, 16, 1024), dp = sdesc_sw128(base + p_off, 16, 1024);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        mma_bf16_ss(RS, dadd(du, k * 32), dadd(dk, k * 2048), ID_S, 1);
        mma_bf16_ss(RS, dadd(du, 16384 + k * 32), dadd(dk, k * 2048), ID_S, 1);
        if (SPLIT) mma_bf16_ss(RS, dadd(du, k * 32), dadd(dkl, k * 2048), ID_S, 1);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) mma_bf16_ss(RO, dadd(du, 32768 + k * 32), dadd(dp, k * 32), ID_KK, 1);
}

// bf16 copy of S (TMEM RS, this thread's row and column half) into the K-major
// tiles at sb_off (two 64-column halves 16 KB apart), then S <- fC S in TMEM.
__device__ __forceinline__ void state_copy(uint8_t *sm, uint32_t sb_off, uint32_t RS, uint32_t lane_off, int half,
                                           int row, float fC) {
    uint32_t r[32];
#pragma unroll
    for (int part = 0; part < 2; ++part) {
        tmem_ld_32x32b_x32(RS + lane_off + 64 * half + 32 * part, r);
        tmem_ld_wait();
        uint8_t *sb = sm + sb_off + half * 16384;
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
        tmem_st_32x32b_x32(RS + lane_off + 64 * half + 32 * part, r);
    }
    tmem_st_wait();
}

// Qg = scale e^{gamma_t} Q (same swizzled geometry as the Q tiles): the two
// 64-column halves at qg_off and qg_off + half_stride; thread i of nthr.
__device__ __forceinline__ void build_qg(uint8_t *sm, uint32_t qg_off, uint32_t half_stride, const float *gam,
                                         float scale, int i, int nthr) {
    for (int e = i; e < 1024; e += nthr) {
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
        *reinterpret_cast<uint4 *>(sm + qg_off + sub * half_stride + off) = w;
    }
}

// Qg = scale e^{gamma_t} Q, formed from the Q tiles (at OFF_KQ + 8192 and + 24576)
// and written straight to global memory in the same swizzled tile layout, at dst
// (j 0-63) and dst + 16 KB (j 64-127).  A warp writes four whole 128-byte rows per
// instruction.
__device__ __forceinline__ void build_qg_image(const uint8_t *sm, uint8_t *dst, const float *gam, float scale,
                                               int tid) {
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
        *reinterpret_cast<uint4 *>(dst + sub * 16384 + off) = w;
    }
}

// -W^T (bf16) from TMEM RW as the MN-major B tile [j][t] at w_off.
__device__ __forceinline__ void convert_w(uint8_t *sm, uint32_t w_off, uint32_t RW, uint32_t lane_off, int half,
                                          int row) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(RW + lane_off + 32 * half, r);
    tmem_ld_wait();
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
        uint4 w;
        w.x = pack2(-__uint_as_float(r[8 * q4 + 0]), -__uint_as_float(r[8 * q4 + 1]));
        w.y = pack2(-__uint_as_float(r[8 * q4 + 2]), -__uint_as_float(r[8 * q4 + 3]));
        w.z = pack2(-__uint_as_float(r[8 * q4 + 4]), -__uint_as_float(r[8 * q4 + 5]));
        w.w = pack2(-__uint_as_float(r[8 * q4 + 6]), -__uint_as_float(r[8 * q4 + 7]));
        *reinterpret_cast<uint4 *>(sm + w_off + sw128(row, 4 * half + q4)) = w;
    }
}

// -W (bf16) from TMEM RW (holding W^T: lane = j, columns = t) as the K-major
// tiles [t][j] of j 0-63 at w_off and j 64-127 at w_off + 8 KB.
__device__ __forceinline__ void convert_w_t(uint8_t *sm, uint32_t w_off, uint32_t RW, uint32_t lane_off, int half,
                                            int row) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(RW + lane_off + 32 * half, r);
    tmem_ld_wait();
    uint8_t *wt = sm + w_off + (row >> 6) * 8192;
    const uint32_t cofs = uint32_t(row & 7) * 2;
    const uint32_t chunk = uint32_t(row & 63) >> 3;
#pragma unroll
    for (int e = 0; e < 32; ++e)
        *reinterpret_cast<__nv_bfloat16 *>(wt + sw128(32 * half + e, chunk) + cofs) =
            __float2bfloat16_rn(-__uint_as_float(r[e]));
}

// U diag(e^{gamma_C - gamma}) (hi + lo) and U (bf16) from TMEM RU as K-major
// tiles [i][t] at xr_off, xr_off + 16 KB and xr_off + 32 KB.
__device__ __forceinline__ void convert_u(uint8_t *sm, uint32_t xr_off, uint32_t RU, uint32_t lane_off, int half,
                                          int row, const float *fu) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(RU + lane_off + 32 * half, r);
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
        *reinterpret_cast<uint4 *>(sm + xr_off + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        *reinterpret_cast<uint4 *>(sm + xr_off + 16384 + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
        *reinterpret_cast<uint4 *>(sm + xr_off + 32768 + off) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
    }
}

// o_t (bf16) from TMEM RO (lane = value channel i, columns = tokens).  A full
// chunk is staged as a [t][i] tile (two 64-channel halves) at stage_off for one
// TMA store; the ragged last chunk is stored element by element, so that no row
// of the next sequence is touched.
template <int DH>
__device__ __forceinline__ void out_chunk(uint8_t *sm, uint32_t stage_off, uint32_t RO, uint32_t lane_off, int half,
                                          int row, __nv_bfloat16 *o, size_t tok0, int clen, size_t v_stride, int h,
                                          bool tile_store, long long o_elems, uint32_t *status) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(RO + lane_off + 32 * half, r);
    tmem_ld_wait();
    if (tile_store) {
        uint8_t *ot = sm + stage_off + (row >> 6) * 8192;
        const uint32_t cofs = uint32_t(row & 7) * 2;
        const uint32_t chunk = uint32_t(row & 63) >> 3;
#pragma unroll
        for (int e = 0; e < 32; ++e)
            *reinterpret_cast<__nv_bfloat16 *>(ot + sw128(32 * half + e, chunk) + cofs) =
                __float2bfloat16_rn(__uint_as_float(r[e]));
        fence_async_smem();
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int t = 32 * half + e;
            const size_t idx = (tok0 + t) * v_stride + size_t(h) * (64 * DH) + row;
            if (t < clen && row < 64 * DH && SR_IN_BOUNDS(idx, o_elems, status))
                o[idx] = __float2bfloat16_rn(__uint_as_float(r[e]));
        }
    }
}

// Initial state (h0, or zero) into TMEM RS: thread -> row `row`, its column half.
// With DH = 1 (d = 64) h0 is [64][64] and the rest of the 128 x 128 state is zero.
template <int DH>
__device__ __forceinline__ void state_init(uint32_t RS, uint32_t lane_off, int half, int row, const float *h0,
                                           size_t sbase, long long s_elems, uint32_t *status) {
    constexpr int d = 64 * DH;
    uint32_t r[32];
#pragma unroll
    for (int part = 0; part < 2; ++part) {
        const int j0 = 64 * half + 32 * part;
        const bool in = h0 && row < d && j0 < d &&
                        SR_IN_BOUNDS(sbase + size_t(row) * d + j0 + 31, s_elems, status);
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(in ? h0[sbase + size_t(row) * d + j0 + e] : 0.f);
        tmem_st_32x32b_x32(RS + lane_off + j0, r);
    }
    tmem_st_wait();
}

// Final state TMEM RS -> s_out (the d x d block of it).
template <int DH>
__device__ __forceinline__ void state_out(uint32_t RS, uint32_t lane_off, int half, int row, float *s_out,
                                          size_t sbase, long long s_elems, uint32_t *status) {
    constexpr int d = 64 * DH;
    uint32_t r[32];
#pragma unroll
    for (int part = 0; part < 2; ++part) {
        const int j0 = 64 * half + 32 * part;
        tmem_ld_32x32b_x32(RS + lane_off + j0, r);
        tmem_ld_wait();
        if (row >= d || j0 >= d) continue;
        if (!SR_IN_BOUNDS(sbase + size_t(row) * d + j0 + 31, s_elems, status)) continue;
        float4 *dst = reinterpret_cast<float4 *>(s_out + sbase + size_t(row) * d + j0);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                 __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
    }
}

// Copies h0 (or zeros) to s_out for an empty sequence.
template <int DH>
__device__ __forceinline__ void state_passthrough(const float *h0, float *s_out, size_t sbase, int tid,
                                                  long long s_elems, uint32_t *status) {
    constexpr int d = 64 * DH;
    for (int e = tid; e < d * d / 4; e += kThreads) {
        if (!SR_IN_BOUNDS(sbase + 4 * size_t(e) + 3, s_elems, status)) continue;
        const float4 v = h0 ? reinterpret_cast<const float4 *>(h0 + sbase)[e] : make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4 *>(s_out + sbase)[e] = v;
    }
}

// ---------------------------------------------------------------- fused form
template <bool SPLIT, int DH>
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
    float *Tf = reinterpret_cast<float *>(sm + oXR + SZ_AT);

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
    constexpr int d = 64 * DH;
    const size_t sbase = (size_t(n) * h_v + h) * d * d;
    const long long s_elems = (long long)p.n_seqs * h_v * d * d, o_elems = (long long)p.total * h_v * d,
                    gate_elems = (long long)p.total * h_v;
    const float *h0 = p.h0[gi];
    float *s_out = p.s_out[gi];

    if (nchunks == 0) {  // empty sequence: the state is h0 (or zero)
        state_passthrough<DH>(h0, s_out, sbase, tid, s_elems, p.status);
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
    if (DH == 1) {  // d = 64: the upper halves of the K, Q and V tiles are never loaded and stay zero
        for (int e = tid; e < 3 * 512; e += kThreads) {
            const uint32_t tile = e < 512 ? OFF_KQ + 16384 : (e < 1024 ? OFF_KQ + 24576 : OFF_V + 8192);
            *reinterpret_cast<uint4 *>(sm + tile + (e & 511) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_async_smem();
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

    state_init<DH>(R2, lane_off, half, row, h0, sbase, s_elems, p.status);

    const CUtensorMap *mq = &p.q[gi], *mk = &p.k[gi], *mv = &p.v[gi], *mkl = &p.kl[gi], *mvl = &p.vl[gi];
    const CUtensorMap *mo = &p.om[gi];
    // Each input is refilled as soon as the last product reading it has completed.
    auto issue_k = [&](int c) {
        const int y = bos + c * C;
        mbar_arrive_expect_tx(bar_k, DH * (SPLIT ? 16384u : 8192u));
        tma_load_2d(sm + OFF_KQ, mk, bar_k, hk * d, y);
        if (DH == 2) tma_load_2d(sm + OFF_KQ + 16384, mk, bar_k, hk * d + 64, y);
        if (SPLIT) {
            tma_load_2d(sm + OFF_KL, mkl, bar_k, hk * d, y);
            if (DH == 2) tma_load_2d(sm + OFF_KL + 8192, mkl, bar_k, hk * d + 64, y);
        }
    };
    auto issue_q = [&](int c) {
        const int y = bos + c * C;
        mbar_arrive_expect_tx(bar_q, DH * 8192u);
        tma_load_2d(sm + OFF_KQ + 8192, mq, bar_q, hk * d, y);
        if (DH == 2) tma_load_2d(sm + OFF_KQ + 24576, mq, bar_q, hk * d + 64, y);
    };
    auto issue_v = [&](int c) {
        const int y = bos + c * C;
        mbar_arrive_expect_tx(bar_v, DH * (SPLIT ? 16384u : 8192u));
        tma_load_2d(sm + OFF_V, mv, bar_v, h * d, y);
        if (DH == 2) tma_load_2d(sm + OFF_V + 8192, mv, bar_v, h * d + 64, y);
        if (SPLIT) {
            tma_load_2d(sm + OFF_VL, mvl, bar_v, h * d, y);
            if (DH == 2) tma_load_2d(sm + OFF_VL + 8192, mvl, bar_v, h * d + 64, y);
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
    const size_t v_stride = size_t(h_v) * d;
    const float scale = p.scale;
    uint32_t kq_phase = 0, v_phase = 0, mma_phase = 0;
    float g_next = 0.f, b_next = 0.f;  // gates of the next chunk (threads tid < C)
    if (tid < C && tid < len && SR_IN_BOUNDS((size_t(bos) + tid) * h_v + h, gate_elems, p.status)) {
        g_next = gh[size_t(tid) * h_v];
        b_next = bh[size_t(tid) * h_v];
    }

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

    for (int c = 0; c < nchunks; ++c) {
        const int clen = min(C, len - c * C);
        // ---- gates of the chunk: gamma = inclusive prefix sum of g; padding has g = beta = 0
        if (tid < C) {
            gam[tid] = g_next;
            bet[tid] = b_next;
            const int t = (c + 1) * C + tid;
            const bool in = t < len && SR_IN_BOUNDS((size_t(bos) + t) * h_v + h, gate_elems, p.status);
            g_next = in ? gh[size_t(t) * h_v] : 0.f;
            b_next = in ? bh[size_t(t) * h_v] : 0.f;
        }
        const bool tma_ok = mbar_wait(bar_k, kq_phase) && mbar_wait(bar_q, kq_phase);
        kq_phase ^= 1;
        if (tid == 0) bulk_wait_read();  // the previous chunk's o tile has left the Qg region
        __syncthreads();
        if (warp == 0) gate_prefix(gam, lane);
        if (check(tma_ok)) break;
        const float gC = gam[C - 1];
        if (tid < C) {  // per-column factors, read after later barriers
            const float e = __expf(gam[tid]);
            fb[tid] = bet[tid] * e;
            fu[tid] = __expf(gC - gam[tid]);
            eg[tid] = e;
            ei[tid] = __expf(-gam[tid]);
        }
        const bool fact = gC > -80.f;

        // ---- MMA 1: [K;Q] K^T -> R0 (and R1)
        if (tid == 0) {
            mma_kqk<SPLIT>(base, R0, R1);
            mma_commit(bar_mma);
        }
        // ---- meanwhile: bf16 copy of S (entering the chunk), S <- e^{gamma_C} S, and Qg
        state_copy(sm, oSB, R2, lane_off, half, row, __expf(gC));
        build_qg(sm, oQG, 8192, gam, scale, tid, kThreads);
        fence_async_smem();
        tc_fence_before();
        if (check(true)) break;
        // ---- O^T = S Qg^T -> R3 (issued now, completes with the next commit)
        if (tid == 0) {
            tc_fence_after();
            mma_sq(base, oSB, oQG, R3);
        }
        const bool m1 = wait_mma();  // MMA 1 done (the O^T product may still run)

        // ---- A (fp32, for the solve) from K K^T and P (bf16 tile) from Q K^T
        build_a_p<SPLIT>(sm, oP, Af, R0, R1, lane_off, quad, half, row, gam, bet, fb, eg, ei, fact, scale);
        tc_fence_before();
        if (check(m1)) break;
        if (tid == 0 && c + 1 < nchunks) issue_q(c + 1);  // Q read by MMA 1 and the Qg copy only

        t_solve(Af, Tf, tid, warp, lane);
        write_t12(sm, Tf, bet, fb, oTR, oTR + 8192, oTR + 16384, tid);
        fence_async_smem();
        tc_fence_before();
        if (check(true)) break;

        // ---- MMA 2: W^T = K^T T1^T -> R1 ; Ut^T = V^T T2^T -> R0
        if (tid == 0) {
            if (!mbar_wait(bar_v, v_phase)) *abort_flag = 1;
            tc_fence_after();
            mma_w<SPLIT>(base, oTR, R1);
            mma_ut<SPLIT>(base, oTR + 8192, oTR + 16384, R0, false);
            mma_commit(bar_mma);
        }
        v_phase ^= 1;
        const bool m2 = wait_mma() && *abort_flag == 0;

        // ---- -W^T (bf16) as the MN-major B tile [j][t] of the next product
        convert_w(sm, oTR, R1, lane_off, half, row);
        fence_async_smem();
        tc_fence_before();
        if (check(m2)) break;
        if (tid == 0 && c + 1 < nchunks) issue_v(c + 1);  // V read by MMA 2 only

        // ---- MMA 3: U^T = Ut^T + S (-W)^T -> R0
        if (tid == 0) {
            tc_fence_after();
            mma_sw(base, oSB, oTR, R0);
            mma_commit(bar_mma);
        }
        const bool m3 = wait_mma();

        // ---- U diag(e^{gamma_C - gamma}) (hi + lo) and U (bf16): K-major tiles [i][t]
        convert_u(sm, oXR, R0, lane_off, half, row, fu);
        fence_async_smem();
        tc_fence_before();
        if (check(m3)) break;

        // ---- MMA 4: S += (U diag)^T K -> R2 ; O^T += U^T P^T -> R3
        if (tid == 0) {
            tc_fence_after();
            mma_update<SPLIT>(base, oXR, oP, R2, R3);
            mma_commit(bar_mma);
        }
        const bool m4 = wait_mma();
        if (check(m4)) break;
        // K is free now: fetch the next chunk's while O is written out
        if (tid == 0 && c + 1 < nchunks) issue_k(c + 1);

        // ---- o_t (bf16) through the (now free) Qg region
        const bool tile_store = o != nullptr && clen == C;
        if (o) out_chunk<DH>(sm, oQG, R3, lane_off, half, row, o, size_t(bos) + size_t(c) * C, clen, v_stride, h, tile_store, o_elems, p.status);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0 && tile_store) {
            tma_store_2d(mo, sm + oQG, h * d, bos + c * C);
            if (DH == 2) tma_store_2d(mo, sm + oQG + 8192, h * d + 64, bos + c * C);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait_all();

    __syncthreads();
    if (*abort_flag == 0) {
        state_out<DH>(R2, lane_off, half, row, s_out, sbase, s_elems, p.status);
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

// ---------------------------------------------------------------- two-phase form: prep
// One CTA per (chunk slot, V head, group).  Slots between two sequences' chunks
// (at most one per sequence) exit at once.
template <bool SPLIT, int DH>
__global__ void __launch_bounds__(kThreads, 3) gdn_prep_kernel(const __grid_constant__ GdnTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t base = smem_u32(sm);
    // split k: T over the low part of K (read by the first product, loaded again for W)
    constexpr uint32_t oT = SPLIT ? OFF_KL_PREP : 32768 + SZ_AT, oA = SPLIT ? OFF_KL_PREP + SZ_AT : 32768;
    constexpr uint32_t oMISC = 32768 + 2 * SZ_AT;
    constexpr uint32_t oP = OFF_KQ + 8192, oT2H = OFF_KQ + 24576;  // the Q tiles
    constexpr uint32_t oT1 = oA, oT2L = oA + 8192;                  // A
    constexpr uint32_t oW = oT;                                     // T
    float *Af = reinterpret_cast<float *>(sm + oA);
    float *Tf = reinterpret_cast<float *>(sm + oT);
    float *gam = reinterpret_cast<float *>(sm + oMISC);  // [64]
    float *bet = gam + C;                                 // [64]
    float *fb = gam + 2 * C;                              // [64] beta_s e^{gamma_s}
    float *eg = gam + 3 * C;                              // [64] e^{gamma_t}
    float *ei = gam + 4 * C;                              // [64] e^{-gamma_t}
    uint64_t *bar_in = reinterpret_cast<uint64_t *>(sm + oMISC + 1280);
    uint64_t *bar_mma = bar_in + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_mma + 1);

    const int slot = blockIdx.x, h = blockIdx.y, gi = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;
    // the state chain (launched as this grid's programmatic dependent) may start
    // its set-up once every CTA of this grid is running; it waits for this whole
    // grid, and its memory, before it reads an image
    grid_launch_dependents();

    // the sequence holding this slot: the largest n with floor(cu[n] / C) + n <= slot
    // (a key that grows with n).  Up to 31 sequences: one load per lane brings
    // cu[0 .. n_seqs], and the sequence's bounds come from the lanes by shuffles.
    // More: every warp narrows [lo, hi) 32-fold per round with one probe per lane,
    // so a few hundred sequences take two rounds of loads.
    int n, bos, eos;
    if (p.n_seqs < 32) {
        const int v = lane <= p.n_seqs ? p.cu[lane] : 0;
        const bool le = lane < p.n_seqs && v / C + lane <= slot;
        n = max(1, __popc(__ballot_sync(0xffffffffu, le))) - 1;
        bos = __shfl_sync(0xffffffffu, v, n);
        eos = __shfl_sync(0xffffffffu, v, n + 1);
        // the checks of seq_bounds on the values in hand
        if (!(bos >= 0 && bos <= eos && eos <= p.total && (n != 0 || bos == 0))) {
            if (tid == 0) atomicOr(p.status, SR_DEV_BAD_CU_SEQLENS);
            return;
        }
        if (eos - bos > p.max_len) {
            if (tid == 0) atomicOr(p.status, SR_DEV_SEQ_TOO_LONG);
            return;
        }
    } else {
        int lo = 0, hi = p.n_seqs;
        while (hi - lo > 1) {
            const int step = (hi - lo + 31) >> 5, m = lo + lane * step;
            const bool le = m < hi && p.cu[m] / C + m <= slot;
            const int k = max(1, __popc(__ballot_sync(0xffffffffu, le)));  // the probes at or below: a prefix
            hi = min(hi, lo + k * step);
            lo += (k - 1) * step;
        }
        n = lo;
        if (!seq_bounds(p.cu, n, p.total, p.max_len, p.status, bos, eos)) return;
    }
    const int len = eos - bos, c = slot - (bos / C + n);
    if (c < 0 || c * C >= len) return;
    if (!SR_IN_BOUNDS(slot, p.slots, p.status)) return;
    const int clen = min(C, len - c * C), y = bos + c * C;
    const int hk = h / (p.h_v / p.h_k);

    // the tiles and the gates are requested first; tensor memory is taken while they load
    if (tid == 0) {
        mbar_init(bar_in, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        const CUtensorMap *mq = &p.q[gi], *mk = &p.k[gi], *mkl = &p.kl[gi];
        constexpr int d = 64 * DH;
        // without o, Q is not needed: P and Qg are neither formed nor stored
        mbar_arrive_expect_tx(bar_in, DH * ((SPLIT ? 24576u : 16384u) - (p.want_o ? 0u : 8192u)));
        tma_load_2d(sm + OFF_KQ, mk, bar_in, hk * d, y);
        if (p.want_o) tma_load_2d(sm + OFF_KQ + 8192, mq, bar_in, hk * d, y);
        if (DH == 2) {
            tma_load_2d(sm + OFF_KQ + 16384, mk, bar_in, hk * d + 64, y);
            if (p.want_o) tma_load_2d(sm + OFF_KQ + 24576, mq, bar_in, hk * d + 64, y);
        }
        if (SPLIT) {
            tma_load_2d(sm + OFF_KL_PREP, mkl, bar_in, hk * d, y);
            if (DH == 2) tma_load_2d(sm + OFF_KL_PREP + 8192, mkl, bar_in, hk * d + 64, y);
        }
    }
    if (DH == 1) {  // d = 64: the upper halves of the K and Q tiles are never loaded and stay zero
        for (int e = tid; e < 2 * 512; e += kThreads) {
            const uint32_t tile = e < 512 ? OFF_KQ + 16384 : OFF_KQ + 24576;
            *reinterpret_cast<uint4 *>(sm + tile + (e & 511) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_async_smem();
    }
    float g0 = 0.f, b0 = 0.f;  // padding has g = beta = 0
    if (tid < clen && SR_IN_BOUNDS(size_t(y + tid) * p.h_v + h, (long long)p.total * p.h_v, p.status)) {
        g0 = p.g[gi][size_t(y + tid) * p.h_v + h];
        b0 = p.beta[gi][size_t(y + tid) * p.h_v + h];
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot, R0 = tmem, R1 = tmem + 64;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    // gates: gamma = inclusive prefix sum of g
    if (tid < C) {
        gam[tid] = g0;
        bet[tid] = b0;
    }
    __syncthreads();
    if (warp == 0) gate_prefix(gam, lane);
    __syncthreads();
    const float gC = gam[C - 1];
    if (tid < C) {
        const float e = __expf(gam[tid]);
        fb[tid] = bet[tid] * e;
        eg[tid] = e;
        ei[tid] = __expf(-gam[tid]);
    }
    const bool fact = gC > -80.f;
    uint32_t mma_phase = 0;
    bool ok = __syncthreads_and(mbar_wait(bar_in, 0)) != 0;
    uint8_t *dst = p.img + ((size_t(gi) * p.slots + slot) * p.h_v + h) * kImg;

    if (ok) {
        // ---- [K;Q] K^T, then A and P
        if (tid == 0) {
            tc_fence_after();
            mma_kqk<SPLIT>(base, R0, R1, OFF_KL_PREP);
            mma_commit(bar_mma);
        }
        // ---- meanwhile: Qg = scale e^{gamma_t} Q and the decay factors, straight to the image
        if (p.want_o) build_qg_image(sm, dst + IMG_QGW, gam, p.scale, tid);
        if (tid < C) reinterpret_cast<float *>(dst + IMG_GATE)[tid] = __expf(gC - gam[tid]);
        if (tid == 0) reinterpret_cast<float *>(dst + IMG_GATE)[C] = __expf(gC);
        __syncthreads();  // every Q read is done before P overwrites the first Q tile
        const bool w = mbar_wait(bar_mma, mma_phase);
        mma_phase ^= 1;
        tc_fence_after();
        build_a_p<SPLIT>(sm, oP, Af, R0, R1, lane_off, quad, half, row, gam, bet, fb, eg, ei, fact, p.scale,
                         p.want_o != 0);
        fence_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(w) != 0;
    }
    // each tile of the image leaves as soon as it is formed
    if (ok && tid == 0 && p.want_o) bulk_store(dst + IMG_P, sm + oP, 8192);
    if (ok) {
        // ---- the solve, T1 and T2, then W^T = K^T T1^T and -W
        t_solve(Af, Tf, tid, warp, lane);
        write_t12(sm, Tf, bet, fb, oT1, oT2H, oT2L, tid);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        bool wk = true;
        if (tid == 0) {
            tc_fence_after();
            if (SPLIT) {  // the low part of K again, over the spent T
                constexpr int d = 64 * DH;
                mbar_arrive_expect_tx(bar_in, DH * 8192u);
                tma_load_2d(sm + OFF_KL_PREP, &p.kl[gi], bar_in, hk * d, y);
                if (DH == 2) tma_load_2d(sm + OFF_KL_PREP + 8192, &p.kl[gi], bar_in, hk * d + 64, y);
                wk = mbar_wait(bar_in, 1);
            }
            if (wk) {
                mma_w<SPLIT>(base, oT1, R0, OFF_KL_PREP);
                mma_commit(bar_mma);
            }
            bulk_store(dst + IMG_T2H, sm + oT2H, 8192);
            bulk_store(dst + IMG_T2L, sm + oT2L, 8192);
        }
        // a failed wait for the reload skips W's product; every thread learns of it here
        if (__syncthreads_or(!wk)) {
            ok = false;
        }
    }
    if (ok) {
        const bool w = mbar_wait(bar_mma, mma_phase);
        mma_phase ^= 1;
        tc_fence_after();
        convert_w_t(sm, oW, R0, lane_off, half, row);
        fence_async_smem();
        ok = __syncthreads_and(w) != 0;
    }
    if (ok) {
        if (tid == 0) {
            bulk_store(dst + IMG_QGW + 8192, sm + oW, 8192);
            bulk_store(dst + IMG_QGW + 24576, sm + oW + 8192, 8192);
            bulk_commit();
            bulk_wait_read();  // shared memory may go; the writes complete with the grid
        }
    } else if (tid == 0) {
        bulk_commit();
        bulk_wait_read();
        atomicOr(p.status, SR_DEV_TIMEOUT);
        mma_commit(bar_mma);
        mbar_wait(bar_mma, mma_phase);
        for (int i = 0; i < 64; ++i) __nanosleep(1000);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// ---------------------------------------------------------------- two-phase form: sequential
// o_t (bf16) of one chunk straight from TMEM RO to global memory: a warp stores
// one token's 32 consecutive value channels per instruction (64 contiguous bytes).
// With `clear`, the columns read are then zeroed, so that the next product group
// into this accumulator can add to it from the start.
template <int DH>
__device__ __forceinline__ void out_direct(uint32_t RO, uint32_t lane_off, int half, int row, __nv_bfloat16 *o,
                                           size_t tok0, int clen, size_t v_stride, int h, long long o_elems,
                                           uint32_t *status, bool clear) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(RO + lane_off + 32 * half, r);
    tmem_ld_wait();
    if (clear) {
        uint32_t z[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) z[e] = 0u;
        tmem_st_32x32b_x32(RO + lane_off + 32 * half, z);
    }
    const size_t first = (tok0 + size_t(32 * half)) * v_stride + size_t(h) * (64 * DH) + row;
    __nv_bfloat16 *dst = o + first;
    int n_out = row < 64 * DH ? min(32, clen - 32 * half) : 0;
    if (n_out > 0 && !SR_IN_BOUNDS(first + size_t(n_out - 1) * v_stride, o_elems, status)) n_out = 0;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        if (e < n_out) *dst = __float2bfloat16_rn(__uint_as_float(r[e]));
        dst += v_stride;
    }
    if (clear) tmem_st_wait();
}

// Zeroes the 64 O columns of an [O | U] accumulator (this thread's lane, its half).
__device__ __forceinline__ void clear_o(uint32_t RO, uint32_t lane_off, int half) {
    uint32_t z[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) z[e] = 0u;
    tmem_st_32x32b_x32(RO + lane_off + 32 * half, z);
    tmem_st_wait();
}

// The state chain keeps every A operand of its products in tensor memory
// (tcgen05.mma with A from TMEM): the bf16 copy of S at RSB (64 columns, row
// i of S in lane i, two values per column), and U's tiles written over U's own
// fp32 columns RU and at RUB.  Only B operands live in shared memory.

// bf16 copy of S (TMEM RS, this thread's row and column half) into RSB, then
// S <- fC S in TMEM.
__device__ __forceinline__ void state_copy_t(uint32_t RS, uint32_t RSB, uint32_t lane_off, int half, float fC) {
    uint32_t r[32], b[16];
#pragma unroll
    for (int part = 0; part < 2; ++part) {
        tmem_ld_32x32b_x32(RS + lane_off + 64 * half + 32 * part, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) b[e] = pack2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
        tmem_st_32x32b_x16(RSB + lane_off + 32 * half + 16 * part, b);
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * fC);
        tmem_st_32x32b_x32(RS + lane_off + 64 * half + 32 * part, r);
    }
    tmem_st_wait();
}

// U's operands from its fp32 columns RU (lane i = value channel, column t =
// token): U diag(e^{gamma_C - gamma}) as hi + lo written back over RU (tokens
// 32 half .. 32 half + 31: hi at RU + 32 half, lo at RU + 32 half + 16, so a
// thread overwrites only the columns it read) and U (bf16) at RUB + 16 half.
__device__ __forceinline__ void convert_u_t(uint32_t RU, uint32_t RUB, uint32_t lane_off, int half, const float *fu) {
    uint32_t r[32], wh[16], wl[16], wb[16];
    tmem_ld_32x32b_x32(RU + lane_off + 32 * half, r);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const int t = 32 * half + 2 * e;
        const float u0 = __uint_as_float(r[2 * e]), u1 = __uint_as_float(r[2 * e + 1]);
        split2(u0 * fu[t], u1 * fu[t + 1], wh[e], wl[e]);
        wb[e] = pack2(u0, u1);
    }
    tmem_st_32x32b_x16(RU + lane_off + 32 * half, wh);
    tmem_st_32x32b_x16(RU + lane_off + 32 * half + 16, wl);
    tmem_st_32x32b_x16(RUB + lane_off + 16 * half, wb);
    tmem_st_wait();
}

// U^T = V^T T2^T -> RU (overwriting) from V at v_off and the hi and lo tiles of T2
// (split: + Vl^T T2h^T, the low part of V at vl_off).
template <bool SPLIT>
__device__ __forceinline__ void mma_ut_s(uint32_t base, uint32_t v_off, uint32_t vl_off, uint32_t o2h, uint32_t o2l,
                                         uint32_t RU) {
    base = fresh(base);
    const uint64_t dv = sdesc_sw128(base + v_off, 8192, 1024);  // V as MN-major A (i blocks 8 KB apart)
    const uint64_t dvl = sdesc_sw128(base + vl_off, 8192, 1024);
    const uint64_t dh = sdesc_sw128(base + o2h, 16, 1024), dl = sdesc_sw128(base + o2l, 16, 1024);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        mma_bf16_ss(RU, dadd(dv, k * 2048), dadd(dh, k * 32), ID_MN_K, k > 0);
        mma_bf16_ss(RU, dadd(dv, k * 2048), dadd(dl, k * 32), ID_MN_K, 1);
        if (SPLIT) mma_bf16_ss(RU, dadd(dvl, k * 2048), dadd(dh, k * 32), ID_MN_K, 1);
    }
}

// [O^T | U^T] += S [Qg ; -W]^T -> RD (128 columns), S bf16 from TMEM RSB.
__device__ __forceinline__ void mma_sqw_t(uint32_t base, uint32_t RSB, uint32_t qgw_off, uint32_t RD) {
    base = fresh(base);
    const uint64_t db = sdesc_sw128(base + qgw_off, 16, 1024);
#pragma unroll
    for (int k = 0; k < 8; ++k)
        mma_bf16_ts(RD, RSB + 8 * k, dadd(db, (k >> 2) * 16384 + (k & 3) * 32), ID_KK128, 1);
}

// S += (U diag)^T K -> RS: hi + lo of U diag from TMEM RU, K at k_off as the
// MN-major B operand (j blocks 8 KB apart); split: + hi times the low part of K.
template <bool SPLIT>
__device__ __forceinline__ void mma_s_update_t(uint32_t base, uint32_t k_off, uint32_t kl_off, uint32_t RU,
                                               uint32_t RS) {
    base = fresh(base);
    const uint64_t dk = sdesc_sw128(base + k_off, 8192, 1024);
    const uint64_t dkl = sdesc_sw128(base + kl_off, 8192, 1024);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t ah = RU + 32 * (k >> 1) + 8 * (k & 1);
        mma_bf16_ts(RS, ah, dadd(dk, k * 2048), ID_S, 1);
        mma_bf16_ts(RS, ah + 16, dadd(dk, k * 2048), ID_S, 1);
        if (SPLIT) mma_bf16_ts(RS, ah, dadd(dkl, k * 2048), ID_S, 1);
    }
}

// O^T += U^T P^T -> RO, U (bf16) from TMEM RUB and P at p_off.
__device__ __forceinline__ void mma_o_update_t(uint32_t base, uint32_t RUB, uint32_t p_off, uint32_t RO) {
    base = fresh(base);
    const uint64_t dp = sdesc_sw128(base + p_off, 16, 1024);
#pragma unroll
    for (int k = 0; k < 4; ++k) mma_bf16_ts(RO, RUB + 8 * k, dadd(dp, k * 32), ID_KK, 1);
}

// Shared memory of the sequential kernel: K (and its low part) single-buffered;
// V (and its low part) and the chunk image double-buffered, so the next chunk's
// inputs stream in during a whole chunk.
constexpr uint32_t SQ_K = 0, SQ_KL = 16384;   // [K_j0][K_j1], [Kl_j0][Kl_j1]
constexpr uint32_t SQ_V = 32768;              // buffer b: [V_i0][V_i1] at SQ_V + 16 KB b
constexpr uint32_t SQ_VL = 65536;             // buffer b: [Vl_i0][Vl_i1] at SQ_VL + 16 KB b
constexpr uint32_t SQ_IMG = 98304;            // buffer b: the chunk image at SQ_IMG + SQ_IMG_STRIDE b
constexpr uint32_t SQ_IMG_STRIDE = (kImg + 1023) / 1024 * 1024;
constexpr uint32_t SQ_MISC = SQ_IMG + 2 * SQ_IMG_STRIDE;
constexpr uint32_t smem_seq() { return SQ_MISC + 1024 + 1024; }
static_assert(smem_seq() <= 232448, "sequential kernel exceeds shared memory");

// The sequential kernel runs 9 warps: warps 0-7 move data between tensor
// memory and registers (warp w takes TMEM lanes 32 (w % 4) .. + 31 and column
// half w / 4), warp 8 only waits for inputs and issues products and copies.
constexpr int kSeqThreads = 288;
constexpr int kIssuer = 256;

// One CTA per (V head, sequence rank, group).  Per chunk c the state chain is
//   S(c) -> bf16 (TMEM);  [O(c) | U^T] += S [Qg ; -W]^T (U^T = V^T T2^T already
//   there);  U -> hi, lo, bf16 (TMEM);  S += (U diag)^T K;
// and the rest runs beside it: V^T T2^T of chunk c is issued while S is
// copied; o of chunk c-1 is written (and its accumulator cleared for chunk
// c+1) and chunk c+1's inputs are requested while the first product group of c
// runs (O alternates between two TMEM accumulators); O(c) += U^T P^T is issued
// right behind the state update and runs beside the next chunk's copy.  The
// chunk image brings Qg and the decay factors, so no gate work is left here.
// Two block barriers per chunk hand work between the warps: after the state
// copy and after U's conversion.
template <bool SPLIT, int DH>
__global__ void __launch_bounds__(kSeqThreads, 1) gdn_seq_kernel(const __grid_constant__ GdnTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t base = smem_u32(sm);
    uint64_t *bar_k = reinterpret_cast<uint64_t *>(sm + SQ_MISC);  // K (+ its low part) landed
    uint64_t *bar_in = bar_k + 1;                                  // [2]: V and the image of buffer b landed
    uint64_t *bar_g1 = bar_k + 3;                                  // [O | U] products done
    uint64_t *bar_s = bar_k + 4;                                   // state update done
    uint64_t *bar_o = bar_k + 5;                                   // output update done
    uint64_t *bar_drain = bar_k + 6;                               // every issued MMA done (abort path)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_k + 7);

    const int h = blockIdx.x, gi = blockIdx.z;
    const int n = longest_first(p.cu, gridDim.y, blockIdx.y, reinterpret_cast<int *>(sm + SQ_IMG));
    const int h_k = p.h_k, h_v = p.h_v;
    const int hk = h / (h_v / h_k);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool mover = warp < 8;              // warps 0-7
    const int quad = warp & 3, half = (warp >> 2) & 1;
    const int row = quad * 32 + lane;
    int bos, eos;
    // every CTA waits for the prep grid before it exits, so that this grid's
    // completion implies the prep's for the work that follows in the stream
    if (!seq_bounds(p.cu, n, p.total, p.max_len, p.status, bos, eos)) {
        grid_dependency_wait();
        return;
    }
    const int len = eos - bos;
    const int nchunks = (len + C - 1) / C;
    constexpr int d = 64 * DH;
    const size_t sbase = (size_t(n) * h_v + h) * d * d;
    const long long s_elems = (long long)p.n_seqs * h_v * d * d, o_elems = (long long)p.total * h_v * d;
    const float *h0 = p.h0[gi];
    float *s_out = p.s_out[gi];

    if (nchunks == 0) {
        if (mover) state_passthrough<DH>(h0, s_out, sbase, tid, s_elems, p.status);
        grid_dependency_wait();
        return;
    }

    if (tid == kIssuer) {
        for (int i = 0; i < 7; ++i) mbar_init(bar_k + i, 1);
        fence_mbar_init();
    }
    if (DH == 1) {  // d = 64: the upper halves of the K and V tiles are never loaded and stay zero
        for (int e = tid; e < 3 * 512; e += kSeqThreads) {
            const uint32_t tile = e < 512 ? SQ_K + 8192 : (e < 1024 ? SQ_V + 8192 : SQ_V + 16384 + 8192);
            *reinterpret_cast<uint4 *>(sm + tile + (e & 511) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_async_smem();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // S fp32 in columns 0-127; per chunk parity a 128-column pair [O | U]; the bf16
    // copy of S in 384-447; U (bf16) in 448-479
    const uint32_t RS = tmem, RO0 = tmem + 128, RO1 = tmem + 256, RSB = tmem + 384, RUB = tmem + 448;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;

    if (mover) {
        state_init<DH>(RS, lane_off, half, row, h0, sbase, s_elems, p.status);
        clear_o(RO0, lane_off, half);
        clear_o(RO1, lane_off, half);
    }

    const CUtensorMap *mk = &p.k[gi], *mv = &p.v[gi], *mkl = &p.kl[gi], *mvl = &p.vl[gi];
    const uint8_t *img = p.img + (size_t(gi) * p.slots * h_v + h) * kImg;
    auto img_of = [&](int c) {
        int sl = chunk_slot(bos, n, c);
        if (!SR_IN_BOUNDS(sl, p.slots, p.status)) sl = 0;  // checked build: a slot past the images reads slot 0
        return img + size_t(sl) * h_v * kImg;
    };
    auto issue_k = [&](int c) {
        const int y = bos + c * C;
        mbar_arrive_expect_tx(bar_k, DH * (SPLIT ? 16384u : 8192u));
        tma_load_2d(sm + SQ_K, mk, bar_k, hk * d, y);
        if (DH == 2) tma_load_2d(sm + SQ_K + 8192, mk, bar_k, hk * d + 64, y);
        if (SPLIT) {
            tma_load_2d(sm + SQ_KL, mkl, bar_k, hk * d, y);
            if (DH == 2) tma_load_2d(sm + SQ_KL + 8192, mkl, bar_k, hk * d + 64, y);
        }
    };
    // V (+ low part) and the chunk image into buffer c & 1, on one barrier; the
    // two halves may be issued apart (the image only after the prep grid is done)
    auto issue_v = [&](int c) {
        const int y = bos + c * C, b = c & 1;
        uint64_t *bar = &bar_in[b];
        mbar_arrive_expect_tx(bar, DH * (SPLIT ? 16384u : 8192u) + (p.want_o ? kImg : 16384u + (kImg - IMG_T2H)));
        tma_load_2d(sm + SQ_V + 16384 * b, mv, bar, h * d, y);
        if (DH == 2) tma_load_2d(sm + SQ_V + 16384 * b + 8192, mv, bar, h * d + 64, y);
        if (SPLIT) {
            tma_load_2d(sm + SQ_VL + 16384 * b, mvl, bar, h * d, y);
            if (DH == 2) tma_load_2d(sm + SQ_VL + 16384 * b + 8192, mvl, bar, h * d + 64, y);
        }
    };
    auto issue_img = [&](int c) {
        const int b = c & 1;
        uint64_t *bar = &bar_in[b];
        if (p.want_o) {
            bulk_load(sm + SQ_IMG + SQ_IMG_STRIDE * b, img_of(c), kImg, bar);
        } else {
            // no o: only -W, T2 (hi and lo) and the decay factors; P and Qg were not formed
            // (the products that read their slots feed only the O accumulator, never output)
            uint8_t *dsm = sm + SQ_IMG + SQ_IMG_STRIDE * b;
            const uint8_t *src = img_of(c);
            bulk_load(dsm + IMG_QGW + 8192, src + IMG_QGW + 8192, 8192, bar);
            bulk_load(dsm + IMG_QGW + 24576, src + IMG_QGW + 24576, 8192, bar);
            bulk_load(dsm + IMG_T2H, src + IMG_T2H, kImg - IMG_T2H, bar);
        }
    };
    auto issue_in = [&](int c) {
        issue_v(c);
        issue_img(c);
    };
    if (tid == kIssuer) {
        prefetch_tmap(mk); prefetch_tmap(mv);
        if (SPLIT) { prefetch_tmap(mkl); prefetch_tmap(mvl); }
        issue_k(0);
        issue_v(0);
        if (nchunks > 1) issue_v(1);
        grid_dependency_wait();  // the images are the prep grid's output
        issue_img(0);
        if (nchunks > 1) issue_img(1);
    }

    __nv_bfloat16 *o = p.o[gi];
    const size_t v_stride = size_t(h_v) * d;

    auto wait_on = [&](uint64_t *bar, int parity) -> bool {
        const bool w = mbar_wait(bar, uint32_t(parity & 1));
        tc_fence_after();
        return w;
    };
    // block barrier that also tells every thread whether any thread's wait failed
    auto check = [&](bool w) -> bool { return __syncthreads_or(!w) != 0; };

    bool ok = true, carry = true;  // carry: this thread's wait for the previous state update
    int c = 0;
    for (; c < nchunks; ++c) {
        const int b = c & 1;
        const uint32_t img_b = SQ_IMG + SQ_IMG_STRIDE * b;
        const float *gate = reinterpret_cast<const float *>(sm + img_b + IMG_GATE);  // e^{gamma_C - gamma_t}, e^{gamma_C}
        const uint32_t RO = (c & 1) ? RO1 : RO0, RO_prev = (c & 1) ? RO0 : RO1, RU = RO + 64;
        // ---- this chunk's V and image: U^T = V^T T2^T (state-free) is issued while
        // the movers copy S to bf16 in tensor memory and decay it
        bool w = wait_on(&bar_in[b], c >> 1) && carry;
        if (tid == kIssuer && w)
            mma_ut_s<SPLIT>(base, SQ_V + 16384 * b, SQ_VL + 16384 * b, img_b + IMG_T2H, img_b + IMG_T2L, RU);
        if (mover && w) state_copy_t(RS, RSB, lane_off, half, gate[C]);
        tc_fence_before();
        if (check(w)) { ok = false; break; }

        // ---- [O(c) | U^T] += S [Qg ; -W]^T  (O(c) starts cleared)
        if (tid == kIssuer) {
            tc_fence_after();
            mma_sqw_t(base, RSB, img_b + IMG_QGW, RO);
            mma_commit(bar_g1);
        }
        // ---- meanwhile: o of the previous chunk, its accumulator cleared for chunk
        // c + 1, and the next chunk's inputs into the other buffer, whose last reader
        // (O(c - 1)'s update) is then done
        w = true;
        if (c > 0) {
            w = wait_on(bar_o, c - 1);
            if (tid == kIssuer && w && c + 1 < nchunks) issue_in(c + 1);
            if (mover && w) {
                if (o) {
                    out_direct<DH>(RO_prev, lane_off, half, row, o, size_t(bos) + size_t(c - 1) * C, C, v_stride, h,
                                   o_elems, p.status, true);
                } else {
                    clear_o(RO_prev, lane_off, half);
                }
            }
        }
        w = wait_on(bar_g1, c) && w;
        // ---- U diag(e^{gamma_C - gamma}) (hi + lo) and U (bf16), in tensor memory
        if (mover && w) convert_u_t(RU, RUB, lane_off, half, gate);
        tc_fence_before();
        if (check(w)) { ok = false; break; }

        // ---- S += (U diag)^T K, then right behind it O(c) += U^T P^T (off the chain)
        if (tid == kIssuer) {
            w = mbar_wait(bar_k, uint32_t(c & 1));
            tc_fence_after();
            if (w) {
                mma_s_update_t<SPLIT>(base, SQ_K, SQ_KL, RU, RS);
                mma_commit(bar_s);
                mma_o_update_t(base, RUB, img_b + IMG_P, RO);
                mma_commit(bar_o);
            }
        }
        if (tid != kIssuer) w = true;
        carry = wait_on(bar_s, c) && w;
        if (tid == kIssuer && carry && c + 1 < nchunks) issue_k(c + 1);  // K's last reader is done
    }
    if (ok) ok = __syncthreads_and(carry) != 0;

    if (ok) {
        const int cl = nchunks - 1;
        const bool w = wait_on(bar_o, cl);
        if (mover && o && w)
            out_direct<DH>(cl & 1 ? RO1 : RO0, lane_off, half, row, o, size_t(bos) + size_t(cl) * C, len - cl * C,
                           v_stride, h, o_elems, p.status, false);
        if (!w && tid == kIssuer) atomicOr(p.status, SR_DEV_TIMEOUT);
        if (mover) state_out<DH>(RS, lane_off, half, row, s_out, sbase, s_elems, p.status);
    } else if (tid == kIssuer) {
        // let every MMA this thread issued, and in-flight copies, finish before tensor
        // and shared memory are released
        atomicOr(p.status, SR_DEV_TIMEOUT);
        mma_commit(bar_drain);
        mbar_wait(bar_drain, 0);
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

template <bool SPLIT, int DH>
cudaError_t launch(const GdnTcParams &p, int n_groups, int n_seqs, cudaStream_t st) {
    if (!p.img) {
        const int smem = int(smem_fused(SPLIT));
        cudaError_t e =
            cudaFuncSetAttribute(gdn_tc_kernel<SPLIT, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        gdn_tc_kernel<SPLIT, DH><<<dim3(p.h_v, n_seqs, n_groups), kThreads, smem, st>>>(p);
        return cudaGetLastError();
    }
    const int s1 = int(smem_prep()), s2 = int(smem_seq());
    cudaError_t e =
        cudaFuncSetAttribute(gdn_prep_kernel<SPLIT, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, s1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gdn_seq_kernel<SPLIT, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, s2);
    if (e != cudaSuccess) return e;
    gdn_prep_kernel<SPLIT, DH><<<dim3(p.slots, p.h_v, n_groups), kThreads, s1, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // the state chain as the prep's programmatic dependent: its CTAs take their
    // SMs, tensor memory, initial state and first K and V tiles while the prep's
    // last units run, and wait for the prep grid only before loading an image
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.h_v, n_seqs, n_groups);
    cfg.blockDim = dim3(kSeqThreads);
    cfg.dynamicSmemBytes = size_t(s2);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, gdn_seq_kernel<SPLIT, DH>, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

int image_slots(int total, int n_seqs) { return total / C + n_seqs; }

}  // namespace

// d = 128 natively; d = 64 runs the same kernels with the upper half of every
// 128-wide K, Q and V tile left at zero, which keeps the upper rows and
// columns of the state, W and U at zero (split precision: d = 128 only).
bool gdn_tc_supported(int d) { return d == 128 || d == 64; }

size_t gdn_tc_image_bytes(int total, int n_seqs, int h_v, int n_groups) {
    return size_t(n_groups) * size_t(image_slots(total, n_seqs)) * size_t(h_v) * kImg;
}

cudaError_t gdn_tc_batch(const GdnBatch &b, int n_groups, int n_seqs, int d, bool split, cudaStream_t st) {
    if (n_seqs == 0 || n_groups == 0 || b.total == 0) return gdn_chunked_batch(b, n_groups, n_seqs, d, split, st);
    if (b.h_v > 65535 || !gdn_tc_supported(d) || (split && d != 128)) return cudaErrorInvalidValue;
    GdnTcParams p{};
    const int T = b.total, qkw = b.h_k * d, vw = b.h_v * d;
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
    p.img = static_cast<uint8_t *>(b.img);
    p.total = b.total;
    p.max_len = b.max_len;
    p.h_k = b.h_k;
    p.h_v = b.h_v;
    p.n_seqs = n_seqs;
    p.slots = image_slots(b.total, n_seqs);
    p.d = d;
    p.want_o = 0;
    for (int g = 0; g < n_groups; ++g) p.want_o |= b.o[g] != nullptr;
    p.scale = b.scale;
    p.status = b.status;
    if (split) return launch<true, 2>(p, n_groups, n_seqs, st);
    return d == 128 ? launch<false, 2>(p, n_groups, n_seqs, st) : launch<false, 1>(p, n_groups, n_seqs, st);
}

cudaError_t gdn_tc(const sr_gdn_args &a, float scale, uint32_t *status, void *img, cudaStream_t st) {
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
    b.img = img;
    b.total = a.total_tokens;
    b.max_len = a.max_seqlen;
    b.h_k = a.h_k;
    b.h_v = a.h_v;
    b.scale = scale;
    b.status = status;
    return gdn_tc_batch(b, 1, a.n_seqs, a.d_k, false, st);
}

}  // namespace sr
