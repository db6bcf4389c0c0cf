// Persistent, warp-specialised tcgen05 GEMM for the replay group's dense
// projections:  C[M, N] = A[M, K] * B[N, K]^T  (bf16 in, fp32 accumulate in
// tensor memory), with the epilogue fused:
//   EPI_STORE         C = A B^T                       bf16 out
//   EPI_RESIDUAL      C = R + A B^T                   bf16 out
//   EPI_SWIGLU        C = SiLU(r A Bg^T) * (r A Bu^T) bf16 out, optional lo part   (MLP gate/up)
//   EPI_F32_ROWSCALE  C = r A B^T                     fp32 out                     (in_proj)
//   EPI_F32_RESIDUAL  C += A B^T                      fp32 in place                (out_proj, down)
//                     and optionally the next RMSNorm's operand from the new C:
//                     C * w as hi + lo, and each row's sum of C^2 over the tile
// r is an optional fp32 per-row scale (the folded RMSNorm factor), given as
// such or formed from the producing GEMM's per-tile sums of squares.  With two
// passes the A operand is an exact hi + lo pair of bf16 matrices
// (A = A_hi + A_lo) and both products accumulate into the same TMEM tile, so
// the result carries ~16 mantissa bits of the activations: the weights are
// exact bf16, so A_hi B^T + A_lo B^T is the product of the unrounded A.
// Roles: warp 0 issues TMA loads (128-byte swizzle) into a 4-stage ring,
// warp 1 allocates TMEM and issues tcgen05.mma (M=128, N=256, K=16) from one
// thread, warps 2-5 drain the double-buffered TMEM accumulator (2 x 256
// columns) with tcgen05.ld and apply the epilogue while the next tile's MMAs
// run; each epilogue warp stages its outputs 32 x 32 at a time in shared
// memory and writes them with TMA stores.  Tiles walk M fastest so CTAs
// running together share the weight tile through L2.  Several problems with
// identical shapes (one per replay group) are scheduled as one launch.  A
// second form (gemm_pair_kernel, below) computes 256 x 256 tiles with a
// cluster of two CTAs and cta_group::2 products.  Every mbarrier wait is
// bounded; on timeout the kernel records SR_DEV_TIMEOUT, drains its MMAs,
// frees TMEM and exits.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

#include <cuda_fp8.h>

namespace sr {

namespace {

constexpr int BM = 128, BK = 64;
constexpr int kTileA = BM * BK * 2;  // 16 KB
constexpr int kThreads = 192;
// Staging of the epilogue's outputs, per epilogue warp (its 32 rows x 32 columns
// per step): fp32 4 KB at 0, bf16 hi 2 KB at 4 KB, low part (<= 2 KB) at 6 KB.
constexpr int kStageWarpBytes = 8192;
constexpr int kEpiStageBytes = 4 * kStageWarpBytes;
// Tile width BN fixes the stage count (the launcher uses 256).
template <int BN> struct Cfg {
    static constexpr int STAGES = BN == 256 ? 4 : 6;
    static constexpr int kTileB = BN * BK * 2;
    static constexpr int kSmemBytes = STAGES * (kTileA + kTileB) + kEpiStageBytes + 1024 /*align*/ + 256 /*barriers*/;
};

struct Problem {
    CUtensorMap a;   // [M, K], box {64, 128}
    CUtensorMap a_lo;  // [M, K] low part of A (second pass), box {64, 128}
    CUtensorMap b0;  // [N, K] box {64, 256}; gate [N, K] box {64, 128} for SwiGLU
    CUtensorMap b1;  // up [N, K] box {64, 128} (SwiGLU only)
    CUtensorMap b0_lo;  // fp8 low pass: e5m2 bytes of b0 * 2^-8, box {128 B, as b0}
    CUtensorMap b1_lo;  // fp8 low pass: e5m2 bytes of b1 * 2^-8 (SwiGLU only)
    // outputs of the staged epilogue, written by TMA stores of 32 x 32 boxes:
    CUtensorMap o_f32;  // fp32 C (EPI_F32_*), 128-byte swizzle; also the residual's loads
    CUtensorMap o_hi;   // bf16 hi part: SwiGLU C, or the next norm's n_hi; 64-byte swizzle
    CUtensorMap o_lo;   // its low part: e4m3 bytes (32-byte swizzle) or bf16 (64-byte swizzle)
    void *c;
    const __nv_bfloat16 *r;
    void *c_lo;              // SwiGLU: low part of the output (bf16, or e4m3 of lo * 2^8; may be null)
    const float *rowscale;   // per-row scale (may be null)
    const float *ssq_in;     // per-row partial sums of squares -> RMSNorm row scale (may be null)
    const __nv_bfloat16 *nw; // EPI_F32_RESIDUAL: next norm weight (may be null)
    __nv_bfloat16 *n_hi;     // x * nw, hi part, row pitch N
    void *n_lo;              // low part (bf16, or e4m3 of lo * 2^8; may be null)
    float *ssq_out;          // [n_tiles, M] sums of x^2 per N-tile
};

struct Params {
    Problem prob[kMaxGemmProblems];
    int n_problems;
    int M, N, K;  // N = output columns
    int ldc;      // row pitch of C and R in elements
    int m_tiles, n_tiles;
    int epi;
    int n_pass;  // 1: A; 2: A_hi then A_lo
    int lo_fp8;  // the A_lo pass on the fp8 tensor cores (128-byte K blocks of 128 elements)
    int ssq_parts;  // partial sums per row in ssq_in
    float eps;      // RMSNorm epsilon of the row scale formed from ssq_in
    int nt_skip_at, nt_skip;  // N tiles nt_skip_at .. + nt_skip - 1 are not computed (n_tiles excludes them)
    int ssq_slots;  // partial sums per row written by the next-norm epilogue: one per 256-column tile
    uint32_t *status;
};

// Problem, N tile and M tile of work item `tile` (M tiles fastest).
__device__ __forceinline__ void decode_tile(const Params &p, int tile, int &pi, int &nt, int &mt) {
    const int tiles_per_prob = p.m_tiles * p.n_tiles;
    pi = tile / tiles_per_prob;
    const int rem = tile % tiles_per_prob;
    nt = rem / p.m_tiles;
    mt = rem % p.m_tiles;
    if (nt >= p.nt_skip_at) nt += p.nt_skip;
}

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ float silu(float x) { return x / (1.f + __expf(-x)); }
// Eight low parts -> eight e4m3 bytes of lo * 2^8 (round to nearest, saturating).
__device__ __forceinline__ uint2 lo8_pack8(const float (&lo)[8]) {
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const __nv_fp8x2_storage_t a = __nv_cvt_float2_to_fp8x2(make_float2(lo[4 * h] * 256.f, lo[4 * h + 1] * 256.f),
                                                               __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t b = __nv_cvt_float2_to_fp8x2(
            make_float2(lo[4 * h + 2] * 256.f, lo[4 * h + 3] * 256.f), __NV_SATFINITE, __NV_E4M3);
        w[h] = uint32_t(a) | (uint32_t(b) << 16);
    }
    return make_uint2(w[0], w[1]);
}

// Abort-aware bounded wait: gives up after tc::kWaitLimitNs, or as soon as
// another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t phase, volatile int *abort_flag) {
    if (tc::mbar_try_wait(bar, phase)) return true;
    const uint64_t t0 = tc::globaltimer_ns();
    for (;;) {
        for (int i = 0; i < 32; ++i)
            if (tc::mbar_try_wait(bar, phase)) return true;
        if (*abort_flag || tc::globaltimer_ns() - t0 > tc::kWaitLimitNs) return false;
    }
}

// Byte offset of 16-byte chunk v of row r in a staging box whose rows are 128,
// 64 or 32 bytes, under the TMA swizzle of that row size (the chunk index XOR
// address bits 7.. of the row start; boxes start 1024-byte aligned).
__device__ __forceinline__ uint32_t sw128(int r, int v) { return uint32_t(r * 128 + ((v ^ (r & 7)) << 4)); }
__device__ __forceinline__ uint32_t sw64(int r, int v) { return uint32_t(r * 64 + ((v ^ ((r >> 1) & 3)) << 4)); }
__device__ __forceinline__ uint32_t sw32(int r, int v) { return uint32_t(r * 32 + ((v ^ ((r >> 2) & 1)) << 4)); }

// RMSNorm row factor of the calling thread's row: from the producer's per-tile
// sums of squares (added in order), or given, or 1.
__device__ __forceinline__ float row_scale(const Params &p, const Problem &pr, int row) {
    if (row >= p.M) return 1.f;
    if (pr.ssq_in) {
        float ss = 0.f;
        for (int t = 0; t < p.ssq_parts; ++t)
            if (SR_IN_BOUNDS(size_t(t) * p.M + row, (long long)p.ssq_parts * p.M, p.status))
                ss += pr.ssq_in[size_t(t) * p.M + row];
        return 1.f / sqrtf(ss / float(p.K) + p.eps);
    }
    return pr.rowscale ? pr.rowscale[row] : 1.f;
}

// x (8 values) -> bf16 hi in `hi` and the low part as bf16 in `lo` and as e4m3
// bytes of lo * 2^8 in `lo8`.
__device__ __forceinline__ void split8(const float (&x)[8], uint4 &hi, uint4 &lo, uint2 &lo8) {
    uint32_t w[4], wl[4];
    float l[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        w[e] = pack2(x[2 * e], x[2 * e + 1]);
        l[2 * e] = x[2 * e] - bf_lo(w[e]);
        l[2 * e + 1] = x[2 * e + 1] - bf_hi(w[e]);
        wl[e] = pack2(l[2 * e], l[2 * e + 1]);
    }
    hi = make_uint4(w[0], w[1], w[2], w[3]);
    lo = make_uint4(wl[0], wl[1], wl[2], wl[3]);
    lo8 = lo8_pack8(l);
}

// Staged epilogue of one output tile for one warp's 32 rows (row0 + lane): per
// 32 accumulator columns, the warp writes its outputs into its staging boxes in
// shared memory and one lane stores each box with a TMA store (coalesced, and
// clipped at the tensor's bounds); the residual of EPI_F32_RESIDUAL comes in by
// a TMA load of the same box.  `width` accumulator columns at tbase (SwiGLU:
// gate products in the first half, up products in the second) produce output
// columns col0..; with the next norm's operand, the row's sum of squares over
// those columns goes to partial-sum slot ssq_slot.  Returns false if the
// residual's load timed out.
__device__ __forceinline__ bool epilogue_staged(const Params &p, const Problem &pr, uint32_t tbase, int row0,
                                                int lane, int width, int col0, int ssq_slot, uint8_t *stg,
                                                uint64_t *rbar, uint32_t &rphase) {
    // a warp whose 32 rows all lie past M has nothing to write (and issues no
    // store that would start outside the tensor)
    if (row0 >= p.M) return true;
    const int row = row0 + lane;
    const float rs = row_scale(p, pr, row);
    uint8_t *sf = stg, *sh = stg + 4096, *sl = stg + 6144;
    const bool f8 = p.lo_fp8 != 0;
    bool ok = true;
    if (p.epi == EPI_SWIGLU) {
        const bool has_lo = pr.c_lo != nullptr;
#pragma unroll 1
        for (int c = 0; c < width / 2 && col0 + c < p.N; c += 32) {
            uint32_t g[32], u[32];
            tc::tmem_ld_32x32b_x32(tbase + c, g);
            tc::tmem_ld_32x32b_x32(tbase + width / 2 + c, u);
            if (lane == 0) tc::bulk_wait_read();  // the previous boxes have left shared memory
            __syncwarp();
            tc::tmem_ld_wait();
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                float h[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    h[e] = silu(rs * __uint_as_float(g[8 * v + e])) * (rs * __uint_as_float(u[8 * v + e]));
                uint4 hi, lo;
                uint2 lo8;
                split8(h, hi, lo, lo8);
                *reinterpret_cast<uint4 *>(sh + sw64(lane, v)) = hi;
                if (has_lo && !f8) *reinterpret_cast<uint4 *>(sl + sw64(lane, v)) = lo;
                if (has_lo && f8) *reinterpret_cast<uint2 *>(sl + sw32(lane, v >> 1) + 8 * (v & 1)) = lo8;
            }
            tc::fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                tc::tma_store_2d(&pr.o_hi, sh, col0 + c, row0);
                if (has_lo) tc::tma_store_2d(&pr.o_lo, sl, col0 + c, row0);
                tc::bulk_commit();
            }
        }
    } else {
        const bool resid = p.epi == EPI_F32_RESIDUAL;
        const bool norm_out = resid && pr.nw != nullptr;
        const bool has_lo = norm_out && pr.n_lo != nullptr;
        float ssq = 0.f;
#pragma unroll 1
        for (int c = 0; c < width && col0 + c < p.N; c += 32) {
            const int col = col0 + c;
            if (lane == 0) {
                tc::bulk_wait_read();  // the previous boxes have left shared memory
                if (resid) {
                    tc::mbar_arrive_expect_tx(rbar, 4096);
                    tc::tma_load_2d(sf, &pr.o_f32, rbar, col, row0);
                }
            }
            __syncwarp();
            uint32_t x[32];
            tc::tmem_ld_32x32b_x32(tbase + c, x);
            tc::tmem_ld_wait();
            float xv[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) xv[e] = rs * __uint_as_float(x[e]);
            if (resid) {
                if (!tc::mbar_wait(rbar, rphase)) ok = false;
                rphase ^= 1;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const float4 r = *reinterpret_cast<const float4 *>(sf + sw128(lane, v));
                    xv[4 * v] += r.x;
                    xv[4 * v + 1] += r.y;
                    xv[4 * v + 2] += r.z;
                    xv[4 * v + 3] += r.w;
                }
            }
#pragma unroll
            for (int v = 0; v < 8; ++v)
                *reinterpret_cast<float4 *>(sf + sw128(lane, v)) =
                    make_float4(xv[4 * v], xv[4 * v + 1], xv[4 * v + 2], xv[4 * v + 3]);
            if (norm_out) {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    // norm weights of columns past N read as zero (N is a multiple of 8)
                    const uint4 wq = col + 8 * v < p.N ? reinterpret_cast<const uint4 *>(pr.nw + col)[v]
                                                       : make_uint4(0u, 0u, 0u, 0u);
                    const uint32_t ww[4] = {wq.x, wq.y, wq.z, wq.w};
                    float h[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float x0 = xv[8 * v + 2 * e], x1 = xv[8 * v + 2 * e + 1];
                        ssq = fmaf(x0, x0, ssq);
                        ssq = fmaf(x1, x1, ssq);
                        h[2 * e] = x0 * bf_lo(ww[e]);
                        h[2 * e + 1] = x1 * bf_hi(ww[e]);
                    }
                    uint4 hi, lo;
                    uint2 lo8;
                    split8(h, hi, lo, lo8);
                    *reinterpret_cast<uint4 *>(sh + sw64(lane, v)) = hi;
                    if (has_lo && !f8) *reinterpret_cast<uint4 *>(sl + sw64(lane, v)) = lo;
                    if (has_lo && f8) *reinterpret_cast<uint2 *>(sl + sw32(lane, v >> 1) + 8 * (v & 1)) = lo8;
                }
            }
            tc::fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                tc::tma_store_2d(&pr.o_f32, sf, col, row0);
                if (norm_out) tc::tma_store_2d(&pr.o_hi, sh, col, row0);
                if (has_lo) tc::tma_store_2d(&pr.o_lo, sl, col, row0);
                tc::bulk_commit();
            }
        }
        const size_t si = size_t(ssq_slot) * p.M + row;
        if (norm_out && row < p.M && SR_IN_BOUNDS(si, (long long)p.ssq_slots * p.M, p.status)) pr.ssq_out[si] = ssq;
    }
    return ok;
}

// Per-thread epilogue of the bf16 test epilogues (EPI_STORE, EPI_RESIDUAL): the
// calling thread's row, `width` accumulator columns at tbase, output columns col0..
__device__ __forceinline__ void epilogue_row_bf16(const Params &p, const Problem &pr, uint32_t tbase, int row,
                                                  int width, int col0) {
    const bool row_ok = row < p.M;
    const float rs = row_scale(p, pr, row);
#pragma unroll 1
    for (int c = 0; c < width; c += 32) {
        uint32_t x[32];
        tc::tmem_ld_32x32b_x32(tbase + c, x);
        tc::tmem_ld_wait();
        const int col = col0 + c;
        const int nvec = min(4, (p.N - col) / 8);
        if (!row_ok || nvec <= 0) continue;
        if (!SR_IN_BOUNDS(size_t(row) * p.ldc + col + 8 * nvec - 1, (long long)p.M * p.ldc, p.status)) continue;
        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(pr.c) + size_t(row) * p.ldc + col);
        const uint4 *res =
            p.epi == EPI_RESIDUAL ? reinterpret_cast<const uint4 *>(pr.r + size_t(row) * p.ldc + col) : nullptr;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            if (v >= nvec) break;
            uint32_t rr[4] = {0u, 0u, 0u, 0u};
            if (res) {
                const uint4 rv = res[v];
                rr[0] = rv.x; rr[1] = rv.y; rr[2] = rv.z; rr[3] = rv.w;
            }
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = v * 8 + e * 2;
                w[e] = pack2(bf_lo(rr[e]) + rs * __uint_as_float(x[j]), bf_hi(rr[e]) + rs * __uint_as_float(x[j + 1]));
            }
            dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// Epilogue of one output tile for one epilogue warp (rows row0 .. row0 + 31).
__device__ __forceinline__ bool epilogue_warp(const Params &p, const Problem &pr, uint32_t tbase, int row0, int lane,
                                              int width, int col0, int ssq_slot, uint8_t *stg, uint64_t *rbar,
                                              uint32_t &rphase) {
    if (p.epi == EPI_STORE || p.epi == EPI_RESIDUAL) {
        epilogue_row_bf16(p, pr, tbase, row0 + lane, width, col0);
        return true;
    }
    return epilogue_staged(p, pr, tbase, row0, lane, width, col0, ssq_slot, stg, rbar, rphase);
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ Params p) {
    constexpr int STAGES = Cfg<BN>::STAGES;
    constexpr int kTileB = Cfg<BN>::kTileB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + STAGES * kTileA;
    uint8_t *stage_out = sB + STAGES * kTileB;  // the epilogue warps' staging boxes (1024-aligned)
    uint64_t *full = reinterpret_cast<uint64_t *>(stage_out + kEpiStageBytes);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint64_t *rbar = drain + 1;  // [4] residual loads of the epilogue warps
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(rbar + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&tfull[b], 1);
            tc::mbar_init(&tempty[b], 4);
        }
        tc::mbar_init(drain, 1);
        for (int w = 0; w < 4; ++w) tc::mbar_init(&rbar[w], 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 2 * BN);
        tc::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < p.n_problems; ++i) {
            tc::prefetch_tmap(&p.prob[i].a);
            if (p.n_pass == 2) tc::prefetch_tmap(&p.prob[i].a_lo);
            if (p.lo_fp8) {
                tc::prefetch_tmap(&p.prob[i].b0_lo);
                if (p.epi == EPI_SWIGLU) tc::prefetch_tmap(&p.prob[i].b1_lo);
            }
            tc::prefetch_tmap(&p.prob[i].b0);
            if (p.epi == EPI_SWIGLU) tc::prefetch_tmap(&p.prob[i].b1);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int tiles_per_prob = p.m_tiles * p.n_tiles;
    const int total = p.n_problems * tiles_per_prob;
    const int kblocks = p.K / BK;
    // k blocks of the low pass: 64 bf16 or 128 fp8 elements, 128 bytes per row either way
    const int kblocks_lo = p.n_pass == 2 ? (p.lo_fp8 ? p.K / (2 * BK) : kblocks) : 0;
    const int kblocks_all = kblocks + kblocks_lo;
    auto fail = [&]() {
        *abort_flag = 1;
        atomicOr(p.status, SR_DEV_TIMEOUT);
    };

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
                int pi, nt, mt;
                decode_tile(p, tile, pi, nt, mt);
                const Problem &pr = p.prob[pi];
                for (int kk = 0; kk < kblocks_all; ++kk) {
                    const bool lo = kk >= kblocks;
                    const bool f8 = lo && p.lo_fp8;
                    const int kb = lo ? kk - kblocks : kk;
                    const int kx = f8 ? kb * 2 * BK : kb * BK;  // element column of the 128-byte block
                    const CUtensorMap *mb0 = f8 ? &pr.b0_lo : &pr.b0, *mb1 = f8 ? &pr.b1_lo : &pr.b1;
                    if (!wait_or_abort(&empty[stage], phase ^ 1, abort_flag)) { fail(); break; }
                    tc::mbar_arrive_expect_tx(&full[stage], kTileA + kTileB);
                    tc::tma_load_2d(sA + stage * kTileA, lo ? &pr.a_lo : &pr.a, &full[stage], kx, mt * BM);
                    if (p.epi == EPI_SWIGLU) {
                        tc::tma_load_2d(sB + stage * kTileB, mb0, &full[stage], kx, nt * (BN / 2));
                        tc::tma_load_2d(sB + stage * kTileB + (BN / 2) * BK * 2, mb1, &full[stage], kx,
                                        nt * (BN / 2));
                    } else {
                        tc::tma_load_2d(sB + stage * kTileB, mb0, &full[stage], kx, nt * BN);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
                // a last N tile narrower than BN runs products of its own width (a multiple of 16)
                int pi, nt, mt;
                decode_tile(p, tile, pi, nt, mt);
                const int ncols = p.epi == EPI_SWIGLU ? BN : min(BN, (p.N - nt * BN + 15) / 16 * 16);
                const uint32_t idesc = tc::idesc_bf16_f32(BM, ncols);
                const uint32_t idesc_f8 = tc::idesc_e4m3_e5m2_f32(BM, ncols);
                if (!wait_or_abort(&tempty[acc], acc_phase ^ 1, abort_flag)) { fail(); break; }
                tc::tc_fence_after();
                const uint32_t d = tmem + uint32_t(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < kblocks_all; ++kb) {
                    if (!wait_or_abort(&full[stage], phase, abort_flag)) { fail(); ok = false; break; }
                    tc::tc_fence_after();
                    const uint32_t a0 = tc::smem_u32(sA + stage * kTileA);
                    const uint32_t b0 = tc::smem_u32(sB + stage * kTileB);
                    // four MMAs per 128-byte block: K = 16 bf16 or K = 32 fp8 elements, 32 bytes apart
                    if (p.lo_fp8 && kb >= kblocks) {
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            tc::mma_f8_ss(d, tc::sdesc_k_sw128(a0 + k * 32), tc::sdesc_k_sw128(b0 + k * 32), idesc_f8,
                                          1);
                    } else {
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k)
                            tc::mma_bf16_ss(d, tc::sdesc_k_sw128(a0 + k * 32), tc::sdesc_k_sw128(b0 + k * 32), idesc,
                                            (kb | k) != 0);
                    }
                    tc::mma_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc::mma_commit(&tfull[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
            // all MMAs issued by this thread complete before TMEM is released
            tc::mma_commit(drain);
            if (!tc::mbar_wait(drain, 0)) atomicOr(p.status, SR_DEV_TIMEOUT);
        }
    } else {
        const int quad = warp & 3;  // TMEM lane quadrant this warp may access
        uint8_t *stg = stage_out + (warp - 2) * kStageWarpBytes;
        uint64_t *rb = &rbar[warp - 2];
        uint32_t rphase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
            int pi, nt, mt;
            decode_tile(p, tile, pi, nt, mt);
            const Problem &pr = p.prob[pi];
            if (!wait_or_abort(&tfull[acc], acc_phase, abort_flag)) { fail(); break; }
            tc::tc_fence_after();
            const bool ok = epilogue_warp(p, pr, tmem + (uint32_t(quad * 32) << 16) + uint32_t(acc * BN),
                                          mt * BM + quad * 32, lane, BN, p.epi == EPI_SWIGLU ? nt * (BN / 2) : nt * BN,
                                          nt, stg, rb, rphase);
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tempty[acc]);
            if (!ok) { fail(); break; }
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
        if (lane == 0) tc::bulk_wait_all();  // the output boxes are written before the CTA leaves
    }

    if (*abort_flag) {
        // let TMA copies already in flight land before the shared memory is released
        for (int i = 0; i < 64; ++i) __nanosleep(1000);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 2 * BN);
    }
}

// ------------------------------------------------------------------ CTA pairs
// The same GEMM with each output tile of 256 rows x 256 columns computed by a
// cluster of two CTAs on two SMs through cta_group::2 products: CTA r of the
// pair loads rows r*128.. of the tile's A rows and its half of the tile's B
// rows (for SwiGLU: the gate rows in CTA 0, the up rows in CTA 1) into its own
// shared memory, and holds rows r*128.. of the accumulator in its own tensor
// memory.  Each SM thus streams 32 KB per 64-deep K block instead of 48 KB,
// for the same tensor work.  The even CTA issues every product; both CTAs'
// loads signal its stage barriers, its commits arrive at both CTAs' stage and
// accumulator barriers, and both CTAs' epilogue warps release its accumulator
// buffers.  The arithmetic of every output element (the K blocks in order,
// fp32 accumulation in tensor memory) is that of the single-CTA form.
constexpr int kPairStages = 6;
constexpr int kPairSmemBytes = kPairStages * 2 * kTileA + kEpiStageBytes + 1024 /*align*/ + 256 /*barriers*/;

__device__ __forceinline__ bool wait_or_abort_cluster(uint64_t *bar, uint32_t phase, volatile int *abort_flag) {
    if (tc::mbar_try_wait_cluster(bar, phase)) return true;
    const uint64_t t0 = tc::globaltimer_ns();
    for (;;) {
        for (int i = 0; i < 32; ++i)
            if (tc::mbar_try_wait_cluster(bar, phase)) return true;
        if (*abort_flag || tc::globaltimer_ns() - t0 > tc::kWaitLimitNs) return false;
    }
}

__global__ void __launch_bounds__(kThreads, 1) gemm_pair_kernel(const __grid_constant__ Params p) {
    constexpr int BN = 256, STAGES = kPairStages, kTileB = kTileA;  // B: this CTA's 128 rows
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + STAGES * kTileA;
    uint8_t *stage_out = sB + STAGES * kTileB;  // the epilogue warps' staging boxes (1024-aligned)
    uint64_t *full = reinterpret_cast<uint64_t *>(stage_out + kEpiStageBytes);  // used in the even CTA
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 2;  // used in the even CTA: 4 epilogue warps of each CTA arrive
    uint64_t *drain = tempty + 2;
    uint64_t *rbar = drain + 1;  // [4] residual loads of the epilogue warps
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(rbar + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = tc::cluster_ctarank();
    const bool leader = rank == 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&tfull[b], 1);
            tc::mbar_init(&tempty[b], 8);
        }
        tc::mbar_init(drain, 1);
        for (int w = 0; w < 4; ++w) tc::mbar_init(&rbar[w], 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc_pair(tmem_slot, 2 * BN);
        tc::tmem_relinquish_pair();
    }
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < p.n_problems; ++i) {
            tc::prefetch_tmap(&p.prob[i].a);
            if (p.n_pass == 2) tc::prefetch_tmap(&p.prob[i].a_lo);
            if (p.lo_fp8) {
                tc::prefetch_tmap(&p.prob[i].b0_lo);
                if (p.epi == EPI_SWIGLU) tc::prefetch_tmap(&p.prob[i].b1_lo);
            }
            tc::prefetch_tmap(&p.prob[i].b0);
            if (p.epi == EPI_SWIGLU) tc::prefetch_tmap(&p.prob[i].b1);
        }
    }
    // the barriers of both CTAs are initialised before either CTA uses its pair's
    __syncwarp();
    tc::tc_fence_before();
    tc::cluster_sync();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int tiles_per_prob = p.m_tiles * p.n_tiles;  // m_tiles counts 256-row tiles here
    const int total = p.n_problems * tiles_per_prob;
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int kblocks = p.K / BK;
    const int kblocks_lo = p.n_pass == 2 ? (p.lo_fp8 ? p.K / (2 * BK) : kblocks) : 0;
    const int kblocks_all = kblocks + kblocks_lo;
    auto fail = [&]() {
        *abort_flag = 1;
        atomicOr(p.status, SR_DEV_TIMEOUT);
    };

    if (warp == 0) {
        if (lane == 0) {
            const uint32_t full0 = tc::mapa_shared(tc::smem_u32(full), 0);  // the even CTA's stage barriers
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = pair; tile < total && !*abort_flag; tile += n_pairs) {
                int pi, nt, mt;
                decode_tile(p, tile, pi, nt, mt);
                const Problem &pr = p.prob[pi];
                for (int kk = 0; kk < kblocks_all; ++kk) {
                    const bool lo = kk >= kblocks;
                    const bool f8 = lo && p.lo_fp8;
                    const int kb = lo ? kk - kblocks : kk;
                    const int kx = f8 ? kb * 2 * BK : kb * BK;
                    const CUtensorMap *mb0 = f8 ? &pr.b0_lo : &pr.b0, *mb1 = f8 ? &pr.b1_lo : &pr.b1;
                    if (!wait_or_abort(&empty[stage], phase ^ 1, abort_flag)) { fail(); break; }
                    // the even CTA's barrier expects both CTAs' bytes of the stage
                    if (leader) tc::mbar_arrive_expect_tx(&full[stage], 2 * (kTileA + kTileB));
                    const uint32_t fb = full0 + uint32_t(stage) * 8u;
                    tc::tma_load_2d_pair(sA + stage * kTileA, lo ? &pr.a_lo : &pr.a, fb, kx,
                                         mt * 2 * BM + int(rank) * BM);
                    if (p.epi == EPI_SWIGLU)
                        tc::tma_load_2d_pair(sB + stage * kTileB, leader ? mb0 : mb1, fb, kx, nt * (BN / 2));
                    else
                        tc::tma_load_2d_pair(sB + stage * kTileB, mb0, fb, kx, nt * BN + int(rank) * (BN / 2));
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            constexpr uint32_t idesc = tc::idesc_bf16_f32(2 * BM, BN);
            constexpr uint32_t idesc_f8 = tc::idesc_e4m3_e5m2_f32(2 * BM, BN);
            for (int tile = pair; tile < total && !*abort_flag; tile += n_pairs) {
                if (!wait_or_abort_cluster(&tempty[acc], acc_phase ^ 1, abort_flag)) { fail(); break; }
                tc::tc_fence_after();
                const uint32_t d = tmem + uint32_t(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < kblocks_all; ++kb) {
                    if (!wait_or_abort(&full[stage], phase, abort_flag)) { fail(); ok = false; break; }
                    tc::tc_fence_after();
                    const uint32_t a0 = tc::smem_u32(sA + stage * kTileA);
                    const uint32_t b0 = tc::smem_u32(sB + stage * kTileB);
                    if (p.lo_fp8 && kb >= kblocks) {
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            tc::mma_f8_ss_pair(d, tc::sdesc_k_sw128(a0 + k * 32), tc::sdesc_k_sw128(b0 + k * 32),
                                               idesc_f8, 1);
                    } else {
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k)
                            tc::mma_bf16_ss_pair(d, tc::sdesc_k_sw128(a0 + k * 32), tc::sdesc_k_sw128(b0 + k * 32),
                                                 idesc, (kb | k) != 0);
                    }
                    tc::mma_commit_pair(&empty[stage], 0x3);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc::mma_commit_pair(&tfull[acc], 0x3);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
            tc::mma_commit_pair(drain, 0x3);
        }
        // in both CTAs: every product writing this CTA's tensor memory has completed
        if (lane == 0 && !tc::mbar_wait(drain, 0)) atomicOr(p.status, SR_DEV_TIMEOUT);
    } else {
        const int quad = warp & 3;  // TMEM lane quadrant this warp may access
        const uint32_t tempty0 = tc::mapa_shared(tc::smem_u32(tempty), 0);
        uint8_t *stg = stage_out + (warp - 2) * kStageWarpBytes;
        uint64_t *rb = &rbar[warp - 2];
        uint32_t rphase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = pair; tile < total && !*abort_flag; tile += n_pairs) {
            int pi, nt, mt;
            decode_tile(p, tile, pi, nt, mt);
            const Problem &pr = p.prob[pi];
            if (!wait_or_abort(&tfull[acc], acc_phase, abort_flag)) { fail(); break; }
            tc::tc_fence_after();
            const bool ok = epilogue_warp(p, pr, tmem + (uint32_t(quad * 32) << 16) + uint32_t(acc * BN),
                                          mt * 2 * BM + int(rank) * BM + quad * 32, lane, BN,
                                          p.epi == EPI_SWIGLU ? nt * (BN / 2) : nt * BN, nt, stg, rb, rphase);
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive_cluster(tempty0 + uint32_t(acc) * 8u);
            if (!ok) { fail(); break; }
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
        if (lane == 0) tc::bulk_wait_all();  // the output boxes are written before the CTA leaves
    }

    if (*abort_flag) {
        // let TMA copies already in flight land before the shared memory is released
        for (int i = 0; i < 64; ++i) __nanosleep(1000);
    }
    __syncwarp();
    tc::tc_fence_before();
    tc::cluster_sync();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc_pair(tmem, 2 * BN);
    }
    // neither CTA leaves while the other may still arrive at its barriers
    __syncwarp();
    tc::cluster_sync();
}

// ------------------------------------------------------------------ host

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    // The driver entry point is looked up once per process.
    static EncodeTiledFn fn = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            ptr = nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

int sm_count() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 1;
}

}  // namespace

// 2-D bf16 tensor map over a row-major [rows, cols] matrix (row pitch `pitch`
// elements), box_cols x box_rows boxes with the 128-byte swizzle.
bool make_map_bf16(CUtensorMap *m, const void *base, int rows, int cols, int pitch, int box_cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(pitch) * 2};
    cuuint32_t box[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)};
    cuuint32_t es[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_u8(CUtensorMap *m, const void *base, int rows, int cols, int pitch, int box_cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(pitch)};
    cuuint32_t box[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)};
    cuuint32_t es[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_f32(CUtensorMap *m, const void *base, int rows, int cols, int pitch, int box_cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(pitch) * 4};
    cuuint32_t box[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)};
    cuuint32_t es[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
bool make_map(CUtensorMap *m, const void *base, int rows, int cols, int pitch, int box_rows) {
    return make_map_bf16(m, base, rows, cols, pitch, 64, box_rows);
}
// Map of an epilogue output [rows, cols] (row pitch `pitch` elements of `esize`
// bytes) in 32 x 32 boxes with the swizzle of the box's row size.
bool make_map_out(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, int rows, int cols,
                  int pitch) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(pitch) * esize};
    cuuint32_t box[2] = {32u, 32u};
    cuuint32_t es[2] = {1u, 1u};
    const CUtensorMapSwizzle sw = esize == 4   ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : esize == 2 ? CU_TENSOR_MAP_SWIZZLE_64B
                                               : CU_TENSOR_MAP_SWIZZLE_32B;
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

namespace {

// Tensor maps and scalars shared by both forms.  b_rows: rows of each weight box.
cudaError_t fill_params(Params &local, const GemmProblemDesc *probs, int n_problems, int M, int N, int K, int ldc,
                        int epi, int n_pass, int lo_fp8, uint32_t *status, GemmOptions norm, int b_rows, int bn_out,
                        int bm_tile) {
    for (int i = 0; i < n_problems; ++i) {
        const GemmProblemDesc &d = probs[i];
        if (!make_map(&local.prob[i].a, d.a, M, K, K, BM)) return cudaErrorInvalidValue;
        if (n_pass == 2) {
            const bool ok = lo_fp8 ? make_map_u8(&local.prob[i].a_lo, d.a_lo, M, K, K, 2 * BK, BM)
                                   : make_map(&local.prob[i].a_lo, d.a_lo, M, K, K, BM);
            if (!ok) return cudaErrorInvalidValue;
        }
        if (!make_map(&local.prob[i].b0, d.b0, N, K, K, b_rows)) return cudaErrorInvalidValue;
        if (epi == EPI_SWIGLU && !make_map(&local.prob[i].b1, d.b1, N, K, K, b_rows)) return cudaErrorInvalidValue;
        if (n_pass == 2 && lo_fp8) {
            if (!d.b0_lo || !make_map_u8(&local.prob[i].b0_lo, d.b0_lo, N, K, K, 2 * BK, b_rows))
                return cudaErrorInvalidValue;
            if (epi == EPI_SWIGLU && (!d.b1_lo || !make_map_u8(&local.prob[i].b1_lo, d.b1_lo, N, K, K, 2 * BK, b_rows)))
                return cudaErrorInvalidValue;
        }
        // outputs of the staged epilogue
        const bool lo8 = n_pass == 2 && lo_fp8;
        bool ok_out = true;
        if (epi == EPI_F32_ROWSCALE || epi == EPI_F32_RESIDUAL)
            ok_out = make_map_out(&local.prob[i].o_f32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d.c, M, N, ldc);
        if (ok_out && epi == EPI_F32_RESIDUAL && d.nw) {
            ok_out = make_map_out(&local.prob[i].o_hi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.n_hi, M, N, N);
            if (ok_out && d.n_lo)
                ok_out = lo8 ? make_map_out(&local.prob[i].o_lo, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d.n_lo, M, N, N)
                                : make_map_out(&local.prob[i].o_lo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.n_lo, M, N, N);
        }
        if (ok_out && epi == EPI_SWIGLU) {
            ok_out = make_map_out(&local.prob[i].o_hi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.c, M, N, ldc);
            if (ok_out && d.c_lo)
                ok_out = lo8 ? make_map_out(&local.prob[i].o_lo, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d.c_lo, M, N, ldc)
                                : make_map_out(&local.prob[i].o_lo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.c_lo, M, N, ldc);
        }
        if (!ok_out) return cudaErrorInvalidValue;
        local.prob[i].c = d.c;
        local.prob[i].r = static_cast<const __nv_bfloat16 *>(d.r);
        local.prob[i].c_lo = d.c_lo;
        local.prob[i].rowscale = d.rowscale;
        local.prob[i].ssq_in = d.ssq_in;
        local.prob[i].nw = static_cast<const __nv_bfloat16 *>(d.nw);
        local.prob[i].n_hi = static_cast<__nv_bfloat16 *>(d.n_hi);
        local.prob[i].n_lo = d.n_lo;
        local.prob[i].ssq_out = d.ssq_out;
    }
    local.n_problems = n_problems;
    local.M = M;
    local.N = N;
    local.K = K;
    local.ldc = ldc;
    local.m_tiles = (M + bm_tile - 1) / bm_tile;
    local.n_tiles = (N + bn_out - 1) / bn_out;
    local.epi = epi;
    local.n_pass = n_pass;
    local.lo_fp8 = n_pass == 2 && lo_fp8;
    local.ssq_parts = norm.ssq_parts;
    local.eps = norm.eps;
    local.nt_skip_at = norm.n_skip_lo / kGemmTileN;
    local.nt_skip = (norm.n_skip_hi - norm.n_skip_lo) / kGemmTileN;
    local.ssq_slots = local.n_tiles;
    local.n_tiles -= local.nt_skip;
    local.status = status;
    return cudaSuccess;
}

template <int BN>
cudaError_t launch_gemm(const GemmProblemDesc *probs, int n_problems, int M, int N, int K, int ldc, int epi,
                        int n_pass, int lo_fp8, uint32_t *status, cudaStream_t st, GemmOptions norm) {
    Params local{};
    const int bn_out = epi == EPI_SWIGLU ? BN / 2 : BN;
    const int bn_rows = epi == EPI_SWIGLU ? BN / 2 : BN;  // rows of each weight box
    cudaError_t e0 = fill_params(local, probs, n_problems, M, N, K, ldc, epi, n_pass, lo_fp8, status, norm, bn_rows,
                                 bn_out, BM);
    if (e0 != cudaSuccess) return e0;
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg<BN>::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int total = n_problems * local.m_tiles * local.n_tiles;
    const int sms = sm_count();
    const int grid = total < sms ? total : sms;
    gemm_tc_kernel<BN><<<grid, kThreads, Cfg<BN>::kSmemBytes, st>>>(local);
    return cudaGetLastError();
}

cudaError_t launch_gemm_pair(const GemmProblemDesc *probs, int n_problems, int M, int N, int K, int ldc, int epi,
                             int n_pass, int lo_fp8, uint32_t *status, cudaStream_t st, GemmOptions norm) {
    constexpr int BN = 256;
    Params local{};
    const int bn_out = epi == EPI_SWIGLU ? BN / 2 : BN;
    // each CTA of a pair loads 128 weight rows: half the tile's B rows, or for
    // SwiGLU the tile's gate rows (even CTA) or up rows (odd CTA)
    cudaError_t e = fill_params(local, probs, n_problems, M, N, K, ldc, epi, n_pass, lo_fp8, status, norm, BN / 2,
                                bn_out, 2 * BM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmemBytes);
    if (e != cudaSuccess) return e;
    const int total = n_problems * local.m_tiles * local.n_tiles;
    const int pairs = sm_count() / 2;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * (total < pairs ? total : pairs), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kPairSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, gemm_pair_kernel, local);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

cudaError_t gemm_tc(const GemmProblemDesc *probs, int n_problems, int M, int N, int K, int ldc, int epi,
                    int n_pass, int lo_fp8, uint32_t *status, cudaStream_t st, GemmOptions norm) {
    if (n_problems <= 0 || n_problems > kMaxGemmProblems || M <= 0 || N <= 0 || K <= 0 || K % BK != 0 ||
        N % 8 != 0 || ldc % 8 != 0 || ldc < N || (n_pass != 1 && n_pass != 2) ||
        (n_pass == 2 && lo_fp8 && K % (2 * BK) != 0))
        return cudaErrorInvalidValue;
    for (int i = 0; i < n_problems; ++i) {
        const GemmProblemDesc &d = probs[i];
        if (d.ssq_in && (norm.ssq_parts <= 0 || !(norm.eps > 0.f) || epi == EPI_F32_RESIDUAL || epi == EPI_STORE ||
                         epi == EPI_RESIDUAL))
            return cudaErrorInvalidValue;
        if (d.nw && (epi != EPI_F32_RESIDUAL || !d.n_hi || !d.ssq_out || (n_pass == 2) != (d.n_lo != nullptr)))
            return cudaErrorInvalidValue;
        if (norm.n_skip_hi > norm.n_skip_lo && d.nw) return cudaErrorInvalidValue;
    }
    if (norm.n_skip_lo < 0 || norm.n_skip_hi < norm.n_skip_lo || norm.n_skip_lo % kGemmTileN ||
        norm.n_skip_hi % kGemmTileN || norm.n_skip_hi >= N || (norm.n_skip_hi > norm.n_skip_lo && epi == EPI_SWIGLU))
        return cudaErrorInvalidValue;
    // 256-wide tiles: measured against 128-wide ones on the group shapes, they stay
    // ahead even where the 128-wide tiling fills the last wave of SMs better
    // (the A tile is then streamed twice as often).
    static_assert(kGemmTileN == 256, "the partial sums of squares come one per 256-wide tile");
    if (norm.form == GEMM_FORM_PAIR)
        return launch_gemm_pair(probs, n_problems, M, N, K, ldc, epi, n_pass, lo_fp8, status, st, norm);
    return launch_gemm<256>(probs, n_problems, M, N, K, ldc, epi, n_pass, lo_fp8, status, st, norm);
}

}  // namespace sr
