// Chunked Mamba2 replay on the 5th-generation tensor cores (head dim 64,
// d_state 128, one B/C group).
//
// Recurrence ("SuffixReplay: Prefix Caching via Suffix Replay for Hybrid
// LLMs", Eq. 4, the per-head-decay instance with no erase term):
//     S_t = exp(dt_t A_h) S_{t-1} + dt_t x_t B_t^T,   y_t = S_t C_t.
// Per chunk of C = 64 tokens with gamma_t = sum_{r<=t} dt_r A_h (chunk
// relative) and entry state S_0:
//     y_t = sum_{s<=t} e^{gamma_t-gamma_s} dt_s (C_t . B_s) x_s + e^{gamma_t} S_0 C_t
//     S_C = e^{gamma_C} S_0 + sum_s dt_s e^{gamma_C-gamma_s} x_s B_s^T.
// A CTA takes one sequence and two heads.  Their states (64 x 128 each) are
// stacked into one 128 x 128 fp32 accumulator in tensor memory, so every
// product is a tcgen05 MMA with M = 128, issued by one thread of a warp that
// does nothing else:
//     [C; B] B^T          -> G = C B^T in rows 0..63 (the B B^T rows are unused)
//     [S_h0; S_h1] C^T    -> e^{-gamma} y's state part for both heads
//     [x_h0^T; x_h1^T] [Gm_h0 | Gm_h1]^T -> the chunk-internal part; the two
//                            diagonal 64 x 64 blocks are the two heads' outputs
//     [x_h0^T; x_h1^T] [D_h0 | D_h1]^T -> x diag(w) for both heads (diagonal blocks),
//                            D_h = diag(w_h) as hi + lo bf16 tiles, w = dt e^{gamma_C-gamma}
//     S += [xw_h0^T; xw_h1^T] B   (xw = x diag(w) as hi + lo)
// with Gm_h = (G o L_h), L_h[t][s] = e^{gamma_t-gamma_s} dt_s for s <= t.  The A
// operands of the state's own products (the bf16 copy of S and xw's hi and lo)
// are written by the other eight warps into tensor memory and read from there;
// A chunk's gates (gamma, e^{gamma}, the diagonal of diag(w)) are formed by the
// data warps during the chunk before it, while that chunk's last products run,
// so the products of a chunk can start as soon as its inputs have landed.
// C, B and x tiles arrive by TMA (double-buffered, two chunks ahead); y goes
// from tensor memory straight to global memory, a warp storing 32 consecutive
// channels of one token per instruction.
// Exponentials only ever see differences gamma_t - gamma_s with s <= t.
// Every mbarrier wait is bounded; a timeout records SR_DEV_TIMEOUT, drains the
// MMAs, frees tensor memory and ends the CTA.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sr {

namespace {

using namespace tc;

constexpr int C = 64, P = 64, NS = 128;
// warps 0-7 move data (warp w: TMEM lanes 32 (w % 4) .. + 31, column half w / 4);
// warp 8 waits for inputs and issues every product and copy
constexpr int kMovers = 256, kThreads = 288, kIssuer = 256;

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t SZ_IN = 49152;        // one input buffer: [C_n0][B_n0][C_n1][B_n1][x_h0][x_h1], 8 KB each
constexpr uint32_t OFF_IN = 0;           // two buffers
constexpr uint32_t OFF_Q = 2 * SZ_IN;    // masked G rows [(h,t)][s], 16 KB
constexpr uint32_t OFF_YS = OFF_Q + 16384;    // G = C B^T staged for the mask rows
// diag(w) per head as hi and lo tiles [t][s]: [h0 hi][h1 hi][h0 lo][h1 lo], one set
// per chunk parity (a chunk's set is formed during the chunk before it)
constexpr uint32_t OFF_DW = OFF_YS + 16384;
constexpr uint32_t SZ_DW = 32768;
constexpr uint32_t OFF_MISC = OFF_DW + 2 * SZ_DW; // gate tables (per chunk parity), barriers
constexpr uint32_t SZ_MISC = 4096;
constexpr uint32_t kSmem = OFF_MISC + SZ_MISC + 1024;

// barrier of the eight data-moving warps only
__device__ __forceinline__ void movers_sync() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }

struct M2TcParams {
    CUtensorMap mc, mb, mx;
    const float *dt;
    const float *A;
    const int32_t *cu;
    const float *h0;
    __nv_bfloat16 *y;
    float *s_out;
    int total, max_len, H, n_seqs;
    uint32_t *status;
};

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

__global__ void __launch_bounds__(kThreads, 1) mamba2_tc_kernel(const __grid_constant__ M2TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t base = smem_u32(sm);
    // per chunk parity and head: gamma, dt (0 beyond the sequence) and e^{gamma}, [2][2][64] each
    float *gam_all = reinterpret_cast<float *>(sm + OFF_MISC);
    float *dts_all = gam_all + 4 * C;
    float *egs_all = gam_all + 8 * C;
    uint64_t *bar_in = reinterpret_cast<uint64_t *>(sm + OFF_MISC + 3072);  // [2] input buffers landed
    uint64_t *bar_g = bar_in + 2;      // C B^T done
    uint64_t *bar_s = bar_in + 3;      // state part of y and the state update done
    uint64_t *bar_y = bar_in + 4;      // chunk-internal part of y done
    uint64_t *bar_drain = bar_in + 5;  // every issued MMA done (abort path)
    uint64_t *bar_xw = bar_in + 6;     // x diag(w) done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_in + 7);
    float *gs = reinterpret_cast<float *>(sm + OFF_YS);      // G = C B^T staged for the mask

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool mover = tid < kMovers;
    const int quad = warp & 3, half = (warp >> 2) & 1;
    const int row = quad * 32 + lane;      // TMEM lane = stacked state row (head row >> 6, p = row & 63)
    const int hrow = row >> 6, prow = row & 63;
    const int pair = blockIdx.x;
    const int n = longest_first(p.cu, gridDim.y, blockIdx.y, reinterpret_cast<int *>(sm + OFF_Q));
    int bos, eos;
    if (!seq_bounds(p.cu, n, p.total, p.max_len, p.status, bos, eos)) return;
    const int len = eos - bos;
    const int nchunks = (len + C - 1) / C;
    const int H = p.H;
    const size_t sbase0 = (size_t(n) * H + 2 * pair) * P * NS;  // state of head 2 pair; the pair is contiguous
    const long long s_elems = (long long)p.n_seqs * H * P * NS, y_elems = (long long)p.total * H * P;
    const float *h0 = p.h0;
    float *s_out = p.s_out;

    if (nchunks == 0) {  // empty sequence: the states are h0 (or zero)
        for (int e = tid; e < 2 * P * NS / 4; e += kThreads) {
            if (!SR_IN_BOUNDS(sbase0 + 4 * size_t(e) + 3, s_elems, p.status)) continue;
            const float4 v = h0 ? reinterpret_cast<const float4 *>(h0 + sbase0)[e] : make_float4(0.f, 0.f, 0.f, 0.f);
            reinterpret_cast<float4 *>(s_out + sbase0)[e] = v;
        }
        return;
    }

    if (tid == kIssuer) {
        for (int i = 0; i < 7; ++i) mbar_init(bar_in + i, 1);
        fence_mbar_init();
    }
    // diag(w) tiles: zero off the diagonal for good; the diagonal is rewritten per chunk
    for (int e = tid; e < 2 * SZ_DW / 16; e += kThreads)
        *reinterpret_cast<uint4 *>(sm + OFF_DW + 16 * e) = make_uint4(0u, 0u, 0u, 0u);
    fence_async_smem();
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // S (fp32) 0-127, G 128-191, the state part of y 192-255, the chunk-internal
    // part 256-383 (before it, x diag(w) in fp32), bf16 S 384-447, xw hi 448-479,
    // xw lo 480-511
    const uint32_t RS = tmem, RG = tmem + 128, RI = tmem + 192, RY = tmem + 256;
    const uint32_t RSB = tmem + 384, RXH = tmem + 448, RXL = tmem + 480;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;

    // ---- initial states into TMEM: row (h, p), columns n in [64 half, 64 half + 64)
    if (mover) {
        uint32_t r[32];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const int n0 = 64 * half + 32 * part;
            const bool in = h0 && SR_IN_BOUNDS(sbase0 + size_t(row) * NS + n0 + 31, s_elems, p.status);
#pragma unroll
            for (int e = 0; e < 32; ++e)
                r[e] = __float_as_uint(in ? h0[sbase0 + size_t(row) * NS + n0 + e] : 0.f);
            tmem_st_32x32b_x32(RS + lane_off + n0, r);
        }
        tmem_st_wait();
    }

    auto issue_in = [&](int c) {
        const int b = c & 1;
        const int y0 = bos + c * C;
        uint8_t *in = sm + OFF_IN + b * SZ_IN;
        mbar_arrive_expect_tx(&bar_in[b], SZ_IN);
        tma_load_2d(in, &p.mc, &bar_in[b], 0, y0);
        tma_load_2d(in + 8192, &p.mb, &bar_in[b], 0, y0);
        tma_load_2d(in + 16384, &p.mc, &bar_in[b], 64, y0);
        tma_load_2d(in + 24576, &p.mb, &bar_in[b], 64, y0);
        tma_load_2d(in + 32768, &p.mx, &bar_in[b], (2 * pair) * P, y0);
        tma_load_2d(in + 40960, &p.mx, &bar_in[b], (2 * pair + 1) * P, y0);
    };
    if (tid == kIssuer) {
        prefetch_tmap(&p.mc); prefetch_tmap(&p.mb); prefetch_tmap(&p.mx);
        issue_in(0);
        if (nchunks > 1) issue_in(1);
    }

    // dt of the next chunk whose gates are formed: thread tid < 128 holds token
    // (tid & 63) of head (tid >> 6) of the pair
    const int dh = (tid >> 6) & 1, dtok = tid & 63;
    const float Ah = p.A[2 * pair + (warp & 1)];  // warps 0 and 1 scan heads 0 and 1
    float dt_next = (tid < 128 && dtok < len &&
                     SR_IN_BOUNDS((size_t(bos) + dtok) * H + 2 * pair + dh, (long long)p.total * H, p.status))
                        ? p.dt[(size_t(bos) + dtok) * H + 2 * pair + dh] : 0.f;
    // ---- the gates of chunk cc into the tables and diag(w) tiles of parity cc & 1
    // (movers only): gamma = inclusive prefix sum of dt A, e^{gamma}, and the
    // diagonal entries w = dt e^{gamma_C - gamma} of diag(w) as hi and lo.  Chunk
    // cc's dt is in dt_next, which then moves on to chunk cc + 1.
    auto gates = [&](int cc) {
        const int gb = cc & 1;
        float *gam = gam_all + gb * 2 * C, *dts = dts_all + gb * 2 * C, *egs = egs_all + gb * 2 * C;
        if (tid < 128) {
            dts[dh * C + dtok] = dt_next;
            const int t = (cc + 1) * C + dtok;
            dt_next = (t < len && SR_IN_BOUNDS((size_t(bos) + t) * H + 2 * pair + dh, (long long)p.total * H,
                                               p.status))
                          ? p.dt[(size_t(bos) + t) * H + 2 * pair + dh] : 0.f;
        }
        movers_sync();
        if (warp < 2) {
            const float *d = dts + warp * C;
            const float a0 = d[2 * lane] * Ah, a1 = d[2 * lane + 1] * Ah;
            float incl = a0 + a1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            const float excl = incl - (a0 + a1);
            gam[warp * C + 2 * lane] = excl + a0;
            gam[warp * C + 2 * lane + 1] = excl + a0 + a1;
        }
        movers_sync();
        if (tid < 128) {
            const float g = gam[dh * C + dtok], gC = gam[dh * C + C - 1];
            const float wv = dts[dh * C + dtok] * __expf(gC - g);
            egs[dh * C + dtok] = __expf(g);
            uint32_t whi, wlo;
            split2(wv, 0.f, whi, wlo);
            const uint32_t off = OFF_DW + gb * SZ_DW + sw128(dtok, dtok >> 3) + (dtok & 7) * 2;
            *reinterpret_cast<uint16_t *>(sm + off + dh * 8192) = uint16_t(whi & 0xffffu);
            *reinterpret_cast<uint16_t *>(sm + off + 16384 + dh * 8192) = uint16_t(wlo & 0xffffu);
        }
        fence_async_smem();
    };
    if (mover) gates(0);
    __syncthreads();  // chunk 0's tables and diag(w) tiles, before the first product reads them

    auto wait_on = [&](uint64_t *bar, int parity) -> bool {
        const bool w = mbar_wait(bar, uint32_t(parity & 1));
        tc_fence_after();
        return w;
    };
    // block barrier that also tells every thread whether any thread's wait failed
    auto check = [&](bool w) -> bool { return __syncthreads_or(!w) != 0; };
    constexpr uint32_t ID_G = idesc_bf16_f32_major(128, 64, 0, 0);      // [C;B] B^T, [S] C^T
    constexpr uint32_t ID_Y = idesc_bf16_f32_major(128, 128, 1, 0);     // x^T (MN-major) Q^T
    constexpr uint32_t ID_S = idesc_bf16_f32_major(128, 128, 0, 1);     // xw^T (TMEM) B (MN-major)
    const bool want_y = p.y != nullptr;

    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
        const int b = c & 1;
        const uint32_t in = base + OFF_IN + b * SZ_IN;
        const int clen = min(C, len - c * C);
        const float *gam = gam_all + b * 2 * C, *dts = dts_all + b * 2 * C, *egs = egs_all + b * 2 * C;
        bool w = wait_on(&bar_in[b], (c >> 1) & 1);
        if (tid == kIssuer && w) {
            // G = [C;B] B^T -> RG, and x diag(w) (hi + lo of w) -> the chunk-internal part's
            // columns: both need only this chunk's inputs and its gates (formed a chunk ago)
            if (want_y) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t a = in + (k >> 2) * 16384 + (k & 3) * 32;
                    mma_bf16_ss(RG, sdesc_sw128(a, 16, 1024), sdesc_sw128(a + 8192, 16, 1024), ID_G, k > 0);
                }
                mma_commit(bar_g);
            }
            const uint32_t dw = base + OFF_DW + b * SZ_DW;
#pragma unroll
            for (int k = 0; k < 4; ++k) {  // [x_h0^T; x_h1^T] (MN-major) [Dh_h0; Dh_h1]^T, then the lo tiles
                const uint64_t ax = sdesc_sw128(in + 32768 + k * 2048, 8192, 1024);
                mma_bf16_ss(RY, ax, sdesc_sw128(dw + k * 32, 16, 1024), ID_Y, k > 0);
                mma_bf16_ss(RY, ax, sdesc_sw128(dw + 16384 + k * 32, 16, 1024), ID_Y, 1);
            }
            mma_commit(bar_xw);
        }
        if (mover) {
            // ---- bf16 copy of S (for y) into TMEM and S <- e^{gamma_C} S
            {
                const float fC = __expf(gam[hrow * C + C - 1]);
                uint32_t r[32], bq[16];
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const int n0 = 64 * half + 32 * part;
                    tmem_ld_32x32b_x32(RS + lane_off + n0, r);
                    tmem_ld_wait();
                    if (want_y) {
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            bq[e] = pack2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
                        tmem_st_32x32b_x16(RSB + lane_off + n0 / 2, bq);
                    }
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * fC);
                    tmem_st_32x32b_x32(RS + lane_off + n0, r);
                }
            }
            // ---- xw (own head's diagonal block of the product) as hi + lo into TMEM:
            // lane (h, p), tokens 32 half .. + 31
            w = wait_on(bar_xw, c) && w;
            {
                uint32_t r[32], hi[16], lo[16];
                tmem_ld_32x32b_x32(RY + lane_off + 64 * hrow + 32 * half, r);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) split2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]), hi[e], lo[e]);
                tmem_st_32x32b_x16(RXH + lane_off + 16 * half, hi);
                tmem_st_32x32b_x16(RXL + lane_off + 16 * half, lo);
            }
            tmem_st_wait();
        }
        tc_fence_before();
        if (check(w)) { ok = false; break; }

        // ---- [S] C^T -> RI and S += xw^T B (hi, lo), one commit
        if (tid == kIssuer) {
            tc_fence_after();
            if (want_y) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t bc = in + (k >> 2) * 16384 + (k & 3) * 32;
                    mma_bf16_ts(RI, RSB + 8 * k, sdesc_sw128(bc, 16, 1024), ID_G, k > 0);
                }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t bmn = sdesc_sw128(in + 8192 + k * 2048, 16384, 1024);  // B as MN-major (n halves 16 KB apart)
                mma_bf16_ts(RS, RXH + 8 * k, bmn, ID_S, 1);
                mma_bf16_ts(RS, RXL + 8 * k, bmn, ID_S, 1);
            }
            mma_commit(bar_s);
        }
        if (want_y) {
            // ---- Gm_h rows: Q[(h, t)][s] = G[t][s] e^{gamma_h,t - gamma_h,s} dt_h,s (s <= t), bf16.
            // G lives in TMEM lanes 0..63, which half of the movers can read: they stage it
            // in shared memory (columns XOR-swizzled by row), then all movers build the rows
            // while the other products run.
            w = true;
            if (mover) {
                w = wait_on(bar_g, c);
                if (quad < 2) {
                    const int t = row;
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(RG + lane_off + 32 * half, r);
                    tmem_ld_wait();
                    const int sw = (t & 7) << 2;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<float4 *>(gs + t * C + ((32 * half + 4 * j) ^ sw)) =
                            make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                        __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
                }
                movers_sync();
                // thread: head hq, token tq, 32 columns s0 .. s0 + 31
                const int hq = tid >> 7, tq = (tid >> 1) & 63, s0 = (tid & 1) * 32;
                const float gt = gam[hq * C + tq];
                const float *gh = gam + hq * C, *dh2 = dts + hq * C;
                const int sw = (tq & 7) << 2;
                uint8_t *qrow = sm + OFF_Q;
#pragma unroll 1
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 ga = *reinterpret_cast<const float4 *>(gs + tq * C + ((s0 + 8 * q4) ^ sw));
                    const float4 gb = *reinterpret_cast<const float4 *>(gs + tq * C + ((s0 + 8 * q4 + 4) ^ sw));
                    const float gv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                    uint32_t wq[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int s = s0 + 8 * q4 + 2 * u;
                        const float d0 = s <= tq ? __expf(gt - gh[s]) * dh2[s] : 0.f;
                        const float d1 = s + 1 <= tq ? __expf(gt - gh[s + 1]) * dh2[s + 1] : 0.f;
                        wq[u] = pack2(d0 * gv[2 * u], d1 * gv[2 * u + 1]);
                    }
                    *reinterpret_cast<uint4 *>(qrow + sw128(hq * C + tq, (s0 >> 3) + q4)) =
                        make_uint4(wq[0], wq[1], wq[2], wq[3]);
                }
                fence_async_smem();
            }
            tc_fence_before();
            if (check(w)) { ok = false; break; }
            if (tid == kIssuer) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k)  // [x_h0^T; x_h1^T] (MN-major, head blocks 8 KB apart) Q^T
                    mma_bf16_ss(RY, sdesc_sw128(in + 32768 + k * 2048, 8192, 1024),
                                sdesc_sw128(base + OFF_Q + k * 32, 16, 1024), ID_Y, k > 0);
                mma_commit(bar_y);
            }
        }

        // ---- the next chunk's gates, while this chunk's last products run (the tables
        // and diag(w) tiles of that parity were last read by chunk c - 1)
        if (mover && c + 1 < nchunks) gates(c + 1);
        // ---- the products of this chunk are done: y out, and the input buffer of
        // chunk c + 2 (this one) can be refilled
        w = wait_on(bar_s, c);
        if (want_y) w = wait_on(bar_y, c) && w;
        if (tid == kIssuer && w && c + 2 < nchunks) issue_in(c + 2);
        if (mover && want_y && w) {
            // y_t = e^{gamma_t} Yi + Y (own head's diagonal block); thread = (h, p), 32 tokens
            // in two passes of 16
            const size_t stride = size_t(H) * P;
            const size_t y_first = (size_t(bos) + size_t(c) * C + 32 * half) * stride + size_t(2 * pair + hrow) * P + prow;
            __nv_bfloat16 *yd = p.y + y_first;
            int n_out = min(32, clen - 32 * half);
            if (n_out > 0 && !SR_IN_BOUNDS(y_first + size_t(n_out - 1) * stride, y_elems, p.status)) n_out = 0;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                uint32_t ri[16], ry[16];
                tmem_ld_32x32b_x16(RI + lane_off + 32 * half + 16 * part, ri);
                tmem_ld_32x32b_x16(RY + lane_off + 64 * hrow + 32 * half + 16 * part, ry);
                tmem_ld_wait();
                const float *eg = egs + hrow * C + 32 * half + 16 * part;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    if (16 * part + e < n_out)
                        *yd = __float2bfloat16_rn(eg[e] * __uint_as_float(ri[e]) + __uint_as_float(ry[e]));
                    yd += stride;
                }
            }
        }
        if (!w) { ok = false; }
        ok = __syncthreads_and(ok) != 0;
        if (!ok) break;
    }

    if (ok) {
        if (mover) {
            uint32_t r[32];
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const int n0 = 64 * half + 32 * part;
                tmem_ld_32x32b_x32(RS + lane_off + n0, r);
                tmem_ld_wait();
                if (!SR_IN_BOUNDS(sbase0 + size_t(row) * NS + n0 + 31, s_elems, p.status)) continue;
                float4 *dst = reinterpret_cast<float4 *>(s_out + sbase0 + size_t(row) * NS + n0);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    dst[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                         __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
            }
        }
    } else if (tid == kIssuer) {
        // let every MMA this thread issued, and in-flight TMA copies, finish before
        // tensor and shared memory are released
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

}  // namespace

cudaError_t mamba2_tc(const sr_mamba2_args &a, uint32_t *status, cudaStream_t st) {
    M2TcParams p{};
    const int T = a.total_tokens, hp = a.n_heads * P;
    if (!make_map_bf16(&p.mc, a.C, T, NS, NS, 64, 64) || !make_map_bf16(&p.mb, a.B, T, NS, NS, 64, 64) ||
        !make_map_bf16(&p.mx, a.x, T, hp, hp, 64, 64))
        return cudaErrorInvalidValue;
    p.dt = a.dt;
    p.A = a.A;
    p.cu = a.cu_seqlens;
    p.h0 = a.h0;
    p.y = static_cast<__nv_bfloat16 *>(a.y);
    p.s_out = a.s_out;
    p.total = a.total_tokens;
    p.max_len = a.max_seqlen;
    p.H = a.n_heads;
    p.n_seqs = a.n_seqs;
    p.status = status;
    cudaError_t e = cudaFuncSetAttribute(mamba2_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem));
    if (e != cudaSuccess) return e;
    dim3 grid(a.n_heads / 2, a.n_seqs);
    mamba2_tc_kernel<<<grid, kThreads, kSmem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace sr
