// Elementwise / reduction kernels of a replay-group layer (HBM-bound; one
// launch covers every replay group of the call through per-group pointers).
//
//   row_prep     A = x * w (as an exact hi + lo bf16 pair when split) and the
//                RMSNorm factor r_t = 1/sqrt(mean(x_t^2) + eps); the GEMM that
//                consumes A applies r_t in its epilogue, so RMSNorm(x) w W^T is
//                formed without rounding the normalised activations.  Row t of
//                x is optionally gathered through an anchor index table.
//   conv_gates   causal depthwise conv (width 4; zero left padding per
//                sequence, or the stored history of a continuation) + SiLU
//                over [q|k|v], per-head L2 norm of q and k,
//                g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b).
//   conv_state   the last (width-1) pre-conv rows of each sequence.
//   gated_norm   y = RMSNorm_head(o) w_g * SiLU(z) (hi + lo when split).
//   to_bf16      fp32 residual stream -> bf16 hidden output.
// The layer math is the Qwen3.5-family Gated DeltaNet block ("Tail-Replay",
// Sec. 2 names Gated DeltaNet as the linear layer of the hybrids replayed).
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sr {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void split2(float a, float b, __nv_bfloat162 &hi, __nv_bfloat162 &lo) {
    hi = __floats2bfloat162_rn(a, b);
    const float2 h = __bfloat1622float2(hi);
    lo = __floats2bfloat162_rn(a - h.x, b - h.y);
}
// hi = bf16 pair; lo8 = e4m3 bytes of (x - hi) * 2^8 (round to nearest, saturating)
__device__ __forceinline__ void split2_lo8(float a, float b, __nv_bfloat162 &hi, uint16_t &lo8) {
    hi = __floats2bfloat162_rn(a, b);
    const float2 h = __bfloat1622float2(hi);
    lo8 = __nv_cvt_float2_to_fp8x2(make_float2((a - h.x) * 256.f, (b - h.y) * 256.f), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + expf(-x)); }
__device__ __forceinline__ float softplusf_(float x) { return x > 20.f ? x : log1pf(expf(x)); }
// SiLU on the per-element hot paths: hardware exp2-based __expf and the fast
// division (a few fp32 ulp; the result is carried on as an fp32 value or an
// exact hi + lo pair, far inside the bf16-level tolerances).  For x -> -inf the
// quotient goes to zero (x times the reciprocal of +inf).
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.f + __expf(-x)); }

// ---------------------------------------------------------------- row_prep
// One warp per row.  H % 8 == 0.
__global__ void __launch_bounds__(256) row_prep_kernel(const __grid_constant__ RowPrepBatch p) {
    const int g = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + warp;
    if (row >= p.T) return;
    const int H = p.H;
    const size_t base = size_t(row) * H;  // destination row (packed token)
    // source row: the token itself, or its entry of the anchor index table
    int src = row;
    bool zero = false;
    if (p.idx) {
        src = p.idx[row];
        if (src < 0 || src >= p.x_rows) {
            zero = true;
            src = 0;
            if (lane == 0) atomicOr(p.status, SR_DEV_BAD_INDEX);
        }
    }
    const size_t sbase = size_t(src) * H;
    float ss = 0.f;
    for (int c = lane * 8; c < H; c += 256) {
        float xv[8];
        if (zero) {
#pragma unroll
            for (int e = 0; e < 8; ++e) xv[e] = 0.f;
        } else if (p.x_f32) {
            const float4 *xs = reinterpret_cast<const float4 *>(static_cast<const float *>(p.x[g]) + sbase + c);
            const float4 a = xs[0], b = xs[1];
            xv[0] = a.x; xv[1] = a.y; xv[2] = a.z; xv[3] = a.w; xv[4] = b.x; xv[5] = b.y; xv[6] = b.z; xv[7] = b.w;
        } else {
            const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.x[g]) + sbase + c);
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                xv[2 * e] = f.x;
                xv[2 * e + 1] = f.y;
            }
        }
        const uint4 wu = *reinterpret_cast<const uint4 *>(p.w[g] + c);
        const __nv_bfloat162 *w2 = reinterpret_cast<const __nv_bfloat162 *>(&wu);
        __nv_bfloat162 hi[4], lo[4];
        uint16_t lo8[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            ss = fmaf(xv[2 * e], xv[2 * e], ss);
            ss = fmaf(xv[2 * e + 1], xv[2 * e + 1], ss);
            const float2 wf = __bfloat1622float2(w2[e]);
            if (p.lo8)
                split2_lo8(xv[2 * e] * wf.x, xv[2 * e + 1] * wf.y, hi[e], lo8[e]);
            else
                split2(xv[2 * e] * wf.x, xv[2 * e + 1] * wf.y, hi[e], lo[e]);
        }
        *reinterpret_cast<uint4 *>(p.a_hi[g] + base + c) = *reinterpret_cast<uint4 *>(hi);
        if (p.a_lo[g]) {
            if (p.lo8)
                *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.a_lo[g]) + base + c) =
                    make_uint2(uint32_t(lo8[0]) | (uint32_t(lo8[1]) << 16), uint32_t(lo8[2]) | (uint32_t(lo8[3]) << 16));
            else
                *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.a_lo[g]) + base + c) =
                    *reinterpret_cast<uint4 *>(lo);
        }
        if (p.x32_out[g]) {
            float4 *d = reinterpret_cast<float4 *>(p.x32_out[g] + base + c);
            d[0] = make_float4(xv[0], xv[1], xv[2], xv[3]);
            d[1] = make_float4(xv[4], xv[5], xv[6], xv[7]);
        }
    }
    ss = warp_sum(ss);
    if (lane == 0) p.r[g][row] = 1.f / sqrtf(ss / float(H) + p.eps);
}

// ---------------------------------------------------------------- conv_gates
constexpr int kConvTok = 32;   // tokens per CTA: 4 warps x 8 consecutive tokens
constexpr int kWarpTok = 8;

// Index n of the sequence holding token t (cu non-decreasing, cu[0] = 0).
__device__ __forceinline__ int seq_of(const int32_t *cu, int n_seqs, int t) {
    int lo = 0, hi = n_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

constexpr int kConvRows = kConvTok + 3;  // the block's tokens and the 3 rows before them

// blockIdx.y < 2 h_k + h_v: one 128-channel head of [q|k|v].  One TMA tile
// load brings the block's 32 rows and the 3 rows before them (rows outside
// [0, T) read as zero) into shared memory; warp w then takes tokens
// t0 + 8w .. t0 + 8w + 7 and lane l channels 4l .. 4l+3, so the per-head L2
// norm is a warp reduction.  blockIdx.y == 2 h_k + h_v: gates.
// At most 51 registers a thread, so that ten CTAs (40 warps) share an SM: 0.527 -> 0.502 ms
// per whole-model step against eight at 64 registers (twelve spill and are slower).
__global__ void __launch_bounds__(128, 10) conv_gates_kernel(const __grid_constant__ ConvBatch p) {
    __shared__ __align__(128) float tile[kConvRows * 128];
    __shared__ __align__(8) uint64_t bar;
    const int g = blockIdx.z;
    const int head = blockIdx.y;
    const int t0 = blockIdx.x * kConvTok;
    const int tid = threadIdx.x;
    const float *P = p.p[g];
    const int n_qk = 2 * p.h_k;
    if (head == n_qk + p.h_v) {
        const int t1 = min(p.T, t0 + kConvTok);
        for (int e = tid; e < (t1 - t0) * p.h_v; e += blockDim.x) {
            const int t = t0 + e / p.h_v, h = e % p.h_v;
            if (!SR_IN_BOUNDS(size_t(t) * p.h_v + h, (long long)p.T * p.h_v, p.status)) continue;
            const float b = P[size_t(t) * p.ld + p.b_off + h];
            const float a = P[size_t(t) * p.ld + p.b_off + p.h_v + h];
            p.gate[g][size_t(t) * p.h_v + h] = -expf(p.a_log[g][h]) * softplusf_(a + p.dt_bias[g][h]);
            p.beta[g][size_t(t) * p.h_v + h] = sigmoidf_(b);
        }
        return;
    }
    if (tid == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(&bar, kConvRows * 128 * 4);
        tc::tma_load_2d(tile, &p.pmap[g], &bar, head * 128, t0 - 3);
    }
    __syncthreads();
    if (!tc::mbar_wait(&bar, 0)) {
        // give the copy a second bounded wait before the block's shared memory goes away
        if (tid == 0) {
            atomicOr(p.status, SR_DEV_TIMEOUT);
            tc::mbar_wait(&bar, 0);
        }
        return;
    }
    const int warp = tid >> 5, lane = tid & 31;
    const int tw = t0 + warp * kWarpTok;  // first token of this warp
    if (tw >= p.T) return;
    const int ch = head * 128 + lane * 4;
    float w[4][4];  // w[channel][tap]
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p.conv_w[g] + size_t(ch + c) * 4);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        w[c][0] = a.x; w[c][1] = a.y; w[c][2] = b.x; w[c][3] = b.y;
    }
    // tile row j holds token t0 - 3 + j; this warp's rows tw-3 .. tw+7 start at row 8 warp
    const float4 *x = reinterpret_cast<const float4 *>(tile) + (warp * kWarpTok) * 32 + lane;
    int n = seq_of(p.cu, p.n_seqs, tw);
    int eos = p.cu[n + 1];
    int bos = max(p.cu[n], 0);
    // SiLU'd conv output of token t -> (L2 norm for q, k) -> bf16 (hi + lo) stores
    auto emit = [&](int t, float (&c)[4]) {
        if (head < n_qk) {
            const float ss = warp_sum(c[0] * c[0] + c[1] * c[1] + c[2] * c[2] + c[3] * c[3]);
            const float inv = rsqrtf(ss + 1e-6f);
#pragma unroll
            for (int e = 0; e < 4; ++e) c[e] *= inv;
        }
        __nv_bfloat162 hi[2], lo[2];
        split2(c[0], c[1], hi[0], lo[0]);
        split2(c[2], c[3], hi[1], lo[1]);
        const uint2 hv = *reinterpret_cast<uint2 *>(hi), lv = *reinterpret_cast<uint2 *>(lo);
        const long long w_out = head < n_qk ? (long long)p.T * p.h_k * 128 : (long long)p.T * p.h_v * 128;
        const size_t o_first = size_t(t) * (head < n_qk ? p.h_k : p.h_v) * 128 +
                               (ch - (head < p.h_k ? 0 : head < n_qk ? p.h_k * 128 : n_qk * 128));
        if (!SR_IN_BOUNDS(o_first + 3, w_out, p.status)) return;
        if (head < p.h_k) {
            *reinterpret_cast<uint2 *>(p.q[g] + size_t(t) * p.h_k * 128 + ch) = hv;
        } else if (head < n_qk) {
            const size_t o = size_t(t) * p.h_k * 128 + (ch - p.h_k * 128);
            *reinterpret_cast<uint2 *>(p.k[g] + o) = hv;
            if (p.k_lo[g]) *reinterpret_cast<uint2 *>(p.k_lo[g] + o) = lv;
        } else {
            const size_t o = size_t(t) * p.h_v * 128 + (ch - n_qk * 128);
            *reinterpret_cast<uint2 *>(p.v[g] + o) = hv;
            if (p.v_lo[g]) *reinterpret_cast<uint2 *>(p.v_lo[g] + o) = lv;
        }
    };
    // fast path: the warp's tokens and the 3 rows before them all lie inside one
    // sequence, so no tap is masked; a rolling window keeps the previous rows in
    // registers (same arithmetic, in the same order, as the general path)
    if (tw - 3 >= bos && tw + kWarpTok <= eos && tw + kWarpTok <= p.T) {
        float4 h3 = x[0], h2 = x[32], h1 = x[64];
#pragma unroll
        for (int i = 0; i < kWarpTok; ++i) {
            const float4 x0 = x[(i + 3) * 32];
            const float a0[4] = {x0.x, x0.y, x0.z, x0.w}, a1[4] = {h1.x, h1.y, h1.z, h1.w};
            const float a2[4] = {h2.x, h2.y, h2.z, h2.w}, a3[4] = {h3.x, h3.y, h3.z, h3.w};
            float c[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float acc = w[e][3] * a0[e];
                acc = fmaf(w[e][2], a1[e], acc);
                acc = fmaf(w[e][1], a2[e], acc);
                acc = fmaf(w[e][0], a3[e], acc);
                c[e] = silu_fast(acc);
            }
            emit(tw + i, c);
            h3 = h2;
            h2 = h1;
            h1 = x0;
        }
        return;
    }
#pragma unroll
    for (int i = 0; i < kWarpTok; ++i) {
        const int t = tw + i;
        if (t >= p.T) break;
        while (t >= eos && n + 1 < p.n_seqs) {
            ++n;
            bos = max(p.cu[n], 0);
            eos = p.cu[n + 1];
        }
        float c[4];
        const float4 x0v = x[(i + 3) * 32];
        const float *x0 = reinterpret_cast<const float *>(&x0v);
        // rows t-1, t-2, t-3: inside the sequence from the tile; before its
        // start zero (replay) or the stored history (continuation)
        float xm[3][4];
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int tj = t - 1 - j;
            const float4 xv = x[(i + 2 - j) * 32];
            const float *xr = reinterpret_cast<const float *>(&xv);
            if (tj >= bos) {
#pragma unroll
                for (int e = 0; e < 4; ++e) xm[j][e] = xr[e];
            } else if (p.conv_in[g]) {
                const size_t hofs = (size_t(n) * p.conv_dim + ch) * 3 + (3 - bos + tj);
                const bool hin = SR_IN_BOUNDS(hofs + 9, (long long)p.n_seqs * p.conv_dim * 3, p.status);
                const __nv_bfloat16 *hp = p.conv_in[g] + hofs;
#pragma unroll
                for (int e = 0; e < 4; ++e) xm[j][e] = hin ? __bfloat162float(hp[e * 3]) : 0.f;
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) xm[j][e] = 0.f;
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float acc = w[e][3] * x0[e];
            acc = fmaf(w[e][2], xm[0][e], acc);
            acc = fmaf(w[e][1], xm[1][e], acc);
            acc = fmaf(w[e][0], xm[2][e], acc);
            c[e] = silu_fast(acc);
        }
        emit(t, c);
    }
}

// conv_state[n, ch, j] = pre-conv row (eos - W + 1 + j) of sequence n; rows
// before its start come from its history (zero, or conv_in on a continuation).
// The history is read before anything is written, so conv_in may alias conv_out.
__global__ void __launch_bounds__(128) conv_state_kernel(const __grid_constant__ ConvBatch p) {
    const int g = blockIdx.z, n = blockIdx.x;
    const int ch = blockIdx.y * 128 + threadIdx.x;
    if (ch >= p.conv_dim) return;
    const int bos = max(p.cu[n], 0), eos = min(p.cu[n + 1], p.T);
    const size_t off = (size_t(n) * p.conv_dim + ch) * 3;
    if (!SR_IN_BOUNDS(off + 2, (long long)p.n_seqs * p.conv_dim * 3, p.status)) return;
    float hist[3] = {0.f, 0.f, 0.f};
    if (p.conv_in[g]) {
#pragma unroll
        for (int j = 0; j < 3; ++j) hist[j] = __bfloat162float(p.conv_in[g][off + j]);
    }
    float val[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int t = eos - 3 + j;
        const int hj = 3 - bos + t;  // history slot of a row before the start (in [0, 3) when t < bos)
        val[j] = t >= bos && SR_IN_BOUNDS(size_t(t) * p.ld + ch, (long long)p.T * p.ld, p.status)
                     ? p.p[g][size_t(t) * p.ld + ch]
                     : (t < bos && hj >= 0 ? hist[hj] : 0.f);
    }
    __nv_bfloat16 *out = p.conv_out[g] + off;
#pragma unroll
    for (int j = 0; j < 3; ++j) out[j] = __float2bfloat16_rn(val[j]);
}

// ---------------------------------------------------------------- gated_norm
// One warp per (token, V head); d = 128 (4 values per lane).
__global__ void __launch_bounds__(256) gated_norm_kernel(const __grid_constant__ GatedNormBatch p) {
    const int g = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int item = blockIdx.x * 8 + warp;  // t * h_v + h
    if (item >= p.T * p.h_v) return;
    const int t = item / p.h_v, h = item % p.h_v;
    const int c = lane * 4;
    if (!SR_IN_BOUNDS(size_t(item) * 128 + c + 3, (long long)p.T * p.h_v * 128, p.status)) return;
    const uint2 ou = *reinterpret_cast<const uint2 *>(p.o[g] + size_t(item) * 128 + c);
    const __nv_bfloat162 *o2 = reinterpret_cast<const __nv_bfloat162 *>(&ou);
    const float2 oa = __bfloat1622float2(o2[0]), ob = __bfloat1622float2(o2[1]);
    const float ov[4] = {oa.x, oa.y, ob.x, ob.y};
    const float ss = warp_sum(ov[0] * ov[0] + ov[1] * ov[1] + ov[2] * ov[2] + ov[3] * ov[3]);
    const float r = rsqrtf(ss / 128.f + p.eps);
    const float4 z = *reinterpret_cast<const float4 *>(p.p[g] + size_t(t) * p.ld + p.z_off + h * 128 + c);
    const float zv[4] = {z.x, z.y, z.z, z.w};
    float y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
        y[e] = ov[e] * r * __bfloat162float(p.w[g][c + e]) * silu_fast(zv[e]);
    __nv_bfloat162 hi[2], lo[2];
    if (p.lo8) {
        uint16_t l8[2];
        split2_lo8(y[0], y[1], hi[0], l8[0]);
        split2_lo8(y[2], y[3], hi[1], l8[1]);
        if (p.y_lo[g])
            *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(p.y_lo[g]) + size_t(item) * 128 + c) =
                uint32_t(l8[0]) | (uint32_t(l8[1]) << 16);
    } else {
        split2(y[0], y[1], hi[0], lo[0]);
        split2(y[2], y[3], hi[1], lo[1]);
        if (p.y_lo[g])
            *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.y_lo[g]) + size_t(item) * 128 + c) =
                *reinterpret_cast<uint2 *>(lo);
    }
    *reinterpret_cast<uint2 *>(p.y_hi[g] + size_t(item) * 128 + c) = *reinterpret_cast<uint2 *>(hi);
}

// ---------------------------------------------------------------- prepare_lo8
// w_lo8[i] = e5m2(w[i] * 2^-8); 8 weights per thread (n % 8 handled by the tail loop).
__global__ void __launch_bounds__(256) prepare_lo8_kernel(const __nv_bfloat16 *__restrict__ w, uint8_t *__restrict__ q,
                                                          int64_t n) {
    const int64_t i = (int64_t(blockIdx.x) * 256 + threadIdx.x) * 8;
    if (i + 8 <= n) {
        const uint4 u = *reinterpret_cast<const uint4 *>(w + i);
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
        uint32_t out[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float2 a = __bfloat1622float2(h2[2 * h]), b = __bfloat1622float2(h2[2 * h + 1]);
            const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a.x * 0.00390625f, a.y * 0.00390625f),
                                                         __NV_SATFINITE, __NV_E5M2);
            const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(b.x * 0.00390625f, b.y * 0.00390625f),
                                                         __NV_SATFINITE, __NV_E5M2);
            out[h] = lo | (hi << 16);
        }
        *reinterpret_cast<uint2 *>(q + i) = make_uint2(out[0], out[1]);
    } else {
        for (int64_t j = i; j < n; ++j)
            q[j] = __nv_cvt_float_to_fp8(__bfloat162float(w[j]) * 0.00390625f, __NV_SATFINITE, __NV_E5M2);
    }
}

// ---------------------------------------------------------------- to_bf16
__global__ void __launch_bounds__(256) to_bf16_kernel(const __grid_constant__ CastBatch p) {
    const int g = blockIdx.y;
    const size_t i = (size_t(blockIdx.x) * 256 + threadIdx.x) * 4;
    if (i >= p.n) return;
    const float4 v = *reinterpret_cast<const float4 *>(p.src[g] + i);
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p.dst[g] + i) = u;
}

}  // namespace

cudaError_t row_prep(const RowPrepBatch &b, int n_groups, cudaStream_t st) {
    if (b.T == 0) return cudaSuccess;
    dim3 grid((b.T + 7) / 8, n_groups);
    row_prep_kernel<<<grid, 256, 0, st>>>(b);
    return cudaGetLastError();
}

cudaError_t conv_gates(const ConvBatch &b_in, int n_groups, cudaStream_t st) {
    if (b_in.T == 0) return cudaSuccess;
    ConvBatch b = b_in;
    for (int g = 0; g < n_groups; ++g)
        if (!make_map_f32(&b.pmap[g], b.p[g], b.T, b.ld, b.ld, 128, kConvRows)) return cudaErrorInvalidValue;
    dim3 grid((b.T + kConvTok - 1) / kConvTok, 2 * b.h_k + b.h_v + 1, n_groups);
    conv_gates_kernel<<<grid, 128, 0, st>>>(b);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || b.n_seqs == 0) return e;
    dim3 g2(b.n_seqs, (b.conv_dim + 127) / 128, n_groups);
    conv_state_kernel<<<g2, 128, 0, st>>>(b);
    return cudaGetLastError();
}

cudaError_t gated_norm(const GatedNormBatch &b, int n_groups, cudaStream_t st) {
    if (b.T == 0) return cudaSuccess;
    dim3 grid((b.T * b.h_v + 7) / 8, n_groups);
    gated_norm_kernel<<<grid, 256, 0, st>>>(b);
    return cudaGetLastError();
}

cudaError_t to_bf16(const CastBatch &b, int n_groups, cudaStream_t st) {
    if (b.n == 0) return cudaSuccess;
    dim3 grid(unsigned((b.n / 4 + 255) / 256), n_groups);
    to_bf16_kernel<<<grid, 256, 0, st>>>(b);
    return cudaGetLastError();
}

cudaError_t prepare_lo8(const void *w, void *w_lo8, int64_t n, cudaStream_t st) {
    if (reinterpret_cast<uintptr_t>(w) % 16 || reinterpret_cast<uintptr_t>(w_lo8) % 8) return cudaErrorInvalidValue;
    const int64_t blocks = (n + 2047) / 2048;
    if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
    prepare_lo8_kernel<<<unsigned(blocks), 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(w),
                                                          static_cast<uint8_t *>(w_lo8), n);
    return cudaGetLastError();
}

}  // namespace sr
