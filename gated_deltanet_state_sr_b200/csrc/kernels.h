// Internal launchers of libsr (not part of the C ABI).  Each returns the
// cudaError_t of its launches; shapes were validated by api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "sr/sr.h"

namespace sr {

// Raw gated-delta replay.
cudaError_t gdn_sequential(const sr_gdn_args &a, float scale, uint32_t *status, cudaStream_t st);
bool gdn_chunked_supported(const sr_gdn_args &a);
size_t gdn_scratch_bytes(const sr_gdn_args &a);
cudaError_t gdn_chunked(const sr_gdn_args &a, float scale, uint32_t *status, void *scratch,
                        cudaStream_t st);

// Chunked replay of several independent problems (replay groups) in one
// launch: grid = (h_v, n_seqs, n_groups); all groups share cu_seqlens and shapes.
constexpr int kMaxGroups = 8;
struct GdnBatch {
    const __nv_bfloat16 *q[kMaxGroups];
    const __nv_bfloat16 *k[kMaxGroups];
    const __nv_bfloat16 *v[kMaxGroups];
    const __nv_bfloat16 *k_lo[kMaxGroups];  // low parts (split precision), else unused
    const __nv_bfloat16 *v_lo[kMaxGroups];
    const float *g[kMaxGroups];
    const float *beta[kMaxGroups];
    const float *h0[kMaxGroups];      // may be null
    __nv_bfloat16 *o[kMaxGroups];     // may be null
    float *s_out[kMaxGroups];
    const int32_t *cu;
    void *img;  // tcgen05 two-phase form: chunk images (gdn_tc_image_bytes); null selects the fused kernel
    int total, max_len, h_k, h_v;
    float scale;
    uint32_t *status;
};
cudaError_t gdn_chunked_batch(const GdnBatch &b, int n_groups, int n_seqs, int d, bool split, cudaStream_t st);
// The same on tcgen05 with the state in tensor memory (d = 128, or d = 64 on
// half-zero tiles; gdn_tc.cu).
bool gdn_tc_supported(int d);
cudaError_t gdn_tc(const sr_gdn_args &a, float scale, uint32_t *status, void *img, cudaStream_t st);
// Scratch of the two-phase form: one 56.5 KB chunk image per (group, chunk slot, V head).
size_t gdn_tc_image_bytes(int total, int n_seqs, int h_v, int n_groups);
cudaError_t gdn_tc_batch(const GdnBatch &b, int n_groups, int n_seqs, int d, bool split, cudaStream_t st);

// 2-D bf16 TMA map (128-byte swizzle) over a row-major [rows, cols] matrix with row pitch `pitch`.
bool make_map_bf16(CUtensorMap *m, const void *base, int rows, int cols, int pitch, int box_cols, int box_rows);
// bytes [rows, cols] (row pitch `pitch` bytes), 128-byte swizzled boxes of box_rows x box_cols.
bool make_map_u8(CUtensorMap *m, const void *base, int rows, int cols, int pitch, int box_cols, int box_rows);
// fp32 [rows, cols] (row pitch `pitch` elements), unswizzled boxes of box_rows x box_cols.
bool make_map_f32(CUtensorMap *m, const void *base, int rows, int cols, int pitch, int box_cols, int box_rows);

// Layer kernels of a replay group (layer_kernels.cu).  Arrays are indexed by group.
struct RowPrepBatch {
    const void *x[kMaxGroups];            // [T, H] fp32 (x_f32) or bf16
    const __nv_bfloat16 *w[kMaxGroups];   // [H] norm weight
    __nv_bfloat16 *a_hi[kMaxGroups];      // [T, H] x * w (hi part)
    void *a_lo[kMaxGroups];               // [T, H] low part (bf16, or e4m3(lo * 2^8) when lo8), may be null
    float *r[kMaxGroups];                 // [T] 1 / sqrt(mean(x^2) + eps)
    float *x32_out[kMaxGroups];           // [T, H] fp32 copy of x, may be null
    const int32_t *idx;                   // [T] row of x that token t reads, may be null (row t)
    uint32_t *status;                     // device status word (bad index flag)
    int T, H, x_f32, x_rows;              // x_rows: rows of x (bounds of idx)
    int lo8;                              // low part as e4m3 bytes of lo * 2^8
    float eps;
};
cudaError_t row_prep(const RowPrepBatch &b, int n_groups, cudaStream_t st);

struct ConvBatch {
    CUtensorMap pmap[kMaxGroups];          // p, boxes of 128 channels x (32 + 3) rows (set by conv_gates)
    const float *p[kMaxGroups];            // [T, ld] fp32 in_proj output
    const __nv_bfloat16 *conv_w[kMaxGroups];  // [conv_dim, 4]
    const float *a_log[kMaxGroups];
    const float *dt_bias[kMaxGroups];
    __nv_bfloat16 *q[kMaxGroups];          // [T, h_k, 128]
    __nv_bfloat16 *k[kMaxGroups];
    __nv_bfloat16 *k_lo[kMaxGroups];       // may be null
    __nv_bfloat16 *v[kMaxGroups];          // [T, h_v, 128]
    __nv_bfloat16 *v_lo[kMaxGroups];       // may be null
    float *gate[kMaxGroups];               // [T, h_v]
    float *beta[kMaxGroups];
    __nv_bfloat16 *conv_out[kMaxGroups];   // [n_seqs, conv_dim, 3]
    const __nv_bfloat16 *conv_in[kMaxGroups];  // [n_seqs, conv_dim, 3] history before each sequence, may be null
    const int32_t *cu;
    uint32_t *status;                      // device status word (timeout flag)
    int n_seqs, T, ld, h_k, h_v, conv_dim, b_off;  // b_off: column of b (a follows at + h_v)
};
cudaError_t conv_gates(const ConvBatch &b, int n_groups, cudaStream_t st);

struct GatedNormBatch {
    const __nv_bfloat16 *o[kMaxGroups];   // [T, h_v, 128]
    const float *p[kMaxGroups];           // [T, ld] (z at column z_off)
    const __nv_bfloat16 *w[kMaxGroups];   // [128]
    __nv_bfloat16 *y_hi[kMaxGroups];      // [T, h_v * 128]
    void *y_lo[kMaxGroups];               // may be null; bf16, or e4m3(lo * 2^8) when lo8
    int T, h_v, ld, z_off, lo8;
    float eps;
    uint32_t *status;                     // device status word (bounds-checked build)
};
cudaError_t gated_norm(const GatedNormBatch &b, int n_groups, cudaStream_t st);

struct CastBatch {
    const float *src[kMaxGroups];
    __nv_bfloat16 *dst[kMaxGroups];
    size_t n;  // elements per group, multiple of 4
};
cudaError_t to_bf16(const CastBatch &b, int n_groups, cudaStream_t st);

// Mamba2 replay.
cudaError_t mamba2_sequential(const sr_mamba2_args &a, uint32_t *status, cudaStream_t st);
size_t mamba2_scratch_bytes(const sr_mamba2_args &a);
cudaError_t mamba2_replay(const sr_mamba2_args &a, uint32_t *status, void *scratch, cudaStream_t st);
cudaError_t mamba2_tc(const sr_mamba2_args &a, uint32_t *status, cudaStream_t st);

// Dense projections on tcgen05 (gemm_tc.cu).  C[M,N] = A[M,K] B[N,K]^T with
// a fused epilogue; all problems of one call share M, N, K and the epilogue.
enum GemmEpilogue { EPI_STORE = 0, EPI_RESIDUAL = 1, EPI_SWIGLU = 2, EPI_F32_ROWSCALE = 3, EPI_F32_RESIDUAL = 4 };
constexpr int kMaxGemmProblems = 8;
struct GemmProblemDesc {
    const void *a;   // [M, K] bf16, row pitch K
    const void *a_lo;  // [M, K] low part of A (two-pass GEMMs): bf16, or e4m3(lo * 2^8) bytes (lo_fp8)
    const void *b0;  // [N, K] bf16 (SwiGLU: gate)
    const void *b1;  // [N, K] bf16 (SwiGLU: up), else unused
    void *c;         // [M, ldc] bf16
    const void *r;   // residual [M, ldc] bf16 (EPI_RESIDUAL), may equal c
    void *c_lo;      // SwiGLU low-part output [M, ldc] (bf16, or e4m3(lo * 2^8) bytes when lo_fp8), may be null
    const float *rowscale;  // [M] fp32 per-row scale, may be null (= 1)
    const void *b0_lo = nullptr;  // lo_fp8: e5m2(b0 * 2^-8) bytes [N, K]
    const void *b1_lo = nullptr;  // lo_fp8: e5m2(b1 * 2^-8) bytes [N, K] (SwiGLU)
    // The next RMSNorm's operand, formed in the EPI_F32_RESIDUAL epilogue from the
    // updated fp32 rows x: n_hi/n_lo = x * nw as hi + lo (lo as bf16, or as
    // e4m3(lo * 2^8) bytes when lo_fp8; null in one-pass mode), row pitch N, and
    // ssq_out[t * M + row] = sum of x^2 over the columns of N-tile t, in column order.
    const void *nw = nullptr;     // [N] bf16 norm weight; null: no operand is formed
    void *n_hi = nullptr;
    void *n_lo = nullptr;
    float *ssq_out = nullptr;     // [ceil(N / kGemmTileN), M]
    // Row scale from such partial sums (in place of rowscale): 1 / sqrt(sum / K + eps),
    // the parts added in order.
    const float *ssq_in = nullptr;  // [ssq_parts, M]
};
// Output columns per GEMM tile (the partial sums of squares come one per tile).
constexpr int kGemmTileN = 256;
// How output tiles map to CTAs: one CTA per 128 x 256 tile (the default), or a
// cluster of two CTAs (two SMs) per 256 x 256 tile sharing cta_group::2
// products, which streams a third fewer operand bytes per SM for the same
// tensor work but pads M to a multiple of 256.
enum GemmForm { GEMM_FORM_DEFAULT = 0, GEMM_FORM_SINGLE = 1, GEMM_FORM_PAIR = 2 };
struct GemmOptions {
    int ssq_parts = 0;  // partial sums per row in ssq_in
    float eps = 0.f;
    int form = GEMM_FORM_DEFAULT;
    // Output columns [n_skip_lo, n_skip_hi) that nobody reads: their tiles are not
    // computed and those columns of C are left as they are.  Both bounds are
    // multiples of kGemmTileN and n_skip_hi < N (not with EPI_SWIGLU or nw).
    int n_skip_lo = 0, n_skip_hi = 0;
};
// n_pass 1: A only; 2: A_hi then A_lo.  lo_fp8: the A_lo pass runs on the fp8
// tensor cores (e4m3 A_lo * 2^8 times e5m2 B * 2^-8); needs K % 128 == 0.
cudaError_t gemm_tc(const GemmProblemDesc *probs, int n_problems, int M, int N, int K, int ldc, int epi,
                    int n_pass, int lo_fp8, uint32_t *status, cudaStream_t st, GemmOptions norm = GemmOptions{});
// fp8 low-pass helpers (layer_kernels.cu): e5m2(w * 2^-8) for n bf16 weights.
cudaError_t prepare_lo8(const void *w, void *w_lo8, int64_t n, cudaStream_t st);

}  // namespace sr
