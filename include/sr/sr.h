/*
 * sr.h -- C ABI of the suffix-replay state-reconstruction library (libsr.so).
 *
 * What it computes.  A hybrid LLM's linear-attention layers carry recurrent
 * states that cannot be rolled back to an arbitrary prefix boundary.  Suffix
 * replay rebuilds them by running the linear state update
 *         S_t = A_t(S_{t-1}) + B_t,  S_0 = 0
 * over only a short recent suffix of the matched prefix
 * ("SuffixReplay: Prefix Caching via Suffix Replay for Hybrid LLMs",
 *  Theoretical Foundation, Eq. 2 and Eq. 4; "Tail-Replay: Escaping the Curse
 *  of Linear Attention in Prefix Caching for Hybrid LLMs", Sec. 3, where the
 *  replay length is k = ceil(r m) for a matched prefix of m tokens and every
 *  group starts its tail from a zero state).
 *
 * Entry points (all asynchronous on the given CUDA stream):
 *   sr_gdn_replay     one Gated DeltaNet layer from raw q/k/v/g/beta
 *   sr_group_replay   whole replay groups from cached anchor hiddens plus
 *                     layer weights (RMSNorm, in_proj, conv, gates, the
 *                     recurrence, gated norm, out_proj, SwiGLU MLP)
 *   sr_mamba2_replay  the Mamba2 per-head-decay variant
 *
 * Conventions shared by every call
 * --------------------------------
 * Memory.  Every pointer in an args struct is a DEVICE pointer unless its
 *   comment says "host".  The caller owns all buffers; the library never
 *   allocates, never frees, and keeps no state between calls except a
 *   thread-local error string.  Scratch memory is the caller's `workspace`
 *   (device, 256-byte aligned) of at least the size the matching
 *   *_workspace() query returns for the same args.
 * Packing.  Sequences are packed token-major and delimited by `cu_seqlens`
 *   (device, int32, n_seqs+1 entries, cu[0] = 0, non-decreasing,
 *   cu[n_seqs] = total_tokens): "Batched replay: multiple hits packed into one
 *   variable-length execution with device-side boundaries" (SuffixReplay,
 *   System Design, Pipelined Replay Path).  The host passes n_seqs,
 *   total_tokens and an upper bound max_seqlen on every sequence length (used
 *   only to size grids).  Zero-length sequences are allowed.
 * Layouts are row-major, last index contiguous.  bf16 is IEEE bfloat16.
 * Asynchrony.  A call validates its host-side arguments, enqueues kernels on
 *   `stream` (a cudaStream_t; NULL = the legacy default stream) and returns.
 *   It never synchronises and never allocates.
 * Errors.  A call returns SR_OK or an error code; sr_last_error() gives a
 *   message for the calling thread's last failure.  Nothing is enqueued when
 *   host-side validation fails.  Device-side checks (a cu_seqlens entry out of
 *   range, a sequence longer than max_seqlen) cannot be seen by the host
 *   without a sync: the kernels skip the offending sequence, leave its outputs
 *   untouched and OR a flag into the workspace's device status word, which
 *   sr_device_status() reads.  Each call clears the status word first.
 */
#ifndef SR_SR_H
#define SR_SR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SR_API __attribute__((visibility("default")))
#else
#define SR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sr_status {
    SR_OK = 0,
    SR_ERR_INVALID_ARG = 1,  /* null pointer, bad size, inconsistent shape  */
    SR_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. head dim)   */
    SR_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small  */
    SR_ERR_CUDA = 4,         /* a CUDA runtime call failed (message says)   */
    SR_ERR_DEVICE = 5        /* reported by sr_device_status only           */
} sr_status;

typedef enum sr_dtype { SR_BF16 = 0, SR_FP32 = 1 } sr_dtype;

/* Device status word flags (sr_device_status). */
#define SR_DEV_BAD_CU_SEQLENS 0x1u  /* cu[n] > cu[n+1], cu[n+1] > total, cu[0] != 0 */
#define SR_DEV_SEQ_TOO_LONG 0x2u    /* a sequence is longer than max_seqlen       */
#define SR_DEV_TIMEOUT 0x4u         /* a bounded on-chip wait gave up (kernel exited early) */
#define SR_DEV_BAD_INDEX 0x8u       /* an anchor or row index outside its table (row read as zero / skipped) */
#define SR_DEV_BAD_ACCESS 0x10u     /* bounds-checked build (libsr_checked.so) only: a global-memory access
                                       outside its buffer was found and skipped */

/* Kernel selection for sr_gdn_replay. */
typedef enum sr_gdn_algo {
    SR_GDN_AUTO = 0,        /* bf16: the tcgen05 two-phase form; fp32: sequential      */
    SR_GDN_SEQUENTIAL = 1,  /* token-by-token fp32 FFMA recurrence (any dtype)          */
    SR_GDN_CHUNKED = 2,     /* chunked WY/UT form, warp-level mma.sync (bf16 only)      */
    SR_GDN_TCGEN05 = 3,     /* chunked WY/UT form on tcgen05, state in tensor memory
                               (bf16; d = 64 runs on 128-wide tiles whose upper halves
                               stay zero), two phases: the state-free part
                               of every chunk (masks, (I + A)^{-1}, W) for all chunks at
                               once, then the per-sequence state chain.  Workspace grows
                               by 56.5 KB per (chunk slot, V head), with
                               floor(total_tokens / 64) + n_seqs slots.                  */
    SR_GDN_TCGEN05_FUSED = 4, /* the same in one kernel per (sequence, V head), every
                               step of a chunk in order; no scratch                     */
} sr_gdn_algo;

/* ------------------------------------------------------------------------
 * sr_gdn_replay -- one Gated DeltaNet layer's recurrence over packed suffixes.
 *
 * For every sequence n and V head h (QK head h / (h_v / h_k)), starting from
 * S = h0[n,h] (or 0 when h0 is NULL), for each token t of the sequence:
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     alpha_t = exp(g_t),   o_t = scale * S_t q_t
 * ("Tail-Replay", Sec. 2: Gated DeltaNet with gate alpha in (0,1] and a rank-1
 * correction; SuffixReplay, Eq. 4 with S_0 = 0).  S is d_v x d_k (row = value
 * channel).  The final S of every (n, h) is written to s_out.
 *
 *   q, k       [total_tokens, h_k, d_k]   bf16 or fp32 (dtype)
 *   v          [total_tokens, h_v, d_v]   same dtype
 *   g          [total_tokens, h_v]        fp32, natural-log decay (<= 0)
 *   beta       [total_tokens, h_v]        fp32
 *   h0         [n_seqs, h_v, d_v, d_k]    fp32, may be NULL (zero state)
 *   o          [total_tokens, h_v, d_v]   dtype, may be NULL (state only)
 *   s_out      [n_seqs, h_v, d_v, d_k]    fp32, required
 *   scale      multiplier of the output; 0 selects 1/sqrt(d_k)
 * Supported: d_k = d_v in {64, 128}; h_v % h_k == 0.  Output buffers must not
 * alias inputs.
 * ---------------------------------------------------------------------- */
typedef struct sr_gdn_args {
    const void *q;
    const void *k;
    const void *v;
    const float *g;
    const float *beta;
    const int32_t *cu_seqlens;
    const float *h0;
    void *o;
    float *s_out;
    int32_t dtype;        /* sr_dtype */
    int32_t algo;         /* sr_gdn_algo */
    int32_t n_seqs;
    int32_t total_tokens;
    int32_t max_seqlen;
    int32_t h_k, h_v, d_k, d_v;
    float scale;
} sr_gdn_args;

SR_API size_t sr_gdn_replay_workspace(const sr_gdn_args *args);
SR_API sr_status sr_gdn_replay(const sr_gdn_args *args, void *workspace, size_t workspace_bytes,
                        void *stream);

/* ------------------------------------------------------------------------
 * sr_mamba2_replay -- Mamba2 variant: per-head scalar decay, no erase.
 *
 *     S_t = exp(dt_t A_h) S_{t-1} + dt_t x_t B_t^T,   y_t = S_t C_t
 * (SuffixReplay, Eq. 4: "per-head decay in Mamba2").  S is P x N_s per head;
 * head h reads B/C group h / (n_heads / n_groups).
 *
 *   x          [total_tokens, n_heads, head_dim]   bf16
 *   B, C       [total_tokens, n_groups, d_state]   bf16
 *   dt         [total_tokens, n_heads]             fp32 (already positive)
 *   A          [n_heads]                           fp32 (negative)
 *   h0         [n_seqs, n_heads, head_dim, d_state] fp32, may be NULL
 *   y          [total_tokens, n_heads, head_dim]   bf16, may be NULL
 *   s_out      [n_seqs, n_heads, head_dim, d_state] fp32, required
 * Supported: head_dim = 64, d_state = 128.
 * algo: SR_MAMBA2_AUTO picks the tcgen05 chunk kernel for one B/C group and
 *   an even head count, the fp32 token-by-token kernel otherwise;
 *   SR_MAMBA2_SEQUENTIAL, SR_MAMBA2_CHUNKED (mma.sync chunk kernel, same
 *   shape limits as the tcgen05 one) and SR_MAMBA2_TCGEN05 force a kernel
 *   (SR_ERR_UNSUPPORTED when the shape does not fit it).
 * ---------------------------------------------------------------------- */
typedef enum sr_mamba2_algo {
    SR_MAMBA2_AUTO = 0,
    SR_MAMBA2_SEQUENTIAL = 1,
    SR_MAMBA2_CHUNKED = 2,
    SR_MAMBA2_TCGEN05 = 3
} sr_mamba2_algo;

typedef struct sr_mamba2_args {
    const void *x;
    const void *B;
    const void *C;
    const float *dt;
    const float *A;
    const int32_t *cu_seqlens;
    const float *h0;
    void *y;
    float *s_out;
    int32_t n_seqs;
    int32_t total_tokens;
    int32_t max_seqlen;
    int32_t n_heads, head_dim, n_groups, d_state;
    int32_t algo;  /* sr_mamba2_algo */
} sr_mamba2_args;

SR_API size_t sr_mamba2_replay_workspace(const sr_mamba2_args *args);
SR_API sr_status sr_mamba2_replay(const sr_mamba2_args *args, void *workspace, size_t workspace_bytes,
                           void *stream);

/* ------------------------------------------------------------------------
 * sr_group_replay -- replay whole linear-attention groups from anchors.
 *
 * A group is a run of consecutive Gated DeltaNet layers between two full-
 * attention layers; its anchor is the cached hidden entering the group (the
 * preceding full-attention layer's output).  Every layer's recurrent state
 * starts at zero and full-attention layers are skipped (SuffixReplay,
 * Algorithm Design 1; Tail-Replay, Sec. 3).  Per layer:
 *     h = RMSNorm(x) w_in_norm;  p = h W_in^T = [q|k|v|z|b|a]
 *     causal depthwise conv (width conv_width, zero left padding per
 *     sequence) + SiLU over [q|k|v]; q, k L2-normalised per head (eps 1e-6)
 *     g = -exp(A_log) softplus(a + dt_bias);  beta = sigmoid(b)
 *     gated-delta recurrence as in sr_gdn_replay (scale 1/sqrt(d_k))
 *     y = RMSNorm_head(o) w_gnorm * SiLU(z);  x = x + y W_out^T
 *     x = x + W_down(SiLU(W_gate hh) * W_up hh),  hh = RMSNorm(x) w_post_norm
 * mode SR_MODE_SKIP stops the group's LAST layer after its recurrence (its
 * gated norm, out_proj and MLP change no state: "Tail-Replay", Sec. 3 omits
 * the final group FFN); SR_MODE_FULL runs every layer to its MLP.
 * Groups are independent; n_groups > 1 replays them group-parallel with the
 * same cu_seqlens (one request's suffix seen by every group).
 *
 * Shapes: proj_dim = 2 h_k d_k + 2 h_v d_v + 2 h_v, conv_dim = 2 h_k d_k + h_v d_v.
 * Supported: n_groups <= 8, d_k = d_v = 128, conv_width = 4, hidden % 64 == 0,
 * inter % 64 == 0, (h_v d_v) % 64 == 0, h_v % h_k == 0.  Workspace: the size
 * sr_group_replay_workspace() returns (it grows linearly with total_tokens
 * and n_groups; about 135-170 KB per token per group at hidden 2560).
 * ---------------------------------------------------------------------- */
typedef struct sr_layer_weights {
    const void *w_in_norm;   /* [hidden] bf16 */
    const void *w_in;        /* [proj_dim, hidden] bf16 */
    const void *conv_w;      /* [conv_dim, conv_width] bf16 */
    const float *a_log;      /* [h_v] fp32 */
    const float *dt_bias;    /* [h_v] fp32 */
    const void *w_gnorm;     /* [d_v] bf16, shared by all V heads */
    const void *w_out;       /* [hidden, h_v d_v] bf16 */
    const void *w_post_norm; /* [hidden] bf16 */
    const void *w_gate;      /* [inter, hidden] bf16 */
    const void *w_up;        /* [inter, hidden] bf16 */
    const void *w_down;      /* [hidden, inter] bf16 */
    /* SR_PREC_SPLIT_FP8 only (NULL otherwise): the low-pass copies of the five
     * projections, same shapes, one byte per weight: e5m2(W * 2^-8), written by
     * sr_prepare_lo8_weights once per model. */
    const void *w_in_lo8;
    const void *w_out_lo8;
    const void *w_gate_lo8;
    const void *w_up_lo8;
    const void *w_down_lo8;
} sr_layer_weights;

typedef struct sr_layer_outputs {
    float *s_out;     /* [n_seqs, h_v, d_v, d_k] fp32, required */
    void *conv_out;   /* [n_seqs, conv_dim, conv_width-1] bf16, oldest row first, required */
    void *hidden_out; /* [total_tokens, hidden] bf16, may be NULL: hidden after the layer's
                         MLP; must be NULL for the last layer in SR_MODE_SKIP */
} sr_layer_outputs;

/* Initial states of one layer, for a continuation.  A replay starts every
 * layer from zero; the unmatched tokens after it are then processed from the
 * rebuilt states ("Tail-Replay", Sec. 3; "SuffixReplay", Pipelined Replay
 * Path: extend consumes the reconstructed state).  With these set, layer l's
 * recurrence starts at s_in and its causal conv reads conv_in's rows as the
 * (conv_width-1) tokens before each sequence, so the call continues exactly
 * where a previous call over the preceding tokens stopped (up to the bf16
 * rounding of the stored conv state).  s_in may equal the layer's s_out and
 * conv_in its conv_out (in-place continuation). */
typedef struct sr_layer_state {
    const float *s_in;    /* [n_seqs, h_v, d_v, d_k] fp32, or NULL: zero state */
    const void *conv_in;  /* [n_seqs, conv_dim, conv_width-1] bf16, oldest row first, or NULL: zero padding */
} sr_layer_state;

typedef enum sr_group_mode { SR_MODE_SKIP = 0, SR_MODE_FULL = 1 } sr_group_mode;

/* Arithmetic of the group's activations.
 * SR_PREC_SPLIT (default): the residual stream, the in_proj output and the
 *   gates are fp32; every activation operand of a tensor-core product (the
 *   normalised hidden, the gated-norm output, the SwiGLU output, k and v) is
 *   carried as an exact pair of bf16 matrices hi + lo, so each projection runs
 *   two bf16 MMA passes (the weights are exact bf16).  The states then track
 *   the fp64 layer math to ~1e-4 of max|S| over a 3-layer group.
 * SR_PREC_BF16: one pass per projection with bf16 activations (the usual bf16
 *   serving arithmetic); about half the tensor-core work, state error a few
 *   1e-3 of max|S| after three layers.
 * SR_PREC_SPLIT_FP8: as SR_PREC_SPLIT, but the low pass of every projection
 *   runs on the fp8 tensor cores: the activation's low part as
 *   e4m3(lo * 2^8) times the prepared weight copy e5m2(W * 2^-8), accumulated
 *   with the bf16 high pass (the powers of two cancel).  The low part's own
 *   rounding (3 mantissa bits) and the weight copy's (2 bits) act on a term
 *   2^-9 of the product, so the states stay within about 5e-4 of max|S| over a
 *   3-layer group, at three quarters of SR_PREC_SPLIT's tensor time.  Needs the
 *   *_lo8 weight pointers, and hidden, inter and h_v d_v multiples of 128. */
typedef enum sr_group_precision { SR_PREC_SPLIT = 0, SR_PREC_BF16 = 1, SR_PREC_SPLIT_FP8 = 2 } sr_group_precision;

/* Optional per-launch timing.  When sr_group_args.profile is non-NULL the
 * call records events[2i] before and events[2i+1] after its i-th kernel
 * launch on `stream` (cudaEvent_t handles the caller created) and stores the
 * launch's kind in kinds[i], for up to `capacity` launches; `count` returns
 * how many launches the call made (it may exceed capacity: the excess is not
 * timed).  Recording events adds no synchronisation. */
typedef enum sr_kernel_kind {
    SR_K_ROW_PREP = 0,   /* RMSNorm factor + activation split            */
    SR_K_GEMM_IN = 1,    /* in_proj                                      */
    SR_K_CONV = 2,       /* conv + SiLU + L2 norm + gates (+ conv state) */
    SR_K_GDN = 3,        /* chunked gated-delta recurrence               */
    SR_K_GATED_NORM = 4, /* gated RMSNorm                                */
    SR_K_GEMM_OUT = 5,   /* out_proj + residual                          */
    SR_K_GEMM_GATEUP = 6,/* MLP gate/up + SwiGLU                         */
    SR_K_GEMM_DOWN = 7,  /* MLP down + residual                          */
    SR_K_CAST = 8,       /* fp32 hidden -> bf16 hidden_out               */
    SR_K_COUNT = 9
} sr_kernel_kind;

typedef struct sr_profile {
    void *const *events;  /* host array [2 * capacity] of cudaEvent_t */
    int32_t *kinds;       /* host array [capacity] */
    int32_t capacity;
    int32_t count;        /* out */
} sr_profile;

typedef struct sr_group_args {
    const void *const *anchors;       /* host array [n_groups] of device [total_tokens, hidden] bf16 */
    const int32_t *cu_seqlens;
    const sr_layer_weights *weights;  /* host array [n_groups * n_layers], group-major */
    const sr_layer_outputs *outputs;  /* host array [n_groups * n_layers], group-major */
    int32_t n_groups, n_layers;
    int32_t n_seqs, total_tokens, max_seqlen;
    int32_t hidden, inter, h_k, h_v, d_k, d_v, conv_width;
    float eps;
    int32_t mode;                     /* sr_group_mode */
    int32_t precision;                /* sr_group_precision */
    sr_profile *profile;              /* host, may be NULL */
    /* Continuation (see sr_layer_state): host array [n_groups * n_layers],
     * group-major, or NULL for a replay from zero. */
    const sr_layer_state *initial;
    /* Token-wise sparse anchors ("SuffixReplay", Algorithm Design 2): when
     * non-NULL, a device int32 array [total_tokens]; replay token t of every
     * group reads row anchor_index[t] of that group's anchor pool
     * anchors[g] ([anchor_rows, hidden] bf16).  An index outside
     * [0, anchor_rows) reads a zero row and sets SR_DEV_BAD_INDEX.  NULL:
     * anchors[g] holds the packed suffix itself ([total_tokens, hidden]). */
    const int32_t *anchor_index;
    int32_t anchor_rows;
    /* Per-layer hand-off ("SuffixReplay", System Design, Pipelined Replay
     * Path: the forward pass waits only at the layer that consumes a rebuilt
     * state): a host array [n_layers] of cudaEvent_t handles the caller
     * created, or NULL; NULL entries are skipped.  layer_done[l] is recorded on
     * `stream` right after the launch that completes layer l's s_out and
     * conv_out for every group, so work on another stream that needs only layer
     * l's rebuilt state can wait on it instead of on the whole call.  It does
     * not cover hidden_out[l], which the layer's MLP writes later.  Recording
     * adds no synchronisation. */
    void *const *layer_done;
} sr_group_args;

SR_API size_t sr_group_replay_workspace(const sr_group_args *args);
SR_API sr_status sr_group_replay(const sr_group_args *args, void *workspace, size_t workspace_bytes,
                          void *stream);

/* ------------------------------------------------------------------------
 * sr_group_replay_noalloc -- sr_group_replay without a caller workspace.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory: a plug-in given only its input and
 * output buffers by the host framework, an engine whose spare HBM is all
 * promised to its KV-cache pool, or a path that cannot afford the implicit
 * synchronisation of cudaMalloc.  The scratch is a fixed device array of
 * SR_GROUP_NOALLOC_SCRATCH_BYTES inside this library, which every GPU that
 * loads the library keeps until the process exits.  The call allocates
 * nothing and computes exactly what sr_group_replay computes.
 *
 * Limit: a replay whose sr_group_replay_workspace() exceeds
 * SR_GROUP_NOALLOC_SCRATCH_BYTES is rejected with SR_ERR_WORKSPACE.  At
 * hidden 2560, intermediate 9216 and 32 V heads a group takes about 169 KB
 * per token with SR_PREC_SPLIT (158 KB with SR_PREC_SPLIT_FP8, 134 KB with
 * SR_PREC_BF16) plus 1.8 MB per sequence for the gated-delta chunk images,
 * so one sequence of up to 191 tokens fits (197 and 241).
 * Set-up: a call made outside a stream capture looks up the array's device
 * address on the current device (cudaGetSymbolAddress), so the first call on
 * a device must come before any stream capture; a call inside a capture
 * reuses the address found by the last call outside one on that device (and
 * fails with SR_ERR_INVALID_ARG if there was none).  Sharing: every call on a device uses the same
 * array, which keeps the previous call's contents, so calls whose kernels
 * overlap on the GPU (for example on two streams) race; serialise them.
 * status_scratch (may be NULL) receives the array's device address, which
 * sr_device_status() accepts in place of a workspace.
 * ---------------------------------------------------------------------- */
#define SR_GROUP_NOALLOC_SCRATCH_BYTES (32u << 20)

SR_API sr_status sr_group_replay_noalloc(const sr_group_args *args, void *stream,
                                         const void **status_scratch);

/* ------------------------------------------------------------------------
 * sr_prepare_lo8_weights -- the low-pass weight copy of SR_PREC_SPLIT_FP8.
 *
 * The paper has no counterpart: this belongs to this library's split
 * arithmetic.  Writes w_lo8[i] = e5m2(w[i] * 2^-8) (round to nearest,
 * saturating) for n bf16 weights, on `stream`.  Run it once per weight matrix
 * when a model is loaded; every replay then reads the copy.  w and w_lo8 are
 * device pointers; returns SR_ERR_INVALID_ARG for n < 0 or a NULL pointer
 * with n > 0.
 * ---------------------------------------------------------------------- */
SR_API sr_status sr_prepare_lo8_weights(const void *w, void *w_lo8, int64_t n, void *stream);

/* ------------------------------------------------------------------------
 * sr_anchor_capture -- write selected hidden rows into an anchor pool.
 *
 * The forward pass that serves a request caches, for each replay group, the
 * hidden entering the group at selected token positions: the anchors that a
 * later replay starts from.  The pages store them in a sidecar pool beside
 * the KV pages, written by indexed copies inside captured CUDA graphs from a
 * destination table prepared on the host ("SuffixReplay", System Design,
 * Anchor Sidecar).  This call is that indexed copy:
 *     pool[dst_rows[i], :] = hidden_states[src_rows[i], :]   for i < n.
 * Layout: hidden_states [src_rows_total, hidden] bf16 and pool [pool_rows,
 * hidden] bf16, row-major, both 16-byte aligned, hidden % 8 == 0; src_rows and
 * dst_rows are device int32 [n].  Two entries with the same dst_rows race
 * (one of them wins).  A pair with an index out of range is skipped and sets
 * SR_DEV_BAD_INDEX in the workspace status word.  Workspace: 256 bytes (the
 * status word).  No allocation, no host synchronisation: the call can be
 * captured into a CUDA graph whose index tables the host rewrites in place
 * between launches.
 * ---------------------------------------------------------------------- */
typedef struct sr_capture_args {
    const void *hidden_states; /* [src_rows_total, hidden] bf16, device */
    void *pool;                /* [pool_rows, hidden] bf16, device */
    const int32_t *src_rows;   /* [n] device */
    const int32_t *dst_rows;   /* [n] device */
    int32_t n, hidden, src_rows_total, pool_rows;
} sr_capture_args;

SR_API sr_status sr_anchor_capture(const sr_capture_args *args, void *workspace, size_t workspace_bytes,
                                   void *stream);

/* ------------------------------------------------------------------------
 * sr_sparse_anchor_plan -- host: which anchors a token-sparse replay reads.
 *
 * Token-wise sparse anchors ("SuffixReplay", Algorithm Design 2): each page
 * of page_size tokens (64 on the pages) keeps anchors_per_page of its
 * positions (density 1/16: 4 per page); SR_ANCHORS_PAGE_TAIL puts them on
 * the page's last positions (the dense sampling near the page boundary that
 * the pages prefer), SR_ANCHORS_UNIFORM at offsets (i+1) page_size /
 * anchors_per_page - 1.  The replay budget is counted in anchors (Algorithm
 * Design 3): k = min(ceil(ratio * n_prefix), k_max, anchors present), and the
 * replay reads the last k anchors of the prefix, oldest first.
 * Outputs (host arrays of `capacity` entries, either may be NULL):
 * positions[j], the token position of replayed anchor j, and pool_rows[j],
 * its row in a page-major pool holding anchors_per_page rows per page:
 * block_table[page] * anchors_per_page + slot (block_table NULL: the page
 * index itself).  *count receives k; capacity < k is SR_ERR_INVALID_ARG
 * (with *count set, so the caller can size its arrays).  Pure host code.
 * ---------------------------------------------------------------------- */
typedef enum sr_anchor_layout { SR_ANCHORS_PAGE_TAIL = 0, SR_ANCHORS_UNIFORM = 1 } sr_anchor_layout;

typedef struct sr_anchor_plan_args {
    int64_t n_prefix;             /* matched prefix length in tokens */
    int32_t page_size;            /* tokens per page (64) */
    int32_t anchors_per_page;     /* page_size * density (4) */
    int32_t layout;               /* sr_anchor_layout */
    int32_t k_max;                /* budget cap in anchors (512 / 256 on the pages) */
    double ratio;                 /* budget ratio (0.05) */
    const int32_t *block_table;   /* host [pages], may be NULL */
} sr_anchor_plan_args;

SR_API sr_status sr_sparse_anchor_plan(const sr_anchor_plan_args *args, int64_t *positions, int32_t *pool_rows,
                                       int64_t capacity, int64_t *count);

/* ------------------------------------------------------------------------
 * sr_checkpoint_plan -- host: where to keep recurrent-state checkpoints.
 *
 * The checkpoint alternative to replay ("Sparse Prefix Caching for Hybrid and
 * Recurrent LLM Serving", Methodology): a retained prefix of n tokens keeps
 * exact states at up to m_max positions C in 1..n; a request overlapping the
 * prefix to depth t resumes from max({0} u {c in C : c <= t}) and recomputes
 * the rest.  Given p[t] (t = 0..n, any non-negative weights: the overlap-depth
 * distribution or a histogram of it), the call returns the placement that
 * minimises sum_t p[t] (t - l(t; C)), by the exact dynamic program of that
 * page, O(n m_max) with the monotone convex-hull trick.
 *   positions  host [m_max] out: the chosen positions, increasing (fewer than
 *              m_max when more checkpoints would not lower the cost)
 *   count      host out: how many positions were written
 *   expected_cost  host out (may be NULL): sum_t p[t] r(t; C) of the result
 * Pure host code.  Errors: SR_ERR_INVALID_ARG for NULL pointers, n < 0,
 * m_max < 0 or a negative weight; SR_ERR_UNSUPPORTED when n (m_max + 1)
 * exceeds 2^31.
 * ---------------------------------------------------------------------- */
SR_API sr_status sr_checkpoint_plan(const double *p, int64_t n, int32_t m_max, int64_t *positions, int32_t *count,
                                    double *expected_cost);

/* ------------------------------------------------------------------------
 * Status and diagnostics.
 * ---------------------------------------------------------------------- */
/* Message for the calling thread's last failed call ("" if none). */
SR_API const char *sr_last_error(void);

/* Copies the device status word of `workspace` (written by the last call that
 * used it) into *flags (SR_DEV_* bits), synchronising `stream`.  Returns
 * SR_ERR_DEVICE when any flag is set, SR_OK when none is. */
SR_API sr_status sr_device_status(const void *workspace, void *stream, uint32_t *flags);

/* Library version, e.g. 0x000100 for 0.1.0. */
SR_API int32_t sr_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SR_SR_H */
