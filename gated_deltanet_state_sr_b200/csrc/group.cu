// sr_group_replay: replay whole linear-attention groups from cached anchors.
//
// A group is a run of Gated DeltaNet layers between two full-attention
// layers; its anchor is the hidden entering it.  Every state starts at zero
// and full-attention layers are skipped ("SuffixReplay", Algorithm Design 1;
// "Tail-Replay", Sec. 3).  Two options widen the replay: anchors gathered
// from a pool through an index table (token-wise sparse anchors,
// "SuffixReplay", Algorithm Design 2), and initial states per layer, which
// continue a previous call exactly (the extend step that follows a replay).
// Per layer, all groups of the call advance together (each launch covers
// every group through per-group pointers):
//   row_prep(x, w_in_norm) -> in_proj GEMM (fp32 out, RMSNorm factor in the
//   epilogue) -> conv + gates (+ conv state) -> chunked gated-delta recurrence
//   -> gated norm -> out_proj GEMM (+= residual) -> gate/up GEMM (SwiGLU
//   epilogue) -> down GEMM (+= residual).
// Only layer 0 runs row_prep (it also gathers the anchors): the out_proj and
// down epilogues form the next RMSNorm's operand (x * w as hi + lo) from the
// updated residual rows, with each row's sum of squares per 256-column tile,
// and the GEMM that consumes the operand adds those sums in order into its
// RMSNorm factor.
// In skip mode the last layer stops after its recurrence: its gated norm,
// out_proj and MLP change no state ("Tail-Replay", Sec. 3 omits the final
// group FFN).  The residual stream is kept in fp32 between layers.
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace sr {

namespace {

struct Dims {
    int G, L, N, T, H, I, hk, hv, d, qd, vd, conv_dim, proj;
    bool split;  // activations carried as hi + lo
    bool lo8;    // the lo parts of the projection operands as e4m3 bytes (fp8 low pass)
};

Dims dims_of(const sr_group_args &a) {
    Dims m;
    m.G = a.n_groups;
    m.L = a.n_layers;
    m.N = a.n_seqs;
    m.T = a.total_tokens;
    m.H = a.hidden;
    m.I = a.inter;
    m.hk = a.h_k;
    m.hv = a.h_v;
    m.d = a.d_k;
    m.qd = a.h_k * a.d_k;
    m.vd = a.h_v * a.d_v;
    m.conv_dim = 2 * m.qd + m.vd;
    m.proj = m.conv_dim + m.vd + 2 * m.hv;
    m.split = a.precision == SR_PREC_SPLIT || a.precision == SR_PREC_SPLIT_FP8;
    m.lo8 = a.precision == SR_PREC_SPLIT_FP8;
    return m;
}

struct GroupBufs {
    float *x32, *r, *ssq, *p, *gate, *beta;
    __nv_bfloat16 *a_hi, *q, *k, *k_lo, *v, *v_lo, *o, *h_hi;
    void *a_lo, *h_lo;  // bf16, or e4m3 bytes with the fp8 low pass
};

// Partial sums of squares per hidden row: one per 256-column GEMM tile.
int ssq_parts(const Dims &m) { return (m.H + kGemmTileN - 1) / kGemmTileN; }

// Carves the per-group scratch buffers, then the chunk images of the two-phase
// gated-delta kernels (shared by the layers; *img), out of the workspace
// (after its header).  Returns the bytes used; with base == nullptr only sizes
// are computed.
size_t carve(const Dims &m, char *base, GroupBufs *out, void **img = nullptr) {
    size_t off = kWsHeader;
    auto take = [&](size_t bytes) {
        char *ptr = base ? base + off : nullptr;
        off += align_up(bytes, kWsAlign);
        return ptr;
    };
    const size_t T = size_t(m.T);
    // A holds the RMSNorm operands [T, H]; the MLP buffer h holds the SwiGLU output
    // [T, I] and, before out_proj, the gated norm's y [T, h_v d_v]
    const size_t hmax = size_t(m.I > m.vd ? m.I : m.vd);
    for (int g = 0; g < m.G; ++g) {
        GroupBufs b;
        b.x32 = reinterpret_cast<float *>(take(T * m.H * 4));
        b.r = reinterpret_cast<float *>(take(T * 4));
        b.ssq = reinterpret_cast<float *>(take(T * ssq_parts(m) * 4));
        b.p = reinterpret_cast<float *>(take(T * m.proj * 4));
        b.gate = reinterpret_cast<float *>(take(T * m.hv * 4));
        b.beta = reinterpret_cast<float *>(take(T * m.hv * 4));
        b.a_hi = reinterpret_cast<__nv_bfloat16 *>(take(T * m.H * 2));
        const size_t lo_elem = m.lo8 ? 1 : 2;
        b.a_lo = m.split ? take(T * m.H * lo_elem) : nullptr;
        b.q = reinterpret_cast<__nv_bfloat16 *>(take(T * m.qd * 2));
        b.k = reinterpret_cast<__nv_bfloat16 *>(take(T * m.qd * 2));
        b.k_lo = m.split ? reinterpret_cast<__nv_bfloat16 *>(take(T * m.qd * 2)) : nullptr;
        b.v = reinterpret_cast<__nv_bfloat16 *>(take(T * m.vd * 2));
        b.v_lo = m.split ? reinterpret_cast<__nv_bfloat16 *>(take(T * m.vd * 2)) : nullptr;
        b.o = reinterpret_cast<__nv_bfloat16 *>(take(T * m.vd * 2));
        b.h_hi = reinterpret_cast<__nv_bfloat16 *>(take(T * hmax * 2));
        b.h_lo = m.split ? take(T * hmax * lo_elem) : nullptr;
        if (out) out[g] = b;
    }
    void *im = take(gdn_tc_supported(m.d) ? gdn_tc_image_bytes(m.T, m.N, m.hv, m.G) : 0);
    if (img) *img = im;
    return off;
}

sr_status validate(const sr_group_args *a) {
    if (!a) return set_error(SR_ERR_INVALID_ARG, "args is NULL");
    if (a->n_groups < 1 || a->n_groups > kMaxGroups)
        return set_error(SR_ERR_UNSUPPORTED, "n_groups must be in [1, %d] (got %d)", kMaxGroups, a->n_groups);
    if (a->n_layers < 1) return set_error(SR_ERR_INVALID_ARG, "n_layers must be >= 1");
    if (!a->anchors || !a->weights || !a->outputs || !a->cu_seqlens)
        return set_error(SR_ERR_INVALID_ARG, "anchors, weights, outputs and cu_seqlens are required");
    if (a->n_seqs < 0 || a->total_tokens < 0 || a->max_seqlen < 0 || a->max_seqlen > a->total_tokens)
        return set_error(SR_ERR_INVALID_ARG, "bad n_seqs / total_tokens / max_seqlen");
    if (a->n_seqs > 65535) return set_error(SR_ERR_UNSUPPORTED, "n_seqs > 65535");
    if (a->d_k != 128 || a->d_v != 128) return set_error(SR_ERR_UNSUPPORTED, "d_k = d_v = 128 required");
    if (a->conv_width != 4) return set_error(SR_ERR_UNSUPPORTED, "conv_width 4 required");
    if (a->h_k <= 0 || a->h_v <= 0 || a->h_v % a->h_k)
        return set_error(SR_ERR_INVALID_ARG, "need h_v %% h_k == 0");
    if (a->hidden <= 0 || a->hidden % 64 || a->inter <= 0 || a->inter % 64)
        return set_error(SR_ERR_UNSUPPORTED, "hidden and inter must be positive multiples of 64");
    if (a->mode != SR_MODE_SKIP && a->mode != SR_MODE_FULL) return set_error(SR_ERR_INVALID_ARG, "bad mode");
    if (a->precision != SR_PREC_SPLIT && a->precision != SR_PREC_BF16 && a->precision != SR_PREC_SPLIT_FP8)
        return set_error(SR_ERR_INVALID_ARG, "bad precision");
    if (a->precision == SR_PREC_SPLIT_FP8 && (a->hidden % 128 || a->inter % 128 || (a->h_v * a->d_v) % 128))
        return set_error(SR_ERR_UNSUPPORTED, "SR_PREC_SPLIT_FP8 needs hidden, inter and h_v d_v multiples of 128");
    if (!(a->eps > 0.f)) return set_error(SR_ERR_INVALID_ARG, "eps must be > 0");
    if (a->anchor_index && a->anchor_rows < 1)
        return set_error(SR_ERR_INVALID_ARG, "anchor_index needs anchor_rows >= 1 (got %d)", a->anchor_rows);
    for (int g = 0; g < a->n_groups; ++g) {
        if (!a->anchors[g]) return set_error(SR_ERR_INVALID_ARG, "anchors[%d] is NULL", g);
        for (int l = 0; l < a->n_layers; ++l) {
            const sr_layer_weights &w = a->weights[g * a->n_layers + l];
            const sr_layer_outputs &o = a->outputs[g * a->n_layers + l];
            if (!w.w_in_norm || !w.w_in || !w.conv_w || !w.a_log || !w.dt_bias || !w.w_gnorm || !w.w_out ||
                !w.w_post_norm || !w.w_gate || !w.w_up || !w.w_down)
                return set_error(SR_ERR_INVALID_ARG, "weights of group %d layer %d incomplete", g, l);
            if (a->precision == SR_PREC_SPLIT_FP8 &&
                (!w.w_in_lo8 || !w.w_out_lo8 || !w.w_gate_lo8 || !w.w_up_lo8 || !w.w_down_lo8))
                return set_error(SR_ERR_INVALID_ARG,
                                 "SR_PREC_SPLIT_FP8: low-pass weights of group %d layer %d missing", g, l);
            if (!o.s_out || !o.conv_out)
                return set_error(SR_ERR_INVALID_ARG, "outputs of group %d layer %d need s_out and conv_out", g, l);
            if (o.hidden_out && a->mode == SR_MODE_SKIP && l == a->n_layers - 1)
                return set_error(SR_ERR_INVALID_ARG, "skip mode produces no hidden for the last layer");
        }
    }
    return SR_OK;
}

// Records caller events around launches when profiling is on.
struct Prof {
    sr_profile *p;
    cudaStream_t st;
    int i = 0;
    cudaError_t begin(int kind) {
        if (!p || i >= p->capacity) return cudaSuccess;
        p->kinds[i] = kind;
        return cudaEventRecord(static_cast<cudaEvent_t>(p->events[2 * i]), st);
    }
    cudaError_t end() {
        cudaError_t e = cudaSuccess;
        if (p && i < p->capacity) e = cudaEventRecord(static_cast<cudaEvent_t>(p->events[2 * i + 1]), st);
        ++i;
        if (p) p->count = i;
        return e;
    }
};

#define SR_TRY(expr)                                                        \
    do {                                                                    \
        cudaError_t e_ = (expr);                                            \
        if (e_ != cudaSuccess) return cuda_error(e_, "sr_group_replay: " #expr); \
    } while (0)

}  // namespace

}  // namespace sr

using namespace sr;

extern "C" size_t sr_group_replay_workspace(const sr_group_args *a) {
    if (validate(a) != SR_OK) return 0;
    return carve(dims_of(*a), nullptr, nullptr);
}

extern "C" sr_status sr_group_replay(const sr_group_args *a, void *ws, size_t ws_bytes, void *stream) {
    if (sr_status s = validate(a)) return s;
    const Dims m = dims_of(*a);
    const size_t need = carve(m, nullptr, nullptr);
    if (!ws) return set_error(SR_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
    if (reinterpret_cast<uintptr_t>(ws) % kWsAlign) return set_error(SR_ERR_WORKSPACE, "workspace not 256-byte aligned");
    if (ws_bytes < need) return set_error(SR_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t *status = static_cast<uint32_t *>(ws);
    SR_TRY(cudaMemsetAsync(status, 0, sizeof(uint32_t), st));
    if (m.T == 0 || m.N == 0) {
        // no tokens: every state is its initial state (zero for a replay)
        const size_t s_bytes = size_t(m.N) * m.hv * m.d * m.d * 4, c_bytes = size_t(m.N) * m.conv_dim * 3 * 2;
        for (int g = 0; g < m.G; ++g)
            for (int l = 0; l < m.L; ++l) {
                const sr_layer_outputs &o = a->outputs[g * m.L + l];
                const sr_layer_state *in = a->initial ? &a->initial[g * m.L + l] : nullptr;
                if (in && in->s_in) {
                    if (in->s_in != o.s_out)
                        SR_TRY(cudaMemcpyAsync(o.s_out, in->s_in, s_bytes, cudaMemcpyDeviceToDevice, st));
                } else {
                    SR_TRY(cudaMemsetAsync(o.s_out, 0, s_bytes, st));
                }
                if (in && in->conv_in) {
                    if (in->conv_in != o.conv_out)
                        SR_TRY(cudaMemcpyAsync(o.conv_out, in->conv_in, c_bytes, cudaMemcpyDeviceToDevice, st));
                } else {
                    SR_TRY(cudaMemsetAsync(o.conv_out, 0, c_bytes, st));
                }
            }
        for (int l = 0; a->layer_done && l < m.L; ++l)
            if (a->layer_done[l]) SR_TRY(cudaEventRecord(static_cast<cudaEvent_t>(a->layer_done[l]), st));
        return SR_OK;
    }
    GroupBufs B[kMaxGroups];
    void *img = nullptr;
    carve(m, static_cast<char *>(ws), B, &img);
    Prof prof{a->profile, st};
    if (a->profile) a->profile->count = 0;
    const int G = m.G, T = m.T;
    const int npass = m.split ? 2 : 1;

    for (int l = 0; l < m.L; ++l) {
        const bool last = l == m.L - 1;
        const bool stop = last && a->mode == SR_MODE_SKIP;
        auto W = [&](int g) -> const sr_layer_weights & { return a->weights[g * m.L + l]; };
        auto O = [&](int g) -> const sr_layer_outputs & { return a->outputs[g * m.L + l]; };
        auto I = [&](int g) -> const sr_layer_state * { return a->initial ? &a->initial[g * m.L + l] : nullptr; };

        // (1) layer 0: A = x * w_in_norm (hi/lo) and r = RMSNorm factor from the anchors
        // (gathered through the index table for sparse anchors), and the fp32 residual
        // stream; later layers find A and the partial sums in place (step 8)
        if (l == 0) {
            RowPrepBatch rp{};
            for (int g = 0; g < G; ++g) {
                rp.x[g] = a->anchors[g];
                rp.w[g] = static_cast<const __nv_bfloat16 *>(W(g).w_in_norm);
                rp.a_hi[g] = B[g].a_hi;
                rp.a_lo[g] = B[g].a_lo;
                rp.r[g] = B[g].r;
                rp.x32_out[g] = B[g].x32;
            }
            rp.T = T; rp.H = m.H; rp.x_f32 = 0; rp.eps = a->eps; rp.lo8 = m.lo8;
            rp.idx = a->anchor_index;
            rp.x_rows = a->anchor_index ? a->anchor_rows : T;
            rp.status = status;
            SR_TRY(prof.begin(SR_K_ROW_PREP));
            SR_TRY(row_prep(rp, G, st));
            SR_TRY(prof.end());
        }
        GemmOptions rn;
        rn.ssq_parts = ssq_parts(m);
        rn.eps = a->eps;
        // Tile form per projection, as measured on the whole-model replay (8 groups of
        // 1639 tokens, hidden 2560): CTA pairs for in_proj, out_proj and down_proj, whose
        // tiles then take 13 % less time per round; one CTA per tile for gate/up, where
        // the pairs' padding of M to 256 rows costs more than their rounds gain.
        GemmOptions pair_opt;
        pair_opt.form = GEMM_FORM_PAIR;

        // (2) p = r * (A W_in^T), fp32.  When the layer stops after its recurrence, the
        // z columns (read only by the gated norm) are not computed where they span
        // whole GEMM tiles.
        GemmProblemDesc gp[kMaxGemmProblems];
        for (int g = 0; g < G; ++g) {
            gp[g] = GemmProblemDesc{B[g].a_hi, B[g].a_lo, W(g).w_in, nullptr, B[g].p, nullptr, nullptr,
                                    l == 0 ? B[g].r : nullptr, W(g).w_in_lo8, nullptr};
            if (l > 0) gp[g].ssq_in = B[g].ssq;
        }
        GemmOptions in_opt = rn;
        in_opt.form = GEMM_FORM_PAIR;
        if (stop && m.conv_dim % kGemmTileN == 0 && m.vd % kGemmTileN == 0) {
            in_opt.n_skip_lo = m.conv_dim;
            in_opt.n_skip_hi = m.conv_dim + m.vd;
        }
        SR_TRY(prof.begin(SR_K_GEMM_IN));
        SR_TRY(gemm_tc(gp, G, T, m.proj, m.H, m.proj, EPI_F32_ROWSCALE, npass, m.lo8, status, st, in_opt));
        SR_TRY(prof.end());

        // (3) conv + SiLU + L2 norm + gates, conv state
        ConvBatch cb{};
        for (int g = 0; g < G; ++g) {
            cb.p[g] = B[g].p;
            cb.conv_w[g] = static_cast<const __nv_bfloat16 *>(W(g).conv_w);
            cb.a_log[g] = W(g).a_log;
            cb.dt_bias[g] = W(g).dt_bias;
            cb.q[g] = B[g].q;
            cb.k[g] = B[g].k;
            cb.k_lo[g] = B[g].k_lo;
            cb.v[g] = B[g].v;
            cb.v_lo[g] = B[g].v_lo;
            cb.gate[g] = B[g].gate;
            cb.beta[g] = B[g].beta;
            cb.conv_out[g] = static_cast<__nv_bfloat16 *>(O(g).conv_out);
            cb.conv_in[g] = I(g) ? static_cast<const __nv_bfloat16 *>(I(g)->conv_in) : nullptr;
        }
        cb.cu = a->cu_seqlens; cb.status = status; cb.n_seqs = m.N; cb.T = T; cb.ld = m.proj; cb.h_k = m.hk; cb.h_v = m.hv;
        cb.conv_dim = m.conv_dim; cb.b_off = m.conv_dim + m.vd;
        SR_TRY(prof.begin(SR_K_CONV));
        SR_TRY(conv_gates(cb, G, st));
        SR_TRY(prof.end());

        // (4) gated-delta recurrence from a zero state (or s_in on a continuation)
        GdnBatch gb{};
        for (int g = 0; g < G; ++g) {
            gb.q[g] = B[g].q;
            gb.k[g] = B[g].k;
            gb.v[g] = B[g].v;
            gb.k_lo[g] = B[g].k_lo;
            gb.v_lo[g] = B[g].v_lo;
            gb.g[g] = B[g].gate;
            gb.beta[g] = B[g].beta;
            gb.h0[g] = I(g) ? I(g)->s_in : nullptr;
            gb.o[g] = stop ? nullptr : B[g].o;
            gb.s_out[g] = O(g).s_out;
        }
        gb.cu = a->cu_seqlens; gb.img = img; gb.total = T; gb.max_len = a->max_seqlen; gb.h_k = m.hk; gb.h_v = m.hv;
        gb.scale = 1.0f / sqrtf(float(m.d)); gb.status = status;
        SR_TRY(prof.begin(SR_K_GDN));
        SR_TRY(gdn_tc_supported(m.d) ? gdn_tc_batch(gb, G, m.N, m.d, m.split, st)
                                     : gdn_chunked_batch(gb, G, m.N, m.d, m.split, st));
        SR_TRY(prof.end());
        // layer l's states (s_out from this launch, conv_out from the conv launch) are final
        if (a->layer_done && a->layer_done[l])
            SR_TRY(cudaEventRecord(static_cast<cudaEvent_t>(a->layer_done[l]), st));
        if (stop) break;

        // (5) y = RMSNorm_head(o) w_gnorm * SiLU(z) (hi/lo), into the MLP activation buffer
        // (free here; the out_proj epilogue writes the next operand into A)
        GatedNormBatch gn{};
        for (int g = 0; g < G; ++g) {
            gn.o[g] = B[g].o;
            gn.p[g] = B[g].p;
            gn.w[g] = static_cast<const __nv_bfloat16 *>(W(g).w_gnorm);
            gn.y_hi[g] = B[g].h_hi;
            gn.y_lo[g] = B[g].h_lo;
        }
        gn.T = T; gn.h_v = m.hv; gn.ld = m.proj; gn.z_off = m.conv_dim; gn.eps = a->eps; gn.lo8 = m.lo8;
        gn.status = status;
        SR_TRY(prof.begin(SR_K_GATED_NORM));
        SR_TRY(gated_norm(gn, G, st));
        SR_TRY(prof.end());

        // (6) x += y W_out^T; the epilogue also forms A = x * w_post_norm (hi/lo) and the
        // partial sums of x^2 of the post-attention RMSNorm
        for (int g = 0; g < G; ++g) {
            gp[g] = GemmProblemDesc{B[g].h_hi, B[g].h_lo, W(g).w_out, nullptr, B[g].x32, nullptr, nullptr, nullptr,
                                    W(g).w_out_lo8, nullptr};
            gp[g].nw = W(g).w_post_norm;
            gp[g].n_hi = B[g].a_hi;
            gp[g].n_lo = B[g].a_lo;
            gp[g].ssq_out = B[g].ssq;
        }
        SR_TRY(prof.begin(SR_K_GEMM_OUT));
        SR_TRY(gemm_tc(gp, G, T, m.H, m.vd, m.H, EPI_F32_RESIDUAL, npass, m.lo8, status, st, pair_opt));
        SR_TRY(prof.end());

        // (7) h = SiLU(r A W_gate^T) * (r A W_up^T) (hi/lo), r from the partial sums
        for (int g = 0; g < G; ++g) {
            gp[g] = GemmProblemDesc{B[g].a_hi, B[g].a_lo, W(g).w_gate, W(g).w_up, B[g].h_hi, nullptr, B[g].h_lo,
                                    nullptr, W(g).w_gate_lo8, W(g).w_up_lo8};
            gp[g].ssq_in = B[g].ssq;
        }
        SR_TRY(prof.begin(SR_K_GEMM_GATEUP));
        SR_TRY(gemm_tc(gp, G, T, m.I, m.H, m.I, EPI_SWIGLU, npass, m.lo8, status, st, rn));
        SR_TRY(prof.end());

        // (8) x += h W_down^T; unless this is the last layer, the epilogue also forms the
        // next layer's A = x * w_in_norm (hi/lo) and partial sums of x^2
        const bool next = l + 1 < m.L;
        for (int g = 0; g < G; ++g) {
            gp[g] = GemmProblemDesc{B[g].h_hi, B[g].h_lo, W(g).w_down, nullptr, B[g].x32, nullptr, nullptr, nullptr,
                                    W(g).w_down_lo8, nullptr};
            if (next) {
                gp[g].nw = a->weights[g * m.L + l + 1].w_in_norm;
                gp[g].n_hi = B[g].a_hi;
                gp[g].n_lo = B[g].a_lo;
                gp[g].ssq_out = B[g].ssq;
            }
        }
        SR_TRY(prof.begin(SR_K_GEMM_DOWN));
        SR_TRY(gemm_tc(gp, G, T, m.H, m.I, m.H, EPI_F32_RESIDUAL, npass, m.lo8, status, st, pair_opt));
        SR_TRY(prof.end());

        // (9) optional bf16 copy of the hidden after this layer
        CastBatch cast{};
        int n_cast = 0;
        for (int g = 0; g < G; ++g)
            if (O(g).hidden_out) ++n_cast;
        if (n_cast == G) {
            for (int g = 0; g < G; ++g) {
                cast.src[g] = B[g].x32;
                cast.dst[g] = static_cast<__nv_bfloat16 *>(O(g).hidden_out);
            }
            cast.n = size_t(T) * m.H;
            SR_TRY(prof.begin(SR_K_CAST));
            SR_TRY(to_bf16(cast, G, st));
            SR_TRY(prof.end());
        } else if (n_cast > 0) {
            for (int g = 0; g < G; ++g) {
                if (!O(g).hidden_out) continue;
                cast.src[0] = B[g].x32;
                cast.dst[0] = static_cast<__nv_bfloat16 *>(O(g).hidden_out);
                cast.n = size_t(T) * m.H;
                SR_TRY(prof.begin(SR_K_CAST));
                SR_TRY(to_bf16(cast, 1, st));
                SR_TRY(prof.end());
            }
        }
    }
    return SR_OK;
}
