/*
 * Oracle: plain fp64 token-by-token recurrences for suffix-replay state
 * reconstruction.  TEST INFRASTRUCTURE ONLY -- the product path never links,
 * loads or calls this file; only the tests, the smoke check and the CPU
 * baseline leg of the benchmark do.
 *
 * Both recurrences are instances of the linear state update
 *     S_t = A_t(S_{t-1}) + B_t,   S_0 = 0 (or a given h0)
 * ("SuffixReplay: Prefix Caching via Suffix Replay for Hybrid LLMs",
 *  Theoretical Foundation, Eq. 4), run over each sequence of a packed
 * varlen batch independently (Pipelined Replay Path, "Batched replay":
 * several hits packed into one variable-length execution).
 *
 * Gated DeltaNet ("Tail-Replay: Escaping the Curse of Linear Attention in
 * Prefix Caching for Hybrid LLMs", Sec. 2: decay gate alpha in (0,1] plus a
 * rank-1 correction):
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = scale * S_t q_t
 * S is d_v x d_k (row = value channel, column = key channel).  Expanding the
 * product gives S_t = alpha_t S_{t-1} + u_t k_t^T with
 * u_t = beta_t (v_t - alpha_t S_{t-1} k_t); the loop below applies exactly
 * those three steps in that order.  V head h reads QK head h / (H_v / H_k).
 *
 * Mamba2 (SuffixReplay, Eq. 4: "per-head decay in Mamba2", no erase term):
 *     S_t = exp(dt_t A_h) S_{t-1} + dt_t x_t B_t^T,   y_t = S_t C_t
 * S is P x N_s; head h reads B/C group h / (H / G).
 *
 * Everything is fp64; inputs arrive as fp64 copies of the (bf16 or fp32)
 * data.  The loop over (sequence, head) units is parallel; each unit is a
 * plain serial loop over its tokens.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* units: optional list of (seq * H + head) indices to compute; NULL = all.
 * o / y may be NULL.  Returns 0 on success, -1 on bad arguments. */
int oracle_gdn(const double *q, const double *k, const double *v,
               const double *g, const double *beta, const long long *cu,
               int n_seqs, int h_k, int h_v, int d_k, int d_v, double scale,
               const double *h0, double *o, double *s_out, const int *units,
               int n_units, int n_threads)
{
    if (h_k <= 0 || h_v <= 0 || h_v % h_k != 0 || d_k <= 0 || d_v <= 0)
        return -1;
    const int group = h_v / h_k;
    const int total = units ? n_units : n_seqs * h_v;
#ifdef _OPENMP
    if (n_threads > 0)
        omp_set_num_threads(n_threads);
#endif
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int idx = 0; idx < total; ++idx) {
        const int unit = units ? units[idx] : idx;
        const int n = unit / h_v, h = unit % h_v, hk = h / group;
        if (n < 0 || n >= n_seqs) {
            bad |= 1;
            continue;
        }
        double *S = (double *)calloc((size_t)d_v * d_k, sizeof(double));
        double *u = (double *)malloc(sizeof(double) * d_v);
        if (h0)
            memcpy(S, h0 + ((size_t)n * h_v + h) * d_v * d_k,
                   sizeof(double) * d_v * d_k);
        for (long long t = cu[n]; t < cu[n + 1]; ++t) {
            const double alpha = exp(g[t * h_v + h]);
            const double b = beta[t * h_v + h];
            const double *kt = k + ((size_t)t * h_k + hk) * d_k;
            const double *qt = q + ((size_t)t * h_k + hk) * d_k;
            const double *vt = v + ((size_t)t * h_v + h) * d_v;
            /* decay */
            for (size_t e = 0; e < (size_t)d_v * d_k; ++e)
                S[e] *= alpha;
            /* u = beta (v - (alpha S_{t-1}) k) */
            for (int i = 0; i < d_v; ++i) {
                double sk = 0.0;
                for (int j = 0; j < d_k; ++j)
                    sk += S[(size_t)i * d_k + j] * kt[j];
                u[i] = b * (vt[i] - sk);
            }
            /* rank-1 write */
            for (int i = 0; i < d_v; ++i)
                for (int j = 0; j < d_k; ++j)
                    S[(size_t)i * d_k + j] += u[i] * kt[j];
            if (o) {
                double *ot = o + ((size_t)t * h_v + h) * d_v;
                for (int i = 0; i < d_v; ++i) {
                    double sq = 0.0;
                    for (int j = 0; j < d_k; ++j)
                        sq += S[(size_t)i * d_k + j] * qt[j];
                    ot[i] = scale * sq;
                }
            }
        }
        memcpy(s_out + ((size_t)n * h_v + h) * d_v * d_k, S,
               sizeof(double) * d_v * d_k);
        free(S);
        free(u);
    }
    return bad ? -1 : 0;
}

int oracle_mamba2(const double *x, const double *B, const double *C,
                  const double *dt, const double *A, const long long *cu,
                  int n_seqs, int H, int P, int G, int Ns, const double *h0,
                  double *y, double *s_out, const int *units, int n_units,
                  int n_threads)
{
    if (H <= 0 || G <= 0 || H % G != 0 || P <= 0 || Ns <= 0)
        return -1;
    const int heads_per_group = H / G;
    const int total = units ? n_units : n_seqs * H;
#ifdef _OPENMP
    if (n_threads > 0)
        omp_set_num_threads(n_threads);
#endif
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int idx = 0; idx < total; ++idx) {
        const int unit = units ? units[idx] : idx;
        const int n = unit / H, h = unit % H, gi = h / heads_per_group;
        if (n < 0 || n >= n_seqs) {
            bad |= 1;
            continue;
        }
        double *S = (double *)calloc((size_t)P * Ns, sizeof(double));
        if (h0)
            memcpy(S, h0 + ((size_t)n * H + h) * P * Ns, sizeof(double) * P * Ns);
        for (long long t = cu[n]; t < cu[n + 1]; ++t) {
            const double d = dt[t * H + h];
            const double a = exp(d * A[h]);
            const double *xt = x + ((size_t)t * H + h) * P;
            const double *Bt = B + ((size_t)t * G + gi) * Ns;
            const double *Ct = C + ((size_t)t * G + gi) * Ns;
            for (int p = 0; p < P; ++p)
                for (int s = 0; s < Ns; ++s)
                    S[(size_t)p * Ns + s] = a * S[(size_t)p * Ns + s] + d * xt[p] * Bt[s];
            if (y) {
                double *yt = y + ((size_t)t * H + h) * P;
                for (int p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int s = 0; s < Ns; ++s)
                        acc += S[(size_t)p * Ns + s] * Ct[s];
                    yt[p] = acc;
                }
            }
        }
        memcpy(s_out + ((size_t)n * H + h) * P * Ns, S, sizeof(double) * P * Ns);
        free(S);
    }
    return bad ? -1 : 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
