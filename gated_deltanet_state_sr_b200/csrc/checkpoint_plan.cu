// Host: distribution-aware checkpoint placement ("Sparse Prefix Caching for
// Hybrid and Recurrent LLM Serving", Methodology, Algorithmic Approach 2).
//
// A retained prefix of N tokens may keep recurrent-state checkpoints at up to
// M positions C = {c_1 < ... < c_m} in 1..N.  A later request that overlaps
// the prefix to depth t resumes from the deepest checkpoint at or below t,
// l(t; C) = max({0} u {c in C : c <= t}), and recomputes r(t; C) = t - l(t; C)
// tokens.  Given the probabilities p_t of the overlap depths t = 0..N, the
// placement minimises E[r(T; C)] = sum_t p_t r(t; C).
//
// With prefix sums P_j = sum_{t<=j} p_t and A_j = sum_{t<=j} t p_t, the cost of
// serving depths s..j from a checkpoint at s is
//     w(s, j) = (A_j - A_{s-1}) - s (P_j - P_{s-1})
// and dp[m][j] (depths 0..j, at most m checkpoints in 1..j) satisfies
//     dp[0][j] = A_j,
//     dp[m][j] = min(dp[m-1][j], min_{1<=s<=j} dp[m-1][s-1] + w(s, j)).
// For fixed m, each s contributes the line y = -s x + (dp[m-1][s-1] - A_{s-1}
// + s P_{s-1}) evaluated at x = P_j; slopes fall as s grows and the query
// points P_j never decrease, so a monotone lower envelope (the convex hull
// trick) answers every j in amortised O(1): O(N M) in all.
#include <stdint.h>
#include <stdlib.h>

#include <vector>

#include "common.cuh"

namespace {

struct Line {
    double k, b;  // y = k x + b
    int64_t s;    // the checkpoint position the line stands for
};

// true when line b is never strictly below both a and c (slopes k_a > k_b > k_c)
bool useless(const Line &a, const Line &b, const Line &c) {
    // intersection x(a, c) <= x(a, b)  <=>  (c.b - a.b) (a.k - b.k) <= (b.b - a.b) (a.k - c.k)
    return (c.b - a.b) * (a.k - b.k) <= (b.b - a.b) * (a.k - c.k);
}

}  // namespace

extern "C" sr_status sr_checkpoint_plan(const double *p, int64_t n, int32_t m_max, int64_t *positions,
                                        int32_t *count, double *expected_cost) {
    if (!p || !count || n < 0 || m_max < 0) return sr::set_error(SR_ERR_INVALID_ARG, "bad arguments");
    if (m_max > 0 && !positions) return sr::set_error(SR_ERR_INVALID_ARG, "positions is required when m_max > 0");
    if (n > (int64_t(1) << 26) || int64_t(m_max) * (n + 1) > (int64_t(1) << 31))
        return sr::set_error(SR_ERR_UNSUPPORTED, "N (M + 1) too large for the planner's tables");
    for (int64_t t = 0; t <= n; ++t)
        if (!(p[t] >= 0.0)) return sr::set_error(SR_ERR_INVALID_ARG, "p[%lld] must be >= 0", (long long)t);
    const int32_t M = int32_t(m_max < n ? m_max : n);
    std::vector<double> P(n + 1), A(n + 1);
    double ps = 0.0, as = 0.0;
    for (int64_t t = 0; t <= n; ++t) {
        ps += p[t];
        as += double(t) * p[t];
        P[t] = ps;
        A[t] = as;
    }
    // dp rows m = 0..M over j = 0..n; arg[m][j] = deepest checkpoint of the optimum (-1: none added at m)
    std::vector<double> prev(A), cur(n + 1);
    std::vector<int64_t> arg(size_t(M + 1) * size_t(n + 1), 0);
    std::vector<Line> hull;
    hull.reserve(size_t(n) + 1);
    for (int32_t m = 1; m <= M; ++m) {
        hull.clear();
        size_t head = 0;
        cur[0] = prev[0];
        arg[size_t(m) * (n + 1)] = -1;  // depth 0 never needs a checkpoint
        for (int64_t j = 1; j <= n; ++j) {
            // add the line of s = j (needs dp[m-1][j-1])
            // lines before `head` are behind every later query; the envelope is hull[head..]
            const Line ln{-double(j), prev[j - 1] - A[j - 1] + double(j) * P[j - 1], j};
            while (hull.size() - head >= 2 && useless(hull[hull.size() - 2], hull.back(), ln)) hull.pop_back();
            hull.push_back(ln);
            const double x = P[j];
            while (hull.size() - head >= 2 && hull[head + 1].k * x + hull[head + 1].b <= hull[head].k * x + hull[head].b)
                ++head;
            const double with = A[j] + hull[head].k * x + hull[head].b;
            if (with < prev[j]) {
                cur[j] = with;
                arg[size_t(m) * (n + 1) + j] = hull[head].s;
            } else {
                cur[j] = prev[j];
                arg[size_t(m) * (n + 1) + j] = -1;  // the optimum uses fewer checkpoints
            }
        }
        prev.swap(cur);
    }
    // walk back from (M, n)
    std::vector<int64_t> picked;
    int64_t j = n;
    for (int32_t m = M; m >= 1 && j >= 1; --m) {
        const int64_t s = arg[size_t(m) * (n + 1) + j];
        if (s <= 0) continue;  // row m adds nothing at depth j: look one row up
        picked.push_back(s);
        j = s - 1;
    }
    *count = int32_t(picked.size());
    for (size_t i = 0; i < picked.size(); ++i) positions[i] = picked[picked.size() - 1 - i];
    if (expected_cost) {
        // evaluate the returned placement directly
        double cost = 0.0;
        size_t k = 0;
        int64_t last = 0;
        for (int64_t t = 0; t <= n; ++t) {
            while (k < picked.size() && positions[k] <= t) last = positions[k++];
            cost += p[t] * double(t - last);
        }
        *expected_cost = cost;
    }
    return SR_OK;
}
