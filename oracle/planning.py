"""fp64 oracle for checkpoint placement.

TEST INFRASTRUCTURE ONLY (see the package docstring).

"Sparse Prefix Caching for Hybrid and Recurrent LLM Serving", Methodology,
Theoretical Formulation: checkpoints C in 1..N; a request overlapping the
prefix to depth t resumes from l(t; C) = max({0} u {c in C : c <= t}) and
recomputes r(t; C) = t - l(t; C) tokens; the objective is sum_t p_t r(t; C).
Algorithmic Approach 2 gives the recurrence
    dp[m, j] = min_{1<=s<=j} (dp[m-1, s-1] + w(s, j)),
w(s, j) = cost of serving depths s..j from a checkpoint at s.

Here: the objective written out (``expected_recompute``), exhaustive search
over every placement for tiny N (``optimal_by_enumeration``), and the
recurrence taken literally in O(N^2 M) with w summed directly
(``optimal_by_recurrence``).  Pinned by the balanced-spacing optimum of the
uniform distribution and by point masses (tests/test_checkpoint_plan.py).
"""
from __future__ import annotations

import itertools

import numpy as np


def expected_recompute(p, positions) -> float:
    """sum_t p_t (t - l(t; C)) over depths t = 0..N."""
    p = np.asarray(p, dtype=np.float64)
    C = sorted(int(c) for c in positions)
    total = 0.0
    for t in range(len(p)):
        deepest = max([0] + [c for c in C if c <= t])
        total += p[t] * (t - deepest)
    return total


def optimal_by_enumeration(p, m):
    """(cost, positions) minimising the objective over every set of at most m
    positions in 1..N (tiny N only)."""
    N = len(p) - 1
    best = (expected_recompute(p, []), ())
    for k in range(1, min(m, N) + 1):
        for C in itertools.combinations(range(1, N + 1), k):
            c = expected_recompute(p, C)
            if c < best[0]:
                best = (c, C)
    return best


def optimal_by_recurrence(p, m) -> float:
    """The page's recurrence, literally: dp[0, j] = cost of depths 0..j with no
    checkpoint; dp[k, j] = min(dp[k-1, j], min_s dp[k-1, s-1] + w(s, j)) with
    w(s, j) = sum_{t=s}^{j} p_t (t - s).  Returns dp[m, N]."""
    p = np.asarray(p, dtype=np.float64)
    N = len(p) - 1
    t = np.arange(N + 1, dtype=np.float64)
    dp = np.cumsum(p * t)  # no checkpoint: every depth recomputes from 0
    for _ in range(min(m, N)):
        new = dp.copy()
        for j in range(1, N + 1):
            s = np.arange(1, j + 1)
            # w(s, j) for every s at once, summed directly from its definition
            w = np.array([np.sum(p[si:j + 1] * (t[si:j + 1] - si)) for si in s])
            new[j] = min(dp[j], np.min(dp[s - 1] + w))
        dp = new
    return float(dp[N])
