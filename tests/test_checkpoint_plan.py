"""Checkpoint placement ("Sparse Prefix Caching for Hybrid and Recurrent LLM
Serving", Methodology): the oracle pinned by the uniform distribution's
balanced optimum and by point masses, then sr_checkpoint_plan (host C, convex
hull trick) against the oracle's exhaustive search and its literal O(N^2 M)
recurrence."""
import itertools

import numpy as np
import pytest

import gated_deltanet_state_sr_b200 as sr
from oracle import planning as PL


# ---------------------------------------------------------------- oracle pins

@pytest.mark.parametrize("N,m", [(9, 2), (11, 3), (7, 1), (12, 4)])
def test_uniform_overlap_optimum_is_balanced(N, m):
    """Uniform depths: the segments [0, c_1), [c_1, c_2), ..., [c_m, N] cost
    L(L-1)/2 each, so the optimum makes their lengths differ by at most one
    (the page's balanced-spacing result)."""
    cost, C = PL.optimal_by_enumeration(np.ones(N + 1), m)
    lengths = np.diff([0, *C, N + 1])
    assert lengths.max() - lengths.min() <= 1
    assert cost == pytest.approx(sum(L * (L - 1) / 2 for L in lengths))


def test_point_masses():
    """All requests at depth d: one checkpoint at d recomputes nothing; with
    no checkpoint every request recomputes d tokens."""
    p = np.zeros(13)
    p[8] = 1.0
    assert PL.optimal_by_enumeration(p, 1) == (0.0, (8,))
    assert PL.expected_recompute(p, []) == 8.0
    p[3] = 2.0  # two masses, one slot: at 3 the depth-8 requests recompute 5, at 8 the
    # depth-3 ones (twice as many) recompute 3 each
    assert PL.optimal_by_enumeration(p, 1) == (5.0, (3,))
    assert PL.optimal_by_enumeration(p, 2) == (0.0, (3, 8))


def test_recurrence_matches_enumeration_on_tiny_cases():
    rng = np.random.default_rng(7)
    for N in range(1, 10):
        for m in range(0, 4):
            p = rng.random(N + 1)
            assert PL.optimal_by_recurrence(p, m) == pytest.approx(PL.optimal_by_enumeration(p, m)[0], rel=1e-12)


# ---------------------------------------------------------------- sr_checkpoint_plan

@pytest.mark.parametrize("seed", range(6))
def test_plan_is_optimal_on_small_cases(seed):
    rng = np.random.default_rng(100 + seed)
    N = int(rng.integers(1, 13))
    p = rng.random(N + 1) ** 3  # skewed weights
    for m in range(0, 5):
        pos, cost = sr.checkpoint_plan(p, m)
        assert len(pos) <= m and pos == sorted(set(pos)) and all(1 <= c <= N for c in pos)
        assert cost == pytest.approx(PL.expected_recompute(p, pos), rel=1e-12, abs=1e-12)
        assert cost == pytest.approx(PL.optimal_by_enumeration(p, m)[0], rel=1e-10, abs=1e-12)


@pytest.mark.parametrize("dist", ["geometric", "bimodal", "uniform"])
def test_plan_matches_the_recurrence_at_scale(dist):
    N, m = 600, 6
    t = np.arange(N + 1)
    if dist == "geometric":
        p = 0.99 ** (N - t)
    elif dist == "bimodal":
        p = np.exp(-0.5 * ((t - 150) / 20.0) ** 2) + 0.5 * np.exp(-0.5 * ((t - 520) / 40.0) ** 2)
    else:
        p = np.ones(N + 1)
    pos, cost = sr.checkpoint_plan(p, m)
    assert cost == pytest.approx(PL.expected_recompute(p, pos), rel=1e-10)
    assert cost == pytest.approx(PL.optimal_by_recurrence(p, m), rel=1e-9)


def test_plan_arguments():
    with pytest.raises(sr.SrError):
        sr.checkpoint_plan([1.0, -1.0, 2.0], 1)
    assert sr.checkpoint_plan([1.0], 3) == ([], 0.0)       # N = 0: nothing to place
    pos, cost = sr.checkpoint_plan(np.zeros(50), 4)         # no weight anywhere: nothing worth placing
    assert pos == [] and cost == 0.0


def test_no_budget_and_full_budget():
    """M = 0 leaves every request at the empty state: the cost is the mean
    depth.  With M >= N every depth can hold a checkpoint: the cost is 0."""
    rng = np.random.default_rng(11)
    p = rng.random(40)
    mean_depth = float(np.dot(np.arange(40), p))
    assert PL.optimal_by_enumeration(p[:9], 0)[0] == pytest.approx(float(np.dot(np.arange(9), p[:9])))
    assert sr.checkpoint_plan(p, 0) == ([], pytest.approx(mean_depth))
    for m in (39, 60):
        pos, cost = sr.checkpoint_plan(p, m)
        assert cost == 0.0 and pos == list(range(1, 40))


def test_plan_on_uniform_depths_is_balanced():
    """The C planner reaches the balanced-spacing optimum on uniform depths."""
    for N, m in [(100, 3), (257, 7), (64, 63)]:
        pos, cost = sr.checkpoint_plan(np.ones(N + 1), m)
        lengths = np.diff([0, *pos, N + 1])
        assert len(pos) == m and lengths.max() - lengths.min() <= 1
        assert cost == pytest.approx(sum(L * (L - 1) / 2 for L in lengths))
