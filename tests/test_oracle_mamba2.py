"""Pins for the fp64 Mamba2 oracle (CPU only).

The Mamba2 instance of "SuffixReplay: Prefix Caching via Suffix Replay for
Hybrid LLMs", Eq. 4 (per-head decay, no erase):
    S_t = exp(dt_t A_h) S_{t-1} + dt_t x_t B_t^T,   y_t = S_t C_t.
"""
import numpy as np
import pytest

import oracle


def _inputs(rng, T, H=3, P=4, G=1, Ns=5):
    x = rng.standard_normal((T, H, P))
    B = rng.standard_normal((T, G, Ns))
    C = rng.standard_normal((T, G, Ns))
    dt = np.log1p(np.exp(rng.standard_normal((T, H))))
    A = -np.exp(rng.uniform(0, 2, H))
    return x, B, C, dt, A


@pytest.mark.parametrize("G", [1, 3])
def test_closed_sum_of_decay_weighted_outer_products(G):
    """S_T = (prod_t a_t) S_0 + sum_t (prod_{s>t} a_s) dt_t x_t B_t^T, and
    y_t = sum_{s<=t} (prod_{s<r<=t} a_r) dt_s x_s (B_s . C_t) + (prod_{r<=t} a_r) S_0 C_t."""
    rng = np.random.default_rng(11)
    T, H, P, Ns = 23, 3, 4, 5
    x, B, C, dt, A = _inputs(rng, T, H, P, G, Ns)
    h0 = rng.standard_normal((1, H, P, Ns))
    y, S = oracle.mamba2_replay(x, B, C, dt, A, [0, T], h0=h0)
    for h in range(H):
        gi = h // (H // G)
        la = dt[:, h] * A[h]                      # log a_t
        cum = np.concatenate([[0.0], np.cumsum(la)])  # cum[t] = sum_{r<t} log a_r
        ref = np.exp(cum[T]) * h0[0, h]
        for t in range(T):
            ref = ref + np.exp(cum[T] - cum[t + 1]) * dt[t, h] * np.outer(x[t, h], B[t, gi])
        np.testing.assert_allclose(S[0, h], ref, rtol=1e-11, atol=1e-12)
        for t in range(T):
            ref_y = np.exp(cum[t + 1]) * h0[0, h] @ C[t, gi]
            for s in range(t + 1):
                ref_y = ref_y + np.exp(cum[t + 1] - cum[s + 1]) * dt[s, h] * x[s, h] * (B[s, gi] @ C[t, gi])
            np.testing.assert_allclose(y[t, h], ref_y, rtol=1e-10, atol=1e-11)


def test_zero_dt_keeps_state():
    """dt = 0: no decay and no write, so S stays h0 and y_t = h0 C_t."""
    rng = np.random.default_rng(12)
    T = 9
    x, B, C, dt, A = _inputs(rng, T)
    dt[:] = 0.0
    h0 = rng.standard_normal((1, 3, 4, 5))
    y, S = oracle.mamba2_replay(x, B, C, dt, A, [0, T], h0=h0)
    np.testing.assert_array_equal(S, h0)
    for t in range(T):
        for h in range(3):
            np.testing.assert_allclose(y[t, h], h0[0, h] @ C[t, 0], rtol=1e-13)


def test_exact_resume_and_packing():
    rng = np.random.default_rng(13)
    lens = [11, 0, 1, 30]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = cu[-1]
    x, B, C, dt, A = _inputs(rng, T)
    y, S = oracle.mamba2_replay(x, B, C, dt, A, cu)
    for n in range(len(lens)):
        s, e = cu[n], cu[n + 1]
        y1, S1 = oracle.mamba2_replay(x[s:e], B[s:e], C[s:e], dt[s:e], A, [0, e - s])
        np.testing.assert_array_equal(S[n], S1[0])
        np.testing.assert_array_equal(y[s:e], y1)
    # resume: replay(a||b) == replay(b, h0 = replay(a))
    s, e = cu[3], cu[4]
    j = s + 13
    _, Sa = oracle.mamba2_replay(x[s:j], B[s:j], C[s:j], dt[s:j], A, [0, j - s])
    yb, Sb = oracle.mamba2_replay(x[j:e], B[j:e], C[j:e], dt[j:e], A, [0, e - j], h0=Sa)
    np.testing.assert_allclose(Sb[0], S[3], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(yb, y[j:e], rtol=1e-12, atol=1e-13)


def test_planted_mistake_is_caught():
    """A decay applied to the write as well (a plausible slip) breaks the closed sum."""
    rng = np.random.default_rng(14)
    T = 6
    x, B, C, dt, A = _inputs(rng, T, H=1)
    _, S = oracle.mamba2_replay(x, B, C, dt, A, [0, T])
    bad = np.zeros((4, 5))
    for t in range(T):
        a = np.exp(dt[t, 0] * A[0])
        bad = a * (bad + dt[t, 0] * np.outer(x[t, 0], B[t, 0]))
    assert np.max(np.abs(bad - S[0, 0])) > 1e-6
