"""Pins for the fp64 Gated DeltaNet oracle (CPU only).

Each test ties ``oracle.gdn_replay`` to something other than itself: a closed
form, an invariant the pages state, or an explicitly unrolled product.  The
recurrence is "SuffixReplay: Prefix Caching via Suffix Replay for Hybrid
LLMs", Eq. 4, with the Gated DeltaNet transition named in "Tail-Replay", Sec. 2
(decay alpha in (0,1] plus a rank-1 erase):
    S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T.
"""
import math

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(1234)


def _rand_inputs(rng, T, hk, hv, dk, dv, unit_k=False, g_lo=-0.5, g_hi=-0.01):
    q = rng.standard_normal((T, hk, dk))
    k = rng.standard_normal((T, hk, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, hv, dv))
    g = rng.uniform(g_lo, g_hi, (T, hv))
    beta = rng.uniform(0, 1, (T, hv))
    return q, k, v, g, beta


# ------------------------------------------------------------ closed forms


def test_beta_zero_is_pure_decay():
    """beta = 0: S_T = (prod alpha) h0 and o_t = scale (prod_{s<=t} alpha_s) h0 q_t."""
    rng = np.random.default_rng(1)
    T, hk, hv, d = 37, 1, 2, 8
    q, k, v, g, _ = _rand_inputs(rng, T, hk, hv, d, d)
    beta = np.zeros((T, hv))
    h0 = rng.standard_normal((1, hv, d, d))
    scale = 0.3
    o, S = oracle.gdn_replay(q, k, v, g, beta, [0, T], scale=scale, h0=h0)
    for h in range(hv):
        cum = np.cumsum(g[:, h])
        np.testing.assert_allclose(S[0, h], np.exp(cum[-1]) * h0[0, h], rtol=1e-13, atol=0)
        for t in range(T):
            ref = scale * np.exp(cum[t]) * h0[0, h] @ q[t, 0]
            np.testing.assert_allclose(o[t, h], ref, rtol=1e-12, atol=1e-14)
    # and from a zero state nothing is ever written
    o0, S0 = oracle.gdn_replay(q, k, v, g, beta, [0, T], scale=scale)
    assert np.all(S0 == 0) and np.all(o0 == 0)


def test_unit_gates_orthonormal_keys_sum_outer_products():
    """alpha = 1, beta = 1, orthonormal keys: S_T = sum_t v_t k_t^T exactly and
    o_t = scale sum_{s<=t} v_s (k_s . q_t)."""
    rng = np.random.default_rng(2)
    d = 16
    T = 12
    # orthonormal keys: Gram-Schmidt on random vectors (fp64)
    basis = []
    for _ in range(T):
        x = rng.standard_normal(d)
        for b in basis:
            x -= (b @ x) * b
        basis.append(x / np.linalg.norm(x))
    k = np.stack(basis)[:, None, :]
    q = rng.standard_normal((T, 1, d))
    v = rng.standard_normal((T, 1, d))
    g = np.zeros((T, 1))
    beta = np.ones((T, 1))
    o, S = oracle.gdn_replay(q, k, v, g, beta, [0, T], scale=1.0)
    ref = sum(np.outer(v[t, 0], k[t, 0]) for t in range(T))
    np.testing.assert_allclose(S[0, 0], ref, atol=1e-12)
    for t in range(T):
        ref_o = sum(v[s, 0] * (k[s, 0] @ q[t, 0]) for s in range(t + 1))
        np.testing.assert_allclose(o[t, 0], ref_o, atol=1e-12)


def test_single_token_from_zero():
    """One token from S_0 = 0: S_1 = beta v k^T, o_1 = scale beta v (k . q)."""
    rng = np.random.default_rng(3)
    q, k, v, g, beta = _rand_inputs(rng, 1, 1, 1, 5, 3)
    o, S = oracle.gdn_replay(q, k, v, g, beta, [0, 1], scale=0.7)
    np.testing.assert_allclose(S[0, 0], beta[0, 0] * np.outer(v[0, 0], k[0, 0]), rtol=1e-14)
    np.testing.assert_allclose(o[0, 0], 0.7 * beta[0, 0] * v[0, 0] * (k[0, 0] @ q[0, 0]),
                               rtol=1e-13)


# ------------------------------------------------------------ brute force


def brute_force_states(q, k, v, g, beta, h0=None):
    """Explicit unrolled transition product for one head:
    S_t = S_0 M_1..M_t + sum_{s<=t} beta_s v_s k_s^T M_{s+1}..M_t,
    M_s = alpha_s (I - beta_s k_s k_s^T).  Returns all S_t."""
    T, dk = k.shape
    dv = v.shape[1]
    M = [math.exp(g[s]) * (np.eye(dk) - beta[s] * np.outer(k[s], k[s])) for s in range(T)]
    out = []
    S0 = np.zeros((dv, dk)) if h0 is None else h0
    for t in range(T):
        acc = S0.copy()
        for s in range(t + 1):
            acc = acc @ M[s]
        for s in range(t + 1):
            term = beta[s] * np.outer(v[s], k[s])
            for r in range(s + 1, t + 1):
                term = term @ M[r]
            acc = acc + term
        out.append(acc)
    return out


@pytest.mark.parametrize("T,dk,dv", [(1, 2, 3), (5, 4, 4), (8, 3, 2)])
def test_brute_force_unrolled_product(T, dk, dv):
    rng = np.random.default_rng(10 + T)
    q, k, v, g, beta = _rand_inputs(rng, T, 1, 1, dk, dv, g_lo=-1.0, g_hi=0.0)
    h0 = rng.standard_normal((1, 1, dv, dk))
    for init in (None, h0):
        o, S = oracle.gdn_replay(q, k, v, g, beta, [0, T], scale=0.5, h0=init)
        ref = brute_force_states(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0],
                                 None if init is None else init[0, 0])
        np.testing.assert_allclose(S[0, 0], ref[-1], atol=1e-12, rtol=1e-12)
        for t in range(T):
            np.testing.assert_allclose(o[t, 0], 0.5 * ref[t] @ q[t, 0], atol=1e-12, rtol=1e-12)


def test_gqa_head_mapping():
    """V head h reads QK head h // (H_v / H_k) (consecutive grouping)."""
    rng = np.random.default_rng(4)
    T, hk, hv, d = 9, 2, 6, 4
    q, k, v, g, beta = _rand_inputs(rng, T, hk, hv, d, d)
    o, S = oracle.gdn_replay(q, k, v, g, beta, [0, T], scale=1.0)
    for h in range(hv):
        hq = h // (hv // hk)
        ref = brute_force_states(q[:, hq], k[:, hq], v[:, h], g[:, h], beta[:, h])
        np.testing.assert_allclose(S[0, h], ref[-1], atol=1e-12)


# ------------------------------------------------------------ invariants


def test_exact_resume_and_superposition():
    """Resuming from an exact state and replaying the suffix reproduces the
    full-prefix state ("Sparse Prefix Caching for Hybrid and Recurrent LLM
    Serving", Implementation Strategy: exactness of resume).  Equivalently
    Replay(a || b) = Replay(b, h0 = Replay(a))."""
    rng = np.random.default_rng(5)
    T, j = 300, 211
    q, k, v, g, beta = _rand_inputs(rng, T, 2, 4, 16, 8, unit_k=True)
    o_full, S_full = oracle.gdn_replay(q, k, v, g, beta, [0, T])
    _, S_a = oracle.gdn_replay(q[:j], k[:j], v[:j], g[:j], beta[:j], [0, j])
    o_b, S_b = oracle.gdn_replay(q[j:], k[j:], v[j:], g[j:], beta[j:], [0, T - j], h0=S_a)
    np.testing.assert_allclose(S_b, S_full, atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(o_b, o_full[j:], atol=1e-12, rtol=1e-12)


def test_varlen_packing_is_independent():
    """Sequences packed in one cu_seqlens batch replay independently."""
    rng = np.random.default_rng(6)
    lens = [7, 1, 0, 20]
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v, g, beta = _rand_inputs(rng, T, 1, 2, 4, 4)
    o, S = oracle.gdn_replay(q, k, v, g, beta, cu)
    for n in range(len(lens)):
        s, e = cu[n], cu[n + 1]
        o1, S1 = oracle.gdn_replay(q[s:e], k[s:e], v[s:e], g[s:e], beta[s:e], [0, e - s])
        np.testing.assert_array_equal(S[n], S1[0])
        np.testing.assert_array_equal(o[s:e], o1)
    assert np.all(S[2] == 0)  # an empty sequence leaves the zero state


@pytest.mark.parametrize("k_rep", [16, 64, 256, 1024])
def test_contraction_bound_of_suffix_replay(k_rep):
    """Suffix approximation (SuffixReplay, Eq. 2): with ||k_t|| = 1 and
    beta in [0, 1] every transition has spectral norm alpha_t, so
    ||S_j - S'_j||_F <= (prod of alpha over the k replayed tokens) ||S_{j-k}||_F,
    and the gap is exactly S_{j-k} propagated through those k transitions."""
    rng = np.random.default_rng(7)
    j, hk, hv, d = 4096, 1, 2, 32
    q, k, v, g, beta = _rand_inputs(rng, j, hk, hv, d, d, unit_k=True, g_lo=-0.1, g_hi=-0.001)
    _, S_j = oracle.gdn_replay(q, k, v, g, beta, [0, j], want_o=False)
    s = j - k_rep
    _, S_jk = oracle.gdn_replay(q[:s], k[:s], v[:s], g[:s], beta[:s], [0, s], want_o=False)
    _, S_rep = oracle.gdn_replay(q[s:], k[s:], v[s:], g[s:], beta[s:], [0, k_rep], want_o=False)
    for h in range(hv):
        gap = np.linalg.norm(S_j[0, h] - S_rep[0, h])
        bound = math.exp(g[s:, h].sum()) * np.linalg.norm(S_jk[0, h])
        assert gap <= bound * (1 + 1e-9) + 1e-12, (h, gap, bound)
        # the bound is attained by the propagated prefix state: replay the
        # suffix with v = 0 starting from S_{j-k}
        _, prop = oracle.gdn_replay(q[s:], k[s:], np.zeros_like(v[s:]), g[s:], beta[s:],
                                    [0, k_rep], h0=S_jk, want_o=False)
        np.testing.assert_allclose(S_j[0, h] - S_rep[0, h], prop[0, h], atol=1e-10)


# ------------------------------------------------------------ planted mistakes


def _numpy_recurrence(q, k, v, g, beta, mutation=None):
    """Independent single-head numpy restatement, with optional planted bugs;
    used only to show that the pins above reject plausible mistakes."""
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk))
    for t in range(T):
        a = math.exp(g[t])
        if mutation == "erase_sign":
            S = a * S @ (np.eye(dk) + beta[t] * np.outer(k[t], k[t])) + beta[t] * np.outer(v[t], k[t])
        elif mutation == "decay_after_erase_term":
            u = beta[t] * (v[t] - S @ k[t])  # forgets alpha inside u
            S = a * S + np.outer(u, k[t])
        elif mutation == "transposed_state":
            u = beta[t] * (v[t] - (a * S).T @ k[t])  # needs dv == dk
            S = a * S + np.outer(u, k[t])
        else:
            u = beta[t] * (v[t] - (a * S) @ k[t])
            S = a * S + np.outer(u, k[t])
    return S


@pytest.mark.parametrize("mutation", ["erase_sign", "decay_after_erase_term", "transposed_state"])
def test_pins_reject_planted_mistakes(mutation):
    rng = np.random.default_rng(8)
    T, d = 8, 4
    q, k, v, g, beta = _rand_inputs(rng, T, 1, 1, d, d, g_lo=-1.0, g_hi=-0.1)
    ref = brute_force_states(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0])[-1]
    good = _numpy_recurrence(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0])
    np.testing.assert_allclose(good, ref, atol=1e-12)
    bad = _numpy_recurrence(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], mutation)
    assert np.max(np.abs(bad - ref)) > 1e-6
