"""Pins for the fp64 layer oracle (CPU only).

The pages give no layer math beyond the recurrence; each primitive is pinned
here by a closed form, and the composition by a scalar per-token restatement
on tiny shapes and by the group invariants the pages state ("SuffixReplay",
Algorithm Design 1: groups replay independently, errors stay in their group;
"Tail-Replay", Sec. 3: the final FFN can be skipped).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import layers as L
import workloads as W


def test_rmsnorm_constant_vector():
    x = np.full((2, 7), -3.0)
    w = np.arange(1, 8, dtype=np.float64)
    out = L.rmsnorm(x, w, 1e-6)
    np.testing.assert_allclose(out, -3.0 / math.sqrt(9.0 + 1e-6) * np.tile(w, (2, 1)), rtol=1e-15)


def test_l2norm_unit_norm():
    x = np.random.default_rng(0).standard_normal((5, 3, 16)) * 10
    n = np.linalg.norm(L.l2norm(x, 1e-6), axis=-1)
    np.testing.assert_allclose(n, 1.0, rtol=1e-8)


def test_scalar_functions():
    assert L.softplus(np.array(0.0)) == pytest.approx(math.log(2.0), rel=1e-15)
    assert L.softplus(np.array(30.0)) == 30.0
    assert L.softplus(np.array(-30.0)) == pytest.approx(math.exp(-30.0), rel=1e-12)
    assert L.sigmoid(np.array(0.0)) == 0.5
    for x in (-5.0, -0.3, 0.0, 1.7, 9.0):
        assert L.silu(np.array(x)) == pytest.approx(x / (1 + math.exp(-x)), rel=1e-14, abs=1e-300)
        assert L.sigmoid(np.array(x)) == pytest.approx(1 / (1 + math.exp(-x)), rel=1e-14)


def test_causal_conv_delta_weights_shift_within_sequences():
    rng = np.random.default_rng(1)
    cu = [0, 5, 6, 10]
    pre = rng.standard_normal((10, 3))
    w = np.zeros((3, 4))
    w[:, 3] = 1.0  # tap on the current token -> identity
    np.testing.assert_array_equal(L.causal_conv(pre, w, cu), pre)
    w = np.zeros((3, 4))
    w[:, 1] = 1.0  # tap two tokens back -> shift by 2, zero at each start
    out = L.causal_conv(pre, w, cu)
    ref = np.zeros_like(pre)
    for s, e in zip(cu[:-1], cu[1:]):
        for t in range(s, e):
            if t - 2 >= s:
                ref[t] = pre[t - 2]
    np.testing.assert_array_equal(out, ref)


def test_conv_state_last_rows_zero_padded():
    pre = np.arange(12, dtype=np.float64).reshape(6, 2)
    st = L.conv_state(pre, [0, 2, 6], 4)
    np.testing.assert_array_equal(st[0], [[0, 0, 2], [0, 1, 3]])  # only 2 tokens
    np.testing.assert_array_equal(st[1], [[6, 8, 10], [7, 9, 11]])


def _tiny_shape():
    return W.LayerShape(hidden=16, inter=24, h_k=2, h_v=4, d_k=4, d_v=4, conv_w=4, eps=1e-6)


def test_gates_closed_form():
    """A_log = 0, a = 0, dt_bias = 0 -> g = -ln 2 (alpha = 1/2); b = 0 -> beta = 1/2."""
    g = -np.exp(0.0) * L.softplus(np.array(0.0) + 0.0)
    assert math.exp(g) == pytest.approx(0.5, rel=1e-15)
    assert L.sigmoid(np.array(0.0)) == 0.5


def _scalar_layer(x, lw, cu, s):
    """Per-token, per-channel scalar restatement of one GDN layer + MLP (tiny
    shapes only).  Written independently of oracle.layers to catch reshape,
    head-order and split mistakes in the vectorised version."""
    f = lambda t: t.double().numpy()
    T = x.shape[0]
    win, conv_w, wout = f(lw.w_in), f(lw.conv_w), f(lw.w_out)
    A_log, dtb = f(lw.a_log), f(lw.dt_bias)
    sig = lambda u: 1.0 / (1.0 + math.exp(-u))
    sp = lambda u: u if u > 20 else math.log1p(math.exp(u))
    p = np.zeros((T, s.proj_dim))
    for t in range(T):
        r = math.sqrt(sum(xi * xi for xi in x[t]) / s.hidden + s.eps)
        hvec = [x[t][i] / r * float(lw.w_in_norm[i]) for i in range(s.hidden)]
        for j in range(s.proj_dim):
            p[t, j] = sum(hvec[i] * win[j, i] for i in range(s.hidden))
    qk, vd, cd = s.h_k * s.d_k, s.h_v * s.d_v, s.conv_dim
    c = np.zeros((T, cd))
    for n in range(len(cu) - 1):
        for t in range(cu[n], cu[n + 1]):
            for ch in range(cd):
                acc = 0.0
                for i in range(s.conv_w):
                    tt = t - (s.conv_w - 1) + i
                    if tt >= cu[n]:
                        acc += conv_w[ch, i] * p[tt, ch]
                c[t, ch] = acc * sig(acc)
    q = np.zeros((T, s.h_k, s.d_k)); k = np.zeros_like(q); v = np.zeros((T, s.h_v, s.d_v))
    g = np.zeros((T, s.h_v)); beta = np.zeros((T, s.h_v))
    for t in range(T):
        for h in range(s.h_k):
            qs = [c[t, h * s.d_k + d] for d in range(s.d_k)]
            ks = [c[t, qk + h * s.d_k + d] for d in range(s.d_k)]
            nq = math.sqrt(sum(u * u for u in qs) + 1e-6)
            nk = math.sqrt(sum(u * u for u in ks) + 1e-6)
            q[t, h] = [u / nq for u in qs]
            k[t, h] = [u / nk for u in ks]
        for h in range(s.h_v):
            v[t, h] = [c[t, 2 * qk + h * s.d_v + d] for d in range(s.d_v)]
            b = p[t, cd + vd + h]
            a = p[t, cd + vd + s.h_v + h]
            beta[t, h] = sig(b)
            g[t, h] = -math.exp(A_log[h]) * sp(a + dtb[h])
    o, S = oracle.gdn_replay(q, k, v, g, beta, cu, scale=1 / math.sqrt(s.d_k))
    wg = f(lw.w_gnorm)
    x1 = np.array(x, dtype=np.float64).copy()
    for t in range(T):
        y = []
        for h in range(s.h_v):
            r = math.sqrt(sum(o[t, h, d] ** 2 for d in range(s.d_v)) / s.d_v + s.eps)
            for d in range(s.d_v):
                z = p[t, cd + h * s.d_v + d]
                y.append(o[t, h, d] / r * wg[d] * z * sig(z))
        for i in range(s.hidden):
            x1[t, i] += sum(y[j] * wout[i, j] for j in range(vd))
    wgate, wup, wdown, wpost = f(lw.w_gate), f(lw.w_up), f(lw.w_down), f(lw.w_post_norm)
    x2 = x1.copy()
    for t in range(T):
        r = math.sqrt(sum(u * u for u in x1[t]) / s.hidden + s.eps)
        hh = [x1[t, i] / r * wpost[i] for i in range(s.hidden)]
        mid = []
        for j in range(s.inter):
            a = sum(hh[i] * wgate[j, i] for i in range(s.hidden))
            b = sum(hh[i] * wup[j, i] for i in range(s.hidden))
            mid.append(a * sig(a) * b)
        for i in range(s.hidden):
            x2[t, i] += sum(mid[j] * wdown[i, j] for j in range(s.inter))
    return S, x2


def test_layer_matches_scalar_restatement():
    s = _tiny_shape()
    gi = W.group_inputs(99, [5, 2, 4], n_layers=1, shape=s)
    # make the norm weights non-trivial so their placement is exercised
    lw = gi.layers[0]
    lw.w_in_norm = W.normal(7, "wn", (s.hidden,), 0.3).add(1.0).to(torch.bfloat16)
    lw.w_gnorm = W.normal(7, "wg", (s.d_v,), 0.3).add(1.0).to(torch.bfloat16)
    lw.w_post_norm = W.normal(7, "wp", (s.hidden,), 0.3).add(1.0).to(torch.bfloat16)
    lw.dt_bias = W.normal(7, "dtb", (s.h_v,), 1.0, dtype=torch.float32)
    # larger weights so gates and conv are far from their small-input regime
    lw.w_in = W.normal(7, "win", (s.proj_dim, s.hidden), 0.5)
    lw.conv_w = W.normal(7, "cw", (s.conv_dim, s.conv_w), 0.5)
    cu = np.asarray(gi.cu_seqlens.tolist())
    r = L.gdn_layer(oracle._f64(gi.anchors), lw, cu, s)
    S_ref, x_ref = _scalar_layer(gi.anchors.double().numpy(), lw, cu.tolist(), s)
    np.testing.assert_allclose(r["S"], S_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r["x_out"], x_ref, rtol=1e-10, atol=1e-10)


def test_residual_path_with_zero_output_weights():
    """W_out = 0 and W_down = 0 leave the hidden unchanged (pure residual)."""
    s = _tiny_shape()
    gi = W.group_inputs(5, [6], n_layers=1, shape=s)
    lw = gi.layers[0]
    lw.w_out = torch.zeros_like(lw.w_out)
    lw.w_down = torch.zeros_like(lw.w_down)
    r = L.gdn_layer(oracle._f64(gi.anchors), lw, np.array([0, 6]), s)
    np.testing.assert_array_equal(r["x_out"], oracle._f64(gi.anchors))


def test_skip_mode_changes_no_state():
    """Skipping the last layer's gated norm / out_proj / MLP changes no state
    ("Tail-Replay", Sec. 3: the final group FFN is omitted)."""
    s = _tiny_shape()
    gi = W.group_inputs(6, [9, 3], n_layers=3, shape=s)
    full = L.group_replay(gi, "full")
    skip = L.group_replay(gi, "skip")
    for a, b in zip(full, skip):
        np.testing.assert_array_equal(a["S"], b["S"])
        np.testing.assert_array_equal(a["conv_state"], b["conv_state"])
    assert skip[-1]["x_out"] is None and full[-1]["x_out"] is not None


def test_groups_are_independent_of_packing():
    """Two sequences packed together replay as if alone (errors and state never
    cross sequence or group boundaries)."""
    s = _tiny_shape()
    gi = W.group_inputs(8, [4, 7], n_layers=2, shape=s)
    both = L.group_replay(gi, "full")
    for n, (a, b) in enumerate([(0, 4), (4, 11)]):
        single = W.GroupInputs(gi.anchors[a:b], W.cu_from_lengths([b - a]), gi.layers, s)
        one = L.group_replay(single, "full")
        for l in range(2):
            np.testing.assert_allclose(both[l]["S"][n], one[l]["S"][0], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(both[l]["x_out"][a:b], one[l]["x_out"], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- continuation
# After a replay rebuilds a layer's recurrent state and conv state, the
# unmatched tokens continue from them ("Tail-Replay", Sec. 3).  Continuing
# from the states of a must give exactly what processing a || b in one pass
# gives ("Sparse Prefix Caching for Hybrid and Recurrent LLM Serving", exact
# resume); in fp64 the two differ only by rounding order.

def test_conv_priming_closed_form():
    """Delta weights turn the conv into a shift; on a continuation the rows
    shifted in at a sequence start are the stored history, oldest first."""
    rng = np.random.default_rng(3)
    cu = [0, 1, 1, 6]  # lengths 1, 0, 5
    D = 2
    pre = rng.standard_normal((6, D))
    hist = rng.standard_normal((3, D, 3))  # [N, D, width-1]
    w = np.zeros((D, 4))
    w[:, 1] = 1.0  # two tokens back
    out = L.causal_conv(pre, w, cu, hist)
    np.testing.assert_array_equal(out[0], hist[0][:, 1])      # t = 0 of seq 0 reads history slot 1
    np.testing.assert_array_equal(out[1], hist[2][:, 1])      # seq 2 starts at row 1
    np.testing.assert_array_equal(out[2], hist[2][:, 2])
    np.testing.assert_array_equal(out[3], pre[1])
    np.testing.assert_array_equal(out[5], pre[3])
    st = L.conv_state(pre, cu, 4, hist)
    np.testing.assert_array_equal(st[0], np.stack([hist[0][:, 1], hist[0][:, 2], pre[0]], axis=1))
    np.testing.assert_array_equal(st[1], hist[1])              # empty sequence keeps its history
    np.testing.assert_array_equal(st[2], pre[3:6].T)


def _split_batch(lengths, cuts):
    """Index arrays of the a-part (first cut_n tokens of every sequence) and
    the b-part (the rest) of a packed batch, plus their cu_seqlens."""
    starts = np.concatenate([[0], np.cumsum(lengths)])
    a_idx = np.concatenate([np.arange(starts[n], starts[n] + c) for n, c in enumerate(cuts)]).astype(np.int64)
    b_idx = np.concatenate([np.arange(starts[n] + c, starts[n + 1]) for n, c in enumerate(cuts)]).astype(np.int64)
    cu_a = np.concatenate([[0], np.cumsum(cuts)])
    cu_b = np.concatenate([[0], np.cumsum(np.asarray(lengths) - np.asarray(cuts))])
    return a_idx, b_idx, cu_a, cu_b


CONT_LENGTHS = [9, 5, 3, 7, 2]
CONT_CUTS = [4, 1, 3, 0, 2]  # b-parts of 5, 4, 0, 7, 0 tokens; a-parts shorter than the conv window too


def test_layer_continuation_is_exact():
    s = _tiny_shape()
    gi = W.group_inputs(31, CONT_LENGTHS, n_layers=1, shape=s)
    lw = gi.layers[0]
    lw.w_in = W.normal(31, "win", (s.proj_dim, s.hidden), 0.5)
    lw.conv_w = W.normal(31, "cw", (s.conv_dim, s.conv_w), 0.5)
    x = oracle._f64(gi.anchors)
    full = L.gdn_layer(x, lw, np.asarray(gi.cu_seqlens.tolist()), s)
    a_idx, b_idx, cu_a, cu_b = _split_batch(CONT_LENGTHS, CONT_CUTS)
    ra = L.gdn_layer(x[a_idx], lw, cu_a, s)
    rb = L.gdn_layer(x[b_idx], lw, cu_b, s, s_in=ra["S"], conv_in=ra["conv_state"])
    np.testing.assert_allclose(rb["S"], full["S"], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(rb["conv_state"], full["conv_state"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(rb["x_out"], full["x_out"][b_idx], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(rb["o"], full["o"][b_idx], rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("mode", ["skip", "full"])
def test_group_continuation_is_exact(mode):
    s = _tiny_shape()
    gi = W.group_inputs(32, CONT_LENGTHS, n_layers=3, shape=s)
    full = L.group_replay(gi, mode)
    a_idx, b_idx, cu_a, cu_b = _split_batch(CONT_LENGTHS, CONT_CUTS)
    ga = W.GroupInputs(gi.anchors[torch.from_numpy(a_idx)], torch.tensor(cu_a, dtype=torch.int32), gi.layers, s)
    gb = W.GroupInputs(gi.anchors[torch.from_numpy(b_idx)], torch.tensor(cu_b, dtype=torch.int32), gi.layers, s)
    ra = L.group_replay(ga, mode)
    rb = L.group_replay(gb, mode, initial=[(r["S"], r["conv_state"]) for r in ra])
    for l in range(3):
        np.testing.assert_allclose(rb[l]["S"], full[l]["S"], rtol=1e-10, atol=1e-13)
        np.testing.assert_allclose(rb[l]["conv_state"], full[l]["conv_state"], rtol=1e-10, atol=1e-13)


def test_continuation_rejects_a_reversed_conv_history(monkeypatch):
    """Planted mistake: a conv state stored newest-first breaks the exact
    continuation, so the test above pins the history's order."""
    s = _tiny_shape()
    gi = W.group_inputs(33, CONT_LENGTHS, n_layers=1, shape=s)
    x = oracle._f64(gi.anchors)
    lw = gi.layers[0]
    lw.conv_w = W.normal(33, "cw", (s.conv_dim, s.conv_w), 0.5)
    full = L.gdn_layer(x, lw, np.asarray(gi.cu_seqlens.tolist()), s)
    a_idx, b_idx, cu_a, cu_b = _split_batch(CONT_LENGTHS, CONT_CUTS)
    good = L.conv_state
    monkeypatch.setattr(L, "conv_state", lambda *a, **k: good(*a, **k)[..., ::-1])
    ra = L.gdn_layer(x[a_idx], lw, cu_a, s)
    rb = L.gdn_layer(x[b_idx], lw, cu_b, s, s_in=ra["S"], conv_in=ra["conv_state"])
    assert np.max(np.abs(rb["S"] - full["S"])) > 1e-6 * np.max(np.abs(full["S"]))


def test_sparse_anchor_gather_reads_pool_rows():
    """Token-wise sparse anchors ("SuffixReplay", Algorithm Design 2): the
    replay batch is the anchor pool's rows in index order."""
    s = _tiny_shape()
    gi = W.group_inputs(34, [6, 3], n_layers=2, shape=s)
    pool = W.normal(34, "pool", (20, s.hidden), 1.0)
    idx = np.array([19, 3, 4, 7, 0, 12, 5, 5, 18])
    a = L.group_replay(gi, "full", anchors=pool, anchor_index=idx)
    b = L.group_replay(W.GroupInputs(pool[torch.from_numpy(idx)], gi.cu_seqlens, gi.layers, s), "full")
    for l in range(2):
        np.testing.assert_array_equal(a[l]["S"], b[l]["S"])
