"""fp64 oracle for the replay group: GDN layers + SwiGLU MLPs, numpy.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages fix ("Tail-Replay: Escaping the Curse of Linear Attention in
Prefix Caching for Hybrid LLMs", Sec. 3; "SuffixReplay: Prefix Caching via
Suffix Replay for Hybrid LLMs", Algorithm Design 1):
  * consecutive linear-attention layers between two full-attention layers
    form a group; a group is replayed from its cached entry hidden (the
    output of the preceding full-attention layer) with every linear state
    starting at zero, and full-attention layers are skipped;
  * the group's final FFN is omitted, because the next group starts from its
    own cached exact hidden.

What the pages leave open, and the reading taken here (the Qwen3.5-family
GDN block, Sec. 2 of Tail-Replay names Gated DeltaNet as the linear layer):
  x_res = x
  h     = RMSNorm(x) * w_in_norm                     eps = 1e-6
  p     = h W_in^T  -> [q_pre | k_pre | v_pre | z | b | a]
  c     = causal depthwise conv, width 4, over [q_pre|k_pre|v_pre], zero
          left padding at every sequence start (replay starts from zero;
          a continuation supplies the rebuilt conv state instead)
  q,k,v = SiLU(c);  q, k L2-normalised per head (eps 1e-6 inside the sqrt)
  g     = -exp(A_log) * softplus(a + dt_bias);  beta = sigmoid(b)
  o     = gated-delta recurrence (oracle.gdn_replay), scale 1/sqrt(d_k)
  y     = RMSNorm_head(o) * w_gnorm * SiLU(z)        per V head
  x     = x_res + y W_out^T
  x     = x + W_down (SiLU(W_gate hh) * (W_up hh)),  hh = RMSNorm(x) * w_post
  conv_state = the last (width-1) pre-conv rows of each sequence, oldest
               first, taken from the padding where the sequence is shorter.
Skip mode (the method): the last layer of the group stops after its
recurrence -- neither its gated norm, out_proj nor MLP can change any state.
Full mode: every layer runs to its MLP.

Each primitive below is pinned by closed forms in ``tests/``; the composition
is parity unpinned by the pages.
"""
from __future__ import annotations

import numpy as np

from . import gdn_replay, _f64


def rmsnorm(x, w, eps):
    """x / sqrt(mean(x^2) + eps) * w over the last axis."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * w


def l2norm(x, eps):
    """x / sqrt(sum(x^2) + eps) over the last axis."""
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def sigmoid(x):
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def silu(x):
    return x * sigmoid(x)


def softplus(x):
    """log(1 + exp(x)), with x returned as is above 20 (overflow guard)."""
    return np.where(x > 20.0, x, np.log1p(np.exp(np.minimum(x, 20.0))))


def _history(conv_in, n, width, D):
    """The (width-1) pre-conv rows that precede sequence n, oldest first:
    zeros for a replay from zero, conv_in[n] (stored [D, width-1]) for a
    continuation from a rebuilt conv state."""
    if conv_in is None:
        return np.zeros((width - 1, D))
    return np.asarray(conv_in[n], dtype=np.float64).T


def causal_conv(pre, w, cu, conv_in=None):
    """Depthwise causal conv: c_t[ch] = sum_i w[ch, i] * pre_{t-W+1+i}[ch] over
    each sequence, never across cu_seqlens.  The W-1 rows before a sequence
    start are zero (replay from zero, "Tail-Replay", Sec. 3), or conv_in[n]
    when the sequence continues from a rebuilt state."""
    T, D = pre.shape
    W = w.shape[1]
    out = np.zeros_like(pre)
    for n in range(len(cu) - 1):
        s, e = int(cu[n]), int(cu[n + 1])
        ext = np.concatenate([_history(conv_in, n, W, D), pre[s:e]], axis=0)
        for t in range(e - s):
            out[s + t] = np.sum(w * ext[t: t + W].T, axis=1)
    return out


def conv_state(pre, cu, width, conv_in=None):
    """Last (width-1) pre-conv rows per sequence -> [N, D, width-1], oldest
    first; rows before the sequence start come from its history (zeros, or
    conv_in[n] on a continuation)."""
    N = len(cu) - 1
    D = pre.shape[1]
    st = np.zeros((N, D, width - 1))
    for n in range(N):
        s, e = int(cu[n]), int(cu[n + 1])
        ext = np.concatenate([_history(conv_in, n, width, D), pre[s:e]], axis=0)
        st[n] = ext[len(ext) - (width - 1):].T
    return st


def gdn_layer(x, lw, cu, shape, *, stop_after_recurrence=False, s_in=None, conv_in=None):
    """One GDN layer (+ its MLP unless stopped).  Returns a dict with the
    final state S, conv_state, the gates, o (None when stopped) and x_out.

    s_in [N, h_v, d_v, d_k] and conv_in [N, conv_dim, width-1] continue the
    layer from rebuilt states (the unmatched tokens after a replay, "Tail-
    Replay", Sec. 3); None starts from zero, as a replay does."""
    s = shape
    T = x.shape[0]
    h = rmsnorm(x, _f64(lw.w_in_norm), s.eps)
    p = h @ _f64(lw.w_in).T
    qd, vd = s.qk_dim, s.v_dim
    pre = p[:, : s.conv_dim]
    z = p[:, s.conv_dim: s.conv_dim + vd]
    b = p[:, s.conv_dim + vd: s.conv_dim + vd + s.h_v]
    a = p[:, s.conv_dim + vd + s.h_v:]
    c = silu(causal_conv(pre, _f64(lw.conv_w), cu, conv_in))
    q = l2norm(c[:, :qd].reshape(T, s.h_k, s.d_k), 1e-6)
    k = l2norm(c[:, qd: 2 * qd].reshape(T, s.h_k, s.d_k), 1e-6)
    v = c[:, 2 * qd:].reshape(T, s.h_v, s.d_v)
    g = -np.exp(_f64(lw.a_log)) * softplus(a + _f64(lw.dt_bias))
    beta = sigmoid(b)
    o, S = gdn_replay(q, k, v, g, beta, cu, scale=1.0 / np.sqrt(s.d_k), h0=s_in,
                      want_o=not stop_after_recurrence)
    out = dict(S=S, conv_state=conv_state(pre, cu, s.conv_w, conv_in), g=g, beta=beta,
               q=q, k=k, v=v, o=o, x_out=None)
    if stop_after_recurrence:
        return out
    y = rmsnorm(o, _f64(lw.w_gnorm), s.eps) * silu(z.reshape(T, s.h_v, s.d_v))
    x1 = x + y.reshape(T, vd) @ _f64(lw.w_out).T
    hh = rmsnorm(x1, _f64(lw.w_post_norm), s.eps)
    mid = silu(hh @ _f64(lw.w_gate).T) * (hh @ _f64(lw.w_up).T)
    out["x_out"] = x1 + mid @ _f64(lw.w_down).T
    out["x_attn"] = x1
    return out


def group_replay(gi, mode="skip", *, initial=None, anchor_index=None, anchors=None):
    """Replay one group from its anchors.

    gi: workloads.GroupInputs.  mode: "skip" (last layer stops after its
    recurrence) or "full".  anchors (default gi.anchors) is the anchor pool;
    with anchor_index, replay token t reads pool row anchor_index[t] (token-
    wise sparse anchors gathered from the sidecar, "SuffixReplay", Algorithm
    Design 2).  initial: None (every state starts at zero: the replay) or a
    per-layer list of (s_in, conv_in) to continue from.  Returns a list of
    per-layer dicts (see gdn_layer).
    """
    assert mode in ("skip", "full")
    cu = np.asarray(gi.cu_seqlens.tolist(), dtype=np.int64)
    x = _f64(gi.anchors if anchors is None else anchors)
    if anchor_index is not None:
        x = x[np.asarray(anchor_index, dtype=np.int64)]
    outs = []
    L = len(gi.layers)
    for l, lw in enumerate(gi.layers):
        stop = mode == "skip" and l == L - 1
        s_in, c_in = (None, None) if initial is None else initial[l]
        r = gdn_layer(x, lw, cu, gi.shape, stop_after_recurrence=stop, s_in=s_in, conv_in=c_in)
        outs.append(r)
        x = r["x_out"]
    return outs
