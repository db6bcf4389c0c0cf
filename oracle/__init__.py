"""fp64 oracle for suffix-replay state reconstruction.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
path (``gated_deltanet_state_sr_b200``) never imports it, and this package
imports nothing from the product: the two share only the seeded input
generators in ``workloads.py``.

Contents
--------
* ``gdn_replay``     Gated DeltaNet recurrence, token by token, fp64 (C).
* ``mamba2_replay``  Mamba2 per-head-decay recurrence, fp64 (C).
* ``layers``         the GDN layer, the SwiGLU MLP and the replay-group
                     schedule in numpy fp64 (``oracle/layers.py``).
* ``planning``       checkpoint placement: the objective, exhaustive search
                     and the literal recurrence (``oracle/planning.py``).

Parity status of each function (what pins it, see ``tests/test_oracle_*``):
* gdn_replay / mamba2_replay: pinned by closed forms (beta = 0 decay,
  orthonormal-key sum, Mamba2 decay-weighted sum), an explicit unrolled
  transition-product brute force, the contraction bound of the suffix
  approximation and the exact-resume identity.
* planning.*: pinned by the balanced optimum of uniform overlap depths and
  by point masses; the recurrence against exhaustive search.
* layers.*: each primitive pinned by closed forms; the *composition* of a
  GDN layer (order of norm, conv, gates, gated norm, MLP) is not printed on
  the pages -- parity unpinned beyond the readings listed in the design
  notes.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        lp = ctypes.POINTER(ctypes.c_longlong)
        L.oracle_gdn.argtypes = [dp, dp, dp, dp, dp, lp, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                 dp, dp, dp, ip, ctypes.c_int, ctypes.c_int]
        L.oracle_gdn.restype = ctypes.c_int
        L.oracle_mamba2.argtypes = [dp, dp, dp, dp, dp, lp, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_int, dp, dp, dp, ip,
                                    ctypes.c_int, ctypes.c_int]
        L.oracle_mamba2.restype = ctypes.c_int
        L.oracle_num_threads.restype = ctypes.c_int
        _LIB = L
    return _LIB


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor -> exact fp64 copy
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a, ctype=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def gdn_replay(q, k, v, g, beta, cu_seqlens, *, scale=None, h0=None, want_o=True,
               units=None, n_threads=0):
    """Gated DeltaNet replay of every packed sequence from S = h0 (else 0).

    q, k: [T, H_k, d_k]; v: [T, H_v, d_v]; g, beta: [T, H_v] (g = log alpha);
    cu_seqlens: [N+1].  Returns (o [T, H_v, d_v] or None, S [N, H_v, d_v, d_k]),
    both fp64.  ``units`` restricts the work to a list of (seq * H_v + head)
    indices (other entries of o / S are left as NaN).
    """
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    T, h_k, d_k = q.shape
    h_v, d_v = v.shape[1], v.shape[2]
    cu = np.ascontiguousarray(np.asarray(cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens), dtype=np.int64)
    n = cu.size - 1
    if scale is None:
        scale = 1.0 / np.sqrt(d_k)
    h0 = _f64(h0)
    o = np.full((T, h_v, d_v), np.nan) if want_o else None
    s = np.full((n, h_v, d_v, d_k), np.nan)
    u = None if units is None else np.ascontiguousarray(units, dtype=np.int32)
    rc = lib().oracle_gdn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                          _ptr(cu, ctypes.c_longlong), n, h_k, h_v, d_k, d_v, float(scale),
                          _ptr(h0), _ptr(o), _ptr(s), _ptr(u, ctypes.c_int),
                          0 if u is None else u.size, n_threads)
    if rc != 0:
        raise ValueError("oracle_gdn: bad arguments")
    return o, s


def mamba2_replay(x, B, C, dt, A, cu_seqlens, *, h0=None, want_y=True, units=None,
                  n_threads=0):
    """Mamba2 replay: S_t = exp(dt_t A_h) S_{t-1} + dt_t x_t B_t^T, y_t = S_t C_t.

    x: [T, H, P]; B, C: [T, G, N_s]; dt: [T, H]; A: [H].  Returns
    (y [T, H, P] or None, S [N, H, P, N_s]) in fp64."""
    x, B, C, dt, A = map(_f64, (x, B, C, dt, A))
    T, H, P = x.shape
    G, Ns = B.shape[1], B.shape[2]
    cu = np.ascontiguousarray(np.asarray(cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens), dtype=np.int64)
    n = cu.size - 1
    h0 = _f64(h0)
    y = np.full((T, H, P), np.nan) if want_y else None
    s = np.full((n, H, P, Ns), np.nan)
    u = None if units is None else np.ascontiguousarray(units, dtype=np.int32)
    rc = lib().oracle_mamba2(_ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A),
                             _ptr(cu, ctypes.c_longlong), n, H, P, G, Ns, _ptr(h0), _ptr(y),
                             _ptr(s), _ptr(u, ctypes.c_int), 0 if u is None else u.size,
                             n_threads)
    if rc != 0:
        raise ValueError("oracle_mamba2: bad arguments")
    return y, s
