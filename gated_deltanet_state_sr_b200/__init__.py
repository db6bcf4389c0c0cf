"""Suffix-replay state reconstruction for hybrid LLMs on B200 (sm_100a).

Thin Python binding of the C-ABI library ``libsr.so`` (declared in
``include/sr/sr.h``).  This module only marshals arguments -- torch tensors to
device pointers, shapes to the C structs, the current CUDA stream -- and
allocates outputs / workspaces with torch when the caller does not pass them.
Every step of the replay runs in the library's CUDA kernels; there is no CPU
or PyTorch fallback: importing fails loudly when ``libsr.so`` is missing.

Entry points mirror the C ABI:
    gdn_replay      one Gated DeltaNet layer from raw q/k/v/g/beta
    mamba2_replay   the Mamba2 per-head-decay variant
    group_replay    whole groups of GDN layers + MLPs from cached anchors
"""
from __future__ import annotations

import ctypes
import math
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
# SR_LIBRARY=libsr_checked.so selects the bounds-checked build (the same
# kernels with every global index checked into the device status word).
_LIB_NAME = os.environ.get("SR_LIBRARY", "libsr.so")
if _LIB_NAME not in ("libsr.so", "libsr_checked.so"):
    raise ImportError(f"SR_LIBRARY must be libsr.so or libsr_checked.so, not {_LIB_NAME!r}")
LIB_PATH = os.path.join(_HERE, _LIB_NAME)
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "sr", "sr.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python gated_deltanet_state_sr_b200/build.py` "
                      "(there is no fallback path)")

_lib = ctypes.CDLL(LIB_PATH)

SR_OK, SR_ERR_INVALID_ARG, SR_ERR_UNSUPPORTED, SR_ERR_WORKSPACE, SR_ERR_CUDA, SR_ERR_DEVICE = range(6)
SR_BF16, SR_FP32 = 0, 1
SR_GDN_AUTO, SR_GDN_SEQUENTIAL, SR_GDN_CHUNKED, SR_GDN_TCGEN05, SR_GDN_TCGEN05_FUSED = 0, 1, 2, 3, 4
SR_MODE_SKIP, SR_MODE_FULL = 0, 1
SR_DEV_BAD_CU_SEQLENS, SR_DEV_SEQ_TOO_LONG, SR_DEV_TIMEOUT, SR_DEV_BAD_INDEX, SR_DEV_BAD_ACCESS = 0x1, 0x2, 0x4, 0x8, 0x10
CHECKED = _LIB_NAME == "libsr_checked.so"
_ALGOS = {"auto": SR_GDN_AUTO, "sequential": SR_GDN_SEQUENTIAL, "chunked": SR_GDN_CHUNKED,
          "tcgen05": SR_GDN_TCGEN05, "tcgen05_fused": SR_GDN_TCGEN05_FUSED}

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32


class GdnArgs(ctypes.Structure):
    _fields_ = [("q", _vp), ("k", _vp), ("v", _vp), ("g", _vp), ("beta", _vp), ("cu_seqlens", _vp),
                ("h0", _vp), ("o", _vp), ("s_out", _vp), ("dtype", _i32), ("algo", _i32),
                ("n_seqs", _i32), ("total_tokens", _i32), ("max_seqlen", _i32), ("h_k", _i32),
                ("h_v", _i32), ("d_k", _i32), ("d_v", _i32), ("scale", ctypes.c_float)]


class Mamba2Args(ctypes.Structure):
    _fields_ = [("x", _vp), ("B", _vp), ("C", _vp), ("dt", _vp), ("A", _vp), ("cu_seqlens", _vp),
                ("h0", _vp), ("y", _vp), ("s_out", _vp), ("n_seqs", _i32), ("total_tokens", _i32),
                ("max_seqlen", _i32), ("n_heads", _i32), ("head_dim", _i32), ("n_groups", _i32),
                ("d_state", _i32), ("algo", _i32)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("w_in_norm", _vp), ("w_in", _vp), ("conv_w", _vp), ("a_log", _vp),
                ("dt_bias", _vp), ("w_gnorm", _vp), ("w_out", _vp), ("w_post_norm", _vp),
                ("w_gate", _vp), ("w_up", _vp), ("w_down", _vp),
                ("w_in_lo8", _vp), ("w_out_lo8", _vp), ("w_gate_lo8", _vp), ("w_up_lo8", _vp), ("w_down_lo8", _vp)]


LO8_FIELDS = ("w_in_lo8", "w_out_lo8", "w_gate_lo8", "w_up_lo8", "w_down_lo8")


class LayerOutputs(ctypes.Structure):
    _fields_ = [("s_out", _vp), ("conv_out", _vp), ("hidden_out", _vp)]


class LayerState(ctypes.Structure):
    _fields_ = [("s_in", _vp), ("conv_in", _vp)]


class Profile(ctypes.Structure):
    _fields_ = [("events", ctypes.POINTER(_vp)), ("kinds", ctypes.POINTER(_i32)), ("capacity", _i32),
                ("count", _i32)]


KERNEL_KINDS = ["row_prep", "gemm_in", "conv", "gdn", "gated_norm", "gemm_out", "gemm_gateup", "gemm_down", "cast"]


class GroupArgs(ctypes.Structure):
    _fields_ = [("anchors", ctypes.POINTER(_vp)), ("cu_seqlens", _vp),
                ("weights", ctypes.POINTER(LayerWeights)), ("outputs", ctypes.POINTER(LayerOutputs)),
                ("n_groups", _i32), ("n_layers", _i32), ("n_seqs", _i32), ("total_tokens", _i32),
                ("max_seqlen", _i32), ("hidden", _i32), ("inter", _i32), ("h_k", _i32), ("h_v", _i32),
                ("d_k", _i32), ("d_v", _i32), ("conv_width", _i32), ("eps", ctypes.c_float),
                ("mode", _i32), ("precision", _i32), ("profile", ctypes.POINTER(Profile)),
                ("initial", ctypes.POINTER(LayerState)), ("anchor_index", _vp), ("anchor_rows", _i32),
                ("layer_done", ctypes.POINTER(_vp))]


def _sig(name, restype, *argtypes):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = list(argtypes)
    return f


_gdn_ws = _sig("sr_gdn_replay_workspace", ctypes.c_size_t, ctypes.POINTER(GdnArgs))
_gdn = _sig("sr_gdn_replay", _i32, ctypes.POINTER(GdnArgs), _vp, ctypes.c_size_t, _vp)
_m2_ws = _sig("sr_mamba2_replay_workspace", ctypes.c_size_t, ctypes.POINTER(Mamba2Args))
_m2 = _sig("sr_mamba2_replay", _i32, ctypes.POINTER(Mamba2Args), _vp, ctypes.c_size_t, _vp)
_grp_ws = _sig("sr_group_replay_workspace", ctypes.c_size_t, ctypes.POINTER(GroupArgs))
_grp = _sig("sr_group_replay", _i32, ctypes.POINTER(GroupArgs), _vp, ctypes.c_size_t, _vp)
_last_error = _sig("sr_last_error", ctypes.c_char_p)
_dev_status = _sig("sr_device_status", _i32, _vp, _vp, ctypes.POINTER(ctypes.c_uint32))
_version = _sig("sr_version", _i32)


def declared_symbols(header=HEADER_PATH):
    """Names of every entry point ``include/sr/sr.h`` declares."""
    txt = open(header).read()
    return sorted(set(re.findall(r"SR_API\s+[\w\s\*]+?\b(sr_\w+)\s*\(", txt)))


def library():
    return _lib


class SrError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"sr status {status}: {msg}")
        self.status = status


def last_error() -> str:
    return (_last_error() or b"").decode()


def _check(status):
    if status != SR_OK:
        raise SrError(status, last_error())


def version() -> int:
    return int(_version())


# ------------------------------------------------------------------ torch glue


def _torch():
    import torch  # plumbing only: device memory and streams
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype=None, ndim=None, device=True):
    torch = _torch()
    if t is None:
        raise ValueError(f"{name} is required")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")
    return t


def workspace(nbytes, device="cuda"):
    """A 256-byte aligned device workspace of at least nbytes (torch-allocated)."""
    torch = _torch()
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def device_status(ws, stream=None) -> int:
    """Device status flags (SR_DEV_*) that the last call on ``ws`` recorded."""
    flags = ctypes.c_uint32(0)
    st = _dev_status(_ptr(ws), _stream_handle(stream), ctypes.byref(flags))
    if st not in (SR_OK, SR_ERR_DEVICE):
        _check(st)
    return int(flags.value)


def gdn_args(q, k, v, g, beta, cu_seqlens, *, n_seqs, max_seqlen, h0=None, o=None, s_out=None,
             scale=0.0, algo="auto") -> GdnArgs:
    torch = _torch()
    T, h_k, d_k = q.shape
    h_v, d_v = v.shape[1], v.shape[2]
    dtype = SR_FP32 if q.dtype == torch.float32 else SR_BF16
    return GdnArgs(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), _ptr(h0),
                   _ptr(o), _ptr(s_out), dtype, _ALGOS[algo], n_seqs, T, max_seqlen, h_k, h_v,
                   d_k, d_v, float(scale))


def gdn_replay(q, k, v, g, beta, cu_seqlens, *, max_seqlen, h0=None, want_o=True, o=None,
               s_out=None, scale=0.0, algo="auto", ws=None, stream=None):
    """Gated DeltaNet replay of every packed sequence (see sr_gdn_replay).

    q, k: [T, H_k, d] bf16/fp32; v: [T, H_v, d]; g, beta: [T, H_v] fp32;
    cu_seqlens: [N+1] int32 (device); max_seqlen: host int >= every length.
    Returns (o or None, s_out [N, H_v, d_v, d_k] fp32)."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, 3)
    _need(g, "g", torch.float32, 2)
    _need(beta, "beta", torch.float32, 2)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    n = cu_seqlens.numel() - 1
    T, _, d_k = q.shape
    h_v, d_v = v.shape[1], v.shape[2]
    if h0 is not None:
        _need(h0, "h0", torch.float32, 4)
    if o is None and want_o:
        o = torch.empty_like(v)
    if s_out is None:
        s_out = torch.empty(n, h_v, d_v, d_k, dtype=torch.float32, device=q.device)
    args = gdn_args(q, k, v, g, beta, cu_seqlens, n_seqs=n, max_seqlen=max_seqlen, h0=h0, o=o,
                    s_out=s_out, scale=scale, algo=algo)
    need = _gdn_ws(ctypes.byref(args))
    if need == 0:
        _check(_gdn(ctypes.byref(args), None, 0, None))  # raises with the validation message
    if ws is None or ws.numel() < need:
        ws = workspace(need, q.device)
    _check(_gdn(ctypes.byref(args), _ptr(ws), ws.numel(), _stream_handle(stream)))
    return o, s_out


def gdn_workspace_bytes(args: GdnArgs) -> int:
    return int(_gdn_ws(ctypes.byref(args)))


def gdn_call(args: GdnArgs, ws, stream=None) -> int:
    """Raw C call with a prepared GdnArgs (returns the sr_status)."""
    return int(_gdn(ctypes.byref(args), _ptr(ws), 0 if ws is None else ws.numel(),
                    _stream_handle(stream) if ws is not None else None))


SR_MAMBA2_AUTO, SR_MAMBA2_SEQUENTIAL, SR_MAMBA2_CHUNKED, SR_MAMBA2_TCGEN05 = 0, 1, 2, 3
_M2_ALGOS = {"auto": SR_MAMBA2_AUTO, "sequential": SR_MAMBA2_SEQUENTIAL, "chunked": SR_MAMBA2_CHUNKED,
             "tcgen05": SR_MAMBA2_TCGEN05}


def mamba2_args(x, B, C, dt, A, cu_seqlens, *, n_seqs, max_seqlen, h0=None, y=None,
                s_out=None, algo="auto") -> Mamba2Args:
    T, H, P = x.shape
    G, Ns = B.shape[1], B.shape[2]
    return Mamba2Args(_ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A), _ptr(cu_seqlens), _ptr(h0),
                      _ptr(y), _ptr(s_out), n_seqs, T, max_seqlen, H, P, G, Ns, _M2_ALGOS[algo])


def mamba2_replay(x, B, C, dt, A, cu_seqlens, *, max_seqlen, h0=None, want_y=True, y=None,
                  s_out=None, ws=None, stream=None, algo="auto"):
    """Mamba2 replay (see sr_mamba2_replay).  Returns (y or None, s_out)."""
    torch = _torch()
    _need(x, "x", torch.bfloat16, 3)
    _need(B, "B", torch.bfloat16, 3)
    _need(C, "C", torch.bfloat16, 3)
    _need(dt, "dt", torch.float32, 2)
    _need(A, "A", torch.float32, 1)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    n = cu_seqlens.numel() - 1
    T, H, P = x.shape
    Ns = B.shape[2]
    if y is None and want_y:
        y = torch.empty_like(x)
    if s_out is None:
        s_out = torch.empty(n, H, P, Ns, dtype=torch.float32, device=x.device)
    args = mamba2_args(x, B, C, dt, A, cu_seqlens, n_seqs=n, max_seqlen=max_seqlen, h0=h0, y=y,
                       s_out=s_out, algo=algo)
    need = _m2_ws(ctypes.byref(args))
    if need == 0:
        _check(_m2(ctypes.byref(args), None, 0, None))
    if ws is None or ws.numel() < need:
        ws = workspace(need, x.device)
    _check(_m2(ctypes.byref(args), _ptr(ws), ws.numel(), _stream_handle(stream)))
    return y, s_out


def mamba2_workspace_bytes(args: Mamba2Args) -> int:
    return int(_m2_ws(ctypes.byref(args)))


def mamba2_call(args: Mamba2Args, ws, stream=None) -> int:
    return int(_m2(ctypes.byref(args), _ptr(ws), 0 if ws is None else ws.numel(),
                   _stream_handle(stream) if ws is not None else None))


def default_scale(d_k):
    return 1.0 / math.sqrt(d_k)


# ------------------------------------------------------------------ test support (include/sr/sr_testing.h)

_test_gemm = _sig("sr_test_gemm", _i32, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp,
                  ctypes.c_size_t, _vp)
EPI_STORE, EPI_RESIDUAL, EPI_SWIGLU = 0, 1, 2
GEMM_FORM_DEFAULT, GEMM_FORM_SINGLE, GEMM_FORM_PAIR = 0, 1, 2


def test_gemm(a, b0, *, b1=None, r=None, epi=EPI_STORE, c=None, ws=None, stream=None, form=GEMM_FORM_DEFAULT):
    """One tcgen05 GEMM through sr_test_gemm: c = a b0^T, r + a b0^T, or
    SiLU(a b0^T) * (a b1^T).  bf16 CUDA tensors, row-major.  form: the
    library default, one CTA per tile, or CTA pairs."""
    torch = _torch()
    m, k = a.shape
    n = b0.shape[0]
    if c is None:
        c = torch.empty(m, n, dtype=torch.bfloat16, device=a.device)
    if ws is None:
        ws = workspace(256, a.device)
    _check(_test_gemm(_ptr(a), _ptr(b0), _ptr(b1), _ptr(c), _ptr(r), m, n, k, epi, int(form), _ptr(ws),
                      ws.numel(), _stream_handle(stream)))
    return c


_test_wait = _sig("sr_test_wait_timeout", _i32, ctypes.c_uint64, _i32, _vp, ctypes.c_size_t, _vp)
WAIT_LIMIT_NS = 500_000_000  # the kernels' own limit on one mbarrier wait


def test_wait_timeout(limit_ns, *, arrive=False, device="cuda", stream=None):
    """sr_test_wait_timeout: one CTA waits on an mbarrier with a limit of
    limit_ns (nothing arrives unless `arrive`), frees its tensor memory and
    exits.  Returns (status flags, the wait's duration in ns) after a sync."""
    torch = _torch()
    ws = workspace(256, device)
    _check(_test_wait(int(limit_ns), 1 if arrive else 0, _ptr(ws), ws.numel(), _stream_handle(stream)))
    flags = device_status(ws, stream)
    elapsed = int(ws[8:16].cpu().view(torch.int64).item())
    return flags, elapsed


def test_wait_call(limit_ns, arrive=0):
    """Raw C call with no workspace (returns the sr_status; validation only)."""
    return int(_test_wait(int(limit_ns), int(arrive), None, 0, None))


# ------------------------------------------------------------------ group replay

SR_PREC_SPLIT, SR_PREC_BF16, SR_PREC_SPLIT_FP8 = 0, 1, 2
_LAYER_FIELDS = [f for f, _ in LayerWeights._fields_]


def group_args(anchors, cu_seqlens, weights, outputs, *, max_seqlen, hidden, inter, h_k, h_v, d=128,
               conv_width=4, eps=1e-6, mode=SR_MODE_SKIP, precision=SR_PREC_SPLIT, profile=None,
               initial=None, anchor_index=None, total_tokens=None, layer_done=None):
    """Builds a GroupArgs (and keeps the ctypes arrays alive on it).

    anchors: list [G] of [T, hidden] bf16 CUDA tensors (the anchor pools
    [rows, hidden] when anchor_index, an int32 CUDA tensor [T], is given);
    weights: list [G] of lists [L] of objects with the sr_layer_weights field
    names (CUDA tensors); outputs: list [G] of lists [L] of (s_out, conv_out,
    hidden_out-or-None); initial: None or list [G] of lists [L] of
    (s_in-or-None, conv_in-or-None) to continue from; layer_done: None or a
    list [L] of torch.cuda.Event (or None), each recorded once that layer's
    states are final."""
    G, L = len(anchors), len(weights[0])
    init_arr = None
    if initial is not None:
        init_arr = (LayerState * (G * L))()
        for g in range(G):
            for l in range(L):
                si, ci = initial[g][l]
                init_arr[g * L + l] = LayerState(None if si is None else si.data_ptr(),
                                                 None if ci is None else ci.data_ptr())
    anc = (_vp * G)(*[t.data_ptr() for t in anchors])
    w_arr = (LayerWeights * (G * L))()
    o_arr = (LayerOutputs * (G * L))()
    for g in range(G):
        for l in range(L):
            lw = weights[g][l]
            w_arr[g * L + l] = LayerWeights(*[None if getattr(lw, f, None) is None else getattr(lw, f).data_ptr()
                                              for f in _LAYER_FIELDS])
            s, c, h = outputs[g][l]
            o_arr[g * L + l] = LayerOutputs(s.data_ptr(), c.data_ptr(), None if h is None else h.data_ptr())
    n = cu_seqlens.numel() - 1
    if total_tokens is not None:
        T = total_tokens
    else:
        T = anchors[0].shape[0] if anchor_index is None else anchor_index.numel()
    a = GroupArgs(anc, cu_seqlens.data_ptr(), w_arr, o_arr, G, L, n, T, max_seqlen, hidden, inter, h_k, h_v,
                  d, d, conv_width, float(eps), mode, precision,
                  ctypes.pointer(profile.struct) if profile is not None else None,
                  init_arr, None if anchor_index is None else anchor_index.data_ptr(),
                  0 if anchor_index is None else anchors[0].shape[0])
    ev_arr = None
    if layer_done is not None:
        assert len(layer_done) == L
        for e in layer_done:
            if e is not None and e.cuda_event == 0:
                e.record()  # torch creates the CUDA event lazily, at its first record
        ev_arr = (_vp * L)(*[None if e is None else e.cuda_event for e in layer_done])
        a.layer_done = ev_arr
    a._keep = (anc, w_arr, o_arr, profile, init_arr, ev_arr)
    return a


class LaunchProfiler:
    """CUDA events for sr_profile: per-launch device time of a group replay,
    recorded on the launching stream."""

    def __init__(self, capacity=256):
        torch = _torch()
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * capacity)]
        for e in self.ev:  # torch creates the CUDA event lazily, at its first record
            e.record()
        self.handles = (_vp * (2 * capacity))(*[e.cuda_event for e in self.ev])
        self.kinds = (_i32 * capacity)()
        self.struct = Profile(self.handles, self.kinds, capacity, 0)

    def times(self):
        """[(kind name, ms)] of the last profiled call (events must have completed)."""
        n = min(self.struct.count, self.struct.capacity)
        return [(KERNEL_KINDS[self.kinds[i]], self.ev[2 * i].elapsed_time(self.ev[2 * i + 1])) for i in range(n)]


def group_workspace_bytes(args: GroupArgs) -> int:
    return int(_grp_ws(ctypes.byref(args)))


def group_call(args: GroupArgs, ws, stream=None) -> int:
    return int(_grp(ctypes.byref(args), None if ws is None else _ptr(ws), 0 if ws is None else ws.numel(),
                    _stream_handle(stream) if ws is not None else None))


def group_replay(anchors, cu_seqlens, weights, *, max_seqlen, hidden, inter, h_k, h_v, d=128, conv_width=4,
                 eps=1e-6, mode=SR_MODE_SKIP, precision=SR_PREC_SPLIT, want_hidden=False, outputs=None,
                 ws=None, stream=None, profile=None, initial=None, anchor_index=None, layer_done=None):
    """Replays every group of the call (see sr_group_replay).  Returns the
    outputs list [G][L] of (s_out, conv_out, hidden_out or None).

    anchor_index (int32 CUDA tensor [T]) gathers the replay tokens from the
    anchor pools ``anchors``; initial ([G][L] of (s_in, conv_in), either may
    be None) continues from earlier states instead of zero."""
    torch = _torch()
    dev = anchors[0].device
    G, L = len(anchors), len(weights[0])
    n = cu_seqlens.numel() - 1
    T = anchors[0].shape[0] if anchor_index is None else anchor_index.numel()
    conv_dim = 2 * h_k * d + h_v * d
    if outputs is None:
        outputs = []
        for g in range(G):
            row = []
            for l in range(L):
                keep_h = want_hidden and not (mode == SR_MODE_SKIP and l == L - 1)
                row.append((torch.empty(n, h_v, d, d, dtype=torch.float32, device=dev),
                            torch.empty(n, conv_dim, conv_width - 1, dtype=torch.bfloat16, device=dev),
                            torch.empty(T, hidden, dtype=torch.bfloat16, device=dev) if keep_h else None))
            outputs.append(row)
    args = group_args(anchors, cu_seqlens, weights, outputs, max_seqlen=max_seqlen, hidden=hidden, inter=inter,
                      h_k=h_k, h_v=h_v, d=d, conv_width=conv_width, eps=eps, mode=mode, precision=precision,
                      profile=profile, initial=initial, anchor_index=anchor_index, layer_done=layer_done)
    need = group_workspace_bytes(args)
    if need == 0:
        _check(group_call(args, None))
    if ws is None or ws.numel() < need:
        ws = workspace(need, dev)
    _check(group_call(args, ws, stream))
    return outputs


# ------------------------------------------------------------------ allocation-free group replay

_grp_noalloc = _sig("sr_group_replay_noalloc", _i32, ctypes.POINTER(GroupArgs), _vp, ctypes.POINTER(_vp))
NOALLOC_SCRATCH_BYTES = 32 << 20


def group_replay_noalloc(anchors, cu_seqlens, weights, outputs, *, max_seqlen, hidden, inter, h_k, h_v, d=128,
                         conv_width=4, eps=1e-6, mode=SR_MODE_SKIP, precision=SR_PREC_SPLIT, stream=None):
    """sr_group_replay_noalloc: the group replay for callers that cannot allocate
    device memory (scratch in the library's own fixed device array).  The caller
    passes the anchors, the weights and preallocated outputs [G][L] of
    (s_out, conv_out, hidden_out or None).  Returns the device address of the
    scratch array (its first word is the status word)."""
    args = group_args(anchors, cu_seqlens, weights, outputs, max_seqlen=max_seqlen, hidden=hidden, inter=inter,
                      h_k=h_k, h_v=h_v, d=d, conv_width=conv_width, eps=eps, mode=mode, precision=precision)
    scratch = _vp()
    _check(_grp_noalloc(ctypes.byref(args), _stream_handle(stream), ctypes.byref(scratch)))
    return scratch.value


def group_noalloc_call(args: GroupArgs, stream=None) -> int:
    """Raw C call (returns the sr_status); no CUDA work before validation passes."""
    return int(_grp_noalloc(ctypes.byref(args), None if stream is None else _stream_handle(stream), None))


# ------------------------------------------------------------------ anchor sidecar

class CaptureArgs(ctypes.Structure):
    _fields_ = [("hidden_states", _vp), ("pool", _vp), ("src_rows", _vp), ("dst_rows", _vp), ("n", _i32),
                ("hidden", _i32), ("src_rows_total", _i32), ("pool_rows", _i32)]


class AnchorPlanArgs(ctypes.Structure):
    _fields_ = [("n_prefix", ctypes.c_int64), ("page_size", _i32), ("anchors_per_page", _i32), ("layout", _i32),
                ("k_max", _i32), ("ratio", ctypes.c_double), ("block_table", ctypes.POINTER(_i32))]


SR_ANCHORS_PAGE_TAIL, SR_ANCHORS_UNIFORM = 0, 1
_capture = _sig("sr_anchor_capture", _i32, ctypes.POINTER(CaptureArgs), _vp, ctypes.c_size_t, _vp)
_plan = _sig("sr_sparse_anchor_plan", _i32, ctypes.POINTER(AnchorPlanArgs), ctypes.POINTER(ctypes.c_int64),
             ctypes.POINTER(_i32), ctypes.c_int64, ctypes.POINTER(ctypes.c_int64))


def capture_args(hidden_states, pool, src_rows, dst_rows) -> CaptureArgs:
    return CaptureArgs(hidden_states.data_ptr(), pool.data_ptr(), src_rows.data_ptr(), dst_rows.data_ptr(),
                       src_rows.numel(), hidden_states.shape[1], hidden_states.shape[0], pool.shape[0])


def capture_call(args: CaptureArgs, ws, stream=None) -> int:
    return int(_capture(ctypes.byref(args), None if ws is None else _ptr(ws), 0 if ws is None else ws.numel(),
                        _stream_handle(stream) if ws is not None else None))


def anchor_capture(hidden_states, pool, src_rows, dst_rows, *, ws=None, stream=None):
    """sr_anchor_capture: pool[dst_rows[i]] = hidden_states[src_rows[i]] (bf16
    CUDA tensors, int32 index tensors on the same device)."""
    if ws is None:
        ws = workspace(256, hidden_states.device)
    _check(capture_call(capture_args(hidden_states, pool, src_rows, dst_rows), ws, stream))
    return ws


def sparse_anchor_plan(n_prefix, *, page_size=64, anchors_per_page=4, layout=SR_ANCHORS_PAGE_TAIL, k_max=512,
                       ratio=0.05, block_table=None):
    """sr_sparse_anchor_plan (host): (positions, pool_rows) of the anchors a
    token-sparse replay of an n_prefix-token prefix reads, as Python lists."""
    bt = None
    if block_table is not None:
        bt = (_i32 * len(block_table))(*block_table)
    a = AnchorPlanArgs(int(n_prefix), page_size, anchors_per_page, layout, k_max, float(ratio), bt)
    count = ctypes.c_int64(0)
    # first call sizes the arrays: *count is set only once the arguments are valid
    st = _plan(ctypes.byref(a), None, None, 0, ctypes.byref(count))
    k = count.value
    if st != SR_OK and k == 0:
        _check(st)
    pos = (ctypes.c_int64 * max(k, 1))()
    rows = (_i32 * max(k, 1))()
    _check(_plan(ctypes.byref(a), pos, rows, k, ctypes.byref(count)))
    return list(pos[:k]), list(rows[:k])


# ------------------------------------------------------------------ fp8 low-pass weights

_prep_lo8 = _sig("sr_prepare_lo8_weights", _i32, _vp, _vp, ctypes.c_int64, _vp)


def prepare_lo8(w, stream=None):
    """sr_prepare_lo8_weights: the low-pass copy e5m2(w * 2^-8) of a bf16 CUDA
    weight tensor, as a uint8 tensor of the same shape."""
    torch = _torch()
    out = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    _check(_prep_lo8(_ptr(w), _ptr(out), w.numel(), _stream_handle(stream)))
    return out


def attach_lo8(layer, stream=None):
    """Adds the five *_lo8 low-pass copies to a layer-weights object (its
    w_in, w_out, w_gate, w_up, w_down CUDA tensors) for SR_PREC_SPLIT_FP8."""
    for f in LO8_FIELDS:
        setattr(layer, f, prepare_lo8(getattr(layer, f[:-4]), stream))
    return layer


# ------------------------------------------------------------------ checkpoint placement (host)

_ckpt = _sig("sr_checkpoint_plan", _i32, ctypes.POINTER(ctypes.c_double), ctypes.c_int64, _i32,
             ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(_i32), ctypes.POINTER(ctypes.c_double))


def checkpoint_plan(p, m_max):
    """sr_checkpoint_plan (host): (positions, expected recompute) of the best
    placement of at most m_max checkpoints for depth weights p[0..N]."""
    import numpy as np
    w = np.ascontiguousarray(p, dtype=np.float64)
    n = w.size - 1
    pos = (ctypes.c_int64 * max(m_max, 1))()
    cnt = _i32(0)
    cost = ctypes.c_double(0.0)
    _check(_ckpt(w.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), n, m_max, pos, ctypes.byref(cnt),
                 ctypes.byref(cost)))
    return list(pos[:cnt.value]), cost.value
