"""Allocation-free group replay (sr_group_replay_noalloc).

Some callers cannot allocate device memory -- a plug-in that only receives
its input and output buffers, or an engine whose spare HBM is all promised
to its KV cache -- so the library offers a group replay whose scratch lives
in a fixed device array inside the library.  These tests call it through the
C ABI and compare it with sr_group_replay (caller workspace) on the same
inputs, twice in a row, since every call reuses the array the previous call
left behind.  This file is collected last on purpose."""
import pytest
import torch

import workloads as W

sr = pytest.importorskip("gated_deltanet_state_sr_b200")

# Longest single-sequence replay whose split-precision scratch fits the array
# at hidden 2560, intermediate 9216, 16/32 heads of 128, three layers.
NOALLOC_SPLIT_MAX_TOKENS = 191


class DevLayer:
    def __init__(self, lw):
        for f in ("w_in_norm", "w_in", "conv_w", "a_log", "dt_bias", "w_gnorm", "w_out", "w_post_norm",
                  "w_gate", "w_up", "w_down"):
            setattr(self, f, getattr(lw, f).cuda().contiguous())


def fresh_outputs(gis, mode, s):
    T = gis[0].anchors.shape[0]
    n = gis[0].cu_seqlens.numel() - 1
    L = len(gis[0].layers)
    out = []
    for _ in gis:
        row = []
        for l in range(L):
            keep_h = not (mode == sr.SR_MODE_SKIP and l == L - 1)
            row.append((torch.full((n, s.h_v, s.d_v, s.d_k), float("nan"), device="cuda"),
                        torch.zeros(n, s.conv_dim, 3, dtype=torch.bfloat16, device="cuda"),
                        torch.zeros(T, s.hidden, dtype=torch.bfloat16, device="cuda") if keep_h else None))
        out.append(row)
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["small_full", "hidden2560_skip", "hidden2560_capacity"])
def test_noalloc_matches_workspace_entry_point_twice(case):
    """The allocation-free call runs the same kernels on the same bytes as
    sr_group_replay, so its results must be bit-identical, on the first call
    and on a second call that finds the first call's leftovers in the array.
    The capacity case is the longest split-precision replay the array holds
    (one sequence of 191 tokens at hidden 2560), whose scratch ends within
    1 MB of the array's end."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if case == "small_full":
        s = W.LayerShape(hidden=256, inter=512, h_k=2, h_v=4, d_k=128, d_v=128)
        gis = [W.group_inputs(70 + g, [40, 1, 0, 77], n_layers=2, shape=s) for g in range(2)]
        mode = sr.SR_MODE_FULL
    elif case == "hidden2560_skip":
        s = W.LayerShape()
        gis = [W.group_inputs(80, [120], n_layers=3, shape=s)]
        mode = sr.SR_MODE_SKIP
    else:
        s = W.LayerShape()
        gis = [W.group_inputs(81, [NOALLOC_SPLIT_MAX_TOKENS], n_layers=3, shape=s)]
        mode = sr.SR_MODE_SKIP
    anchors = [gi.anchors.cuda().contiguous() for gi in gis]
    weights = [[DevLayer(lw) for lw in gi.layers] for gi in gis]
    cu = gis[0].cu_seqlens.cuda()
    kw = dict(max_seqlen=max(gis[0].lengths), hidden=s.hidden, inter=s.inter, h_k=s.h_k, h_v=s.h_v,
              d=s.d_k, eps=s.eps, mode=mode, precision=sr.SR_PREC_SPLIT)
    if case == "hidden2560_capacity":
        need = sr.group_workspace_bytes(sr.group_args(anchors, cu, weights, fresh_outputs(gis, mode, s), **kw))
        assert sr.NOALLOC_SCRATCH_BYTES - (1 << 20) < need <= sr.NOALLOC_SCRATCH_BYTES
    ref = sr.group_replay(anchors, cu, weights, want_hidden=True, **kw)
    for call in range(2):  # the second call finds the first call's leftovers in the array
        out = fresh_outputs(gis, mode, s)
        scratch = sr.group_replay_noalloc(anchors, cu, weights, out, **kw)
        torch.cuda.synchronize()
        assert scratch
        for g in range(len(gis)):
            for l in range(len(gis[0].layers)):
                (s1, c1, h1), (s0, c0, h0) = out[g][l], ref[g][l]
                assert torch.equal(s1, s0), f"call {call} group {g} layer {l} state"
                assert torch.equal(c1, c0), f"call {call} group {g} layer {l} conv state"
                if h1 is not None:
                    assert torch.equal(h1, h0), f"call {call} group {g} layer {l} hidden"
        flags = ctypes_status(scratch)
        assert flags == 0


def ctypes_status(scratch_addr):
    import ctypes
    flags = ctypes.c_uint32(0)
    st = sr.library().sr_device_status(ctypes.c_void_p(scratch_addr),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                        ctypes.byref(flags))
    assert st in (sr.SR_OK, sr.SR_ERR_DEVICE)
    return flags.value


def _host_args(T, precision=None):
    """Group arguments with placeholder pointers: enough for the host-side size
    checks, which run before any GPU work."""
    import ctypes
    s = W.LayerShape()
    fake = 0x100000
    L, G = 3, 1
    w_arr = (sr.LayerWeights * (G * L))(*[sr.LayerWeights(*([fake] * 16)) for _ in range(G * L)])
    o_arr = (sr.LayerOutputs * (G * L))(*[sr.LayerOutputs(fake, fake, None) for _ in range(G * L)])
    anc = (ctypes.c_void_p * G)(fake)
    prec = sr.SR_PREC_SPLIT if precision is None else precision
    return sr.GroupArgs(anc, fake, w_arr, o_arr, G, L, 1, T, T, s.hidden, s.inter, s.h_k, s.h_v, 128, 128, 4,
                        1e-6, sr.SR_MODE_SKIP, prec, None)


def test_noalloc_rejects_replays_too_large_for_the_array():
    """A replay whose scratch would exceed the built-in array is refused before
    any GPU work (no device needed for this check)."""
    a = _host_args(4096)  # ~169 KB per token: far beyond 32 MiB
    assert sr.group_workspace_bytes(a) > sr.NOALLOC_SCRATCH_BYTES
    assert sr.group_noalloc_call(a) == sr.SR_ERR_WORKSPACE
    assert "built-in array" in sr.last_error()


def test_noalloc_capacity_edge():
    """The stated capacity at hidden 2560: 191 tokens fit in split precision,
    192 do not and are refused before any GPU work; with the fp8 low pass
    197 fit and 198 do not, in bf16 241 and 242."""
    for prec, fits in ((sr.SR_PREC_SPLIT, NOALLOC_SPLIT_MAX_TOKENS), (sr.SR_PREC_SPLIT_FP8, 197),
                       (sr.SR_PREC_BF16, 241)):
        assert sr.group_workspace_bytes(_host_args(fits, prec)) <= sr.NOALLOC_SCRATCH_BYTES
        too_big = _host_args(fits + 1, prec)
        assert sr.group_workspace_bytes(too_big) > sr.NOALLOC_SCRATCH_BYTES
        assert sr.group_noalloc_call(too_big) == sr.SR_ERR_WORKSPACE
