"""Representative calls of every default kernel path, run against the
bounds-checked library (SR_LIBRARY=libsr_checked.so): every global-memory
index the custom kernels use is checked into the device status word, so a
clean run must end with no SR_DEV_BAD_ACCESS flag and results that still match
the oracle.  Run as a script by tests/test_checked_gpu.py (it exits non-zero on
the first failure); it needs a CUDA device."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import torch  # noqa: E402

import gated_deltanet_state_sr_b200 as sr  # noqa: E402
import oracle  # noqa: E402
import workloads as W  # noqa: E402
from oracle import layers as OL  # noqa: E402
from _util import OUT_TOL_BF16, STATE_TOL, assert_close  # noqa: E402


def flags(ws):
    f = sr.device_status(ws)
    assert f == 0, f"device status 0x{f:x} (0x10: an access outside its buffer)"


def gdn_cases():
    for d in (64, 128):
        x = W.gdn_inputs(77 + d, [1, 2, 0, 3, 64, 65, 127, 200, 0, 129], 2, 4, d, d, h0_std=0.5)
        dv = lambda t: None if t is None else t.cuda().contiguous()
        for algo in ("tcgen05", "tcgen05_fused", "chunked", "sequential"):
            ws = sr.workspace(64 << 20)
            o, s = sr.gdn_replay(dv(x.q), dv(x.k), dv(x.v), dv(x.g), dv(x.beta), dv(x.cu_seqlens),
                                 max_seqlen=x.max_seqlen, h0=dv(x.h0), algo=algo, ws=ws)
            flags(ws)
            o_ref, s_ref = oracle.gdn_replay(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, h0=x.h0)
            assert_close(s, s_ref, STATE_TOL, f"gdn d={d} {algo} state")
            assert_close(o, o_ref, OUT_TOL_BF16, f"gdn d={d} {algo} o")


class DevLayer:
    def __init__(self, lw):
        for f in ("w_in_norm", "w_in", "conv_w", "a_log", "dt_bias", "w_gnorm", "w_out", "w_post_norm",
                  "w_gate", "w_up", "w_down"):
            setattr(self, f, getattr(lw, f).cuda().contiguous())


def group_cases():
    s = W.LayerShape(hidden=256, inter=512, h_k=2, h_v=4, d_k=128, d_v=128)
    gis = [W.group_inputs(31 + g, [5, 1, 0, 70, 130, 2], n_layers=2, shape=s) for g in range(2)]
    anchors = [gi.anchors.cuda().contiguous() for gi in gis]
    cu = gis[0].cu_seqlens.cuda()
    for prec in (sr.SR_PREC_SPLIT, sr.SR_PREC_SPLIT_FP8, sr.SR_PREC_BF16):
        for mode, name in ((sr.SR_MODE_FULL, "full"), (sr.SR_MODE_SKIP, "skip")):
            weights = [[DevLayer(lw) for lw in gi.layers] for gi in gis]
            if prec == sr.SR_PREC_SPLIT_FP8:
                for row in weights:
                    for lw in row:
                        sr.attach_lo8(lw)
            kw = dict(max_seqlen=130, hidden=s.hidden, inter=s.inter, h_k=s.h_k, h_v=s.h_v, d=s.d_k, eps=s.eps,
                      mode=mode, precision=prec)
            ws = sr.workspace(256 << 20)
            out = sr.group_replay(anchors, cu, weights, want_hidden=True, ws=ws, **kw)
            flags(ws)
            if prec != sr.SR_PREC_BF16:
                ref = OL.group_replay(gis[1], name)
                for l in range(2):
                    assert_close(out[1][l][0], ref[l]["S"], STATE_TOL, f"group {prec} {name} layer {l} state")


def mamba2_cases():
    m = W.mamba2_inputs(17, [1, 0, 63, 64, 65, 300], H=4, h0_std=0.3)
    dv = lambda t: None if t is None else t.cuda().contiguous()
    for algo in ("tcgen05", "chunked", "sequential"):
        ws = sr.workspace(64 << 20)
        y, s = sr.mamba2_replay(dv(m.x), dv(m.B), dv(m.C), dv(m.dt), dv(m.A), dv(m.cu_seqlens), max_seqlen=300,
                                h0=dv(m.h0), algo=algo, ws=ws)
        flags(ws)
        y_ref, s_ref = oracle.mamba2_replay(m.x, m.B, m.C, m.dt, m.A, m.cu_seqlens, h0=m.h0)
        assert_close(s, s_ref, STATE_TOL, f"mamba2 {algo} state")
        assert_close(y, y_ref, OUT_TOL_BF16, f"mamba2 {algo} y")


if __name__ == "__main__":
    assert sr.CHECKED, "run with SR_LIBRARY=libsr_checked.so"
    gdn_cases()
    group_cases()
    mamba2_cases()
    torch.cuda.synchronize()
    print("checked build: every case clean")
