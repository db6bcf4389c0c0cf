"""Host-side tests of the C ABI (no GPU needed, no kernel launched).

The library must load, export every entry point ``include/sr/sr.h`` declares,
and reject bad arguments during host validation -- before any CUDA call."""
import ctypes

import pytest

sr = pytest.importorskip("gated_deltanet_state_sr_b200")

FAKE = 0x10000  # an aligned, never-dereferenced address: validation fails first


def test_exports_every_declared_symbol():
    import glob
    import os
    headers = sorted(glob.glob(os.path.join(os.path.dirname(sr.HEADER_PATH), "*.h")))
    assert len(headers) >= 2
    names = sorted({n for h in headers for n in sr.declared_symbols(h)})
    assert {"sr_gdn_replay", "sr_group_replay", "sr_mamba2_replay", "sr_last_error", "sr_device_status",
            "sr_group_replay_noalloc", "sr_test_gemm", "sr_test_wait_timeout"} <= set(names)
    for n in names:
        assert hasattr(sr.library(), n), f"libsr.so does not export {n}"


def test_checked_build_exports_the_same_entry_points():
    """The bounds-checked build (libsr_checked.so) is built beside libsr.so and
    exports every entry point the headers declare."""
    import ctypes as C
    import glob
    import os
    lib = C.CDLL(os.path.join(os.path.dirname(sr.LIB_PATH), "libsr_checked.so"))
    for h in glob.glob(os.path.join(os.path.dirname(sr.HEADER_PATH), "*.h")):
        for n in sr.declared_symbols(h):
            assert hasattr(lib, n), n


def test_wait_timeout_validation():
    """The test-only bounded-wait entry point refuses a zero limit, a limit
    above the kernels' own, and a missing workspace, before any CUDA call."""
    assert sr.test_wait_call(0) == sr.SR_ERR_INVALID_ARG
    assert sr.test_wait_call(sr.WAIT_LIMIT_NS + 1) == sr.SR_ERR_INVALID_ARG
    assert sr.test_wait_call(10_000) == sr.SR_ERR_WORKSPACE


def test_version():
    assert sr.version() == 0x000100


def _gdn(**kw):
    a = sr.GdnArgs(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, cu_seqlens=FAKE, h0=None, o=FAKE,
                   s_out=FAKE, dtype=sr.SR_BF16, algo=sr.SR_GDN_AUTO, n_seqs=2, total_tokens=100,
                   max_seqlen=60, h_k=2, h_v=4, d_k=64, d_v=64, scale=0.0)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("field,value,status", [
    ("q", None, sr.SR_ERR_INVALID_ARG),
    ("s_out", None, sr.SR_ERR_INVALID_ARG),
    ("cu_seqlens", None, sr.SR_ERR_INVALID_ARG),
    ("h_v", 5, sr.SR_ERR_INVALID_ARG),          # h_v % h_k != 0
    ("h_k", 0, sr.SR_ERR_INVALID_ARG),
    ("d_k", 96, sr.SR_ERR_UNSUPPORTED),
    ("d_v", 128, sr.SR_ERR_UNSUPPORTED),        # d_k != d_v
    ("n_seqs", -1, sr.SR_ERR_INVALID_ARG),
    ("max_seqlen", 101, sr.SR_ERR_INVALID_ARG),  # longer than total
    ("dtype", 7, sr.SR_ERR_INVALID_ARG),
    ("algo", 9, sr.SR_ERR_INVALID_ARG),
    ("s_out", FAKE + 4, sr.SR_ERR_INVALID_ARG),  # misaligned
    ("scale", float("nan"), sr.SR_ERR_INVALID_ARG),
])
def test_gdn_validation(field, value, status):
    a = _gdn(**{field: value})
    assert sr.gdn_workspace_bytes(a) == 0
    assert sr.gdn_call(a, None) == status
    assert sr.last_error() != ""


def test_gdn_chunked_requires_bf16():
    a = _gdn(dtype=sr.SR_FP32, algo=sr.SR_GDN_CHUNKED)
    assert sr.gdn_call(a, None) == sr.SR_ERR_UNSUPPORTED


def test_gdn_workspace_required():
    a = _gdn()
    need = sr.gdn_workspace_bytes(a)
    assert need >= 256
    assert sr.gdn_call(a, None) == sr.SR_ERR_WORKSPACE
    assert "workspace" in sr.last_error()


def test_gdn_two_phase_workspace_holds_the_chunk_images():
    """The default tcgen05 form keeps one 56.5 KB chunk image per (chunk slot, V
    head), with floor(T / 64) + n_seqs slots, at d = 128 and at d = 64 alike;
    the fused form and the other kernels need only the 256-byte header."""
    kw = dict(d_k=128, d_v=128, h_k=16, h_v=32, n_seqs=8, total_tokens=8917, max_seqlen=2048)
    slots = 8917 // 64 + 8
    want = 256 + slots * 32 * 57856
    assert sr.gdn_workspace_bytes(_gdn(**kw)) == want
    assert sr.gdn_workspace_bytes(_gdn(algo=sr.SR_GDN_TCGEN05, **kw)) == want
    assert sr.gdn_workspace_bytes(_gdn(algo=sr.SR_GDN_TCGEN05_FUSED, **kw)) == 256
    assert sr.gdn_workspace_bytes(_gdn(algo=sr.SR_GDN_SEQUENTIAL, **kw)) == 256
    # d = 64 (100 tokens, 2 sequences, 4 V heads) takes the two-phase form too
    assert sr.gdn_workspace_bytes(_gdn()) == 256 + (100 // 64 + 2) * 4 * 57856
    assert sr.gdn_workspace_bytes(_gdn(algo=sr.SR_GDN_CHUNKED)) == 256
    assert sr.gdn_workspace_bytes(_gdn(algo=sr.SR_GDN_TCGEN05_FUSED)) == 256
    # the tcgen05 forms take bf16 only
    assert sr.gdn_workspace_bytes(_gdn(algo=sr.SR_GDN_TCGEN05_FUSED, dtype=sr.SR_FP32, **kw)) == 0


def test_group_workspace_holds_the_chunk_images():
    """A replay group's workspace grows by the chunk images of its gated-delta
    layers: 56.5 KB per (group, chunk slot, V head)."""
    a16, a80 = _fake_group_args(total_tokens=16, max_seqlen=16), _fake_group_args(total_tokens=80, max_seqlen=80)
    grow = sr.group_workspace_bytes(a80) - sr.group_workspace_bytes(a16)
    # 64 more tokens: one more slot (80 // 64 - 16 // 64) of 4 V heads, plus the per-token buffers
    assert grow >= 1 * 4 * 57856


def test_gdn_workspace_too_small_and_misaligned():
    import torch
    a = _gdn()
    lib = sr.library()
    small = ctypes.c_void_p(FAKE)
    st = lib.sr_gdn_replay(ctypes.byref(a), small, 16, None)
    assert st == sr.SR_ERR_WORKSPACE and "too small" in sr.last_error()
    st = lib.sr_gdn_replay(ctypes.byref(a), ctypes.c_void_p(FAKE + 16), 1 << 30, None)
    assert st == sr.SR_ERR_WORKSPACE and "aligned" in sr.last_error()


def _m2(**kw):
    a = sr.Mamba2Args(x=FAKE, B=FAKE, C=FAKE, dt=FAKE, A=FAKE, cu_seqlens=FAKE, h0=None, y=FAKE,
                      s_out=FAKE, n_seqs=3, total_tokens=50, max_seqlen=40, n_heads=8, head_dim=64,
                      n_groups=1, d_state=128)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("field,value,status", [
    ("x", None, sr.SR_ERR_INVALID_ARG),
    ("n_groups", 3, sr.SR_ERR_INVALID_ARG),
    ("head_dim", 32, sr.SR_ERR_UNSUPPORTED),
    ("d_state", 64, sr.SR_ERR_UNSUPPORTED),
    ("total_tokens", -5, sr.SR_ERR_INVALID_ARG),
])
def test_mamba2_validation(field, value, status):
    a = _m2(**{field: value})
    assert sr.mamba2_workspace_bytes(a) == 0
    assert sr.mamba2_call(a, None) == status


def test_mamba2_workspace_required():
    a = _m2()
    assert sr.mamba2_workspace_bytes(a) >= 256
    assert sr.mamba2_call(a, None) == sr.SR_ERR_WORKSPACE


def test_device_status_needs_workspace():
    flags = ctypes.c_uint32(0)
    st = sr.library().sr_device_status(None, None, ctypes.byref(flags))
    assert st == sr.SR_ERR_INVALID_ARG


def test_ctypes_structs_match_the_c_header(tmp_path):
    """The binding's ctypes structs have the C header's sizes and field offsets
    (compiled here with gcc from include/sr/sr.h)."""
    import os
    import subprocess
    structs = {"sr_gdn_args": sr.GdnArgs, "sr_mamba2_args": sr.Mamba2Args,
               "sr_layer_weights": sr.LayerWeights, "sr_layer_outputs": sr.LayerOutputs,
               "sr_group_args": sr.GroupArgs, "sr_profile": sr.Profile, "sr_layer_state": sr.LayerState,
               "sr_capture_args": sr.CaptureArgs, "sr_anchor_plan_args": sr.AnchorPlanArgs}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "sr/sr.h"', 'int main(void) {']
    for cname, py in structs.items():
        lines.append(f'printf("{cname} %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            lines.append(f'printf("{cname}.{f} %zu\\n", offsetof({cname}, {f}));')
    lines.append("return 0; }")
    src = tmp_path / "abi.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "abi"
    inc = os.path.join(os.path.dirname(sr.HEADER_PATH), "..")
    subprocess.run(["gcc", "-I", inc, str(src), "-o", str(exe)], check=True)
    out = dict(l.split() for l in subprocess.run([str(exe)], capture_output=True, text=True,
                                                 check=True).stdout.splitlines())
    for cname, py in structs.items():
        assert int(out[cname]) == ctypes.sizeof(py), cname
        for f, _ in py._fields_:
            assert int(out[f"{cname}.{f}"]) == getattr(py, f).offset, f"{cname}.{f}"


def _fake_group_args(**over):
    """A GroupArgs over fake (never dereferenced) device pointers: host
    validation runs before any CUDA work, so no GPU is needed."""
    fake = 0x10000
    anc = (ctypes.c_void_p * 1)(fake)
    w = (sr.LayerWeights * 1)(sr.LayerWeights(*([fake] * 11)))
    o = (sr.LayerOutputs * 1)(sr.LayerOutputs(fake, fake, None))
    a = sr.GroupArgs(anc, fake, w, o, 1, 1, 1, 16, 16, 256, 512, 2, 4, 128, 128, 4, 1e-6, sr.SR_MODE_SKIP, 0,
                     None, None, None, 0)
    for k, v in over.items():
        setattr(a, k, v)
    a._keep = (anc, w, o)
    return a


def test_group_sparse_anchors_need_pool_rows():
    a = _fake_group_args(anchor_index=0x20000, anchor_rows=0)
    assert sr.group_workspace_bytes(a) == 0
    assert sr.group_call(a, None) == sr.SR_ERR_INVALID_ARG
    assert "anchor_rows" in sr.last_error()
    a = _fake_group_args(anchor_index=0x20000, anchor_rows=5)
    assert sr.group_workspace_bytes(a) > 0


def test_group_workspace_independent_of_continuation():
    """Initial states are read in place: a continuation needs no extra scratch."""
    init = (sr.LayerState * 1)(sr.LayerState(0x30000, 0x40000))
    assert sr.group_workspace_bytes(_fake_group_args(initial=init)) == sr.group_workspace_bytes(_fake_group_args())


def test_prepare_lo8_validation_runs_without_a_gpu():
    f = sr.library().sr_prepare_lo8_weights
    assert f(ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000), ctypes.c_int64(-1), None) == sr.SR_ERR_INVALID_ARG
    assert f(None, ctypes.c_void_p(0x20000), ctypes.c_int64(8), None) == sr.SR_ERR_INVALID_ARG
    assert f(None, None, ctypes.c_int64(0), None) == sr.SR_OK


def test_group_fp8_low_pass_needs_its_weights_and_shapes():
    a = _fake_group_args(precision=sr.SR_PREC_SPLIT_FP8)
    assert sr.group_call(a, None) == sr.SR_ERR_INVALID_ARG
    assert "low-pass weights" in sr.last_error()
    w = a._keep[1]
    for f in sr.LO8_FIELDS:
        setattr(w[0], f, 0x50000)
    assert sr.group_workspace_bytes(a) > 0
    a.hidden = 192  # a multiple of 64 but not of 128
    assert sr.group_call(a, None) == sr.SR_ERR_UNSUPPORTED
