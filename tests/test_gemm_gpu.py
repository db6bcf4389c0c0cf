"""GPU parity of the tcgen05 projection GEMM (sr_test_gemm) against fp64.

The GEMM carries every dense projection of the replay group (in_proj,
out_proj + residual, SwiGLU gate/up, down + residual); it is checked on its
own here, at the group's full shapes (T = 1638 rows: ragged last M tile;
N = 12352: ragged last N tile) and on small ragged shapes."""
import numpy as np
import pytest
import torch

import workloads as W
from _util import OUT_TOL_BF16, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_deltanet_state_sr_b200 as m
    return m


def f64(t):
    return t.double().cpu().numpy()


def silu(x):
    return x / (1.0 + np.exp(-x))


@pytest.mark.parametrize("m,n,k", [(1, 32, 64), (130, 96, 128), (257, 544, 192), (1638, 12352, 2560)])
def test_store(sr, m, n, k):
    a = W.normal(1, "a", (m, k)).cuda()
    b = W.normal(1, "b", (n, k), 0.02).cuda()
    c = sr.test_gemm(a, b)
    torch.cuda.synchronize()
    assert_close(c, f64(a) @ f64(b).T, OUT_TOL_BF16, "a b^T")


@pytest.mark.parametrize("m,n,k", [(70, 64, 64), (1638, 2560, 4096)])
def test_residual(sr, m, n, k):
    a = W.normal(2, "a", (m, k)).cuda()
    b = W.normal(2, "b", (n, k), 0.02).cuda()
    r = W.normal(2, "r", (m, n)).cuda()
    c = sr.test_gemm(a, b, r=r, epi=sr.EPI_RESIDUAL)
    torch.cuda.synchronize()
    assert_close(c, f64(r) + f64(a) @ f64(b).T, OUT_TOL_BF16, "r + a b^T")


def test_residual_in_place(sr):
    m, n, k = 300, 256, 320
    a = W.normal(3, "a", (m, k)).cuda()
    b = W.normal(3, "b", (n, k), 0.02).cuda()
    x = W.normal(3, "x", (m, n)).cuda()
    ref = f64(x) + f64(a) @ f64(b).T
    sr.test_gemm(a, b, r=x, c=x, epi=sr.EPI_RESIDUAL)
    torch.cuda.synchronize()
    assert_close(x, ref, OUT_TOL_BF16, "x += a b^T")


@pytest.mark.parametrize("m,n,k", [(5, 128, 64), (1638, 9216, 2560)])
def test_swiglu(sr, m, n, k):
    a = W.normal(4, "a", (m, k)).cuda()
    bg = W.normal(4, "bg", (n, k), 0.02).cuda()
    bu = W.normal(4, "bu", (n, k), 0.02).cuda()
    c = sr.test_gemm(a, bg, b1=bu, epi=sr.EPI_SWIGLU)
    torch.cuda.synchronize()
    A = f64(a)
    ref = silu(A @ f64(bg).T) * (A @ f64(bu).T)
    assert_close(c, ref, OUT_TOL_BF16, "SiLU(a bg^T) * (a bu^T)")
    ws = sr.workspace(256)
    sr.test_gemm(a, bg, b1=bu, epi=sr.EPI_SWIGLU, ws=ws)
    assert sr.device_status(ws) == 0


@pytest.mark.parametrize("epi,m,n,k", [
    ("store", 130, 96, 128),      # one pair tile, the odd CTA's rows past m
    ("store", 64, 256, 128),      # one pair tile, the odd CTA's rows all past m
    ("store", 257, 544, 192),     # ragged M across two pair tiles, ragged N
    ("residual", 300, 352, 320),  # residual epilogue, ragged N in the odd CTA's half
    ("swiglu", 5, 128, 64),       # gate rows in the even CTA, up rows in the odd one
    ("swiglu", 1638, 9216, 2560),
    ("store", 1638, 12352, 2560),
])
def test_cta_pair_form_is_bit_identical_to_single_cta_form(sr, epi, m, n, k):
    """Both forms run the same K blocks in the same order into fp32 tensor
    memory, so every output element must come out bit-identical; the pair
    form is also checked against fp64 like the default path above."""
    a = W.normal(6, "a", (m, k)).cuda()
    b0 = W.normal(6, "b0", (n, k), 0.02).cuda()
    b1 = W.normal(6, "b1", (n, k), 0.02).cuda() if epi == "swiglu" else None
    r = W.normal(6, "r", (m, n)).cuda() if epi == "residual" else None
    e = {"store": sr.EPI_STORE, "residual": sr.EPI_RESIDUAL, "swiglu": sr.EPI_SWIGLU}[epi]
    out = {}
    for form in (sr.GEMM_FORM_SINGLE, sr.GEMM_FORM_PAIR):
        ws = sr.workspace(256)
        out[form] = sr.test_gemm(a, b0, b1=b1, r=r, epi=e, ws=ws, form=form)
        assert sr.device_status(ws) == 0
    torch.cuda.synchronize()
    assert torch.equal(out[sr.GEMM_FORM_SINGLE], out[sr.GEMM_FORM_PAIR])
    A = f64(a)
    if epi == "swiglu":
        ref = silu(A @ f64(b0).T) * (A @ f64(b1).T)
    else:
        ref = A @ f64(b0).T + (f64(r) if r is not None else 0.0)
    assert_close(out[sr.GEMM_FORM_PAIR], ref, OUT_TOL_BF16, f"pair form, {epi}")
