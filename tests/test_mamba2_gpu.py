"""GPU parity of sr_mamba2_replay against the fp64 oracle.

Full-size Mamba2 workload (64 varlen suffixes of U{256..4096} tokens, 64
heads, P=64, N=128) on sampled (sequence, head) units that the oracle computes
one by one, plus a small case checked everywhere and edge lengths, for each
kernel: the tcgen05 chunk kernel (the default), the mma.sync chunk kernel and
the fp32 token-by-token kernel."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from _util import OUT_TOL_BF16, STATE_TOL, assert_close

pytestmark = pytest.mark.gpu

ALGOS = ["tcgen05", "chunked"]


@pytest.fixture(scope="module")
def sr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_deltanet_state_sr_b200 as m
    return m


def run_gpu(sr, m: W.Mamba2Inputs, algo="auto"):
    d = lambda a: None if a is None else a.cuda().contiguous()
    y, s = sr.mamba2_replay(d(m.x), d(m.B), d(m.C), d(m.dt), d(m.A), d(m.cu_seqlens),
                            max_seqlen=max(m.max_seqlen, 1), h0=d(m.h0), algo=algo)
    torch.cuda.synchronize()
    return y, s


@pytest.mark.parametrize("algo", ALGOS + ["sequential"])
def test_small_case(sr, algo):
    m = W.mamba2_inputs(21, [1, 2, 0, 63, 64, 65, 300, 128], H=8, h0_std=0.2)
    y, s = run_gpu(sr, m, algo)
    y_ref, s_ref = oracle.mamba2_replay(m.x, m.B, m.C, m.dt, m.A, m.cu_seqlens, h0=m.h0)
    assert_close(s, s_ref, STATE_TOL, "state")
    assert_close(y, y_ref, OUT_TOL_BF16, "y")
    np.testing.assert_array_equal(s[2].cpu().numpy(), m.h0[2].numpy())


@pytest.mark.parametrize("algo", ALGOS)
def test_full_workload_sampled_units(sr, algo):
    m = W.mamba2()
    y, s = run_gpu(sr, m, algo)
    H = 64
    rng = np.random.default_rng(0)
    seqs = rng.choice(64, 6, replace=False)
    units = [int(n) * H + int(h) for n in seqs for h in rng.choice(H, 2, replace=False)]
    y_ref, s_ref = oracle.mamba2_replay(m.x, m.B, m.C, m.dt, m.A, m.cu_seqlens, units=units)
    cu = m.cu_seqlens.tolist()
    for u in units:
        n, h = divmod(u, H)
        assert_close(s[n, h], s_ref[n, h], STATE_TOL, f"state seq {n} head {h}")
        assert_close(y[cu[n]:cu[n + 1], h], y_ref[cu[n]:cu[n + 1], h], OUT_TOL_BF16,
                     f"y seq {n} head {h}")
    assert torch.isfinite(s).all() and torch.isfinite(y.float()).all()


@pytest.mark.parametrize("H,G", [(3, 1), (4, 2)])
def test_sequential_fallback_shapes(sr, H, G):
    """Several B/C groups or an odd head count take the token-by-token kernel."""
    m = W.mamba2_inputs(22, [9, 0, 130], H=H, G=G, h0_std=0.1)
    y, s = run_gpu(sr, m)
    y_ref, s_ref = oracle.mamba2_replay(m.x, m.B, m.C, m.dt, m.A, m.cu_seqlens, h0=m.h0)
    assert_close(s, s_ref, STATE_TOL, "state")
    assert_close(y, y_ref, OUT_TOL_BF16, "y")


@pytest.mark.parametrize("algo", ALGOS)
def test_state_only_and_strong_decay(sr, algo):
    m = W.mamba2_inputs(23, [200, 64, 1], H=4)
    m.A = m.A * 8.0  # dt A down to ~ -60 per token: exp(gamma) leaves the fp32 range inside a chunk
    d = lambda a: None if a is None else a.cuda().contiguous()
    _, s = sr.mamba2_replay(d(m.x), d(m.B), d(m.C), d(m.dt), d(m.A), d(m.cu_seqlens), max_seqlen=200,
                            want_y=False, algo=algo)
    torch.cuda.synchronize()
    _, s_ref = oracle.mamba2_replay(m.x, m.B, m.C, m.dt, m.A, m.cu_seqlens, want_y=False)
    assert_close(s, s_ref, STATE_TOL, "state")


@pytest.mark.parametrize("algo", ALGOS)
def test_exact_resume_on_gpu(sr, algo):
    """Continuation from a replayed state: Replay(a || b) = Replay(b, h0 = Replay(a))."""
    T, j = 250, 90
    m = W.mamba2_inputs(24, [T], H=4)
    d = lambda a: a.cuda().contiguous()
    y, s = sr.mamba2_replay(d(m.x), d(m.B), d(m.C), d(m.dt), d(m.A), d(m.cu_seqlens), max_seqlen=T, algo=algo)
    cu = lambda n: torch.tensor([0, n], dtype=torch.int32, device="cuda")
    _, sa = sr.mamba2_replay(d(m.x[:j]), d(m.B[:j]), d(m.C[:j]), d(m.dt[:j]), d(m.A), cu(j), max_seqlen=j,
                             algo=algo)
    yb, sb = sr.mamba2_replay(d(m.x[j:]), d(m.B[j:]), d(m.C[j:]), d(m.dt[j:]), d(m.A), cu(T - j),
                              max_seqlen=T - j, h0=sa, algo=algo)
    torch.cuda.synchronize()
    assert_close(sb, s.double().cpu().numpy(), STATE_TOL, "resumed state")
    assert_close(yb, y[j:].double().cpu().numpy(), OUT_TOL_BF16, "resumed outputs")


def test_replay_call_captures_in_a_cuda_graph(sr):
    """As for the gated-delta call: captured in a CUDA graph, the Mamba2 replay
    gives the eager call's results bit for bit."""
    m = W.mamba2_inputs(23, [300, 65, 1, 128], H=8, h0_std=0.2)
    d = lambda a: a.cuda().contiguous()
    x, B, C, dt, A, cu, h0 = map(d, (m.x, m.B, m.C, m.dt, m.A, m.cu_seqlens, m.h0))
    y, s = torch.empty_like(x), torch.empty(4, 8, x.shape[2], B.shape[2], dtype=torch.float32, device="cuda")
    args = sr.mamba2_args(x, B, C, dt, A, cu, n_seqs=4, max_seqlen=m.max_seqlen, h0=h0, y=y, s_out=s)
    ws = sr.workspace(sr.mamba2_workspace_bytes(args))
    call = lambda: sr.mamba2_replay(x, B, C, dt, A, cu, max_seqlen=m.max_seqlen, h0=h0, y=y, s_out=s, ws=ws)
    call()
    torch.cuda.synchronize()
    y_eager, s_eager = y.clone(), s.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    y.zero_()
    s.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y_eager) and torch.equal(s, s_eager)
