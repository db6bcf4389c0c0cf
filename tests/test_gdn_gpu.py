"""GPU parity of sr_gdn_replay against the fp64 oracle (same seeded inputs).

Covers the raw-replay workloads at full size (one GDN layer, 1 x 256 tokens at
2/4 heads d=64, and 8 varlen suffixes of U{512..2048} tokens at 16/32 heads
d=128), plus edge cases: length-1 and length-2 sequences, empty sequences,
ragged chunk tails, a nonzero initial state, strong decay, state-only mode,
the fp32-input mode and device-side rejection of bad cu_seqlens."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from _util import OUT_TOL_BF16, STATE_TOL, TOL_FP32, assert_close

pytestmark = pytest.mark.gpu

ALGOS = ["sequential", "chunked", "tcgen05", "tcgen05_fused"]


@pytest.fixture(scope="module")
def sr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_deltanet_state_sr_b200 as m
    return m


def run_gpu(sr, x: W.GdnInputs, algo, want_o=True, dev="cuda"):
    t = lambda a: None if a is None else a.to(dev).contiguous()
    o, s = sr.gdn_replay(t(x.q), t(x.k), t(x.v), t(x.g), t(x.beta), t(x.cu_seqlens),
                         max_seqlen=max(x.max_seqlen, 1), h0=t(x.h0), want_o=want_o, algo=algo)
    torch.cuda.synchronize()
    return o, s


def run_oracle(x: W.GdnInputs, want_o=True, units=None):
    return oracle.gdn_replay(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, h0=x.h0, want_o=want_o,
                             units=units)


@pytest.mark.parametrize("algo", ALGOS)
def test_raw_small_workload(sr, algo):
    x = W.raw_small()
    o, s = run_gpu(sr, x, algo)
    o_ref, s_ref = run_oracle(x)
    assert_close(s, s_ref, STATE_TOL, "state")
    assert_close(o, o_ref, OUT_TOL_BF16, "o")


@pytest.mark.parametrize("algo", ALGOS)
def test_raw_qwen_workload_full_size(sr, algo):
    x = W.raw_qwen()
    o, s = run_gpu(sr, x, algo)
    o_ref, s_ref = run_oracle(x)
    assert_close(s, s_ref, STATE_TOL, "state")
    assert_close(o, o_ref, OUT_TOL_BF16, "o")
    # per-sequence state check, so one good long sequence cannot hide a bad short one
    for n in range(x.n_seqs):
        assert_close(s[n], s_ref[n], STATE_TOL, f"state seq {n}")


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("d", [64, 128])
def test_edge_lengths_with_initial_state(sr, algo, d):
    lengths = [1, 2, 0, 3, 64, 65, 127, 200, 0, 129]
    x = W.gdn_inputs(77 + d, lengths, 2, 4, d, d, h0_std=0.5)
    o, s = run_gpu(sr, x, algo)
    o_ref, s_ref = run_oracle(x)
    for n in range(len(lengths)):
        assert_close(s[n], s_ref[n], STATE_TOL, f"state seq {n} (len {lengths[n]})")
    assert_close(o, o_ref, OUT_TOL_BF16, "o")
    # empty sequences return their initial state
    np.testing.assert_array_equal(s[2].cpu().numpy(), x.h0[2].numpy())


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("d", [64, 128])
def test_strong_decay(sr, algo, d):
    """Gates of the group workload: g down to about -11 per token, so the
    cumulative decay over a chunk leaves the fp32 exp range."""
    x = W.gdn_inputs(5, [300, 77], 2, 4, d, d, g_range=(-12.0, -0.5), norm_q=True)
    o, s = run_gpu(sr, x, algo)
    o_ref, s_ref = run_oracle(x)
    assert_close(s, s_ref, STATE_TOL, "state")
    assert_close(o, o_ref, OUT_TOL_BF16, "o")


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("d", [64, 128])
def test_decay_around_the_factorisation_bound(sr, algo, d):
    """g ~ U(-2.6, -0.001): a chunk's decay e^{gamma_C} lands on both sides of
    e^{-80}, so one sequence mixes chunks whose masks the tcgen05 kernels form as
    e^{gamma_t} e^{-gamma_s} with chunks that take an exponential per masked
    difference (23 and 17 of the 40 (chunk, head) pairs here); q not normalised."""
    x = W.gdn_inputs(9, [300, 77, 130], 2, 4, d, d, g_range=(-2.6, -0.001), norm_q=False, h0_std=0.2)
    o, s = run_gpu(sr, x, algo)
    o_ref, s_ref = run_oracle(x)
    assert_close(s, s_ref, STATE_TOL, "state")
    assert_close(o, o_ref, OUT_TOL_BF16, "o")


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("d", [64, 128])
def test_state_only_mode(sr, algo, d):
    x = W.gdn_inputs(6, [150, 40], 2, 4, d, d)
    o, s = run_gpu(sr, x, algo, want_o=False)
    assert o is None
    _, s_ref = run_oracle(x, want_o=False)
    assert_close(s, s_ref, STATE_TOL, "state")


def test_fp32_input_mode(sr):
    x = W.gdn_inputs(8, [1, 70, 333], 2, 4, 128, 128, dtype=torch.float32, h0_std=0.3)
    o, s = run_gpu(sr, x, "auto")
    assert o.dtype == torch.float32
    o_ref, s_ref = run_oracle(x)
    assert_close(s, s_ref, TOL_FP32, "state (fp32 mode)")
    assert_close(o, o_ref, TOL_FP32, "o (fp32 mode)")


def test_fp32_input_mode_full_size(sr):
    """The fp32-input mode at the 8-suffix workload's full size (the same values
    as fp32 q, k, v; 16/32 heads, d = 128): states and outputs within the fp32
    tolerance, every sequence on its own."""
    x = W.raw_qwen()
    x.q, x.k, x.v = x.q.float(), x.k.float(), x.v.float()
    o, s = run_gpu(sr, x, "auto")
    assert o.dtype == torch.float32
    o_ref, s_ref = run_oracle(x)
    assert_close(o, o_ref, TOL_FP32, "o (fp32 mode)")
    for n in range(x.n_seqs):
        assert_close(s[n], s_ref[n], TOL_FP32, f"state seq {n} (fp32 mode)")


@pytest.mark.parametrize("algo", ALGOS)
def test_bad_cu_seqlens_flagged_on_device(sr, algo):
    """A decreasing cu_seqlens entry is caught by the kernel's own bounds check:
    that sequence is skipped (its output untouched) and a flag is recorded."""
    x = W.gdn_inputs(9, [10, 10, 10], 2, 4, 128, 128)
    dev = lambda a: a.cuda().contiguous()
    cu = torch.tensor([0, 10, 5, 30], dtype=torch.int32, device="cuda")  # seq 1 runs backwards
    s_out = torch.full((3, 4, 128, 128), 7.0, device="cuda")
    ws = sr.workspace(1 << 20)
    sr.gdn_replay(dev(x.q), dev(x.k), dev(x.v), dev(x.g), dev(x.beta), cu, max_seqlen=25,
                  s_out=s_out, want_o=False, algo=algo, ws=ws)
    flags = sr.device_status(ws)
    assert flags & sr.SR_DEV_BAD_CU_SEQLENS
    assert torch.all(s_out[1] == 7.0)
    # too-long sequence against max_seqlen
    cu = x.cu_seqlens.cuda()
    sr.gdn_replay(dev(x.q), dev(x.k), dev(x.v), dev(x.g), dev(x.beta), cu, max_seqlen=5,
                  s_out=s_out, want_o=False, algo=algo, ws=ws)
    assert sr.device_status(ws) & sr.SR_DEV_SEQ_TOO_LONG
    # and a good call clears the word
    sr.gdn_replay(dev(x.q), dev(x.k), dev(x.v), dev(x.g), dev(x.beta), cu, max_seqlen=10,
                  s_out=s_out, want_o=False, algo=algo, ws=ws)
    assert sr.device_status(ws) == 0


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("split_at", [64, 100])
@pytest.mark.parametrize("dh", [64, 128])
def test_exact_resume_on_gpu(sr, algo, split_at, dh):
    """Continuation: replaying b from h0 = Replay(a) gives Replay(a || b) ("Sparse
    Prefix Caching for Hybrid and Recurrent LLM Serving", exactness of resume; the
    replayed state hands over to the continuing tokens).  Split on and off a chunk
    boundary."""
    T = 300
    x = W.gdn_inputs(15, [T], 2, 4, dh, dh)
    d = lambda a: a.cuda().contiguous()
    full_o, full_s = sr.gdn_replay(d(x.q), d(x.k), d(x.v), d(x.g), d(x.beta), d(x.cu_seqlens), max_seqlen=T,
                                   algo=algo)
    cu_a = torch.tensor([0, split_at], dtype=torch.int32, device="cuda")
    cu_b = torch.tensor([0, T - split_at], dtype=torch.int32, device="cuda")
    sl = lambda t, a, b: d(t[a:b])
    _, s_a = sr.gdn_replay(sl(x.q, 0, split_at), sl(x.k, 0, split_at), sl(x.v, 0, split_at),
                           sl(x.g, 0, split_at), sl(x.beta, 0, split_at), cu_a, max_seqlen=split_at, algo=algo)
    o_b, s_b = sr.gdn_replay(sl(x.q, split_at, T), sl(x.k, split_at, T), sl(x.v, split_at, T),
                             sl(x.g, split_at, T), sl(x.beta, split_at, T), cu_b, max_seqlen=T - split_at,
                             h0=s_a, algo=algo)
    torch.cuda.synchronize()
    ref = full_s.double().cpu().numpy()
    assert_close(s_b, ref, STATE_TOL, "resumed state vs full replay")
    assert_close(o_b, full_o[split_at:].double().cpu().numpy(), OUT_TOL_BF16, "resumed outputs")


def test_two_phase_matches_fused(sr):
    """The two-phase tcgen05 form (state-free chunk work for all chunks first,
    then the state chain) forms the same products as the fused kernel; only the
    order in which S (-W)^T and V^T T2^T enter the fp32 accumulator of U differs.
    That moves a few bf16 roundings of the state copy, which the recurrence
    carries on: the two agree far inside the tolerance each meets against the
    oracle (a tenth of it here)."""
    x = W.raw_qwen()
    o2, s2 = run_gpu(sr, x, "tcgen05")
    o1, s1 = run_gpu(sr, x, "tcgen05_fused")
    assert_close(s2, s1.double().cpu().numpy(), STATE_TOL / 10, "state, two-phase vs fused")
    assert_close(o2, o1.double().cpu().numpy(), OUT_TOL_BF16 / 2, "o, two-phase vs fused")


def test_default_path_at_d64_is_tcgen05(sr):
    """The small raw workload (d = 64) runs the tcgen05 two-phase kernels by
    default, on 128-wide tiles whose upper halves stay zero: it agrees with the
    explicitly selected two-phase form bit for bit and with the mma.sync chunk
    kernel to a small fraction of the oracle tolerance."""
    x = W.raw_small()
    o0, s0 = run_gpu(sr, x, "auto")
    o1, s1 = run_gpu(sr, x, "tcgen05")
    o2, s2 = run_gpu(sr, x, "chunked")
    assert torch.equal(s0, s1) and torch.equal(o0, o1)
    assert_close(s1, s2.double().cpu().numpy(), STATE_TOL / 4, "state, tcgen05 vs mma.sync")


@pytest.mark.parametrize("algo", ["tcgen05", "tcgen05_fused"])
@pytest.mark.parametrize("d", [64, 128])
def test_many_short_sequences(sr, algo, d):
    """More sequences than the longest-first ranking handles (300), lengths
    0..140 with empty ones between: every chunk finds its image slot."""
    gen = torch.Generator().manual_seed(31)
    lengths = torch.randint(0, 141, (300,), generator=gen).tolist()
    for i in range(0, 300, 37):
        lengths[i] = 0
    x = W.gdn_inputs(31, lengths, 1, 2, d, d, h0_std=0.2)
    o, s = run_gpu(sr, x, algo)
    units = [n * 2 + h for n in range(0, 300, 7) for h in range(2)]
    o_ref, s_ref = run_oracle(x, units=units)
    cu = x.cu_seqlens.tolist()
    for u in units:
        n, h = divmod(u, 2)
        assert_close(s[n, h], s_ref[n, h], STATE_TOL, f"state seq {n} head {h}")
        assert_close(o[cu[n]:cu[n + 1], h], o_ref[cu[n]:cu[n + 1], h], OUT_TOL_BF16, f"o seq {n} head {h}")


@pytest.mark.parametrize("want_o", [True, False])
def test_replay_call_captures_in_a_cuda_graph(sr, want_o):
    """The replay call issues only stream work (a status clear and its kernels)
    with no host synchronisation, so a serving engine can capture it in a CUDA
    graph: replaying the graph gives the eager call's results bit for bit,
    also after the inputs change in place between replays."""
    x = W.raw_qwen()
    d = lambda a: a.cuda().contiguous()
    q, k, v, g, b, cu = map(d, (x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens))
    o = torch.empty_like(v) if want_o else None
    s = torch.empty(x.n_seqs, v.shape[1], v.shape[2], v.shape[2], dtype=torch.float32, device="cuda")
    args = sr.gdn_args(q, k, v, g, b, cu, n_seqs=x.n_seqs, max_seqlen=x.max_seqlen, o=o, s_out=s)
    ws = sr.workspace(sr.gdn_workspace_bytes(args))
    call = lambda: sr.gdn_replay(q, k, v, g, b, cu, max_seqlen=x.max_seqlen, want_o=want_o, o=o, s_out=s, ws=ws)
    call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for scale in (1.0, 0.5):
        v.mul_(scale)
        call()
        torch.cuda.synchronize()
        s_eager = s.clone()
        o_eager = o.clone() if want_o else None
        s.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(s, s_eager)
        if want_o:
            assert torch.equal(o, o_eager)
    assert sr.device_status(ws) == 0
