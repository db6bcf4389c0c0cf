"""GPU parity of the two widenings of sr_group_replay.

Continuation: after a replay rebuilds every layer's state, the unmatched
tokens continue from it ("Tail-Replay", Sec. 3; "SuffixReplay", Pipelined
Replay Path).  The call with initial states must match the fp64 oracle's
continuation, agree with one pass over the concatenated tokens, and give the
same bits when it updates its states in place.

Token-wise sparse anchors ("SuffixReplay", Algorithm Design 2): the replay
batch gathered from an anchor pool through an index table must give exactly
the bits of a replay over the pre-gathered rows, and a bad index is flagged
on the device."""
import numpy as np
import pytest
import torch

from oracle import layers as OL
import workloads as W
from _util import OUT_TOL_BF16, STATE_TOL, assert_close

pytestmark = pytest.mark.gpu

LENGTHS = [70, 5, 130, 3, 0, 9]
CUTS = [40, 5, 64, 1, 0, 2]  # b-parts of 30, 0, 66, 2, 0, 7 tokens


@pytest.fixture(scope="module")
def sr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_deltanet_state_sr_b200 as m
    return m


class DevLayer:
    def __init__(self, lw):
        for f in ("w_in_norm", "w_in", "conv_w", "a_log", "dt_bias", "w_gnorm", "w_out", "w_post_norm",
                  "w_gate", "w_up", "w_down"):
            setattr(self, f, getattr(lw, f).cuda().contiguous())


def small_shape():
    return W.LayerShape(hidden=256, inter=512, h_k=2, h_v=4, d_k=128, d_v=128)


def split_batch(lengths, cuts):
    starts = np.concatenate([[0], np.cumsum(lengths)])
    a_idx = np.concatenate([np.arange(starts[n], starts[n] + c) for n, c in enumerate(cuts)]).astype(np.int64)
    b_idx = np.concatenate([np.arange(starts[n] + c, starts[n + 1]) for n, c in enumerate(cuts)]).astype(np.int64)
    cu_a = torch.tensor(np.concatenate([[0], np.cumsum(cuts)]), dtype=torch.int32)
    cu_b = torch.tensor(np.concatenate([[0], np.cumsum(np.asarray(lengths) - np.asarray(cuts))]), dtype=torch.int32)
    return torch.from_numpy(a_idx), torch.from_numpy(b_idx), cu_a, cu_b


def call(sr, anchors, cu, weights, s, mode, **kw):
    lens = (cu[1:] - cu[:-1]).tolist()
    out = sr.group_replay([anchors.cuda().contiguous()], cu.cuda(), [weights], max_seqlen=max(max(lens), 1),
                          hidden=s.hidden, inter=s.inter, h_k=s.h_k, h_v=s.h_v, d=s.d_k, eps=s.eps, mode=mode,
                          **kw)
    torch.cuda.synchronize()
    return out[0]


@pytest.mark.parametrize("mode", ["skip", "full"])
def test_continuation_matches_oracle_and_one_pass(sr, mode):
    s = small_shape()
    gi = W.group_inputs(41, LENGTHS, n_layers=3, shape=s)
    weights = [DevLayer(lw) for lw in gi.layers]
    m = sr.SR_MODE_SKIP if mode == "skip" else sr.SR_MODE_FULL
    a_idx, b_idx, cu_a, cu_b = split_batch(LENGTHS, CUTS)
    out_a = call(sr, gi.anchors[a_idx], cu_a, weights, s, m)
    out_b = call(sr, gi.anchors[b_idx], cu_b, weights, s, m,
                 initial=[[(st, cv) for st, cv, _ in out_a]])
    one = call(sr, gi.anchors, gi.cu_seqlens, weights, s, m)
    # oracle: the a-part from zero, then the b-part from its states; the conv
    # state is handed over in its stored format (bf16, round to nearest even)
    ga = W.GroupInputs(gi.anchors[a_idx], cu_a, gi.layers, s)
    gb = W.GroupInputs(gi.anchors[b_idx], cu_b, gi.layers, s)
    ref_a = OL.group_replay(ga, mode)
    stored = lambda c: torch.from_numpy(c).to(torch.bfloat16).double().numpy()
    ref_b = OL.group_replay(gb, mode, initial=[(r["S"], stored(r["conv_state"])) for r in ref_a])
    for l in range(3):
        s_b, c_b, _ = out_b[l]
        assert_close(s_b, ref_b[l]["S"], STATE_TOL, f"layer {l} continued state vs oracle")
        assert_close(c_b, ref_b[l]["conv_state"], OUT_TOL_BF16, f"layer {l} continued conv state vs oracle")
        assert_close(s_b, one[l][0].double().cpu().numpy(), STATE_TOL, f"layer {l} continued vs one pass")
    # sequences with no b tokens keep their a-states exactly
    for n in (1, 4):
        for l in range(3):
            assert torch.equal(out_b[l][0][n], out_a[l][0][n])
            assert torch.equal(out_b[l][1][n], out_a[l][1][n])


def test_in_place_continuation_gives_the_same_bits(sr):
    s = small_shape()
    gi = W.group_inputs(42, LENGTHS, n_layers=2, shape=s)
    weights = [DevLayer(lw) for lw in gi.layers]
    a_idx, b_idx, cu_a, cu_b = split_batch(LENGTHS, CUTS)
    out_a = call(sr, gi.anchors[a_idx], cu_a, weights, s, sr.SR_MODE_FULL)
    out_b = call(sr, gi.anchors[b_idx], cu_b, weights, s, sr.SR_MODE_FULL,
                 initial=[[(st, cv) for st, cv, _ in out_a]])
    # in place: the outputs are the initial states
    state = [(st.clone(), cv.clone(), None) for st, cv, _ in out_a]
    call(sr, gi.anchors[b_idx], cu_b, weights, s, sr.SR_MODE_FULL, outputs=[state],
         initial=[[(st, cv) for st, cv, _ in state]])
    for l in range(2):
        assert torch.equal(state[l][0], out_b[l][0])
        assert torch.equal(state[l][1], out_b[l][1])


def test_continuation_with_no_tokens_returns_the_initial_states(sr):
    s = small_shape()
    gi = W.group_inputs(43, [4, 4], n_layers=2, shape=s)
    weights = [DevLayer(lw) for lw in gi.layers]
    n = 2
    init = [(torch.randn(n, s.h_v, 128, 128, device="cuda"),
             torch.randn(n, s.conv_dim, 3, device="cuda").to(torch.bfloat16)) for _ in range(2)]
    outputs = [(torch.full_like(a, 7.0), torch.zeros_like(c), None) for a, c in init]
    cu = torch.zeros(n + 1, dtype=torch.int32, device="cuda")
    args = sr.group_args([gi.anchors.cuda()], cu, [weights], [outputs], max_seqlen=0, hidden=s.hidden,
                         inter=s.inter, h_k=s.h_k, h_v=s.h_v, eps=s.eps, initial=[init], total_tokens=0)
    ws = sr.workspace(sr.group_workspace_bytes(args))
    assert sr.group_call(args, ws) == sr.SR_OK
    torch.cuda.synchronize()
    for (st, cv, _), (si, ci) in zip(outputs, init):
        assert torch.equal(st, si) and torch.equal(cv, ci)


def test_sparse_anchor_gather_is_bit_exact(sr):
    s = small_shape()
    gi = W.group_inputs(44, [100, 37, 1], n_layers=2, shape=s)
    weights = [DevLayer(lw) for lw in gi.layers]
    pool = W.normal(44, "pool", (400, s.hidden), 1.0)
    gen = torch.Generator().manual_seed(44)
    idx = torch.randint(0, 400, (138,), generator=gen, dtype=torch.int64)
    idx[5] = idx[4]  # a repeated row
    idx32 = idx.to(torch.int32).cuda()
    for prec in (sr.SR_PREC_SPLIT, sr.SR_PREC_BF16):
        gathered = call(sr, pool, gi.cu_seqlens, weights, s, sr.SR_MODE_FULL, anchor_index=idx32,
                        precision=prec, want_hidden=True)
        packed = call(sr, pool[idx], gi.cu_seqlens, weights, s, sr.SR_MODE_FULL, precision=prec,
                      want_hidden=True)
        for l in range(2):
            for a, b in zip(gathered[l], packed[l]):
                assert torch.equal(a, b)
    ref = OL.group_replay(gi, "full", anchors=pool, anchor_index=idx.numpy())
    for l in range(2):
        assert_close(gathered[l][0], ref[l]["S"], 1e-2, f"layer {l} state (bf16 mode) vs oracle")


def test_bad_anchor_index_reads_zero_and_is_flagged(sr):
    s = small_shape()
    gi = W.group_inputs(45, [20, 12], n_layers=1, shape=s)
    weights = [DevLayer(lw) for lw in gi.layers]
    pool = W.normal(45, "pool", (50, s.hidden), 1.0)
    idx = torch.arange(32, dtype=torch.int32) + 3
    idx[7] = 50   # one past the pool
    idx[20] = -1  # negative
    ws = sr.workspace(64 << 20)
    got = call(sr, pool, gi.cu_seqlens, weights, s, sr.SR_MODE_SKIP, anchor_index=idx.cuda(), ws=ws)
    assert sr.device_status(ws) & sr.SR_DEV_BAD_INDEX
    rows = pool[idx.clamp(0, 49).long()].clone()
    rows[7] = 0
    rows[20] = 0
    want = call(sr, rows, gi.cu_seqlens, weights, s, sr.SR_MODE_SKIP, ws=ws)
    assert sr.device_status(ws) == 0
    assert torch.equal(got[0][0], want[0][0]) and torch.equal(got[0][1], want[0][1])
