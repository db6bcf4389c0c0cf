"""GPU checks of the anchor sidecar path ("SuffixReplay: Prefix Caching via
Suffix Replay for Hybrid LLMs", System Design, Anchor Sidecar; Algorithm
Design 2): sr_anchor_capture is an exact indexed row copy, it runs inside a
captured CUDA graph whose index tables are rewritten between launches, and a
capture -> plan -> gathered replay round trip gives the bits of a replay
over the same hidden rows packed by hand."""
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_deltanet_state_sr_b200 as m
    return m


def test_capture_is_an_exact_row_copy(sr):
    H = 2560
    hidden = W.normal(51, "h", (300, H), 1.0).cuda()
    pool = torch.full((700, H), 3.0, dtype=torch.bfloat16, device="cuda")
    gen = torch.Generator().manual_seed(51)
    src = torch.randint(0, 300, (257,), generator=gen).to(torch.int32)
    dst = torch.randperm(700, generator=gen)[:257].to(torch.int32)
    ws = sr.anchor_capture(hidden, pool, src.cuda(), dst.cuda())
    assert sr.device_status(ws) == 0
    want = torch.full((700, H), 3.0, dtype=torch.bfloat16)
    want[dst.long()] = hidden.cpu()[src.long()]
    assert torch.equal(pool.cpu(), want)


def test_capture_skips_and_flags_bad_rows(sr):
    H = 256
    hidden = W.normal(52, "h", (10, H), 1.0).cuda()
    pool = torch.zeros(20, H, dtype=torch.bfloat16, device="cuda")
    src = torch.tensor([0, 10, 2, -1, 4], dtype=torch.int32)
    dst = torch.tensor([1, 2, 20, 3, 5], dtype=torch.int32)
    ws = sr.anchor_capture(hidden, pool, src.cuda(), dst.cuda())
    assert sr.device_status(ws) & sr.SR_DEV_BAD_INDEX
    want = torch.zeros(20, H, dtype=torch.bfloat16)
    want[1] = hidden[0].cpu()
    want[5] = hidden[4].cpu()
    assert torch.equal(pool.cpu(), want)


def test_capture_inside_a_cuda_graph(sr):
    H = 512
    hidden = W.normal(53, "h", (64, H), 1.0).cuda()
    pool = torch.zeros(128, H, dtype=torch.bfloat16, device="cuda")
    src = torch.arange(16, dtype=torch.int32, device="cuda")
    dst = torch.arange(16, dtype=torch.int32, device="cuda")
    ws = sr.workspace(256)
    args = sr.capture_args(hidden, pool, src, dst)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside the capture
        assert sr.capture_call(args, ws, s) == sr.SR_OK
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        assert sr.capture_call(args, ws, torch.cuda.current_stream()) == sr.SR_OK
    for rep in range(2):
        # the host rewrites the destination table in place, then relaunches the graph
        src.copy_(torch.arange(16, dtype=torch.int32) * 2 + rep)
        dst.copy_(torch.arange(16, dtype=torch.int32) + 16 * (rep + 1))
        g.replay()
        torch.cuda.synchronize()
        got = pool[16 * (rep + 1): 16 * (rep + 2)]
        assert torch.equal(got, hidden[torch.arange(16, device="cuda") * 2 + rep])
    assert sr.device_status(ws) == 0


def test_capture_plan_and_gathered_replay_round_trip(sr):
    """The forward pass captures every anchor of a 1000-token prefix into a
    page-major pool (through a shuffled block table); the replay reads the
    last k = min(ceil(0.05 n), k_max) anchors through the plan's pool rows.
    That equals replaying the captured hidden rows packed by hand."""
    s = W.LayerShape(hidden=256, inter=512, h_k=2, h_v=4, d_k=128, d_v=128)
    n = 1000
    pages = (n + 63) // 64
    block_table = torch.randperm(pages, generator=torch.Generator().manual_seed(54)).tolist()
    hidden = W.normal(54, "fwd", (n, s.hidden), 1.0).cuda()
    pool = torch.zeros(pages * 4, s.hidden, dtype=torch.bfloat16, device="cuda")
    # every anchor of the prefix: plan with an unbounded budget
    pos_all, rows_all = sr.sparse_anchor_plan(n, ratio=1.0, k_max=10 ** 6, block_table=block_table)
    assert len(pos_all) == (n // 64) * 4 + sum(1 for o in range(60, 64) if (n // 64) * 64 + o < n)
    sr.anchor_capture(hidden, pool, torch.tensor(pos_all, dtype=torch.int32, device="cuda"),
                      torch.tensor(rows_all, dtype=torch.int32, device="cuda"))
    pos, rows = sr.sparse_anchor_plan(n, ratio=0.05, k_max=40, block_table=block_table)
    assert len(pos) == 40
    gi = W.group_inputs(54, [len(pos)], n_layers=2, shape=s)

    class Dev:
        def __init__(self, lw):
            for f in ("w_in_norm", "w_in", "conv_w", "a_log", "dt_bias", "w_gnorm", "w_out", "w_post_norm",
                      "w_gate", "w_up", "w_down"):
                setattr(self, f, getattr(lw, f).cuda().contiguous())

    weights = [Dev(lw) for lw in gi.layers]
    kw = dict(max_seqlen=len(pos), hidden=s.hidden, inter=s.inter, h_k=s.h_k, h_v=s.h_v, eps=s.eps,
              mode=sr.SR_MODE_SKIP)
    cu = gi.cu_seqlens.cuda()
    got = sr.group_replay([pool], cu, [weights], anchor_index=torch.tensor(rows, dtype=torch.int32,
                                                                             device="cuda"), **kw)
    want = sr.group_replay([hidden[torch.tensor(pos, device="cuda")].contiguous()], cu, [weights], **kw)
    torch.cuda.synchronize()
    for l in range(2):
        assert torch.equal(got[0][l][0], want[0][l][0])
        assert torch.equal(got[0][l][1], want[0][l][1])
