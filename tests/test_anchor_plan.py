"""Host logic of the token-sparse replay ("SuffixReplay: Prefix Caching via
Suffix Replay for Hybrid LLMs", Algorithm Design 2 and 3): which prefix
positions carry anchors and which of them a replay of k = min(ratio n, k_max)
anchors reads.  sr_sparse_anchor_plan is checked against a brute-force
enumeration of every position, and against the figures the pages give
(4 anchors per 64-token page at density 1/16; k_max 512)."""
import math

import pytest

import gated_deltanet_state_sr_b200 as sr


def brute(n, page, m, layout, ratio, k_max, block_table=None):
    if layout == sr.SR_ANCHORS_PAGE_TAIL:
        offs = [page - m + i for i in range(m)]
    else:
        offs = [(i + 1) * (page // m) - 1 for i in range(m)]
    anchors = [(p, offs.index(p % page)) for p in range(n) if p % page in offs]
    k = min(math.ceil(ratio * n - 1e-9), k_max, len(anchors))
    chosen = anchors[len(anchors) - k:]
    pos = [p for p, _ in chosen]
    rows = [(block_table[p // page] if block_table else p // page) * m + slot for p, slot in chosen]
    return pos, rows


@pytest.mark.parametrize("layout", [sr.SR_ANCHORS_PAGE_TAIL, sr.SR_ANCHORS_UNIFORM])
@pytest.mark.parametrize("n", [0, 1, 50, 61, 63, 64, 65, 127, 1000, 4096, 8192 + 62])
@pytest.mark.parametrize("ratio,k_max", [(0.05, 512), (0.05, 8), (1.0, 10 ** 6), (0.0, 512)])
def test_plan_matches_brute_force(layout, n, ratio, k_max):
    got = sr.sparse_anchor_plan(n, page_size=64, anchors_per_page=4, layout=layout, k_max=k_max, ratio=ratio)
    assert got == brute(n, 64, 4, layout, ratio, k_max)


def test_block_table_maps_pages_to_pool_blocks():
    bt = [9, 3, 7, 0, 5]
    pos, rows = sr.sparse_anchor_plan(300, k_max=6, ratio=0.05, block_table=bt)
    assert (pos, rows) == brute(300, 64, 4, sr.SR_ANCHORS_PAGE_TAIL, 0.05, 6, bt)
    # page 4 holds tokens 256..299 only, so its page-end slots do not exist yet:
    # the last anchor is slot 3 of page 3 (position 255), which lives in block 0
    assert pos[-1] == 255 and rows[-1] == 0 * 4 + 3
    # k = 6: slots 2, 3 of page 2 (block 7), then the four slots of page 3
    assert pos == [190, 191, 252, 253, 254, 255] and rows == [30, 31, 0, 1, 2, 3]


def test_paper_budget_at_32k():
    """32K prefix, density 1/16 on 64-token pages: 2048 anchors; k = min(0.05 n,
    512) = 512, all at page ends, the last one at position 32767."""
    pos, rows = sr.sparse_anchor_plan(32768, k_max=512, ratio=0.05)
    assert len(pos) == 512
    assert pos[-1] == 32767 and pos[0] == 32768 - 128 * 64 + 60
    assert all(p % 64 >= 60 for p in pos) and pos == sorted(pos)
    assert rows == list(range(2048 - 512, 2048))


def test_invalid_arguments_are_rejected():
    with pytest.raises(sr.SrError):
        sr.sparse_anchor_plan(100, page_size=64, anchors_per_page=0)
    with pytest.raises(sr.SrError):
        sr.sparse_anchor_plan(100, page_size=64, anchors_per_page=5, layout=sr.SR_ANCHORS_UNIFORM)
    with pytest.raises(sr.SrError):
        sr.sparse_anchor_plan(100, ratio=1.5)


def test_capture_validation_runs_without_a_gpu():
    import ctypes
    a = sr.CaptureArgs(0x10000, 0x20000, 0x30000, 0x40000, 4, 2560, 10, 10)
    assert sr.capture_call(a, None) == sr.SR_ERR_WORKSPACE
    a.hidden = 2561
    assert sr.capture_call(a, None) == sr.SR_ERR_UNSUPPORTED
    a.hidden = 2560
    a.pool = 0x20008  # not 16-byte aligned
    assert sr.capture_call(a, None) == sr.SR_ERR_INVALID_ARG
    a.pool, a.src_rows = 0x20000, None
    assert sr.capture_call(a, None) == sr.SR_ERR_INVALID_ARG
