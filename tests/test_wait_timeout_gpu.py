"""Failure detection on the GPU without a fault: a bounded mbarrier wait that
runs out.

Every tcgen05 / TMA kernel of the library waits on mbarriers with a time
limit, after which it records SR_DEV_TIMEOUT in the status word, frees its
tensor memory and returns.  sr_test_wait_timeout runs that path on purpose
(an mbarrier that nothing arrives at, a limit of microseconds): the flag must
be set, the wait must have lasted at least its limit and not much longer, and
the context must stay usable -- a tcgen05 replay right after it still matches
the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from _util import OUT_TOL_BF16, STATE_TOL, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_deltanet_state_sr_b200 as m
    return m


@pytest.mark.parametrize("limit_us", [5, 200, 2000])
def test_wait_runs_out_and_reports(sr, limit_us):
    flags, elapsed = sr.test_wait_timeout(limit_us * 1000)
    assert flags == sr.SR_DEV_TIMEOUT
    assert limit_us * 1000 <= elapsed < limit_us * 1000 + 50_000_000


def test_wait_that_completes_sets_no_flag(sr):
    flags, elapsed = sr.test_wait_timeout(2_000_000, arrive=True)
    assert flags == 0
    assert elapsed < 2_000_000


def test_context_usable_after_timeouts(sr):
    """Several timed-out CTAs in a row, then an ordinary tcgen05 replay (which
    allocates tensor memory itself): the tensor memory was returned and the
    results still match the oracle."""
    for _ in range(4):
        flags, _ = sr.test_wait_timeout(10_000)
        assert flags == sr.SR_DEV_TIMEOUT
    x = W.gdn_inputs(91, [130, 64, 1], 2, 4, 128, 128)
    d = lambda t: t.cuda().contiguous()
    o, s = sr.gdn_replay(d(x.q), d(x.k), d(x.v), d(x.g), d(x.beta), d(x.cu_seqlens), max_seqlen=x.max_seqlen,
                         algo="tcgen05")
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.gdn_replay(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens)
    assert_close(s, s_ref, STATE_TOL, "state")
    assert_close(o, o_ref, OUT_TOL_BF16, "output")
