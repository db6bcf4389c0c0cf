"""The bounds-checked build (libsr_checked.so, compiled with -DSR_CHECKED):
every global-memory index of the custom kernels is tested before use and a
bad one is skipped and reported as SR_DEV_BAD_ACCESS, never trapped.  The
default paths of all three replay calls run under it on ragged inputs (empty,
length-1 and chunk-straddling sequences, initial states, every precision mode
of the group replay) with clean status words and oracle-matching results."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_checked_build_runs_clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, SR_LIBRARY="libsr_checked.so")
    r = subprocess.run([sys.executable, os.path.join(HERE, "_checked_cases.py")], env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    assert "every case clean" in r.stdout
