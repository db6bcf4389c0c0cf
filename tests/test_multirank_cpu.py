"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The replay shards by request: every rank replays its own, independent batch
(seeded per rank), there is no collective on the data path, and the job time
is the slowest rank's.  These tests run that host logic in two real
processes over gloo."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    w, r, l = bench.dist_setup()
    # each rank times a different amount of work; the job time is the max
    ms = bench.max_over_ranks(10.0 + 5.0 * r, w, torch.device("cpu"))
    tput = bench.job_throughput(1000, w, 4, ms)
    # per-rank workloads are independent draws (no shared data between ranks)
    x = W.raw_small(seed=0x5EED0000 + r)
    digest = float(x.v.float().sum())
    gathered = [None] * w
    dist.all_gather_object(gathered, digest)
    out[rank] = (w, r, ms, tput, gathered)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_timing_and_independent_shards():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank, (w, r, ms, tput, gathered) in res.items():
        assert (w, r) == (2, rank)
        assert ms == 15.0                      # slowest rank
        assert tput == pytest.approx(1000 * 2 * 4 / 0.015)
        assert gathered[0] != gathered[1]      # each rank replays its own request
