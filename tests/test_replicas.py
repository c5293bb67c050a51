"""Replica bookkeeping on several ranks, as world-size-2 gloo process groups on
the CPU: the job time is the slowest rank's, the job rate counts every rank's
tokens, and a rank that never joins makes the others fail within the
process-group timeout instead of hanging."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from persistent_decode_b200 import replicas


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    replicas.init("gloo", timeout_s=60)
    r, w, _ = replicas.dist_env()
    t = replicas.max_over_ranks(times[r])
    out[r] = (t, replicas.job_rate(256, t, w))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_on_two_gloo_ranks():
    world = 2
    times = [1.25, 2.0]     # seconds measured by each rank
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), times, out), nprocs=world, join=True)
        got = dict(out)
    for r in range(world):
        assert got[r][0] == pytest.approx(2.0)
        assert got[r][1] == pytest.approx(256 * 2 / 2.0)


def test_single_rank_needs_no_process_group():
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.job_rate(100, 2.0, 1) == 50.0


def _lonely(rank, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    try:
        replicas.init("gloo", timeout_s=3)
        out["joined"] = True
    except Exception as e:   # the other rank never came
        out["error"] = type(e).__name__


def test_missing_rank_fails_within_timeout():
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_lonely, args=(_free_port(), out), nprocs=1, join=True)
        got = dict(out)
    assert "error" in got and "joined" not in got
