"""The N>1 host logic on CPU: two gloo ranks in separate processes.

The TTQ path shards by prompt (each prompt has its own s and codes), so ranks run
independent prompt streams; the only cross-rank steps are a barrier and the max of
the per-rank times. These tests run that plumbing with world_size 2.
"""

import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp

from online_activation_aware_b200 import dist as D


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    try:
        assert D.init("gloo", timeout_s=60) == world
        D.barrier()
        # per-rank "step times": the job time is the slowest rank's
        t = 10.0 + 5.0 * rank
        tmax = D.max_over_ranks(t)
        tsum = D.sum_over_ranks(1.0)
        lo, hi = D.shard(1000, rank, world)
        seed = D.rank_seed(3, rank)
        q.put((rank, tmax, tsum, lo, hi, seed))
        D.barrier()
        D.finalize()
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for o in out:
        assert o[1] != "error", o
    assert all(o[1] == 15.0 for o in out)          # max over ranks
    assert all(o[2] == 2.0 for o in out)           # world size seen by the reduction
    assert out[0][3:5] == (0, 500) and out[1][3:5] == (500, 1000)
    assert out[0][5] != out[1][5]                  # each rank draws its own prompts


@pytest.mark.parametrize("n,world", [(10, 3), (7, 8), (1000, 2), (5, 1)])
def test_shard_partitions(n, world):
    seen = []
    for r in range(world):
        lo, hi = D.shard(n, r, world)
        seen.extend(range(lo, hi))
    assert seen == list(range(n))


def test_single_process_defaults():
    assert D.max_over_ranks(3.5) == 3.5
    assert D.sum_over_ranks(2.0) == 2.0


def test_whole_job_throughput_formula():
    import bench

    # two ranks, 4096 tokens each per step, 10 steps, slowest rank 20 ms
    assert bench.whole_job_ktoks(4096, 10, 2, 20.0) == pytest.approx(2 * 4096 * 10 / 0.02 / 1e3)
