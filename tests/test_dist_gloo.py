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


# ------------------------------------------------------------------ one linear split by output rows


class _OracleBlock:
    """A rank's block of a TTQ linear computed by the CPU oracle (stands in for the CUDA
    layer in these CPU tests): prefill keeps s and the codes, decode reuses them."""

    def __init__(self, W_block, q, g, alpha, lam):
        self.W, self.q, self.g, self.alpha, self.lam = W_block, q, g, alpha, lam

    def prefill(self, X):
        from oracle import ttq_oracle as O

        out = O.prefill(X.numpy(), self.W, self.q, self.g, self.alpha, self.lam)
        self.s32, self.codes, self.scale, self.zero = out["s32"], out["codes"], out["scale"], out["zero"]
        return torch.from_numpy(out["Y"])

    def decode(self, X):
        from oracle import ttq_oracle as O

        return torch.from_numpy(O.linear(X.numpy(), self.s32, self.codes, self.scale, self.zero, self.g))


def _split_worker(rank, world, port, q_):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    try:
        import numpy as np

        from online_activation_aware_b200 import synthetic
        from online_activation_aware_b200.tensor_parallel import ColumnParallelTTQLinear, shard_rows

        assert D.init("gloo", timeout_s=60) == world
        T, d, d_out, q, g = 48, 256, 96, 4, 64
        X, W = synthetic.draw_layer(T, d, d_out, seed=17)
        Xv = synthetic.bf16_values(synthetic.as_bf16(X))
        Wv = synthetic.bf16_values(synthetic.as_bf16(W))
        lo, hi = shard_rows(d_out, rank, world)
        layer = ColumnParallelTTQLinear(local=_OracleBlock(Wv[lo:hi], q, g, 0.5, 0.4))
        Y = layer.prefill(torch.from_numpy(Xv)).numpy()
        xt = synthetic.bf16_values(synthetic.as_bf16(synthetic.draw_tokens(3, d, seed=18)))
        Yd = layer.decode(torch.from_numpy(xt)).numpy()
        blk = layer.local
        q_.put((rank, Y, Yd, blk.s32, blk.codes, lo, hi))
        D.barrier()
        D.finalize()
    except Exception as e:
        q_.put((rank, "error", repr(e)))


def test_column_split_two_gloo_ranks_matches_whole_layer():
    # each rank re-quantizes its 48 of 96 rows from its own (identical) statistic; the
    # gathered Y and decode rows equal the whole layer's, and each rank's codes are the
    # whole layer's codes of its rows
    import numpy as np

    from online_activation_aware_b200 import synthetic
    from oracle import ttq_oracle as O

    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, q_)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted([q_.get(timeout=180) for _ in range(world)], key=lambda o: o[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for o in out:
        assert not (isinstance(o[1], str) and o[1] == "error"), o
    X, W = synthetic.draw_layer(48, 256, 96, seed=17)
    Xv = synthetic.bf16_values(synthetic.as_bf16(X))
    Wv = synthetic.bf16_values(synthetic.as_bf16(W))
    full = O.prefill(Xv, Wv, 4, 64, 0.5, 0.4)
    xt = synthetic.bf16_values(synthetic.as_bf16(synthetic.draw_tokens(3, 256, seed=18)))
    Yd_full = O.linear(xt, full["s32"], full["codes"], full["scale"], full["zero"], 64)
    for rank, Y, Yd, s32, codes, lo, hi in out:
        np.testing.assert_allclose(Y, full["Y"], rtol=1e-12, atol=1e-12 * np.abs(full["Y"]).max())
        np.testing.assert_allclose(Yd, Yd_full, rtol=1e-12, atol=1e-12 * np.abs(Yd_full).max())
        np.testing.assert_array_equal(s32, full["s32"])
        np.testing.assert_array_equal(codes, full["codes"][lo:hi])


def test_shard_rows_blocks():
    from online_activation_aware_b200.tensor_parallel import shard_rows

    assert [shard_rows(8192, r, 4) for r in range(4)] == [(0, 2048), (2048, 4096), (4096, 6144), (6144, 8192)]
    for d_out, world in ((100, 2), (96, 5), (8, 2)):
        with pytest.raises(ValueError):
            shard_rows(d_out, 0, world)
