"""The premise of the column split (``tensor_parallel``) on the CUDA path: a TTQ linear over
a block of W's output rows computes the same statistic, the same codes for its rows and
the same columns of Y as the whole layer (the statistic reduces in a fixed order and the
re-quantization is per row), so gathering the blocks of N ranks gives the whole layer's
output. The blocks run one after another on one GPU here; the gather across ranks is
tested with gloo ranks on CPU (tests/test_dist_gloo.py)."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import online_activation_aware_b200 as ttq
from online_activation_aware_b200 import synthetic
from online_activation_aware_b200.tensor_parallel import ColumnParallelTTQLinear, shard_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,T,d,d_out,q,g,r", [(2, 256, 1024, 768, 4, 64, 0), (4, 4096, 5120, 8192, 4, 128, 0),
                                                   (2, 300, 512, 384, 3, 32, 16)])
def test_row_blocks_reproduce_the_whole_layer(world, T, d, d_out, q, g, r):
    X, W = synthetic.draw_layer(T, d, d_out, seed=world + T)
    Xg = synthetic.as_bf16(X).cuda()
    Wg = synthetic.as_bf16(W).cuda()
    A = B = None
    if r > 0:
        from online_activation_aware_b200.lowrank_setup import lowrank_factors

        B, A, Wg = (t.cuda() for t in lowrank_factors(Wg, r))
    whole = ttq.TTQLinear(Wg, q, g, 0.5, 0.4, r=r, A=A, B=B)
    Y = whole.prefill(Xg)
    xt = synthetic.as_bf16(synthetic.draw_tokens(2, d, seed=5)).cuda()
    Yd = whole.decode(xt)
    words = whole.codes.view(d_out, -1)
    for rank in range(world):
        lo, hi = shard_rows(d_out, rank, world)
        blk = ColumnParallelTTQLinear(Wg[lo:hi].contiguous(), q, g, 0.5, 0.4, r=r, A=A,
                                      B_block=None if B is None else B[lo:hi].contiguous())
        Yb = blk.prefill(Xg)            # one process: no group, the block's columns alone
        assert torch.equal(blk.local.s, whole.s)
        assert torch.equal(blk.local.codes.view(hi - lo, -1), words[lo:hi])
        assert torch.equal(blk.local.scale, whole.scale[lo:hi]) and torch.equal(blk.local.zero, whole.zero[lo:hi])
        assert torch.equal(Yb, Y[:, lo:hi])
        assert torch.equal(blk.decode(xt), Yd[:, lo:hi])
    assert ttq.device_status() == 0
