"""One TTQ linear layer split by output rows across the ranks of a process group.

Groups of the quantizer run along the input channels of one output row, so splitting W by
rows never splits a group, and the re-quantization of each row is independent of every
other row. Each rank therefore holds a contiguous block of d'/N output rows of W (of the
residual R with its block of B when r > 0; A is replicated), computes the statistic s
itself from the replicated prompt X (no communication: every rank gets the same s, since
the kernels reduce in a fixed order), re-quantizes and multiplies its rows only, and one
all-gather joins the column blocks of Y. Decode steps reuse each rank's codes the same way.
(The paper-daily.com deep reading of TTQ, section 2, defines the per-row re-quantization
and the statistic; the split is this library's multi-GPU form.)

The communication per call is one all-gather of T x d' x 2 bytes of bf16 Y ((N - 1)/N of it
crosses the links per rank); a row-parallel layer after this one could consume the blocks
without it.
"""

from __future__ import annotations


def shard_rows(d_out: int, rank: int, world: int):
    """[lo, hi) output rows of one rank: equal blocks whose size is a multiple of 8 (the
    library's alignment of code and scale rows)."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError(f"rank {rank} outside a world of {world}")
    n = d_out // world
    if n * world != d_out or n % 8 != 0:
        raise ValueError(f"d_out = {d_out} does not split into {world} blocks of a multiple of 8 rows")
    return rank * n, (rank + 1) * n


class ColumnParallelTTQLinear:
    """A TTQ linear whose output rows are split across the ranks of `group`.

    `local` is this rank's own layer over its row block: an object with ``prefill(X)`` and
    ``decode(X)`` returning that block's columns of Y, by default a ``TTQLinear`` built
    from `W_block` (the rank's rows of W, or of the residual R with `B_block`, its rows of
    B, and the replicated A). ``prefill`` and ``decode`` return the whole Y [rows, d_out]
    on every rank (one all-gather).
    """

    def __init__(self, W_block=None, q: int = 4, g: int = 128, alpha: float = 0.5, lam: float = 0.4, p: int = 2,
                 r: int = 0, A=None, B_block=None, group=None, local=None):
        import torch.distributed as dist

        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        if local is None:
            import online_activation_aware_b200 as ttq

            local = ttq.TTQLinear(W_block, q, g, alpha, lam, p, r, A, B_block)
        self.local = local

    def _gather(self, Y_block):
        import torch
        import torch.distributed as dist

        if self.world == 1:
            return Y_block
        Y_block = Y_block.contiguous()
        parts = [torch.empty_like(Y_block) for _ in range(self.world)]
        dist.all_gather(parts, Y_block, group=self.group)
        return torch.cat(parts, dim=1)

    def prefill(self, X):
        """Statistic of X (on every rank), re-quantization and projection of this rank's rows,
        then Y [T, d_out] on every rank."""
        return self._gather(self.local.prefill(X))

    def decode(self, X):
        """Decode rows with every rank's stored codes; Y [b, d_out] on every rank."""
        return self._gather(self.local.decode(X))
