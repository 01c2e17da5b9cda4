"""Host set-up of the static low-rank side path of a TTQ linear layer.

This runs once per weight, before any prompt, on the host (untimed): it is not part of
the per-prompt hot path, which the CUDA library runs. TTQ can keep a small static
low-rank term next to the re-quantized weight, W_hat = W_q + B A, with the factors taken
from a truncated SVD of W and the quantized part W_q the residual R = W - B A that is
re-quantized for every prompt (paper-daily.com deep reading of TTQ, section 2: low-rank
decomposition, r = 16; gist.science French summary, section 2B: decomposition en rang
faible; gist.science German summary, section 2: static B, A).

Reading of the split: B = U_r S_r^(1/2) and A = S_r^(1/2) V_r^T (the square root of
the singular values on each side), both rounded to bf16; R = bf16(W - B A) with the
product of the rounded factors taken in fp64.
"""

from __future__ import annotations


def lowrank_factors(W, r: int, device="cpu"):
    """Returns bf16 tensors (B [d_out, r], A [r, d], R [d_out, d]) for a weight W
    [d_out, d] (any torch tensor, read in fp64) and rank r >= 1. ``device`` is where the
    fp64 SVD runs and the results live (the host by default; a CUDA device shortens the
    set-up of large weights, with the same fp64 arithmetic)."""
    import torch

    if r < 1 or r > min(W.shape):
        raise ValueError(f"rank r = {r} must be in 1 .. {min(W.shape)}")
    Wd = W.detach().to(device, torch.float64)
    U, S, Vh = torch.linalg.svd(Wd, full_matrices=False)
    root = S[:r].sqrt()
    Bf = (U[:, :r] * root[None, :]).to(torch.bfloat16)
    Af = (root[:, None] * Vh[:r, :]).to(torch.bfloat16)
    R = (Wd - Bf.to(torch.float64) @ Af.to(torch.float64)).to(torch.bfloat16)
    return Bf.contiguous(), Af.contiguous(), R.contiguous()
