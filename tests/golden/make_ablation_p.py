"""Writes ablation_p.json: the activation-weighted loss of TTQ against the statistic's
exponent p and strength alpha, computed by the oracle alone on the seeded synthetic
workloads (no GPU, no product code).

The loss is L = ||(W - W_hat) X^T||_F^2 (paper-daily.com deep reading of TTQ, section 2: the
loss activation-aware scaling targets), reported relative to ||W X^T||_F^2. W_hat is the
TTQ weight Q[W D^(1/2)] D^(-1/2) with s = D^(1/2) = (mean_t |x_t|^p + lambda)^(alpha/p)
(nubint.ai review, "proposed method": alpha, lambda and p fixed ahead of time; the
paper-daily.com deep reading, section 2, argues for the squared, p = 2, statistic over the
mean-|x|, p = 1, one); alpha = 0 is plain round-to-nearest. With a rank-r side path the
weight is W_hat = B A + Q[R D^(1/2)] D^(-1/2) with R = W - B A.

Rows:
  small      the 512 -> 512 layer, T = 128, q = 3, g = 32 (all of it);
  qwen3_1p7b the six Qwen3-1.7B-shaped linears, q = 3, g = 32, r = 16 (SVD factors), on
             the first `--tokens` tokens of T = 4096 and every output row.

Usage: python tests/golden/make_ablation_p.py [--tokens 1024]
"""

from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from oracle import ttq_oracle as O  # noqa: E402
from online_activation_aware_b200 import synthetic  # noqa: E402

SETTINGS = [(2, 0.0), (1, 0.5), (2, 0.5), (1, 0.75), (2, 0.75)]  # (p, alpha); alpha = 0 is RTN for any p
LAMBDA = 0.4


def bf16(a):
    return O.round_bf16(np.asarray(a, dtype=np.float32))


def layer_losses(X, W, q, g, r, settings=SETTINGS):
    """Relative loss L / ||W X^T||^2 for each (p, alpha), X [T, d] and W [d', d] bf16 values."""
    A = B = None
    Wq = W
    if r > 0:
        B, A, Wq = O.lowrank_split(W, r)
    ref = float(np.sum((X @ W.T) ** 2))
    out = {}
    for p, alpha in settings:
        _, s32 = O.act_stats(X, alpha, LAMBDA, p)
        codes, scale, zero = O.requant(Wq, s32, q, g)
        W_hat = O.dequant_original(codes, scale, zero, g, s32)
        if r > 0:
            W_hat = W_hat + B @ A
        out[f"p{p}_a{alpha}"] = O.activation_loss(W, W_hat, X) / ref
    return out


def small_rows():
    wl = synthetic.WORKLOADS["single_512"]
    lin = wl.layers[0]
    X, W = synthetic.draw_layer(wl.T, lin.d, lin.d_out, wl.seed)
    return {"linear": layer_losses(bf16(X), bf16(W), wl.q, wl.g, 0)}


def qwen_rows(tokens: int):
    wl = synthetic.WORKLOADS["qwen3_1p7b_set"]
    rows = {}
    for i, lin in enumerate(wl.layers):
        X, W = synthetic.draw_layer(wl.T, lin.d, lin.d_out, wl.layer_seed(i))
        rows[lin.name] = layer_losses(bf16(X[:tokens]), bf16(W), wl.q, wl.g, wl.r)
    return rows


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--tokens", type=int, default=1024)
    args = ap.parse_args()
    out = {
        "what": "relative activation-weighted loss ||(W - W_hat) X^T||^2 / ||W X^T||^2, oracle only",
        "lambda": LAMBDA,
        "settings": [f"p{p}_a{a}" for p, a in SETTINGS],
        "small": {"workload": "512 -> 512, T = 128, q = 3, g = 32, r = 0, seed 0", "rows": small_rows()},
        "qwen3_1p7b": {"workload": f"Qwen3-1.7B-shaped set, first {args.tokens} of 4096 tokens, q = 3, g = 32, "
                                   "r = 16 (SVD factors), seeds 2000 + layer",
                       "tokens": args.tokens, "rows": qwen_rows(args.tokens)},
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "ablation_p.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
