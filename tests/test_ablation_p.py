"""The p-ablation of the statistic (tests/golden/ablation_p.json, written by
tests/golden/make_ablation_p.py from the oracle alone): the relative activation-weighted
loss ||(W - W_hat) X^T||^2 / ||W X^T||^2 of TTQ for p in {1, 2} and alpha in {0, 0.5,
0.75} (paper-daily.com deep reading of TTQ, section 2; nubint.ai review, "proposed
method"). Recomputed from the seeds here (the small layer in full, one Qwen3-1.7B-shaped
linear) and checked against the stored table; every activation-aware setting must lower
the loss against plain round-to-nearest (alpha = 0). CPU only."""

import json
import os
import sys

import numpy as np
import pytest

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
sys.path.insert(0, HERE)

import make_ablation_p as M  # noqa: E402


@pytest.fixture(scope="module")
def table():
    with open(os.path.join(HERE, "ablation_p.json")) as f:
        return json.load(f)


def test_small_layer_reproduces(table):
    got = M.small_rows()["linear"]
    want = table["small"]["rows"]["linear"]
    for k, v in want.items():
        assert abs(got[k] - v) <= 1e-6 * v, (k, got[k], v)


def test_qwen3_1p7b_q_proj_reproduces(table):
    from online_activation_aware_b200 import synthetic

    wl = synthetic.WORKLOADS["qwen3_1p7b_set"]
    lin = wl.layers[0]
    X, W = synthetic.draw_layer(wl.T, lin.d, lin.d_out, wl.layer_seed(0))
    n = table["qwen3_1p7b"]["tokens"]
    got = M.layer_losses(M.bf16(X[:n]), M.bf16(W), wl.q, wl.g, wl.r)
    for k, v in table["qwen3_1p7b"]["rows"][lin.name].items():
        assert abs(got[k] - v) <= 1e-6 * v, (k, got[k], v)


def test_activation_aware_settings_beat_rtn(table):
    for part in ("small", "qwen3_1p7b"):
        for name, row in table[part]["rows"].items():
            rtn = row["p2_a0.0"]
            for k, v in row.items():
                if k != "p2_a0.0":
                    assert v < rtn, (part, name, k, v, rtn)
