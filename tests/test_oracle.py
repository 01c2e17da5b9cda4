"""Pins for the CPU oracle: each test checks it against something other than itself
(hand-derived worked cases, closed forms, brute force, exact rational arithmetic,
library routines, invariants of the mathematics). CPU only."""

import json
import os
from fractions import Fraction
from itertools import product

import numpy as np
import pytest

from oracle import ttq_oracle as O
from online_activation_aware_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- number formats


def test_round_bf16_matches_torch_on_fp32_inputs():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    # include exact ties: values halfway between two bf16 numbers
    ties = (np.arange(1, 200, dtype=np.float32) * 2 + 1) * np.float32(2.0 ** -9)
    x = np.concatenate([x, 1 + ties, -(1 + ties)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(x), ref)


def test_round_bf16_exact_rational():
    # fp64 inputs rounded in one step: compare with the nearest bf16 found by exact
    # rational arithmetic among the two neighbours
    rng = np.random.default_rng(12)
    for x in rng.standard_normal(300) * 10:
        r = O.round_bf16(x)
        fx = Fraction(float(x))
        m, e = np.frexp(x)
        q = Fraction(2) ** (int(e) - 8)
        lo = (fx / q).__floor__() * q
        hi = lo + q
        dlo, dhi = fx - lo, hi - fx
        if dlo < dhi:
            want = lo
        elif dhi < dlo:
            want = hi
        else:
            want = lo if (lo / q) % 2 == 0 else hi
        assert Fraction(float(r)) == want


def _fp16_table():
    bits = np.arange(1, 0x7C00, dtype=np.uint16)
    return np.sort(bits.view(np.float16).astype(np.float64))


def test_round_fp16_up_bruteforce():
    table = _fp16_table()
    rng = np.random.default_rng(13)
    x = np.exp(rng.uniform(np.log(1e-9), np.log(6e4), 50000)).astype(np.float32).astype(np.float64)
    x = np.concatenate([x, table[::97]])  # exact fp16 values map to themselves
    idx = np.searchsorted(table, x, side="left")
    want = table[np.minimum(idx, len(table) - 1)]
    np.testing.assert_array_equal(O.round_fp16_up(x), want)


def test_round_fp16_up_saturates():
    assert O.round_fp16_up(1e9) == 65504.0
    assert O.round_fp16_up(1e-30) == 2.0 ** -24


# ---------------------------------------------------------------- statistics


def test_act_stats_golden():
    for case in _load("act_stats_examples.json")["cases"]:
        s64, s32 = O.act_stats(np.array(case["X"]), case["alpha"], case["lambda"], case["p"])
        np.testing.assert_allclose(s64, case["s"], rtol=1e-15)
        np.testing.assert_array_equal(s32, np.float32(s64))


def test_act_stats_alpha_zero_is_one_and_permutation_invariant():
    X, _ = synthetic.draw_layer(64, 96, 8, seed=5)
    s, _ = O.act_stats(X, 0.0, 0.4)
    np.testing.assert_array_equal(s, np.ones(96))
    s1, _ = O.act_stats(X, 0.5, 0.4)
    perm = np.random.default_rng(0).permutation(64)
    s2, _ = O.act_stats(X[perm], 0.5, 0.4)
    np.testing.assert_allclose(s1, s2, rtol=1e-14)


def test_act_stats_constant_columns_closed_form():
    c = np.array([0.0, 1.5, -2.0, 7.0])
    X = np.tile(c, (33, 1))
    s, _ = O.act_stats(X, 0.75, 0.4)
    # (c^2 + lambda)^(alpha/2), evaluated by hand for each column
    want = np.array([0.4 ** 0.375, 2.65 ** 0.375, 4.4 ** 0.375, 49.4 ** 0.375])
    np.testing.assert_allclose(s, want, rtol=1e-14)


# ---------------------------------------------------------------- quantizer


def test_requant_golden_groups():
    for case in _load("requant_examples.json")["cases"]:
        c, sg, z = O.quantize_group(np.array(case["v"], dtype=np.float32), case["q"])
        assert list(c) == case["codes"], case
        assert sg == case["scale"], case
        assert int(np.float16(sg).view(np.uint16)) == int(case["scale_bits"], 16), case
        assert z == case["zero"], case


def _groups(seed, n, g, spread=1.0):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((n, g)) * np.exp(rng.uniform(-3, 3, (n, 1))) * spread
    v = v + rng.standard_normal((n, 1)) * rng.choice([0.0, 0.3, 3.0], (n, 1)) * np.abs(v).max(1, keepdims=True)
    return O.round_bf16(v).astype(np.float32)


@pytest.mark.parametrize("q", [2, 3])
def test_codes_bruteforce_optimal_tiny_groups(q):
    # For the chosen (sigma, z), the code vector attains the least squared error over
    # all (2^q)^g code vectors.
    g = 4
    N = 2 ** q - 1
    allc = np.array(list(product(range(N + 1), repeat=g)), dtype=np.float64)
    V = _groups(21 + q, 60, g)
    for v in V:
        c, sg, z = O.quantize_group(v, q)
        err = np.sum(((allc - z) * sg - v.astype(np.float64)) ** 2, axis=1)
        best = err.min()
        mine = np.sum(((c - z) * sg - v.astype(np.float64)) ** 2)
        assert mine <= best * (1 + 1e-12) + 1e-300


@pytest.mark.parametrize("q", [2, 3, 4])
def test_scale_and_zero_bruteforce(q):
    # sigma is the smallest fp16 value >= fl32(range/N); z is the integer in
    # [-2048, 2048] that puts the grid point (0 - z) sigma nearest to the group minimum.
    table = _fp16_table()
    N = 2 ** q - 1
    V = _groups(31 + q, 200, 32)
    for v in V:
        c, sg, z = O.quantize_group(v, q)
        rng = np.float32(v.max() - v.min())
        target = float(np.float32(rng / np.float32(N)))
        want = table[np.searchsorted(table, target, side="left")]
        assert sg == want
        zs = np.arange(-2048, 2049, dtype=np.float64)
        # distance measured in units of sigma on the fp32 quotient -min/sigma
        qv = float(np.float32(-v.min()) / np.float32(sg))
        dist = np.abs(zs - qv)
        cand = zs[dist == dist.min()]
        zwant = cand[0] if len(cand) == 1 else cand[cand % 2 == 0][0]
        assert z == zwant


@pytest.mark.parametrize("q,g", [(2, 32), (3, 32), (4, 64), (4, 128)])
def test_error_within_half_step(q, g):
    X, W = synthetic.draw_layer(64, 256, 48, seed=q * 10 + g)
    W = O.round_bf16(W)
    _, s32 = O.act_stats(O.round_bf16(X), 0.5, 0.4)
    codes, scale, zero = O.requant(W, s32, q, g)
    v = (W.astype(np.float32) * s32[None, :]).astype(np.float64)
    wq = O.dequant_scaled(codes, scale, zero, g)
    half = np.repeat(scale.astype(np.float64), g, axis=1) / 2
    assert np.all(np.abs(wq - v) <= half * (1 + 2.0 ** -20))
    assert codes.min() >= 0 and codes.max() <= 2 ** q - 1


def test_power_of_two_equivariance():
    X, W = synthetic.draw_layer(16, 128, 16, seed=41)
    W = O.round_bf16(W)
    s32 = np.ones(128, dtype=np.float32)
    c0, sc0, z0 = O.requant(W, s32, 4, 32)
    for k in (-3, 2, 5):
        c1, sc1, z1 = O.requant(W * 2.0 ** k, s32, 4, 32)
        np.testing.assert_array_equal(c0, c1)
        np.testing.assert_array_equal(z0, z1)
        np.testing.assert_array_equal(sc0.astype(np.float64) * 2.0 ** k, sc1.astype(np.float64))


@pytest.mark.parametrize("q", [2, 3, 4])
def test_exact_grid_roundtrip(q):
    rng = np.random.default_rng(50 + q)
    N = 2 ** q - 1
    n, g = 40, 32
    c = rng.integers(0, N + 1, (n, g))
    c[:, 0] = 0
    c[:, 1] = N
    sg = O.round_fp16_up(np.exp(rng.uniform(-8, 0, n))).astype(np.float32)
    z = rng.integers(-5, N + 5, n).astype(np.float64)
    v = ((c - z[:, None]) * sg[:, None].astype(np.float64)).astype(np.float32)
    codes, scale, zero = O.requant(v, np.ones(g, np.float32), q, g)
    np.testing.assert_array_equal(codes, c)
    np.testing.assert_array_equal(scale[:, 0].astype(np.float32), sg)
    np.testing.assert_array_equal(zero[:, 0].astype(np.float64), z)


def test_alpha_zero_reduces_to_rtn():
    # alpha = 0 makes D = I: the codes are those of plain round-to-nearest of W, i.e.
    # every weight sits on the grid point nearest to it.
    X, W = synthetic.draw_layer(32, 64, 12, seed=61)
    X, W = O.round_bf16(X), O.round_bf16(W)
    out = O.prefill(X, W, 3, 32, alpha=0.0, lam=0.4)
    np.testing.assert_array_equal(out["s32"], np.ones(64, np.float32))
    sg = np.repeat(out["scale"].astype(np.float64), 32, axis=1)
    zz = np.repeat(out["zero"].astype(np.float64), 32, axis=1)
    grid = (np.arange(8)[None, None, :] - zz[:, :, None]) * sg[:, :, None]
    nearest = np.argmin(np.abs(grid - W[:, :, None]), axis=2)
    dq = O.dequant_scaled(out["codes"], out["scale"], out["zero"], 32)
    best = np.take_along_axis(grid, nearest[:, :, None], 2)[:, :, 0]
    np.testing.assert_allclose(np.abs(dq - W), np.abs(best - W), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- packing


def test_packing_golden():
    for case in _load("packing_examples.json")["cases"]:
        codes = np.array(case["codes"], dtype=np.int64)[None, :]
        words = O.pack_codes(codes, case["q"])
        assert [int(w) for w in words[0]] == [int(h, 16) for h in case["words"]]
        np.testing.assert_array_equal(O.unpack_codes(words, case["q"], codes.shape[1]), codes)


@pytest.mark.parametrize("q", [2, 3, 4])
def test_packing_roundtrip(q):
    rng = np.random.default_rng(q)
    c = rng.integers(0, 2 ** q, (7, 256))
    w = O.pack_codes(c, q)
    assert w.shape == (7, 256 * q // 32)
    np.testing.assert_array_equal(O.unpack_codes(w, q, 256), c)


# ---------------------------------------------------------------- projection


def test_fold_associativity():
    # (w' diag(1/s)) X^T equals w' (diag(1/s) X^T) up to fp64 rounding
    X, W = synthetic.draw_layer(24, 128, 40, seed=71)
    X, W = O.round_bf16(X), O.round_bf16(W)
    out = O.prefill(X, W, 4, 32, 0.5, 0.4)
    Y1 = out["Y"]
    What = O.dequant_original(out["codes"], out["scale"], out["zero"], 32, out["s32"])
    Y2 = X @ What.T
    np.testing.assert_allclose(Y1, Y2, rtol=1e-11, atol=1e-11 * np.abs(Y1).max())


def test_linear_bruteforce_loops():
    rng = np.random.default_rng(72)
    T, d, d_out, g = 2, 32, 3, 32
    X = O.round_bf16(rng.standard_normal((T, d)))
    s = np.float32(rng.uniform(0.5, 2.0, d))
    codes = rng.integers(0, 16, (d_out, d))
    scale = np.float16(rng.uniform(0.01, 0.1, (d_out, 1)))
    zero = np.float16(rng.integers(0, 16, (d_out, 1)))
    A = O.round_bf16(rng.standard_normal((2, d)))
    B = O.round_bf16(rng.standard_normal((d_out, 2)))
    Y = O.linear(X, s, codes, scale, zero, g, A, B)
    for t in range(T):
        for i in range(d_out):
            acc = 0.0
            for k in range(d):
                w = (float(codes[i, k]) - float(zero[i, 0])) * float(scale[i, 0])
                acc += float(X[t, k]) / float(s[k]) * w
            for r in range(2):
                u = sum(float(A[r, k]) * float(X[t, k]) for k in range(d))
                acc += float(B[i, r]) * u
            assert abs(Y[t, i] - acc) <= 1e-12 * max(1.0, abs(acc))


def test_lowrank_split_eckart_young():
    X, W = synthetic.draw_layer(8, 96, 64, seed=81)
    B, A, R = O.lowrank_split(W, 16)
    sv = np.linalg.svd(W, compute_uv=False)
    tail = np.sum(sv[16:] ** 2)
    err = np.sum((W - B @ A) ** 2)
    assert abs(err - tail) <= 0.02 * tail
    assert np.allclose(R, O.round_bf16(R))


def test_lowrank_exact_rank_residual_is_small_and_output_matches():
    rng = np.random.default_rng(82)
    B0 = rng.standard_normal((48, 8))
    A0 = rng.standard_normal((8, 64))
    W = B0 @ A0
    B, A, R = O.lowrank_split(W, 8)
    assert np.linalg.norm(R) <= 2.0 ** -7 * np.linalg.norm(W)
    X = O.round_bf16(rng.standard_normal((5, 64)))
    out = O.prefill(X, R, 4, 32, 0.5, 0.4, A=A, B=B)
    np.testing.assert_allclose(out["Y"], X @ W.T, rtol=0, atol=2e-2 * np.abs(X @ W.T).max())


def test_overhead_rho_law():
    for T, d, dp in [(16, 5120, 8192), (4096, 5120, 8192), (128, 768, 3072)]:
        c = O.overhead_counts(T, d, dp)
        assert Fraction(c["stats"] + c["requant"], c["gemm"]) == Fraction(1, dp) + Fraction(3, T)
    # the overhead falls as 1/T at fixed shape (the 3/T term dominates for large d')
    r = [O.overhead_counts(T, 5120, 8192)["rho"] for T in (128, 1024, 4096)]
    assert r[0] > r[1] > r[2]


def test_ttq_lowers_activation_loss_against_rtn():
    # The pages' method-level claim: activation-aware scaling lowers ||(W - W_hat) X||
    # against plain RTN on outlier-heavy activations. Reported, and checked on the
    # small synthetic layer.
    X, W = synthetic.draw_layer(128, 512, 512, seed=0)
    X, W = O.round_bf16(X), O.round_bf16(W)
    losses = {}
    for name, alpha in (("rtn", 0.0), ("ttq", 0.5)):
        out = O.prefill(X, W, 3, 32, alpha, 0.4)
        What = O.dequant_original(out["codes"], out["scale"], out["zero"], 32, out["s32"])
        losses[name] = O.activation_loss(W, What, X)
    assert losses["ttq"] < losses["rtn"]


# ---------------------------------------------------------------- activation-weighted loss


def test_activation_loss_golden():
    # hand-worked cases: a transposed operand, a dropped square, a missing cross term or a
    # mean instead of a sum each gives one of the recorded wrong values instead
    for case in _load("activation_loss_examples.json")["cases"]:
        L = O.activation_loss(np.array(case["W"]), np.array(case["W_hat"]), np.array(case["X"]))
        assert L == case["loss"], case
        for wrong in case.get("wrong_readings", {}).values():
            assert wrong != case["loss"]


def test_activation_loss_equals_per_token_output_error():
    # L sums, over tokens, the squared output error of the layer: ||W x_t - W_hat x_t||^2
    rng = np.random.default_rng(91)
    W, Wh = rng.standard_normal((5, 7)), rng.standard_normal((5, 7))
    X = rng.standard_normal((4, 7))
    want = sum(float(np.sum((W @ X[t] - Wh @ X[t]) ** 2)) for t in range(4))
    assert abs(O.activation_loss(W, Wh, X) - want) <= 1e-12 * want


# ---------------------------------------------------------------- fold


def test_fold_exact_rational():
    # X' = RN_bf16(x / s): against the nearest bf16 value to the exact rational quotient,
    # found among its two neighbours, ties to the even significand
    rng = np.random.default_rng(92)
    x = O.round_bf16(rng.standard_normal(400) * np.exp(rng.uniform(-6, 6, 400)))
    s = rng.uniform(0.05, 20.0, 400).astype(np.float32)
    got = O.fold(x[None, :], s)[0]
    for xi, si, gi in zip(x, s, got):
        fq = Fraction(float(xi)) / Fraction(float(si))
        if fq == 0:
            assert gi == 0
            continue
        _, e = np.frexp(float(fq))
        q = Fraction(2) ** (int(e) - 8)
        lo = (fq / q).__floor__() * q
        hi = lo + q
        if fq - lo < hi - fq:
            want = lo
        elif hi - fq < fq - lo:
            want = hi
        else:
            want = lo if (lo / q) % 2 == 0 else hi
        assert Fraction(float(gi)) == want, (xi, si)


def test_fold_hand_values():
    # 1/3 = 1.0101010101...b x 2^-2: the ninth significant bit and those after it are more
    # than half an ulp, so it rounds up to 1.0101011b x 2^-2 = 0.333984375; 6/4 = 1.5 is exact;
    # 1 / 1.0078125 lies between 0.9921875 and 0.99609375, nearer the former
    X = np.array([[1.0, 6.0, 1.0]])
    s = np.array([3.0, 4.0, 1.0078125], dtype=np.float32)
    np.testing.assert_array_equal(O.fold(X, s), [[0.333984375, 1.5, 0.9921875]])
