"""The measured overhead ratio against the pages' count rho = (dT + 3d'd) / (d'dT) =
1/d' + 3/T (gist.science French summary, section 2A: O(dT + 3d'd) extra against O(d'dT);
German summary, section 2: rho ~ O(1/d' + 3/T)).

Measured times weight the kinds of operation differently (statistic and fold stream X,
the requant streams W, the projection runs on tensor cores), so the count holds, as
times, in its structure: the overhead t_stats + t_fold_requant is a constant (the 3d'd
requant) plus a term linear in T (dT), the projection's time is proportional to T, and
rho falls with T. (rho alone cannot tell 1/T from, say, 1/sqrt(T) over a 16x range of T
once the constant term is in.) The check is pinned on CPU against the count itself and
against cost structures that break it; the GPU test measures the stages through the
library's stage events at T = 2048 .. 16384 (5120 -> 8192), where the projection runs at
its tensor-core rate.
"""

import statistics

import pytest


def rho_model(T, d_out):
    return 1.0 / d_out + 3.0 / T


def affine_fit(xs, ys):
    """Least-squares y = a + b x with relative residuals (each point weighted by 1 / y).
    Returns (a, b, largest relative residual)."""
    import numpy as np

    x = np.asarray(xs, dtype=np.float64)
    y = np.asarray(ys, dtype=np.float64)
    A = np.stack([np.ones_like(x), x], axis=1) / y[:, None]
    (a, b), *_ = np.linalg.lstsq(A, np.ones_like(y), rcond=None)
    return float(a), float(b), float(np.max(np.abs(a + b * x - y) / y))


def follows_count(stages, tol=0.1, tol_proj=0.25):
    """stages: {T: (t_overhead, t_projection)} at fixed shape. The count (dT + 3d'd) / (d'dT)
    holds, as times, when the overhead is an affine function of T (within `tol`) whose
    constant (the 3d'd requant) and linear part (the dT statistic and fold) both carry at
    least a tenth of the overhead at the ends of the range, the projection's time per token
    is constant (within `tol_proj`: clocks drift over long runs), and so rho = overhead /
    projection falls with T."""
    Ts = sorted(stages)
    over = [stages[T][0] for T in Ts]
    a, b, res = affine_fit(Ts, over)
    per_token = [stages[T][1] / T for T in Ts]
    rho = [stages[T][0] / stages[T][1] for T in Ts]
    both_terms = a >= 0.1 * over[0] and b * Ts[-1] >= 0.1 * over[-1]
    return (both_terms and res <= tol and max(per_token) / min(per_token) <= 1 + tol_proj
            and all(x > y for x, y in zip(rho, rho[1:])))


TS = (2048, 4096, 8192, 16384)


def test_pages_count_as_times_follows_the_count():
    # the count itself, each operation costing one unit (5120 -> 8192)
    d, dp = 5120, 8192
    assert follows_count({T: (d * T + 3 * dp * d, dp * d * T) for T in TS})


def test_measured_like_costs_follow_the_count():
    # per-op costs like the measured ones: 35 us of requant, 5.6 ns per token of statistic
    # and fold, 75 ns per token of projection
    assert follows_count({T: (35.0 + 5.6e-3 * T, 75e-3 * T) for T in TS})


@pytest.mark.parametrize("stages", [
    {T: (40.0, 75e-3 * T) for T in TS},                       # overhead without a dT term
    {T: (5.6e-3 * T, 75e-3 * T) for T in TS},                 # overhead without the constant
    {T: (35.0 + 4e-7 * T * T, 75e-3 * T) for T in TS},        # overhead growing as T^2
    {T: (35.0 + 5.6e-3 * T, 2e-5 * T ** 1.5) for T in TS},    # projection not linear in T
])
def test_costs_off_the_count_fail(stages):
    assert not follows_count(stages)


@pytest.mark.gpu
def test_measured_rho_follows_the_count():
    torch = pytest.importorskip("torch")
    import online_activation_aware_b200 as ttq
    from online_activation_aware_b200 import synthetic

    d, d_out, q, g = 5120, 8192, 4, 128
    cfg = ttq.make_config(q, g, 0.5, 0.4)
    W = synthetic.as_bf16(synthetic.draw_layer(1, d, d_out, seed=3)[1]).cuda()
    stages = {}
    for T in TS:
        X = synthetic.as_bf16(synthetic.draw_layer(T, d, 1, seed=600 + T)[0]).cuda()
        ws = ttq.alloc_workspace(T, d, d_out, cfg)
        out = ttq.linear_prefill(X, W, cfg, ws=ws)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(8)]
        for e in evs:
            ttq.set_trace_events(e)
            ttq.linear_prefill(X, W, cfg, out=out, ws=ws)
        torch.cuda.synchronize()
        ttq.set_trace_events(None)
        med = lambda a, b: statistics.median(e[a].elapsed_time(e[b]) for e in evs)  # noqa: E731
        stages[T] = (med(0, 1) + med(2, 3), med(3, 5))
        del X, ws, out
    assert ttq.device_status() == 0
    assert follows_count(stages), stages
