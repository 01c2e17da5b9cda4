"""The host set-up of the low-rank side path (``lowrank_setup.lowrank_factors``, run once
per weight before any prompt) against the oracle's split (``oracle.lowrank_split``): the
same truncated SVD with the square root of the singular values on each side, factors and
residual rounded to bf16. CPU only."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from online_activation_aware_b200 import synthetic
from online_activation_aware_b200.lowrank_setup import lowrank_factors
from oracle import ttq_oracle as O


def _ulp_bf16(x):
    # spacing of bf16 numbers at |x| (8 significant bits)
    _, e = np.frexp(np.abs(x))
    return np.ldexp(1.0, e - 8)


@pytest.mark.parametrize("d_out,d,r", [(64, 96, 16), (200, 128, 8), (96, 320, 24)])
def test_lowrank_factors_match_oracle_split(d_out, d, r):
    _, W = synthetic.draw_layer(4, d, d_out, seed=d_out + d + r)
    Wb = synthetic.as_bf16(W)
    Wv = synthetic.bf16_values(Wb)
    B, A, R = (synthetic.bf16_values(t) for t in lowrank_factors(Wb, r))
    Bo, Ao, Ro = O.lowrank_split(Wv, r)
    assert B.shape == (d_out, r) and A.shape == (r, d) and R.shape == (d_out, d)
    # singular vectors are unique up to a joint sign per component: align them first
    sign = np.sign(np.sum(B * Bo, axis=0))
    assert np.all(sign != 0)
    B, A = B * sign[None, :], A * sign[:, None]
    # two LAPACK calls may differ in the last bits before the bf16 rounding, so a value
    # may land one bf16 step away; nearly all agree exactly
    for got, want in ((B, Bo), (A, Ao), (R, Ro)):
        diff = np.abs(got - want)
        assert np.all(diff <= _ulp_bf16(np.maximum(np.abs(got), np.abs(want))) * (1 + 1e-12) + 1e-30)
        assert np.mean(diff == 0) >= 0.99
    # the split reconstructs W to the rank-r residual plus bf16 rounding
    np.testing.assert_allclose(B @ A + R, Wv, rtol=0, atol=4 * np.abs(Wv).max() * 2.0 ** -8)


def test_lowrank_factors_rejects_bad_rank():
    W = torch.zeros(8, 16, dtype=torch.bfloat16)
    for r in (0, 9):
        with pytest.raises(ValueError):
            lowrank_factors(W, r)
