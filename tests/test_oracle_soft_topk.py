"""Pins of the oracle's SoftTop-k ("SLA2: Sparse-Linear Attention with Learnable
Routing and QAT", §4 Learnable Router and §6 Training with SLA2: a sigmoid with
temperature tau and a per-row threshold lambda_i found by binary search, so that
every row keeps the Top-k row sum).

Each pin holds independently of the oracle's bisection: an independent root
finder (Brent's method) for lambda_i, the closed form of a constant row, the
hard Top-k (pinned in test_oracle_pins.py) as tau -> 0, and the scale
invariance that a misplaced tau would break.
"""
import numpy as np
import pytest
from scipy.optimize import brentq
from scipy.special import expit

import oracle as O


def _rows(seed, R=6, T=48, scale=2.0):
    g = np.random.default_rng(seed)
    return O.compressed_attention(g.standard_normal((R, T)) * scale)


@pytest.mark.parametrize("tau", [0.002, 0.01, 0.1])
@pytest.mark.parametrize("n_h", [1, 5, 20])
def test_lambda_is_the_root_brent_finds(tau, n_h):
    P = _rows(3)
    M, lam = O.soft_topk(P, n_h, tau)
    for r in range(P.shape[0]):
        g = lambda x: expit((P[r] - x) / tau).sum() - n_h  # noqa: E731
        ref = brentq(g, P[r].min() - 60 * tau, P[r].max() + 60 * tau, xtol=1e-15, rtol=1e-15)
        # lambda is only as determined as f's slope allows (a row whose top
        # value stands far above the rest leaves f flat around its root): the
        # difference times the slope is what moves the row sum
        s = expit((P[r] - ref) / tau)
        slope = (s * (1 - s)).sum() / tau
        assert abs(lam[r] - ref) * slope <= 1e-9
        np.testing.assert_allclose(M[r], s, atol=1e-9)
        assert abs(M[r].sum() - n_h) < 1e-8


def test_constant_row_closed_form():
    # sigmoid((c - lambda) / tau) = n_h / T  =>  lambda = c - tau * logit(n_h / T)
    T, n_h, tau, c = 64, 7, 0.05, 0.3
    M, lam = O.soft_topk(np.full((1, T), c), n_h, tau)
    q = n_h / T
    np.testing.assert_allclose(M, q, atol=1e-12)
    assert abs(lam[0] - (c - tau * np.log(q / (1 - q)))) < 1e-12


def test_small_tau_gives_the_hard_topk():
    P = _rows(5, R=8, T=64)
    n_h = 6
    hard = O.classify(P, n_h, 0) == 1
    srt = -np.sort(-P, axis=1)
    gap = (srt[:, n_h - 1] - srt[:, n_h]).min()  # distinct values around the cut in every row
    assert gap > 0
    M, _ = O.soft_topk(P, n_h, gap / 400)
    np.testing.assert_allclose(M, hard.astype(np.float64), atol=1e-12)


def test_temperature_is_on_the_score_scale():
    # (P - lambda) / tau is unchanged when P and tau are scaled together
    P = _rows(7)
    M1, l1 = O.soft_topk(P, 4, 0.01)
    M2, l2 = O.soft_topk(3.0 * P, 4, 0.03)
    np.testing.assert_allclose(M2, M1, atol=1e-10)
    np.testing.assert_allclose(l2, 3.0 * l1, rtol=1e-9)


def test_order_preserving_and_bounded():
    P = _rows(11, R=4, T=100)
    M, _ = O.soft_topk(P, 10, 0.02)
    assert np.all((M > 0) & (M < 1))
    for r in range(P.shape[0]):
        o = np.argsort(P[r])
        assert np.all(np.diff(M[r, o]) >= 0)


def test_all_blocks_kept_and_bad_tau():
    P = _rows(13, R=2, T=16)
    M, _ = O.soft_topk(P, 16, 0.01)  # n_h = T: every weight -> 1
    assert np.all(M > 1 - 1e-12)
    with pytest.raises(ValueError):
        O.soft_topk(P, 3, 0.0)
