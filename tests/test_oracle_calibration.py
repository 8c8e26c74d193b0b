"""Pins of the temperature-scaling oracle (oracle/calibration.py)."""
import numpy as np
import pytest
from scipy.optimize import minimize_scalar
from scipy.special import expit

from oracle.calibration import (BETA_HI, BETA_LO, calibrate_ref, fit_temperature_ref,
                                outcomes_from_accept)


def test_tau_one_is_the_logistic_function_and_symmetric():
    rng = np.random.default_rng(0)
    l = rng.normal(0, 4, size=(50, 5)).astype(np.float32)
    np.testing.assert_allclose(calibrate_ref(l, np.ones(5)), expit(l.astype(np.float64)),
                               rtol=1e-6)
    tau = np.array([0.5, 1, 2, 4, 8], np.float32)
    c, cm = calibrate_ref(l, tau), calibrate_ref(-l, tau)
    np.testing.assert_allclose(c + cm, 1.0, atol=1e-6)
    # a larger temperature pulls every confidence towards 1/2
    big = calibrate_ref(l, tau * 10)
    assert np.all(np.abs(big - 0.5) <= np.abs(c - 0.5) + 1e-7)


def test_outcomes_follow_the_accepted_prefix():
    y = outcomes_from_accept([5, 5, 3, 0, 2], [2, 5, 0, 0, 2], 5)
    np.testing.assert_array_equal(y, [[1, 1, 0, -1, -1], [1, 1, 1, 1, 1], [0, -1, -1, -1, -1],
                                      [-1, -1, -1, -1, -1], [1, 1, -1, -1, -1]])


def _simulate(tau_true, n, rng, K=5):
    """Requests whose drafts survive position k with probability sigmoid(l_true); the head
    reports l_raw = l_true * tau_true (over-confident for tau_true > 1)."""
    l_true = rng.normal(1.5, 1.5, size=(n, K)) - 0.3 * np.arange(K)
    l_raw = (l_true * np.asarray(tau_true)[None, :]).astype(np.float32)
    p = expit(l_raw.astype(np.float64) / np.asarray(tau_true)[None, :])
    acc_draw = rng.random((n, K)) < p
    L = rng.integers(0, K + 1, size=n)
    a = np.zeros(n, dtype=np.int64)
    for i in range(n):
        while a[i] < L[i] and acc_draw[i, a[i]]:
            a[i] += 1
    return l_raw, L, a


def test_planted_temperature_is_recovered():
    rng = np.random.default_rng(1)
    tau_true = np.array([1.0, 1.5, 2.0, 2.5, 3.0])
    l_raw, L, a = _simulate(tau_true, 200_000, rng)
    tau = fit_temperature_ref(l_raw, L, a, 5)
    np.testing.assert_allclose(tau, tau_true, rtol=0.04)


def test_fit_is_the_likelihood_minimiser_of_a_library_routine():
    rng = np.random.default_rng(2)
    l_raw, L, a = _simulate([2.0] * 5, 3000, rng)
    tau = fit_temperature_ref(l_raw, L, a, 5)
    y = outcomes_from_accept(L, a, 5)
    for k in range(5):
        obs = y[:, k] >= 0
        l = l_raw[obs, k].astype(np.float64)
        s = np.where(y[obs, k] == 1, 1.0, -1.0)
        nll = lambda b: np.logaddexp(0.0, -s * b * l).sum()
        best = minimize_scalar(nll, bounds=(BETA_LO, BETA_HI), method="bounded",
                               options={"xatol": 1e-10})
        np.testing.assert_allclose(1.0 / tau[k], best.x, rtol=1e-6)


def test_censoring_ignores_positions_never_verified():
    rng = np.random.default_rng(3)
    l_raw, L, a = _simulate([1.5] * 5, 5000, rng)
    tau = fit_temperature_ref(l_raw, L, a, 5)
    l2 = l_raw.copy()
    y = outcomes_from_accept(L, a, 5)
    l2[y < 0] = rng.normal(0, 50, size=int((y < 0).sum()))   # unobserved entries: anything
    np.testing.assert_array_equal(fit_temperature_ref(l2, L, a, 5), tau)


def test_degenerate_positions_keep_tau_one_or_hit_the_bounds():
    L = np.array([1, 1, 1, 1])
    a = np.array([1, 1, 1, 1])                 # position 1 always accepted, 2..5 never observed
    l = np.ones((4, 5), np.float32)
    tau = fit_temperature_ref(l, L, a, 5)
    assert tau[0] == pytest.approx(1.0 / BETA_HI)   # separable: as confident as allowed
    np.testing.assert_array_equal(tau[1:], 1.0)
    l0 = np.zeros((4, 5), np.float32)
    np.testing.assert_array_equal(fit_temperature_ref(l0, L, a, 5), 1.0)
