"""Temporal temperature scaling of the confidence head — oracle (TEST INFRASTRUCTURE ONLY).

[P1] section "2. 置信度调度验证": the confidence head estimates each draft token's survival
probability given its prefix, and after training a post-hoc calibration, "temporal temperature
scaling" (时序温度缩放), corrects the raw head's over-confidence.  [P2] §3.2: the confidence of
block position k is the probability that the token is accepted given that the prefix before it
was accepted.

Readings (the pages give only the name; listed in the design notes):
  * one temperature per block position k ("temporal" = along the draft block):
    c_k = sigmoid(l_k / tau_k) for the raw confidence logit l_k;
  * tau_k is fitted by maximum likelihood on observed accept outcomes: a request verified with
    L drafts of which a were accepted observes position k (1-based) iff k <= min(a + 1, L);
    the outcome is "accepted" for k <= a and "rejected" for k = a + 1 <= L; later positions are
    censored (the verifier never saw them with an accepted prefix);
  * the fit is over beta = 1 / tau in [1/64, 64] (the negative log-likelihood is convex in
    beta); a position with no observations, or whose observed logits are all zero, keeps tau = 1.

Parity: calibrate_ref within float32 rounding; fit_temperature_ref is the exact minimiser
(bisection on the monotone derivative to 1e-13 in beta), the GPU's bracketed Newton iteration
must land within 1e-5 relative.  Pinned by tests/test_oracle_calibration.py (tau = 1 equals the
library logistic function, symmetry, recovery of a planted temperature from 2e5 synthetic
outcomes, the derivative of the likelihood computed by a library minimiser, censoring).
"""
from __future__ import annotations

import numpy as np

BETA_LO, BETA_HI = 1.0 / 64.0, 64.0


def calibrate_ref(logits, tau) -> np.ndarray:
    """c[r, k] = sigmoid(logits[r, k] / tau[k]) in float64 (returned as float32)."""
    l = np.asarray(logits, dtype=np.float32).astype(np.float64)
    t = np.asarray(tau, dtype=np.float32).astype(np.float64)
    x = l / t[None, :]
    return (1.0 / (1.0 + np.exp(-x))).astype(np.float32)


def outcomes_from_accept(verify_len, accepted_len, K: int) -> np.ndarray:
    """y[i, k] = 1 (position k+1 accepted), 0 (rejected), -1 (not observed)."""
    L = np.asarray(verify_len, dtype=np.int64)
    a = np.asarray(accepted_len, dtype=np.int64)
    y = np.full((len(L), K), -1, dtype=np.int8)
    for i in range(len(L)):
        for k in range(1, K + 1):
            if k <= a[i]:
                y[i, k - 1] = 1
            elif k == a[i] + 1 and k <= L[i]:
                y[i, k - 1] = 0
    return y


def _nll_grad(beta: float, l: np.ndarray, s: np.ndarray) -> float:
    # NLL(beta) = sum log(1 + exp(-s * beta * l)); d/dbeta = -sum s * l * sigmoid(-s * beta * l)
    z = -s * beta * l
    sig = np.exp(-np.logaddexp(0.0, -z))     # sigmoid(z) without overflow
    return float(-(s * l * sig).sum())


def fit_temperature_ref(logits, verify_len, accepted_len, K: int) -> np.ndarray:
    """tau[k] minimising the observed outcomes' negative log-likelihood under
    c = sigmoid(l / tau), per block position, beta = 1 / tau clamped to [BETA_LO, BETA_HI]."""
    l_all = np.asarray(logits, dtype=np.float32).astype(np.float64)
    y = outcomes_from_accept(verify_len, accepted_len, K)
    tau = np.ones(K, dtype=np.float64)
    for k in range(K):
        obs = y[:, k] >= 0
        l = l_all[obs, k]
        s = np.where(y[obs, k] == 1, 1.0, -1.0)
        if l.size == 0 or not np.any(l != 0.0):
            continue
        lo, hi = BETA_LO, BETA_HI
        if _nll_grad(lo, l, s) >= 0.0:
            beta = lo
        elif _nll_grad(hi, l, s) <= 0.0:
            beta = hi
        else:
            while hi - lo > 1e-13 * hi:
                mid = 0.5 * (lo + hi)
                if _nll_grad(mid, l, s) < 0.0:
                    lo = mid
                else:
                    hi = mid
            beta = 0.5 * (lo + hi)
        tau[k] = 1.0 / beta
    return tau
