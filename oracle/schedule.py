"""Oracle: survival scan, greedy marginal-gain prefix scheduler, flattening with markers.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

What the pages fix and the readings taken:
  * [P2 §3.2] The confidence at draft position k answers "given that every earlier token was
    accepted, how likely is this one to be accepted" — a conditional survival probability.
    [P4 "置信度计划、负载感知验证"] calls the calibrated prefix estimate a survival
    probability.  Reading: S[r,k] = c[r,1] * ... * c[r,k], multiplied left to right.
  * [P2 §3.2] The scheduler's inputs are the load, the per-position confidences and the
    engine's throughput curve over batch sizes.  [P3 "DSpark的神奇之处"] it measures the
    engine's speed at each batch size ahead of time, queues every request's draft tokens by
    score from high to low, and keeps adding the next ones while the time they cost is paid
    for by the correct tokens they are expected to add.  Reading: per-candidate greedy over
    the candidates sorted by S (descending; ties by position k ascending, then request r
    ascending), objective f(n) = (R + top-n sum of S) / t_ms[R + n]; add candidate n+1 iff
    f(n+1) > f(n) strictly, stop at the first non-improvement.  R counts the one correction
    or bonus token every request emits; T = R + n tokens are verified.
  * [P1 engineering table, "GPU流水线停滞"] the asynchronous scheduler uses the confidences
    of two rounds earlier.  Rounds 0 and 1 use round 0's.
  * [P1 engineering table, "内核利用率暴跌"] all verify tokens are flattened into independent
    elements and a marker tensor carries sequence membership and position.  Reading:
    markers[t] = (request r, absolute position kv_len[r] + j) for the j-th verify token of r;
    requests are laid out contiguously in request order.

Parity: decisions pinned by brute force over all length assignments (R <= 4), closed forms
(flat table -> every candidate, per-token cost >= 1 -> none) and invariants.
"""
from __future__ import annotations

import itertools

import numpy as np

CONF_LAG = 2            # confidences are consumed two rounds after they are produced
# A scan comparison is flagged when f(n+1) and f(n) lie closer than any two float64 summation
# orders of the (positive) survival terms could move them apart: every order's prefix sum is
# within gamma_N * P of the exact one (gamma_N = N u / (1 - N u), u = 2**-53), so two orders
# differ by at most 2 gamma_N P, plus the rounding of the division.  For N <= 16384 candidates
# that is below 1e-11 relative.
FLAG_REL = 1e-11


def lagged_round(round_idx: int) -> int:
    """Round whose confidences round `round_idx` is scheduled with."""
    return max(round_idx - CONF_LAG, 0)


def survival_ref(conf) -> np.ndarray:
    """S[r,k] = prod_{j<=k} c[r,j] in float64, multiplied left to right."""
    c = np.asarray(conf, dtype=np.float32).astype(np.float64)
    if c.ndim != 2:
        raise ValueError("conf must be [R][K]")
    if not np.all((c >= 0.0) & (c <= 1.0)):
        raise ValueError("confidences must lie in [0, 1]")
    S = np.empty_like(c)
    acc = np.ones(c.shape[0], dtype=np.float64)
    for k in range(c.shape[1]):
        acc = acc * c[:, k]
        S[:, k] = acc
    return S


def candidate_order(S: np.ndarray):
    """All (r, k) candidates sorted by S descending, then k ascending, then r ascending.

    Candidate index i = k * R + r.  Returns (order, s, r_of, k_of) with s[i] = S[r, k].
    """
    R, K = S.shape
    r_of = np.tile(np.arange(R), K)
    k_of = np.repeat(np.arange(K), R)
    s = S.T.reshape(-1)
    order = np.lexsort((r_of, k_of, -s))
    return order, s, r_of, k_of


def flatten_ref(verify_len, kv_len):
    """q_offsets = exclusive scan of Q_r = 1 + L_r; markers[q_offsets[r] + j] = (r, kv_len[r] + j)."""
    L = np.asarray(verify_len, dtype=np.int64)
    n = np.asarray(kv_len, dtype=np.int64)
    R = len(L)
    q_offsets = np.zeros(R + 1, dtype=np.int32)
    q_offsets[1:] = np.cumsum(1 + L)
    T = int(q_offsets[-1])
    markers = np.zeros((T, 2), dtype=np.int32)
    for r in range(R):
        for j in range(int(L[r]) + 1):
            markers[q_offsets[r] + j] = (r, n[r] + j)
    return q_offsets, markers


def schedule_ref(conf, kv_len, t_ms, T_cap: int) -> dict:
    """Greedy marginal-gain prefix schedule of one verify round.

    conf: float32 [R][K], the (already lagged) confidences; kv_len: int [R];
    t_ms: float64 step-time table for T = 0..T_cap; T_cap: largest verifiable batch.
    Returns verify_len, q_offsets, markers, T, n_star, objective f(n*), the f curve and the
    flag: True when any comparison the scan made lies within FLAG_REL of a tie.
    """
    S = survival_ref(conf)
    R, K = S.shape
    t = np.asarray(t_ms, dtype=np.float64)
    if T_cap < R:
        raise ValueError("T_cap must allow one verify token per request")
    if len(t) < T_cap + 1 or not np.all(t[:T_cap + 1] > 0):
        raise ValueError("t_ms must hold positive times for T = 0..T_cap")
    order, s, r_of, _ = candidate_order(S)
    s_sorted = s[order]
    n_max = min(R * K, T_cap - R)

    P = np.zeros(n_max + 1, dtype=np.float64)     # P[n] = s_(1) + ... + s_(n), left to right
    for n in range(1, n_max + 1):
        P[n] = P[n - 1] + s_sorted[n - 1]
    f = np.empty(n_max + 1, dtype=np.float64)
    for n in range(n_max + 1):
        f[n] = (float(R) + P[n]) / t[R + n]

    n_star = n_max
    flagged = False
    for n in range(n_max):
        if abs(f[n + 1] - f[n]) < FLAG_REL * f[n]:
            flagged = True
        if not (f[n + 1] > f[n]):
            n_star = n
            break

    L = np.zeros(R, dtype=np.int32)
    for i in order[:n_star]:
        L[r_of[i]] += 1
    q_offsets, markers = flatten_ref(L, kv_len)
    return dict(S=S, verify_len=L, q_offsets=q_offsets, markers=markers,
                T=int(q_offsets[-1]), n_star=int(n_star), objective=float(f[n_star]),
                f=f, flagged=flagged)


def schedule_bruteforce(conf, t_ms, T_cap: int):
    """Exhaustive maximum of F(L) = (R + sum_r sum_{k<=L_r} S[r,k]) / t_ms[R + sum L] over
    every assignment L in [0, K]^R with R + sum L <= T_cap (use for R <= 4)."""
    S = survival_ref(conf)
    R, K = S.shape
    t = np.asarray(t_ms, dtype=np.float64)
    prefix = np.concatenate([np.zeros((R, 1)), np.cumsum(S, axis=1)], axis=1)
    best, best_L = -np.inf, None
    for L in itertools.product(range(K + 1), repeat=R):
        T = R + sum(L)
        if T > T_cap:
            continue
        F = (R + sum(prefix[r, L[r]] for r in range(R))) / t[T]
        if F > best:
            best, best_L = F, np.array(L, dtype=np.int32)
    return float(best), best_L
