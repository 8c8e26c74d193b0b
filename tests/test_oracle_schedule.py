"""Pins for the scheduler oracle: closed forms, brute force, invariants, the pages' worked scores."""
import math

import numpy as np
import pytest

from oracle.schedule import (candidate_order, flatten_ref, lagged_round, schedule_bruteforce,
                             schedule_ref, survival_ref)
from workloads.configs import SWEEP_LEVELS, TINY, sweep_config
from workloads.generate import confidences, kv_lengths, step_time_table


def _rand_conf(rng, R, K, lo=0.05, hi=0.99):
    return rng.uniform(lo, hi, size=(R, K)).astype(np.float32)


def test_survival_is_product_of_conditionals():
    rng = np.random.default_rng(1)
    c = _rand_conf(rng, 50, 5)
    S = survival_ref(c)
    # independent closed form: exp of the summed logs
    want = np.exp(np.cumsum(np.log(c.astype(np.float64)), axis=1))
    assert np.allclose(S, want, rtol=1e-13, atol=0)
    assert np.array_equal(S[:, 0], c[:, 0].astype(np.float64))
    assert np.all(np.diff(S, axis=1) <= 0)


def test_survival_rejects_out_of_range():
    with pytest.raises(ValueError):
        survival_ref(np.array([[0.5, 1.5]], dtype=np.float32))
    with pytest.raises(ValueError):
        survival_ref(np.array([[0.5, np.nan]], dtype=np.float32))


def test_candidate_order_tiebreak():
    # exact ties in S: order must be k ascending, then r ascending
    c = np.array([[0.5, 1.0], [0.5, 1.0], [0.25, 1.0]], dtype=np.float32)
    S = survival_ref(c)
    order, s, r_of, k_of = candidate_order(S)
    got = [(int(r_of[i]), int(k_of[i])) for i in order]
    assert got == [(0, 0), (1, 0), (0, 1), (1, 1), (2, 0), (2, 1)]


def test_lag_two_rounds():
    assert [lagged_round(i) for i in range(6)] == [0, 0, 0, 1, 2, 3]


def test_flat_table_takes_everything():
    # t constant: any candidate with s > 0 strictly raises expected tokens per time
    rng = np.random.default_rng(2)
    c = _rand_conf(rng, 7, 5)
    res = schedule_ref(c, np.full(7, 10), np.full(43, 3.0), 42)
    assert np.all(res["verify_len"] == 5)
    assert res["T"] == 42


def test_unit_cost_per_token_takes_nothing():
    # t(T) = T: adding s <= 1 at cost 1 never raises (R + A) / (R + n)   (closed form)
    rng = np.random.default_rng(3)
    c = _rand_conf(rng, 9, 5)
    t = np.arange(55, dtype=np.float64)
    t[0] = 1.0
    res = schedule_ref(c, np.zeros(9, dtype=np.int32), t, 54)
    assert np.all(res["verify_len"] == 0)
    assert res["T"] == 9 and res["n_star"] == 0


@pytest.mark.parametrize("lam,want_L", [(0.1, 3), (0.3, 2), (0.95, 0), (0.0, 4)])
def test_worked_scores_from_the_pages(lam, want_L):
    """One request whose draft tokens score 90, 80, 60 and 30 (the illustration in
    "DeepSeek服务器不再卡顿！DSpark加速60% - 80%，推理成本降40%", section "DSpark的神奇之处"),
    read as conditional confidences, with step time t(T) = 1 + lam * (T - 1).

    Hand derivation: adding the n+1-th token raises (1 + A_n) / (1 + lam*n) iff
    s_{n+1} * (1 + lam*n) > lam * (1 + A_n).  S = 0.9, 0.72, 0.432, 0.1296.
      lam = 0.1: 0.9 > 0.1; 0.792 > 0.19; 0.5184 > 0.262; 0.16848 < 0.3052  -> L = 3
      lam = 0.3: 0.9 > 0.3; 0.936 > 0.57; 0.6912 < 0.786                    -> L = 2
      lam = 0.95: 0.9 < 0.95                                                   -> L = 0
      lam = 0:    flat table                                                   -> L = 4
    """
    c = np.array([[0.9, 0.8, 0.6, 0.3]], dtype=np.float32)
    t = 1.0 + lam * (np.arange(6, dtype=np.float64) - 1.0)
    t[0] = 1.0
    res = schedule_ref(c, np.array([100]), t, 5)
    assert int(res["verify_len"][0]) == want_L


@pytest.mark.parametrize("seed", range(12))
def test_greedy_matches_bruteforce(seed):
    rng = np.random.default_rng(100 + seed)
    R = int(rng.integers(1, 5))
    K = 5
    c = _rand_conf(rng, R, K, 0.02, 0.999)
    T_cap = R * (K + 1)
    kind = seed % 3
    T = np.arange(T_cap + 1, dtype=np.float64)
    if kind == 0:
        t = 1.0 + rng.uniform(0.01, 0.4) * np.maximum(0.0, T - rng.integers(1, T_cap))
    elif kind == 1:
        t = 0.5 + rng.uniform(0.01, 0.3) * T
    else:
        t = 2.0 + rng.uniform(0.0, 0.2) * np.maximum(0.0, T - R) ** 1.5
    res = schedule_ref(c, np.zeros(R, dtype=np.int32), t, T_cap)
    best, best_L = schedule_bruteforce(c, t, T_cap)
    gap = (best - res["objective"]) / best
    assert gap <= 1e-12, f"greedy objective below the exhaustive optimum by {gap:.3e}"
    if not res["flagged"]:
        S = survival_ref(c)
        F = lambda L: (R + sum(S[r, :L[r]].sum() for r in range(R))) / t[R + int(np.sum(L))]
        assert math.isclose(F(res["verify_len"]), best, rel_tol=1e-12)


def test_invariants_and_markers():
    rng = np.random.default_rng(5)
    cfg = TINY.with_(R=37)
    kv = kv_lengths(cfg, rng)
    conf = confidences(cfg, rng, 1)[0]
    t = step_time_table(cfg)
    res = schedule_ref(conf, kv, t, cfg.T_cap)
    L = res["verify_len"]
    assert np.all((L >= 0) & (L <= cfg.K))
    assert res["T"] == cfg.R + L.sum()
    S = res["S"]
    # the chosen set is the top-n* candidates, hence a prefix per request
    chosen = np.concatenate([S[r, :L[r]] for r in range(cfg.R)])
    rest = np.concatenate([S[r, L[r]:] for r in range(cfg.R)])
    if len(chosen) and len(rest):
        assert chosen.min() >= rest.max()
    qo, mk = res["q_offsets"], res["markers"]
    for r in range(cfg.R):
        seg = mk[qo[r]:qo[r + 1]]
        assert np.all(seg[:, 0] == r)
        assert np.array_equal(seg[:, 1], kv[r] + np.arange(L[r] + 1))


def test_flatten_layout():
    qo, mk = flatten_ref([0, 2, 5], [3, 0, 7])
    assert list(qo) == [0, 1, 4, 10]
    assert mk.tolist() == [[0, 3], [1, 0], [1, 1], [1, 2],
                           [2, 7], [2, 8], [2, 9], [2, 10], [2, 11], [2, 12]]


def test_verify_length_shrinks_with_load():
    """Low concurrency verifies (nearly) the whole block; the budget shrinks as load grows."""
    means = []
    for R in SWEEP_LEVELS:
        cfg = sweep_config(R)
        rng = np.random.default_rng(0)
        kv_lengths(cfg, rng)
        conf = confidences(cfg, rng, 1)[0]
        res = schedule_ref(conf, np.zeros(R, dtype=np.int32), step_time_table(cfg), cfg.T_cap)
        means.append(res["verify_len"].mean())
    assert means[0] == 5 and means[1] == 5
    assert all(b <= a + 1e-12 for a, b in zip(means, means[1:]))
    assert means[-1] < 3
