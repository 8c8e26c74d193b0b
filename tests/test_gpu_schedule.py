"""GPU scheduler parity: bit-exact verify lengths, offsets and markers against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_support import (assert_schedule_equal, binding, gpu_schedule, host, new_step,
                               oracle_schedule)
from workloads.configs import CONFIGS, TINY, SWEEP_LEVELS, sweep_config
from workloads.generate import (CONF_RING, conf_ring, confidences, kv_lengths, step_time_table)

pytestmark = pytest.mark.gpu


class _SchedInputs:
    """Only what the scheduler reads (no bulk tensors)."""

    def __init__(self, cfg, seed=0, rounds=4, conf=None, t=None, kv=None):
        rng = np.random.default_rng(seed)
        self.cfg = cfg
        kvl = kv_lengths(cfg, rng) if kv is None else np.asarray(kv, np.int32)
        hist = confidences(cfg, rng, rounds) if conf is None else conf
        self.round_idx = hist.shape[0] - 1
        self.conf_history = hist
        dev = "cuda"
        self.conf_ring = torch.as_tensor(conf_ring(hist, self.round_idx)).to(dev)
        self.kv_len = torch.as_tensor(kvl).to(dev)
        tt = step_time_table(cfg) if t is None else t
        self.t_ms = torch.as_tensor(np.asarray(tt, np.float64)).to(dev)


def _check(cfg, **kw):
    inp = _SchedInputs(cfg, **kw)
    step = new_step(cfg)
    gpu = gpu_schedule(step, inp)
    ref = oracle_schedule(inp)
    flagged = assert_schedule_equal(gpu, ref)
    assert binding().dspark_read_error() == 0
    return gpu, ref, flagged


@pytest.mark.parametrize("name", ["tiny", "qwen3-4b-64req", "mixed-256req", "lognormal-1024req"]
                         + [f"sweep-{R}req" for R in SWEEP_LEVELS])
def test_workload_schedules(name):
    gpu, ref, flagged = _check(CONFIGS[name])
    assert flagged == 0


@pytest.mark.parametrize("seed", range(8))
def test_random_small_vs_bruteforce(seed):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(1, 5))
    cfg = TINY.with_(R=R)
    conf = rng.uniform(0.02, 0.999, size=(1, R, cfg.K)).astype(np.float32)
    T = np.arange(cfg.T_cap + 1, dtype=np.float64)
    t = 1.0 + rng.uniform(0.01, 0.4) * np.maximum(0.0, T - rng.integers(1, cfg.T_cap))
    gpu, ref, _ = _check(cfg, conf=conf, t=t)
    best, _ = oracle.schedule_bruteforce(conf[0], t, cfg.T_cap)
    assert (best - gpu["objective"]) / best <= 1e-12


def test_exact_ties_follow_position_then_request():
    cfg = TINY.with_(R=300)
    conf = np.full((1, 300, 5), 0.8, dtype=np.float32)
    conf[0, ::7] = 1.0          # exact survival 1.0 ties
    conf[0, ::11, 2:] = 0.0     # exact zeros
    T = np.arange(cfg.T_cap + 1, dtype=np.float64)
    t = 4.0 + 0.004 * np.maximum(0.0, T - 500)
    _check(cfg, conf=conf, t=t)


def test_largest_candidate_count_and_edge_tables():
    R = 16384 // 5
    cfg = TINY.with_(R=R)
    rng = np.random.default_rng(1)
    conf = rng.uniform(0.05, 0.99, size=(1, R, 5)).astype(np.float32)
    T = np.arange(cfg.T_cap + 1, dtype=np.float64)
    for t in (np.full(cfg.T_cap + 1, 2.0),                 # flat: take everything
              1.0 + T,                                       # unit cost: take nothing
              5.0 + 0.004 * np.maximum(0.0, T - 256)):       # knee
        _check(cfg, conf=conf, t=t, kv=np.zeros(R, np.int32))


def test_lag_reads_the_round_two_steps_back():
    cfg = sweep_config(128)
    rng = np.random.default_rng(3)
    hist = confidences(cfg, rng, 6)
    for rounds in (1, 2, 3, 4, 6):
        _check(cfg, conf=hist[:rounds])


def test_one_request_and_K1():
    for K in (1, 5, 16):
        cfg = TINY.with_(R=1, K=K)
        rng = np.random.default_rng(K)
        conf = rng.uniform(0.1, 0.99, size=(3, 1, K)).astype(np.float32)
        T = np.arange(cfg.T_cap + 1, dtype=np.float64)
        _check(cfg, conf=conf, t=1.0 + 0.05 * T)


def test_invalid_confidence_sets_error_word():
    d = binding()
    cfg = TINY
    inp = _SchedInputs(cfg)
    bad = inp.conf_ring.clone()
    bad[:, 0, 1] = float("nan")
    bad[:, 2, 0] = 1.5
    step = new_step(cfg)
    step.schedule(bad, inp.round_idx, inp.kv_len, inp.t_ms)
    code = d.dspark_read_error()
    assert code & 1
    assert d.dspark_read_error() == 0   # cleared
    L = host(step.verify_len)
    assert np.all((L >= 0) & (L <= cfg.K))
