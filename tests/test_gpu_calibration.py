"""GPU temperature scaling against the oracle: calibrated confidences within one float32 ulp,
fitted temperatures within 1e-5 relative, error bits for invalid inputs, and the scheduler fed
with calibrated confidences."""
import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from oracle.calibration import BETA_HI
from tests.gpu_support import binding, host, new_step
from workloads.configs import QWEN3_4B
from workloads.generate import build_step_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seed", range(3))
def test_calibrated_confidences_match(seed):
    d = binding()
    rng = np.random.default_rng(seed)
    R, K = 300, 5
    l = rng.normal(0, 6, size=(R, K)).astype(np.float32)
    tau = rng.uniform(0.3, 4.0, size=K).astype(np.float32)
    conf = torch.empty((R, K), dtype=torch.float32, device="cuda")
    d.dspark_calibrate_confidence(torch.as_tensor(l).cuda(), torch.as_tensor(tau).cuda(), conf)
    got = host(conf)
    want = oracle.calibrate_ref(l, tau)
    assert np.all(np.abs(got - want) <= np.spacing(np.maximum(got, want)))
    assert d.dspark_read_error() == 0


def test_invalid_temperature_and_nan_logit_give_zero_and_set_the_bit():
    d = binding()
    l = torch.ones((4, 5), dtype=torch.float32, device="cuda")
    l[2, 1] = float("nan")
    tau = torch.tensor([1.0, 1.0, 0.0, -2.0, float("inf")], device="cuda")
    conf = torch.empty_like(l)
    d.dspark_calibrate_confidence(l, tau, conf)
    c = host(conf)
    assert np.all(c[:, 2:] == 0) and c[2, 1] == 0
    np.testing.assert_allclose(c[[0, 1, 3], :2], expit(1.0), rtol=1e-6)
    assert d.dspark_read_error() & 1


def _simulate(tau_true, n, rng, K=5):
    l_true = rng.normal(1.5, 1.5, size=(n, K)) - 0.3 * np.arange(K)
    l_raw = (l_true * np.asarray(tau_true)[None, :]).astype(np.float32)
    p = expit(l_true)
    acc_draw = rng.random((n, K)) < p
    L = rng.integers(0, K + 1, size=n)
    a = np.zeros(n, dtype=np.int64)
    for i in range(n):
        while a[i] < L[i] and acc_draw[i, a[i]]:
            a[i] += 1
    return l_raw, L, a


@pytest.mark.parametrize("n", [37, 5000, 60000])
def test_fitted_temperatures_match(n):
    d = binding()
    rng = np.random.default_rng(n)
    l, L, a = _simulate([0.7, 1.3, 2.0, 2.8, 3.5], n, rng)
    tau = torch.empty(5, dtype=torch.float32, device="cuda")
    d.dspark_fit_temperature(torch.as_tensor(l).cuda(), torch.as_tensor(L.astype(np.int32)).cuda(),
                             torch.as_tensor(a.astype(np.int32)).cuda(), tau)
    want = oracle.fit_temperature_ref(l, L, a, 5)
    np.testing.assert_allclose(host(tau), want, rtol=1e-5)
    assert d.dspark_read_error() == 0


def test_fit_degenerate_and_invalid_samples():
    d = binding()
    L = np.array([1, 1, 1, 1, 9], np.int32)          # last sample invalid (L > K)
    a = np.array([1, 1, 1, 1, 0], np.int32)
    l = np.ones((5, 5), np.float32)
    tau = torch.empty(5, dtype=torch.float32, device="cuda")
    d.dspark_fit_temperature(torch.as_tensor(l).cuda(), torch.as_tensor(L).cuda(),
                             torch.as_tensor(a).cuda(), tau)
    t = host(tau)
    assert t[0] == pytest.approx(1.0 / BETA_HI) and np.all(t[1:] == 1.0)
    assert d.dspark_read_error() & (1 << 10)


def test_scheduler_runs_on_calibrated_confidences():
    """Over-confident raw logits, calibrated on the GPU into the ring slot the scheduler reads;
    the schedule matches the oracle's on the same confidences."""
    d = binding()
    cfg = QWEN3_4B.with_(R=48, V=64)
    inp = build_step_inputs(cfg, "cuda", seed=3, layers=1)
    rng = np.random.default_rng(3)
    slot = max(inp.round_idx - 2, 0) % inp.conf_ring.shape[0]
    raw = torch.as_tensor(rng.normal(2.0, 3.0, size=(cfg.R, cfg.K)).astype(np.float32)).cuda()
    tau = torch.tensor([1.5, 1.8, 2.1, 2.4, 2.7], dtype=torch.float32, device="cuda")
    d.dspark_calibrate_confidence(raw, tau, inp.conf_ring[slot])
    step = new_step(cfg)
    step.schedule(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms)
    torch.cuda.synchronize()
    ref = oracle.schedule_ref(host(inp.conf_ring[slot]), host(inp.kv_len), host(inp.t_ms), cfg.T_cap)
    if not ref["flagged"]:
        np.testing.assert_array_equal(host(step.verify_len), ref["verify_len"])
    assert d.dspark_read_error() == 0
