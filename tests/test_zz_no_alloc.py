"""dspark_accept_noalloc: the acceptance entry point for callers that cannot allocate.

Some users of this library run where device allocation is off limits (a serving engine whose
memory pool already owns the GPU, a plugin host that forbids allocation after start-up, a loop
that cannot afford an allocation's implicit synchronisation).  This entry point takes no
workspace; its scratch is a fixed array inside the library.  The test calls it through the C
ABI twice in a row and requires exactly the results of dspark_accept with a caller workspace
(the outputs are integers, so "within tolerance" means equal), and checks the size limit.
It lives in its own file so that it runs after every other test.
"""
import numpy as np
import pytest
import torch

from tests.gpu_support import binding, flat_target, host, new_step, set_schedule
from workloads.configs import TINY, QWEN3_4B
from workloads.generate import build_step_inputs

pytestmark = pytest.mark.gpu


def _outputs(R, K, dev):
    return (torch.full((R,), -7, dtype=torch.int32, device=dev),
            torch.full((R, K + 1), -7, dtype=torch.int32, device=dev),
            torch.full((R,), -7, dtype=torch.int32, device=dev))


@pytest.mark.parametrize("cfg,tau", [(TINY.with_(R=64), 1.0), (TINY.with_(R=64), 0.0),
                                     (QWEN3_4B.with_(R=48, V=20000), 1.0),
                                     (QWEN3_4B.with_(R=48, V=20000), 0.7)])
def test_noalloc_matches_workspace_entry_point(cfg, tau):
    d = binding()
    inp = build_step_inputs(cfg, "cuda", seed=21, layers=1)
    rng = np.random.default_rng(5)
    L = rng.integers(0, cfg.K + 1, size=cfg.R)
    step = new_step(cfg)
    set_schedule(step, L, host(inp.kv_len))
    tflat = flat_target(inp, L)
    dlog = inp.draft_logits if tau > 0 else None
    ref = _outputs(cfg.R, cfg.K, "cuda")
    d.dspark_accept(tflat, dlog, inp.draft_tokens, step.verify_len, step.q_offsets, inp.u_acc,
                    inp.u_res, tau, *ref, step.accept_ws)
    for _ in range(2):                      # two calls in a row share the fixed scratch
        got = _outputs(cfg.R, cfg.K, "cuda")
        d.dspark_accept_noalloc(tflat, dlog, inp.draft_tokens, step.verify_len, step.q_offsets,
                                inp.u_acc, inp.u_res, tau, *got)
        torch.cuda.synchronize()
        for a, b in zip(ref, got):
            assert torch.equal(a, b)
    assert d.dspark_read_error() == 0


def test_noalloc_rejects_sizes_beyond_its_array():
    d = binding()
    R, K = 8192, 5                          # T_cap + R*K = 49152 + 40960 > 65536
    T_cap = R * (K + 1)
    dev = "cuda"
    tl = torch.zeros(T_cap, 8, dtype=torch.float32, device=dev)
    dt = torch.zeros(R, K, dtype=torch.int32, device=dev)
    vl = torch.zeros(R, dtype=torch.int32, device=dev)
    qo = torch.zeros(R + 1, dtype=torch.int32, device=dev)
    out = _outputs(R, K, dev)
    with pytest.raises(d.DSparkError) as e:
        d.dspark_accept_noalloc(tl, None, dt, vl, qo, None, None, 0.0, *out)
    assert e.value.status == -6
