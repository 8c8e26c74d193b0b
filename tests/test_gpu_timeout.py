"""The bounded in-kernel wait gives up, reports DSPARK_DERR_TIMEOUT and leaves the context
usable: a barrier that nothing arrives at, waited on with a short limit (no fault, no trap)."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_support import ATTN_MAX_ABS, ATTN_MEAN_ABS, binding, host, new_step, set_schedule
from workloads.configs import QWEN3_4B
from workloads.generate import build_step_inputs

pytestmark = pytest.mark.gpu


def test_wait_on_a_barrier_nobody_arrives_at_times_out_and_the_context_survives():
    d = binding()
    assert d.dspark_read_error() == 0
    res = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    d.dspark_selftest_wait_timeout(2_000_000, res)          # about a millisecond
    torch.cuda.synchronize()
    assert res.tolist() == [0, 1]
    assert d.dspark_read_error() & (1 << 9)                # DSPARK_DERR_TIMEOUT, then cleared
    assert d.dspark_read_error() == 0
    # the context keeps working: a tensor-core attention call right after
    cfg = QWEN3_4B.with_(R=4, kv_dist=("uniform", 50, 300), V=64)
    inp = build_step_inputs(cfg, "cuda", seed=2, layers=1)
    step = new_step(cfg)
    qo, mk = set_schedule(step, [2, 0, 5, 3], host(inp.kv_len))
    out = torch.empty_like(inp.q[0])
    step.plan(inp.kv_len)
    step.attention(inp.q[0], inp.k_new[0], inp.v_new[0], inp.kv_caches[0], inp.block_table,
                   inp.kv_len, out)
    torch.cuda.synchronize()
    T = int(qo[-1])
    ref = oracle.attn_ref_flat(host(inp.q[0, :T]), host(inp.k_new[0, :T]), host(inp.v_new[0, :T]),
                               host(inp.kv_caches[0]), host(inp.block_table), host(inp.kv_len),
                               mk, qo, step.scale, cfg.page_size)
    err = np.abs(host(out[:T]) - ref)
    assert err.max() <= ATTN_MAX_ABS and err.mean() <= ATTN_MEAN_ABS
    assert d.dspark_read_error() == 0
