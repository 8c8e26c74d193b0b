"""Whole verify step on the GPU (schedule -> plan -> attention per layer -> accept) against the
oracle chain on the same inputs."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_support import (ATTN_MAX_ABS, ATTN_MEAN_ABS, F32_ATTN_MAX_ABS,
                               assert_accept_equal, assert_schedule_equal, binding, flat_target,
                               host, new_step, oracle_accept_chunked, oracle_schedule)
from workloads.configs import TINY, QWEN3_4B
from workloads.generate import build_step_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg,tau", [(TINY, 1.0), (TINY, 0.0),
                                     (QWEN3_4B.with_(R=9, V=5000, layers=2), 1.0)])
def test_step_matches_oracle_chain(cfg, tau):
    inp = build_step_inputs(cfg, "cuda", seed=11, layers=cfg.layers)
    step = new_step(cfg)
    ref_s = oracle_schedule(inp)
    L = ref_s["verify_len"]
    tflat = flat_target(inp, L)
    outs = [torch.empty_like(inp.q[i]) for i in range(cfg.layers)]
    step.schedule(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms)
    step.plan(inp.kv_len)
    for i in range(cfg.layers):
        step.attention(inp.q[i], inp.k_new[i], inp.v_new[i], inp.kv_caches[0], inp.block_table,
                       inp.kv_len, outs[i])
    step.accept(tflat, inp.draft_logits if tau > 0 else None, inp.draft_tokens, inp.u_acc,
                inp.u_res, tau)
    torch.cuda.synchronize()
    T = int(step.T.item())
    gpu_s = dict(verify_len=host(step.verify_len), q_offsets=host(step.q_offsets),
                 markers=host(step.markers)[:T], T=T, objective=float(step.objective.item()))
    assert assert_schedule_equal(gpu_s, ref_s) == 0
    qo, mk = ref_s["q_offsets"], ref_s["markers"]
    for i in range(cfg.layers):
        ref_a = oracle.attn_ref_flat(host(inp.q[i, :T]), host(inp.k_new[i, :T]),
                                     host(inp.v_new[i, :T]), host(inp.kv_caches[0]),
                                     host(inp.block_table), host(inp.kv_len), mk, qo, step.scale,
                                     cfg.page_size)
        err = np.abs(host(outs[i][:T]) - ref_a)
        lim = F32_ATTN_MAX_ABS if cfg.dtype == "f32" else ATTN_MAX_ABS
        assert err.max() <= lim and err.mean() <= ATTN_MEAN_ABS
    gpu_a = dict(accepted_len=host(step.accepted_len), out_tokens=host(step.out_tokens),
                 n_out=host(step.n_out))
    ref_acc = oracle_accept_chunked(tflat, inp.draft_logits, host(inp.draft_tokens), L, qo,
                                    host(inp.u_acc), host(inp.u_res), tau)
    assert_accept_equal(gpu_a, ref_acc)
    assert binding().dspark_read_error() == 0


@pytest.mark.parametrize("tau", [1.0, 0.0])
def test_step_from_host_matches_device_resident_step(tau):
    """run_from_host (inputs copied from pinned host memory on a copy stream, per-layer events)
    gives the same results as the same step on device-resident inputs."""
    cfg = QWEN3_4B.with_(R=10, V=3000, layers=3)
    inp = build_step_inputs(cfg, "cuda", seed=4, layers=cfg.layers)
    step = new_step(cfg)
    L = oracle_schedule(inp)["verify_len"]
    tflat = flat_target(inp, L)
    dlog = inp.draft_logits if tau > 0 else None
    caches = [inp.kv_caches[0]] * cfg.layers
    out_a = torch.empty_like(inp.q[0])
    step.run(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms,
             [(inp.q[i], inp.k_new[i], inp.v_new[i]) for i in range(cfg.layers)], caches,
             inp.block_table, out_a, tflat, dlog, inp.draft_tokens, inp.u_acc, inp.u_res, tau)
    torch.cuda.synchronize()
    want = {k: getattr(step, k).clone() for k in ("verify_len", "accepted_len", "out_tokens", "n_out")}
    pin = lambda t: t.cpu().pin_memory() if t is not None else None
    hst = dict(conf=pin(inp.conf_ring), kv_len=pin(inp.kv_len), t_ms=pin(inp.t_ms), q=pin(inp.q),
               k_new=pin(inp.k_new), v_new=pin(inp.v_new), target_logits=pin(tflat),
               draft_logits=pin(dlog), draft_tokens=pin(inp.draft_tokens), u_acc=pin(inp.u_acc),
               u_res=pin(inp.u_res))
    dev = {k: (torch.zeros_like(v, device="cuda") if v is not None else None) for k, v in hst.items()}
    host_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in want.items()}
    for k in want:
        getattr(step, k).zero_()
    out_b = torch.empty_like(inp.q[0])
    step.run_from_host(hst, dev, inp.round_idx, inp.block_table, caches, out_b, tau,
                       torch.cuda.Stream(), host_out)
    torch.cuda.synchronize()
    for k, v in want.items():
        assert torch.equal(host_out[k], v.cpu()), k
    assert torch.equal(out_a, out_b)   # the last layer's attention
