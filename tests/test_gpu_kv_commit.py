"""GPU KV commit (dspark_kv_commit) against the oracle, byte for byte.

Small cases compare whole caches (page size 8 so the kept rows cross pages, several layers in
one call, f32 and bf16); the qwen3-like case compares the whole cache as raw 16-bit words; the
chain case runs schedule -> attention -> accept -> commit and checks the next round's attention
over the committed cache against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_support import (ATTN_MAX_ABS, ATTN_MEAN_ABS, binding, host, new_step,
                               set_schedule)
from workloads.configs import QWEN3_4B, TINY
from workloads.generate import build_step_inputs

pytestmark = pytest.mark.gpu


def _raw(t):
    """Bit pattern of a tensor as a NumPy array (bf16 -> int16 words)."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy()
    return t.cpu().numpy()


def _commit_case(cfg, seed, layers, acc_fn, corrupt=None):
    d = binding()
    rng = np.random.default_rng(seed)
    inp = build_step_inputs(cfg, "cuda", seed=seed, layers=layers, kv_copies=1)
    step = new_step(cfg)
    L = rng.integers(0, cfg.K + 1, size=cfg.R)
    kv = host(inp.kv_len).astype(np.int64)
    qo, _ = set_schedule(step, L, kv)
    acc = np.asarray(acc_fn(rng, L), dtype=np.int32)
    step.accepted_len.copy_(torch.as_tensor(acc))
    caches = torch.stack([inp.kv_caches[0].clone() for _ in range(layers)])
    bt = inp.block_table.clone()
    if corrupt is not None:
        corrupt(step, bt, kv)
    before = caches.clone()
    kv_out = torch.full_like(inp.kv_len, -7)
    d.dspark_kv_commit(inp.k_new, inp.v_new, caches, bt, inp.kv_len, step.q_offsets,
                       step.accepted_len, cfg.K, kv_out)
    torch.cuda.synchronize()
    want, want_len, skipped = oracle.kv_commit_ref(
        _raw(inp.k_new), _raw(inp.v_new), _raw(before), host(bt), kv, host(step.q_offsets),
        host(step.accepted_len), cfg.K, cfg.T_cap)
    np.testing.assert_array_equal(_raw(caches), want)
    np.testing.assert_array_equal(host(kv_out), want_len)
    return d.dspark_read_error(), skipped


@pytest.mark.parametrize("seed", range(3))
def test_tiny_f32_page8_three_layers(seed):
    err, skipped = _commit_case(TINY, seed, 3, lambda rng, L: [rng.integers(0, l + 1) for l in L])
    assert err == 0 and skipped == []


def test_bf16_qwen3_like_whole_cache():
    cfg = QWEN3_4B.with_(R=16, kv_dist=("uniform", 60, 700), V=64)
    err, skipped = _commit_case(cfg, 4, 2, lambda rng, L: [rng.integers(0, l + 1) for l in L])
    assert err == 0 and skipped == []


def test_all_accepted_and_none_accepted():
    for fn in (lambda rng, L: L, lambda rng, L: np.zeros_like(L)):
        err, skipped = _commit_case(TINY, 7, 1, fn)
        assert err == 0 and skipped == []


def test_malformed_requests_set_bits_and_stay_untouched():
    def corrupt(step, bt, kv):
        step.accepted_len[1] = 99                         # beyond the verify length
        n2 = int(kv[2])
        bt[2, n2 // TINY.page_size] = 10 ** 7             # page outside the cache
    err, skipped = _commit_case(TINY, 3, 2, lambda rng, L: [rng.integers(0, l + 1) for l in L],
                                corrupt=corrupt)
    assert 1 in skipped and 2 in skipped
    assert err & (1 << 10) and err & (1 << 3)


def test_chain_schedule_attention_accept_commit_next_round():
    """Round 1 on the GPU (schedule, attention, accept, commit); round 2's attention over the
    committed cache matches the oracle run on the oracle-committed cache."""
    cfg = QWEN3_4B.with_(R=6, kv_dist=("uniform", 30, 400), V=512)
    d = binding()
    inp = build_step_inputs(cfg, "cuda", seed=21, layers=1)
    step = new_step(cfg)
    step.schedule(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms)
    step.plan(inp.kv_len)
    out = torch.empty_like(inp.q[0])
    step.attention(inp.q[0], inp.k_new[0], inp.v_new[0], inp.kv_caches[0], inp.block_table,
                   inp.kv_len, out)
    from workloads.generate import flatten_target
    torch.cuda.synchronize()
    L = host(step.verify_len).astype(np.int64)
    tflat = flatten_target(inp.target_block, L, cfg.T_cap)
    step.accept(tflat, inp.draft_logits, inp.draft_tokens, inp.u_acc, inp.u_res, cfg.temperature)
    cache = inp.kv_caches[0].clone()
    before = cache.clone()
    kv_out = torch.empty_like(inp.kv_len)
    step.commit(inp.k_new[0], inp.v_new[0], cache, inp.block_table, inp.kv_len, kv_out)
    torch.cuda.synchronize()
    assert d.dspark_read_error() == 0
    kv = host(inp.kv_len).astype(np.int64)
    want, want_len, _ = oracle.kv_commit_ref(
        _raw(inp.k_new[:1]), _raw(inp.v_new[:1]), _raw(before)[None], host(inp.block_table), kv,
        host(step.q_offsets), host(step.accepted_len), cfg.K, cfg.T_cap)
    np.testing.assert_array_equal(_raw(cache), want[0])
    np.testing.assert_array_equal(host(kv_out), want_len)
    # round 2: one fresh verify token per request over the committed cache
    step2 = new_step(cfg)
    qo2, mk2 = set_schedule(step2, np.zeros(cfg.R, dtype=np.int64), host(kv_out))
    g = torch.Generator(device="cuda").manual_seed(5)
    q2 = torch.randn(inp.q[0].shape, generator=g, device="cuda").to(torch.bfloat16)
    k2 = torch.randn(inp.k_new[0].shape, generator=g, device="cuda").to(torch.bfloat16)
    v2 = torch.randn(inp.v_new[0].shape, generator=g, device="cuda").to(torch.bfloat16)
    out2 = torch.empty_like(q2)
    step2.plan(kv_out)
    step2.attention(q2, k2, v2, cache, inp.block_table, kv_out, out2)
    torch.cuda.synchronize()
    T2 = int(qo2[-1])
    ref = oracle.attn_ref_flat(host(q2[:T2]), host(k2[:T2]), host(v2[:T2]), host(cache),
                               host(inp.block_table), host(kv_out), mk2, qo2, step2.scale,
                               cfg.page_size)
    err = np.abs(host(out2[:T2]).astype(np.float64) - ref)
    assert err.max() <= ATTN_MAX_ABS and err.mean() <= ATTN_MEAN_ABS
    assert d.dspark_read_error() == 0
