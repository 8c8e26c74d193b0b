"""Verify rounds as CUDA-graph replays (pipeline.RoundPipeline): against the oracle chain
(schedule on the lagged confidences, attention per layer, acceptance, KV commit, committed
lengths carried forward), and against the same rounds run eagerly (bit-identical outputs round
after round, with the committed cache lengths and pages carried on the device); plus a whole
step captured with VerifyStep.capture."""
import numpy as np
import pytest
import torch

from tests.gpu_support import assert_accept_equal, binding, host, new_step
from workloads.configs import QWEN3_4B
from workloads.generate import build_step_inputs, flatten_target

pytestmark = pytest.mark.gpu


def _state(cfg, seed, layers, overlap=False):
    from speculative_decoding_verification_survival_b200 import RoundPipeline
    inp = build_step_inputs(cfg, "cuda", seed=seed, layers=layers, kv_copies=1,
                            reserve_tokens=8 * (cfg.K + 1))
    step = new_step(cfg)
    caches = torch.stack([inp.kv_caches[0].clone() for _ in range(layers)])
    attn_out = torch.zeros_like(inp.q)
    tflat = torch.empty((cfg.T_cap, cfg.V), dtype=inp.target_block.dtype, device="cuda")
    pipe = RoundPipeline(step, inp.conf_ring.clone(), inp.t_ms, inp.kv_len.clone(),
                         inp.block_table, inp.q.clone(), inp.k_new.clone(), inp.v_new.clone(),
                         caches, attn_out, tflat, inp.draft_logits.clone(), inp.draft_tokens.clone(),
                         inp.u_acc.clone(), inp.u_res.clone(), cfg.temperature,
                         overlap=overlap)
    return inp, pipe


def _refill(pipe, inp, cfg, rnd):
    """New inputs for round `rnd` (the engine's job): queries, new K/V, drafts, uniforms,
    logits laid out for the lengths the round will schedule, a fresh confidence slot."""
    g = torch.Generator(device="cuda").manual_seed(100 + rnd)
    for t in (pipe.q, pipe.k_new, pipe.v_new):
        t.copy_(torch.randn(t.shape, generator=g, device="cuda").to(t.dtype))
    pipe.u_acc.copy_(torch.rand(pipe.u_acc.shape, generator=g, device="cuda"))
    pipe.u_res.copy_(torch.rand(pipe.u_res.shape, generator=g, device="cuda"))
    pipe.draft_tokens.copy_(torch.randint(0, cfg.V, pipe.draft_tokens.shape, generator=g,
                                          device="cuda", dtype=torch.int32))
    pipe.draft_logits.copy_(torch.randn(pipe.draft_logits.shape, generator=g, device="cuda")
                            .to(pipe.draft_logits.dtype) * 3)
    pipe.target_logits.copy_(torch.randn(pipe.target_logits.shape, generator=g, device="cuda")
                             .to(pipe.target_logits.dtype) * 3)
    pipe.conf_ring[rnd % pipe.ring_depth].copy_(
        torch.sigmoid(torch.randn(pipe.conf_ring.shape[1:], generator=g, device="cuda") + 2))


def test_graph_rounds_match_eager_rounds_bit_for_bit():
    cfg = QWEN3_4B.with_(R=12, kv_dist=("uniform", 40, 700), V=256, layers=3)
    inp_a, eager = _state(cfg, 7, 3)
    inp_b, graph = _state(cfg, 7, 3)
    for rnd in range(5):
        _refill(eager, inp_a, cfg, rnd)
        _refill(graph, inp_b, cfg, rnd)
        eager.enqueue(rnd)
        graph.round(rnd)
        torch.cuda.synchronize()
        for name in ("kv_len", "attn_out", "kv_caches"):
            assert torch.equal(getattr(eager, name), getattr(graph, name)), (rnd, name)
        for name in ("verify_len", "accepted_len", "out_tokens", "n_out", "markers"):
            assert torch.equal(getattr(eager.step, name), getattr(graph.step, name)), (rnd, name)
    # the cache lengths advanced by the kept tokens each round
    assert torch.all(graph.kv_len > inp_b.kv_len)
    assert binding().dspark_read_error() == 0


def test_captured_step_replays_the_eager_step():
    cfg = QWEN3_4B.with_(R=20, kv_dist=("uniform", 100, 900), V=512)
    inp = build_step_inputs(cfg, "cuda", seed=3, layers=2)
    step = new_step(cfg)
    step.schedule(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms)
    torch.cuda.synchronize()
    tflat = flatten_target(inp.target_block, host(step.verify_len).astype(np.int64), cfg.T_cap)
    outs = [torch.empty_like(inp.q[0]) for _ in range(2)]

    def enqueue():
        step.schedule(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms)
        step.plan(inp.kv_len)
        for layer in range(2):
            step.attention(inp.q[layer], inp.k_new[layer], inp.v_new[layer], inp.kv_caches[0],
                           inp.block_table, inp.kv_len, outs[layer])
        step.accept(tflat, inp.draft_logits, inp.draft_tokens, inp.u_acc, inp.u_res,
                    cfg.temperature)

    enqueue()
    torch.cuda.synchronize()
    ref = [o.clone() for o in outs] + [step.accepted_len.clone(), step.out_tokens.clone()]
    for o in outs:
        o.zero_()
    step.accepted_len.zero_()
    step.out_tokens.zero_()
    g = step.capture(enqueue)
    g.replay()
    torch.cuda.synchronize()
    got = outs + [step.accepted_len, step.out_tokens]
    for a, b in zip(ref, got):
        assert torch.equal(a, b)


@pytest.mark.parametrize("overlap", [False, True])
def test_graph_rounds_follow_the_oracle_chain(overlap):
    """Five rounds replayed as CUDA graphs, each checked against the oracle chain run on the
    same input bits: schedule_ref on the confidences of two rounds earlier, attn_ref_flat per
    layer over the oracle's own cache, accept_ref, kv_commit_ref, and the committed lengths
    carried into the next round.  Lengths, markers and tokens are bit-exact (a request the
    oracle flags may differ; the chain then continues from the GPU's decision, the only other
    valid one), attention is within the stated bf16 tolerance and the caches are byte-exact."""
    import math

    import oracle
    from tests.gpu_support import (ATTN_MAX_ABS, ATTN_MEAN_ABS, assert_schedule_equal)

    cfg = QWEN3_4B.with_(R=10, kv_dist=("uniform", 40, 700), V=512, layers=3)
    inp, pipe = _state(cfg, 11, 3, overlap=overlap)
    layers = 3
    scale = 1.0 / math.sqrt(cfg.D)
    t_ms = host(inp.t_ms)
    table = host(inp.block_table)
    kv_len = host(pipe.kv_len).astype(np.int64)
    caches = host(pipe.kv_caches)                      # the oracle's own copy, float32 bits
    flagged_total = 0
    for rnd in range(5):
        _refill(pipe, inp, cfg, rnd)
        torch.cuda.synchronize()
        ring = host(pipe.conf_ring)
        q, kn, vn = host(pipe.q), host(pipe.k_new), host(pipe.v_new)
        tl, dl = host(pipe.target_logits), host(pipe.draft_logits)
        xt, ua, ur = host(pipe.draft_tokens), host(pipe.u_acc), host(pipe.u_res)

        pipe.round(rnd)
        torch.cuda.synchronize()
        st = pipe.step_of(rnd)

        # schedule on the lagged confidence slot, with the lengths the chain has committed
        conf = ring[oracle.lagged_round(rnd) % pipe.ring_depth]
        sref = oracle.schedule_ref(conf, kv_len, t_ms, cfg.T_cap)
        T = int(st.T.item())
        sgpu = dict(verify_len=host(st.verify_len), q_offsets=host(st.q_offsets),
                    markers=host(st.markers)[:T], T=T, objective=float(st.objective.item()))
        assert assert_schedule_equal(sgpu, sref) == 0, f"round {rnd}: schedule flagged"
        L, qo, mk = sref["verify_len"], sref["q_offsets"], sref["markers"]

        # attention of every layer over the oracle's cache
        for layer in range(layers):
            ref = oracle.attn_ref_flat(q[layer, :T], kn[layer, :T], vn[layer, :T], caches[layer],
                                       table, kv_len, mk, qo, scale, cfg.page_size)
            err = np.abs(host(pipe.attn_out[layer, :T]).astype(np.float64) - ref)
            assert err.max() <= ATTN_MAX_ABS and err.mean() <= ATTN_MEAN_ABS, \
                (rnd, layer, err.max(), err.mean())

        # acceptance, exact modulo flags
        aref = oracle.accept_ref(tl[:T], dl, xt, L, qo, ua, ur, cfg.temperature)
        agpu = dict(accepted_len=host(st.accepted_len), out_tokens=host(st.out_tokens),
                    n_out=host(st.n_out))
        nflag, _ = assert_accept_equal(agpu, aref)
        flagged_total += nflag
        accepted = np.where(aref["flagged"], agpu["accepted_len"], aref["accepted_len"])

        # commit into the oracle's cache; the GPU's caches and lengths must match byte for byte
        caches, kv_out, skipped = oracle.kv_commit_ref(kn, vn, caches, table, kv_len, qo,
                                                       accepted, cfg.K, cfg.T_cap)
        assert skipped == []
        assert np.array_equal(host(pipe.kv_len), kv_out), rnd
        assert np.array_equal(host(pipe.kv_caches), caches), rnd
        assert np.all(kv_out == kv_len + accepted + 1)
        kv_len = kv_out.astype(np.int64)
    print(f"five chained rounds match the oracle chain; flagged requests: {flagged_total}")
    assert binding().dspark_read_error() == 0


def test_overlapped_rounds_equal_serial_rounds():
    """Round i + 1's scheduling decision on a side stream, concurrent with round i, gives the
    serial chain's results bit for bit, as graphs and eagerly."""
    cfg = QWEN3_4B.with_(R=14, kv_dist=("uniform", 40, 900), V=256, layers=2)
    inp_a, serial = _state(cfg, 5, 2)
    inp_b, overlap = _state(cfg, 5, 2, overlap=True)
    inp_c, eager = _state(cfg, 5, 2, overlap=True)
    for rnd in range(6):
        for p, i in ((serial, inp_a), (overlap, inp_b), (eager, inp_c)):
            _refill(p, i, cfg, rnd)
        serial.round(rnd)
        overlap.round(rnd)
        eager.round(rnd, graph=False)
        torch.cuda.synchronize()
        for other in (overlap, eager):
            for name in ("kv_len", "attn_out", "kv_caches"):
                assert torch.equal(getattr(serial, name), getattr(other, name)), (rnd, name)
            for name in ("verify_len", "q_offsets", "accepted_len", "out_tokens", "n_out"):
                assert torch.equal(getattr(serial.step, name),
                                   getattr(other.step_of(rnd), name)), (rnd, name)
            T = int(serial.step.T.item())
            assert torch.equal(serial.step.markers[:T], other.step_of(rnd).markers[:T])
    assert binding().dspark_read_error() == 0
