"""GPU verify-attention parity against the float64 oracle on identical bf16 / f32 inputs.

Small cases compare every output element (several 64-key tiles, ragged tails, empty caches,
zero-length schedules, page crossings, all GQA group sizes used by the workloads); the full
workloads compare sampled (token, head) rows computed one by one by the oracle (every row when
the workload has few verify tokens), and every output element against a closed form on
structured keys and values that make any misrouted page, head, d-half or split piece visible.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_support import (ATTN_MAX_ABS, ATTN_MEAN_ABS, F32_ATTN_MAX_ABS, binding, host,
                               new_step, oracle_attn_rows, set_schedule)
from tests.structured_attn import install_structured, structured_expected
from workloads.configs import CONFIGS, TINY, QWEN3_4B
from workloads.generate import build_step_inputs

pytestmark = pytest.mark.gpu


def _run_attn(step, inp, layer=0, cache=None):
    cache = inp.kv_caches[0] if cache is None else cache
    out = torch.full_like(inp.q[layer], float("nan"))
    step.plan(inp.kv_len)
    step.attention(inp.q[layer], inp.k_new[layer], inp.v_new[layer], cache, inp.block_table,
                   inp.kv_len, out)
    torch.cuda.synchronize()
    return out


def _full_compare(cfg, verify_len, seed=0, tol=None):
    inp = build_step_inputs(cfg, "cuda", seed=seed, layers=1)
    step = new_step(cfg)
    kv = host(inp.kv_len)
    qo, mk = set_schedule(step, verify_len, kv)
    out = _run_attn(step, inp)
    T = int(qo[-1])
    ref = oracle.attn_ref_flat(host(inp.q[0, :T]), host(inp.k_new[0, :T]), host(inp.v_new[0, :T]),
                               host(inp.kv_caches[0]), host(inp.block_table), kv, mk, qo,
                               step.scale, cfg.page_size)
    got = host(out[:T]).astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got))
    if cfg.dtype == "f32":
        assert err.max() <= (tol or F32_ATTN_MAX_ABS), err.max()
    else:
        assert err.max() <= ATTN_MAX_ABS and err.mean() <= ATTN_MEAN_ABS, (err.max(), err.mean())
    assert binding().dspark_read_error() == 0
    return err


@pytest.mark.parametrize("seed", range(4))
def test_tiny_f32_all_rows(seed):
    rng = np.random.default_rng(seed)
    L = rng.integers(0, TINY.K + 1, size=TINY.R)
    _full_compare(TINY, L, seed=seed)


@pytest.mark.parametrize("G,R,lo,hi", [(4, 6, 0, 300), (5, 5, 60, 200), (8, 4, 1, 129),
                                       (8, 3, 0, 0)])
def test_bf16_all_rows_several_tiles(G, R, lo, hi):
    cfg = QWEN3_4B.with_(R=R, Hq=2 * G, Hkv=2, kv_dist=("uniform", lo, hi), V=64)
    rng = np.random.default_rng(G * 100 + R)
    L = rng.integers(0, cfg.K + 1, size=R)
    L[0] = 0
    L[-1] = cfg.K
    _full_compare(cfg, L, seed=G)


def test_bf16_small_pages_and_f32_head_dim_64():
    cfg = QWEN3_4B.with_(R=5, Hq=8, Hkv=2, page_size=16, kv_dist=("uniform", 1, 150), V=64)
    _full_compare(cfg, [5, 0, 3, 1, 2], seed=3)
    cfg = TINY.with_(R=3, Hq=6, Hkv=3, D=64, page_size=32, kv_dist=("uniform", 40, 140))
    _full_compare(cfg, [2, 5, 0], seed=4)


def test_f32_long_cache_many_split_pieces():
    # one request much longer than the rest: its segments are cut across many CTAs
    cfg = TINY.with_(R=3, kv_dist=("uniform", 5000, 5000), D=32, page_size=8)
    _full_compare(cfg, [5, 5, 5], seed=5)


@pytest.mark.parametrize("name", ["qwen3-4b-64req", "mixed-256req", "lognormal-1024req",
                                  "sweep-1req", "sweep-2048req"])
def test_full_workload_sampled_rows(name):
    cfg = CONFIGS[name]
    inp = build_step_inputs(cfg, "cuda", seed=0, layers=1)
    step = new_step(cfg)
    step.schedule(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms)
    out = _run_attn(step, inp)
    T = int(step.T.item())
    qo = host(step.q_offsets)
    mk = host(step.markers)[:T]
    rng = np.random.default_rng(1)
    toks = set(rng.integers(0, T, size=40).tolist()) | {0, T - 1}
    # include the longest request's tokens and a zero-length request if any
    kv = host(inp.kv_len)
    r_long = int(np.argmax(kv))
    toks |= {int(qo[r_long]), int(qo[r_long + 1]) - 1}
    rows = [(t, int(rng.integers(0, cfg.Hq))) for t in sorted(toks)]
    if T * cfg.Hq <= 4096:   # few verify tokens (sweep-1req: one request cut into many pieces)
        rows = [(t, h) for t in range(T) for h in range(cfg.Hq)]
    ref = oracle_attn_rows(inp, 0, inp.kv_caches[0], qo, mk, rows, step.scale)
    errs = np.concatenate([np.abs(host(out[t, h]).astype(np.float64) - ref[(t, h)])
                           for t, h in rows])
    assert errs.max() <= ATTN_MAX_ABS and errs.mean() <= ATTN_MEAN_ABS, (errs.max(), errs.mean())
    # rows past the scheduled total are never written
    if T < cfg.T_cap:
        assert torch.isnan(out[T:]).all()
    assert binding().dspark_read_error() == 0


def test_repeated_calls_reuse_plan_and_counters():
    cfg = QWEN3_4B.with_(R=7, kv_dist=("uniform", 100, 2000), V=64)
    inp = build_step_inputs(cfg, "cuda", seed=9, layers=3)
    step = new_step(cfg)
    rng = np.random.default_rng(2)
    qo, mk = set_schedule(step, rng.integers(0, 6, size=7), host(inp.kv_len))
    step.plan(inp.kv_len)
    outs = []
    for layer in range(3):
        out = torch.empty_like(inp.q[layer])
        step.attention(inp.q[layer], inp.k_new[layer], inp.v_new[layer], inp.kv_caches[0],
                       inp.block_table, inp.kv_len, out)
        outs.append(out)
    out0b = torch.empty_like(inp.q[0])
    step.attention(inp.q[0], inp.k_new[0], inp.v_new[0], inp.kv_caches[0], inp.block_table,
                   inp.kv_len, out0b)
    torch.cuda.synchronize()
    T = int(qo[-1])
    assert torch.equal(outs[0][:T], out0b[:T])   # deterministic, counters reset
    kv = host(inp.kv_len)
    for layer in (1, 2):
        ref = oracle.attn_ref_flat(host(inp.q[layer, :T]), host(inp.k_new[layer, :T]),
                                   host(inp.v_new[layer, :T]), host(inp.kv_caches[0]),
                                   host(inp.block_table), kv, mk, qo, step.scale, cfg.page_size)
        err = np.abs(host(outs[layer][:T]) - ref)
        assert err.max() <= ATTN_MAX_ABS and err.mean() <= ATTN_MEAN_ABS


def test_corrupt_marker_and_page_set_error_bits():
    d = binding()
    cfg = QWEN3_4B.with_(R=4, kv_dist=("uniform", 10, 300), V=64)
    inp = build_step_inputs(cfg, "cuda", seed=1, layers=1)
    step = new_step(cfg)
    set_schedule(step, [1, 2, 0, 3], host(inp.kv_len))
    step.markers[1, 1] += 1            # wrong position for request 0's second token
    _run_attn(step, inp)
    assert d.dspark_read_error() & (1 << 4)
    set_schedule(step, [1, 2, 0, 3], host(inp.kv_len))
    bt = inp.block_table.clone()
    bt[2, 0] = 10 ** 7                 # page outside the cache
    out = torch.empty_like(inp.q[0])
    step.plan(inp.kv_len)
    step.attention(inp.q[0], inp.k_new[0], inp.v_new[0], inp.kv_caches[0], bt, inp.kv_len, out)
    assert d.dspark_read_error() & (1 << 3)
    assert d.dspark_read_error() == 0


def _compare_with_scale(cfg, verify_len, seed, scale, kv_transform=None):
    inp = build_step_inputs(cfg, "cuda", seed=seed, layers=1)
    if kv_transform is not None:
        kv_transform(inp)
    step = new_step(cfg)
    kv = host(inp.kv_len)
    qo, mk = set_schedule(step, verify_len, kv)
    out = torch.full_like(inp.q[0], float("nan"))
    d = binding()
    step.plan(inp.kv_len)
    d.dspark_verify_attn(inp.q[0], inp.k_new[0], inp.v_new[0], inp.kv_caches[0], inp.block_table,
                         inp.kv_len, step.markers, step.q_offsets, cfg.K, scale, out, step.attn_ws)
    torch.cuda.synchronize()
    T = int(qo[-1])
    ref = oracle.attn_ref_flat(host(inp.q[0, :T]), host(inp.k_new[0, :T]), host(inp.v_new[0, :T]),
                               host(inp.kv_caches[0]), host(inp.block_table), kv, mk, qo, scale,
                               cfg.page_size)
    err = np.abs(host(out[:T]).astype(np.float64) - ref)
    assert np.all(np.isfinite(host(out[:T])))
    assert err.max() <= ATTN_MAX_ABS and err.mean() <= ATTN_MEAN_ABS, (err.max(), err.mean())
    assert d.dspark_read_error() == 0


@pytest.mark.parametrize("G", [4, 5, 8, 16])
def test_tensor_core_path_group_sizes(G):
    # bf16, D 128, page 64: the tcgen05 kernel; G*(K+1) spans the 4-, 2- and 1-copy layouts
    cfg = QWEN3_4B.with_(R=6, Hq=2 * G, Hkv=2, kv_dist=("uniform", 1, 700), V=64)
    L = np.array([5, 0, 3, 5, 1, 4])
    _compare_with_scale(cfg, L, seed=G, scale=1.0 / math.sqrt(128))


def test_tensor_core_rescale_path():
    # scale 1 and keys that grow along the cache make the running maximum jump by far more than
    # 2^8 from tile to tile, so O is rescaled in tensor memory
    cfg = QWEN3_4B.with_(R=4, Hq=16, Hkv=2, kv_dist=("uniform", 300, 900), V=64)

    def grow(inp):
        P, _, Hkv, page, D = inp.kv_caches[0].shape
        table = inp.block_table.cpu().numpy()
        kvl = inp.kv_len.cpu().numpy()
        for r in range(cfg.R):
            for p in range(-(-int(kvl[r]) // page)):
                pg = int(table[r, p])
                f = 1.0 + 0.02 * p * page
                inp.kv_caches[0][pg, 0] = (inp.kv_caches[0][pg, 0].float() * f).to(torch.bfloat16)

    _compare_with_scale(cfg, np.array([5, 2, 0, 4]), seed=3, scale=1.0, kv_transform=grow)


def test_tensor_core_pages_of_128():
    cfg = QWEN3_4B.with_(R=5, page_size=128, kv_dist=("uniform", 1, 1000), V=64)
    _compare_with_scale(cfg, np.array([5, 4, 3, 2, 1]), seed=6, scale=1.0 / math.sqrt(128))


@pytest.mark.parametrize("name", ["qwen3-4b-64req", "lognormal-1024req", "mixed-256req",
                                  "sweep-1req", "sweep-2048req"])
def test_full_workload_structured_keys_and_values(name):
    cfg = CONFIGS[name]
    inp = build_step_inputs(cfg, "cuda", seed=0, layers=1)
    install_structured(inp)
    step = new_step(cfg)
    kv = host(inp.kv_len).astype(np.int64)
    sref = oracle.schedule_ref(inp.conf_history[oracle.lagged_round(inp.round_idx)], kv,
                               host(inp.t_ms), cfg.T_cap)
    qo, mk = set_schedule(step, sref["verify_len"], kv)
    out = _run_attn(step, inp)
    T = int(qo[-1])
    ref = structured_expected(inp, qo, kv)                    # [T][Hkv][D]
    got = host(out[:T]).astype(np.float64).reshape(T, cfg.Hkv, cfg.G, cfg.D)
    err = np.abs(got - ref[:, :, None, :])
    bound = 2.0 ** -8 * np.abs(ref)[:, :, None, :] + 1e-5     # the final bf16 rounding
    bad = err > bound
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} elements off, worst "
                           f"{float((err - bound).max()):.3e} at {np.argwhere(bad)[0].tolist()}")
    assert binding().dspark_read_error() == 0


# ---- the plan's cost-balanced ranges ----------------------------------------------------------
_COST_NEW, _COST_PIECE, _COST_MERGE, _SEG_TAIL = 4.0, 7.0, 6.0, 8


def _plan_ranges(step, cfg):
    """The tensor-core kernel's CTA ranges as the plan wrote them into the workspace (layout of
    the workspace: header, unit prefix, counters, request records, CTA start records, CTA
    range starts, each 256-byte aligned)."""
    al = lambda x: (x + 255) // 256 * 256
    ws = step.attn_ws.cpu().numpy()
    hdr = ws[:32].view(np.int32)
    total, ctas = int(hdr[5]), int(hdr[6])
    bound = float(ws[28:32].view(np.float32)[0])
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    off = al(32)
    prefix = ws[off:off + 4 * (cfg.R + 1)].view(np.int32).astype(np.int64)
    off += al(4 * (cfg.R + 1)) + al(4 * cfg.R * cfg.Hkv) + al(16 * cfg.R) + al(16 * 4 * sms)
    begin = ws[off:off + 4 * (ctas + 1)].view(np.int32).astype(np.int64)
    return total, ctas, bound, prefix, begin


def _range_costs(prefix, Hkv, begin):
    """Modelled cost of every CTA's range (cache pages + verify tile + per piece + merge of a
    split segment's head piece)."""
    seg_units = np.diff(prefix) // Hkv
    starts = np.concatenate([prefix[r] + g * seg_units[r] + np.zeros(1, np.int64)
                             for r in range(len(seg_units)) for g in range(Hkv)])
    lens = np.repeat(seg_units, Hkv)
    costs = np.zeros(len(begin) - 1)
    for c in range(len(begin) - 1):
        u0, u1 = begin[c], begin[c + 1]
        if u0 >= u1:
            continue
        for s0, n in zip(starts, lens):
            a, b = max(u0, s0), min(u1, s0 + n)
            if a >= b:
                continue
            cache = n - _SEG_TAIL
            pages = min(b, s0 + cache) - min(a, s0 + cache)
            cost = pages + _COST_PIECE + (_COST_NEW if b == s0 + n else 0.0)
            if a == s0 and b < s0 + n:
                cost += _COST_MERGE          # the head piece of a split segment merges
            costs[c] += cost
    return costs, starts, lens


@pytest.mark.parametrize("name", ["qwen3-4b-64req", "sweep-1req", "sweep-128req"])
def test_plan_ranges_are_cost_balanced(name):
    cfg = CONFIGS[name]
    inp = build_step_inputs(cfg, "cuda", seed=0, layers=1)
    step = new_step(cfg)
    step.schedule(inp.conf_ring, inp.round_idx, inp.kv_len, inp.t_ms)
    step.plan(inp.kv_len)
    torch.cuda.synchronize()
    total, ctas, bound, prefix, begin = _plan_ranges(step, cfg)
    assert begin[0] == 0 and begin[-1] == total and np.all(np.diff(begin) >= 0)
    costs, starts, lens = _range_costs(prefix, cfg.Hkv, begin)
    # no range boundary inside a segment's verify-token units
    for b in begin[1:-1]:
        k = np.searchsorted(starts, b, side="right") - 1
        assert b - starts[k] <= lens[k] - _SEG_TAIL or b == starts[k] + lens[k]
    assert costs.max() <= bound + 1e-3
    # about as good as equal ranges under the same model or better (the greedy fill is not
    # exactly optimal: a head piece costs a merge, so the cost of a range is not monotone in
    # its end; 2% and the spacing of the bounds the plan tries cover that)
    W = -(-total // ctas)
    equal = np.minimum(np.arange(ctas + 1) * W, total)
    eq_costs, _, _ = _range_costs(prefix, cfg.Hkv, equal)
    spacing = ((lens - _SEG_TAIL).max() + _COST_NEW + 2 * _COST_PIECE + _COST_MERGE) / 1024
    assert costs.max() <= 1.02 * eq_costs.max() + spacing, (costs.max(), eq_costs.max())
    print(f"{name}: largest modelled CTA cost {costs.max():.1f} (equal ranges "
          f"{eq_costs.max():.1f}), mean {costs.sum() / ctas:.1f}")
