"""GPU acceptance parity: bit-exact accepted lengths and emitted tokens against the oracle
(requests the oracle flags as within 1e-6 of a decision threshold are counted, not failed),
and the chi-square test of the emitted distribution run through the C ABI."""
import zlib

import numpy as np
import pytest
import torch
from scipy.stats import chisquare

from tests.accept_harness import build_trials, logits_of, target_probs
from tests.gpu_support import (assert_accept_equal, binding, flat_target, gpu_accept, host,
                               new_step, oracle_accept_chunked, oracle_schedule, set_schedule)
from workloads.configs import CONFIGS, TINY, QWEN3_4B
from workloads.generate import build_step_inputs

pytestmark = pytest.mark.gpu


def _workload_accept(cfg, seed=0, verify_len=None, temperature=None):
    inp = build_step_inputs(cfg, "cuda", seed=seed, layers=1)
    tau = cfg.temperature if temperature is None else temperature
    step = new_step(cfg)
    if verify_len is None:
        verify_len = oracle_schedule(inp)["verify_len"]
    qo, _ = set_schedule(step, verify_len, host(inp.kv_len))
    tflat = flat_target(inp, verify_len)
    dt = inp.draft_tokens
    gpu = gpu_accept(step, tflat, inp.draft_logits, dt, inp.u_acc, inp.u_res, tau)
    ref = oracle_accept_chunked(tflat, inp.draft_logits, host(dt), np.asarray(verify_len), qo,
                                host(inp.u_acc), host(inp.u_res), tau)
    nflag, nflag_diff = assert_accept_equal(gpu, ref)
    assert binding().dspark_read_error() == 0
    return gpu, ref, nflag, nflag_diff


@pytest.mark.parametrize("tau", [1.0, 0.7, 0.0])
@pytest.mark.parametrize("seed", range(3))
def test_tiny_f32(seed, tau):
    _workload_accept(TINY.with_(R=64), seed=seed, temperature=tau)


@pytest.mark.parametrize("name,tau", [("qwen3-4b-64req", 1.0), ("mixed-256req", 1.0),
                                      ("lognormal-1024req", 0.7), ("lognormal-1024req", 0.0),
                                      ("sweep-2048req", 1.0)])
def test_full_workloads(name, tau):
    gpu, ref, nflag, nflag_diff = _workload_accept(CONFIGS[name], temperature=tau)
    print(f"{name} tau={tau}: flagged {nflag}, flagged-and-different {nflag_diff}, "
          f"mean accepted {gpu['accepted_len'].mean():.3f}")


def test_edge_lengths_odd_vocab():
    cfg = QWEN3_4B.with_(R=40, V=1000 + 3)          # V % 8 != 0: unaligned rows, scalar path
    L = np.array([0, 5] * 20)
    _workload_accept(cfg, verify_len=L, temperature=1.0)
    _workload_accept(cfg, verify_len=L, temperature=0.0)
    _workload_accept(cfg, verify_len=np.zeros(40, int), temperature=0.9)


@pytest.mark.parametrize("V", [151936, 20000 + 3, 4096 + 1])
def test_draw_split_across_cluster(V):
    # few requests over a long vocabulary: each request's draw is shared by a cluster of CTAs
    # (8 CTAs for 75 chunks; 8 CTAs over 10 chunks, an uneven split, on the unaligned scalar
    # path; 3 CTAs of one chunk each)
    cfg = QWEN3_4B.with_(R=12, V=V)
    for tau in (1.0, 0.6):
        gpu, ref, _, _ = _workload_accept(cfg, seed=V % 7, temperature=tau)
        assert np.all(gpu["out_tokens"][np.arange(12), gpu["accepted_len"]] >= 0)


def test_empty_residual_falls_back_to_p_across_cluster():
    # draft rows equal to the target rows of the same positions: p == q, every ratio is 1, so
    # u = 1 rejects and leaves a residual that is zero everywhere; the draw then falls back to
    # p, in the oracle and in the cluster of CTAs alike
    cfg = QWEN3_4B.with_(R=12)
    inp = build_step_inputs(cfg, "cuda", seed=5, layers=1)
    verify_len = oracle_schedule(inp)["verify_len"]
    step = new_step(cfg)
    qo, _ = set_schedule(step, verify_len, host(inp.kv_len))
    tflat = flat_target(inp, verify_len)
    dl = inp.target_block[:, :cfg.K].contiguous()
    u_acc = inp.u_acc.clone()
    u_acc[::2, 0] = 1.0
    gpu = gpu_accept(step, tflat, dl, inp.draft_tokens, u_acc, inp.u_res, 1.0)
    ref = oracle_accept_chunked(tflat, dl, host(inp.draft_tokens), np.asarray(verify_len), qo,
                                host(u_acc), host(inp.u_res), 1.0)
    assert_accept_equal(gpu, ref)
    assert binding().dspark_read_error() == 0
    L = np.asarray(verify_len)
    assert np.all(gpu["accepted_len"][::2][L[::2] > 0] == 0)   # rejected at once
    assert np.all(gpu["accepted_len"][1::2] == L[1::2])         # every ratio 1: all accepted
    assert np.all(gpu["out_tokens"][np.arange(12), gpu["accepted_len"]] >= 0)
    # u = 1 sits on the acceptance threshold, so the oracle flags those requests; their draws
    # from p are still compared wherever the draw itself is not near a boundary
    even = (np.arange(12) % 2 == 0) & ~ref["flag_sample"]
    assert even.sum() >= 4
    assert np.array_equal(gpu["out_tokens"][even], ref["out_tokens"][even])
    assert np.array_equal(gpu["accepted_len"][even], ref["accepted_len"][even])


def _gpu_trials(tr, tau=1.0):
    d = binding()
    n = len(tr["verify_len"])
    K = tr["draft_tokens"].shape[1]
    dev = "cuda"
    tl = torch.as_tensor(np.ascontiguousarray(tr["target_logits"])).to(dev)
    dlg = torch.as_tensor(np.ascontiguousarray(tr["draft_logits"])).to(dev)
    T_cap = tl.shape[0]
    acc = torch.zeros(n, dtype=torch.int32, device=dev)
    out = torch.zeros(n, K + 1, dtype=torch.int32, device=dev)
    nout = torch.zeros(n, dtype=torch.int32, device=dev)
    ws = torch.zeros(d.dspark_accept_workspace_bytes(n, K, T_cap), dtype=torch.uint8, device=dev)
    d.dspark_accept(tl, dlg, torch.as_tensor(tr["draft_tokens"]).to(dev),
                    torch.as_tensor(tr["verify_len"]).to(dev), torch.as_tensor(tr["q_offsets"]).to(dev),
                    torch.as_tensor(np.ascontiguousarray(tr["u_acc"])).to(dev),
                    torch.as_tensor(np.ascontiguousarray(tr["u_res"])).to(dev),
                    tau, acc, out, nout, ws)
    torch.cuda.synchronize()
    return host(acc), host(out), host(nout)


CHI_CASES = {
    "v4": ([0.1, 0.2, 0.3, 0.4], [0.4, 0.3, 0.2, 0.1]),
    "v2": ([0.7, 0.3], [0.5, 0.5]),
    "q_zero_where_p_pos": ([0.2, 0.2, 0.1, 0.1, 0.1, 0.1, 0.1, 0.1],
                           [0.5, 0.5, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0]),
    "p_zero_where_q_pos": ([0.5, 0.5, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0],
                           [0.1, 0.1, 0.2, 0.1, 0.1, 0.1, 0.2, 0.1]),
    "onehot_p": ([0.0, 0.0, 0.0, 1.0], [0.25, 0.25, 0.25, 0.25]),
}


@pytest.mark.parametrize("name", list(CHI_CASES))
def test_chi_square_first_token_one_million_trials(name):
    p, q = CHI_CASES[name]
    K = 5
    zt = np.tile(logits_of(p), (K + 1, 1))
    zd = np.tile(logits_of(q), (K, 1))
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    tr = build_trials(zt, zd, 5, 1_000_000, rng, round_idx=17)
    _, out, _ = _gpu_trials(tr)
    counts = np.bincount(out[:, 0], minlength=len(p))
    probs = target_probs(zt[0])
    zero = probs == 0
    assert np.all(counts[zero] == 0)
    if np.count_nonzero(~zero) > 1:
        assert chisquare(counts[~zero], probs[~zero] * counts.sum()).pvalue > 0.01


def test_chi_square_v32_and_gpu_equals_oracle_on_trials():
    import oracle
    rng0 = np.random.default_rng(42)
    K, V = 5, 32
    zt = rng0.normal(0, 1.5, size=(K + 1, V)).astype(np.float32)
    zd = (zt[:K] + rng0.normal(0, 1.0, size=(K, V))).astype(np.float32)
    rng = np.random.default_rng(8)
    tr = build_trials(zt, zd, 5, 1_000_000, rng, round_idx=5)
    acc, out, nout = _gpu_trials(tr)
    counts = np.bincount(out[:, 0], minlength=V)
    assert chisquare(counts, target_probs(zt[0]) * counts.sum()).pvalue > 0.01
    sub = slice(0, 50_000)
    ref = oracle.accept_ref(tr["target_logits"][:50_000 * 6], tr["draft_logits"][sub],
                            tr["draft_tokens"][sub], tr["verify_len"][sub],
                            tr["q_offsets"][:50_001], tr["u_acc"][sub], tr["u_res"][sub], 1.0)
    assert_accept_equal(dict(accepted_len=acc[sub], out_tokens=out[sub], n_out=nout[sub]), ref)


def test_invalid_draft_token_sets_error_word():
    d = binding()
    cfg = TINY.with_(R=8)
    inp = build_step_inputs(cfg, "cuda", seed=2, layers=1)
    step = new_step(cfg)
    L = np.full(8, 5)
    set_schedule(step, L, host(inp.kv_len))
    dt = inp.draft_tokens.clone()
    dt[3, 0] = cfg.V + 7
    gpu_accept(step, flat_target(inp, L), inp.draft_logits, dt, inp.u_acc, inp.u_res, 1.0)
    assert d.dspark_read_error() & (1 << 7)
    assert host(step.accepted_len)[3] == 0
