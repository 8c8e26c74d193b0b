"""Pins for the acceptance oracle.

The pages fix one property exactly: the emitted tokens follow the target distribution
("DSpark 的 661% 提速，是真突破还是数字游戏？" §一; "DeepSeek服务器不再卡顿！…" section
"成本与质量的考量").  Chi-square goodness of fit (scipy, run as a library routine) checks it;
deterministic cases and greedy argmax pin the control flow.
"""
import zlib

import numpy as np
import pytest
from scipy.stats import chisquare

from oracle.accept import accept_ref
from tests.accept_harness import build_trials, logits_of, target_probs

K = 5


def _run(tr, tau=1.0):
    return accept_ref(tr["target_logits"], tr["draft_logits"], tr["draft_tokens"],
                      tr["verify_len"], tr["q_offsets"], tr["u_acc"], tr["u_res"], tau)


def _chi2_ok(counts, probs, min_p=0.01):
    probs = np.asarray(probs)
    zero = probs == 0
    assert np.all(counts[zero] == 0), "a zero-probability token was emitted"
    if np.count_nonzero(~zero) == 1:
        return
    exp = probs[~zero] * counts.sum()
    stat = chisquare(counts[~zero], exp)
    assert stat.pvalue > min_p, f"chi-square p-value {stat.pvalue:.4g}"


def _first_token_counts(zt, zd, L, n_total, seed, chunk=100_000):
    V = zt.shape[1]
    rng = np.random.default_rng(seed)
    counts = np.zeros(V, dtype=np.int64)
    acc = []
    for c0 in range(0, n_total, chunk):
        n = min(chunk, n_total - c0)
        tr = build_trials(zt, zd, L, n, rng, round_idx=seed, r_base=c0)
        res = _run(tr)
        counts += np.bincount(res["out_tokens"][:, 0], minlength=V)
        acc.append(res["accepted_len"])
    return counts, np.concatenate(acc)


CASES = {
    "v4": ([0.1, 0.2, 0.3, 0.4], [0.4, 0.3, 0.2, 0.1]),
    "v2": ([0.7, 0.3], [0.5, 0.5]),
    "q_zero_where_p_pos": ([0.2, 0.2, 0.1, 0.1, 0.1, 0.1, 0.1, 0.1],
                           [0.5, 0.5, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0]),
    "p_zero_where_q_pos": ([0.5, 0.5, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0],
                           [0.1, 0.1, 0.2, 0.1, 0.1, 0.1, 0.2, 0.1]),
    "onehot_p": ([0.0, 0.0, 0.0, 1.0], [0.25, 0.25, 0.25, 0.25]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_first_token_follows_target(name):
    p, q = CASES[name]
    zt = np.tile(logits_of(p), (K + 1, 1))
    zd = np.tile(logits_of(q), (K, 1))
    n = 1_000_000 if name == "v4" else 200_000
    counts, _ = _first_token_counts(zt, zd, 5, n, seed=zlib.crc32(name.encode()) % 1000)
    _chi2_ok(counts, target_probs(zt[0]))


def test_first_token_follows_the_tempered_target():
    """At temperature tau the verifier's distribution is p = softmax(z_target / tau) and the
    drafts come from q = softmax(z_draft / tau): the first emitted token must follow p, not
    softmax(z_target) (the lognormal workloads sample at tau = 0.7)."""
    tau, V = 0.7, 8
    g = np.random.default_rng(21)
    zt = np.tile(g.normal(0, 1.0, V).astype(np.float32), (K + 1, 1))
    zd = np.tile(g.normal(0, 1.0, V).astype(np.float32), (K, 1))
    rng = np.random.default_rng(5)
    counts = np.zeros(V, dtype=np.int64)
    n, chunk = 300_000, 100_000
    for c0 in range(0, n, chunk):
        tr = build_trials(zt, zd / tau, 5, chunk, rng, round_idx=11, r_base=c0)
        tr["draft_logits"] = np.broadcast_to(zd, tr["draft_logits"].shape)
        counts += np.bincount(_run(tr, tau)["out_tokens"][:, 0], minlength=V)
    _chi2_ok(counts, target_probs(zt[0] / tau))
    # the untempered distribution is far from what was drawn
    exp1 = target_probs(zt[0]) * counts.sum()
    assert chisquare(counts, exp1).pvalue < 1e-6


def test_first_token_v32_position_dependent():
    rng = np.random.default_rng(42)
    V = 32
    zt = rng.normal(0, 1.5, size=(K + 1, V)).astype(np.float32)
    zd = (zt[:K] + rng.normal(0, 1.0, size=(K, V))).astype(np.float32)
    counts, acc = _first_token_counts(zt, zd, 5, 300_000, seed=7)
    _chi2_ok(counts, target_probs(zt[0]))
    assert 0 < acc.mean() < 5


def test_zero_length_emits_bonus_from_first_position():
    zt = np.tile(logits_of([0.1, 0.6, 0.3]), (K + 1, 1))
    zt[1:] = logits_of([0.9, 0.05, 0.05])        # later positions must not matter
    zd = np.tile(logits_of([0.3, 0.3, 0.4]), (K, 1))
    counts, acc = _first_token_counts(zt, zd, 0, 200_000, seed=3)
    assert np.all(acc == 0)
    _chi2_ok(counts, target_probs(zt[0]))


def test_equal_distributions_accept_everything():
    z = logits_of([0.1, 0.2, 0.3, 0.4])
    zt = np.tile(z, (K + 1, 1))
    zd = np.tile(z, (K, 1))
    rng = np.random.default_rng(5)
    tr = build_trials(zt, zd, 5, 100_000, rng, round_idx=0)
    res = _run(tr)
    assert np.all(res["accepted_len"] == 5)
    # the bonus token at position 6 follows p
    _chi2_ok(np.bincount(res["out_tokens"][:, 5], minlength=4), target_probs(z))


def test_three_token_joint_under_stationary_distributions():
    """Run verify steps until three tokens exist; the triple must follow p x p x p."""
    p = np.array([0.15, 0.25, 0.35, 0.25])
    q = np.array([0.4, 0.1, 0.1, 0.4])
    V = 4
    zt = np.tile(logits_of(p), (K + 1, 1))
    zd = np.tile(logits_of(q), (K, 1))
    pe = target_probs(zt[0])
    rng = np.random.default_rng(11)
    n = 1_000_000
    counts = np.zeros(V ** 3, dtype=np.int64)
    chunk = 100_000
    for c0 in range(0, n, chunk):
        seqs = [[] for _ in range(chunk)]
        pending = np.arange(chunk)
        step = 0
        while len(pending):
            tr = build_trials(zt, zd, 2, len(pending), rng, round_idx=1000 * step + c0 // chunk)
            res = _run(tr)
            for i, tid in enumerate(pending):
                seqs[tid].extend(res["out_tokens"][i, :res["n_out"][i]].tolist())
            pending = np.array([t for t in pending if len(seqs[t]) < 3], dtype=np.int64)
            step += 1
        idx = np.array([s[0] * 16 + s[1] * 4 + s[2] for s in seqs])
        counts += np.bincount(idx, minlength=V ** 3)
    joint = np.einsum("i,j,k->ijk", pe, pe, pe).reshape(-1)
    _chi2_ok(counts, joint)


def test_deterministic_decisions():
    """Ratios 0 or >= 1 make every decision independent of the uniforms."""
    V = 4
    zt = np.stack([logits_of([0.5, 0.5, 0.0, 0.0]),    # position 1: x=0, p/q = 1 -> accept
                   logits_of([0.25, 0.75, 0.0, 0.0]),  # position 2: x=2, p(2) = 0 -> reject
                   logits_of([0.25, 0.25, 0.25, 0.25]),
                   logits_of([0.25, 0.25, 0.25, 0.25]),
                   logits_of([0.25, 0.25, 0.25, 0.25]),
                   logits_of([0.25, 0.25, 0.25, 0.25])])
    zd = np.stack([logits_of([0.5, 0.5, 0.0, 0.0]),
                   logits_of([0.25, 0.25, 0.5, 0.0]),  # residual at 2 = (0, 0.5, 0, 0)
                   logits_of([0.25, 0.25, 0.25, 0.25]),
                   logits_of([0.25, 0.25, 0.25, 0.25]),
                   logits_of([0.25, 0.25, 0.25, 0.25])])
    rng = np.random.default_rng(0)
    tr = build_trials(zt, zd, 5, 2000, rng, round_idx=9)
    tr["draft_tokens"][:, 0] = 0
    tr["draft_tokens"][:, 1] = 2
    res = _run(tr)
    assert np.all(res["accepted_len"] == 1)
    assert np.all(res["out_tokens"][:, 0] == 0)
    assert np.all(res["out_tokens"][:, 1] == 1)
    assert np.all(res["out_tokens"][:, 2:] == -1)
    assert np.all(res["n_out"] == 2)


def test_greedy_matches_argmax_loop():
    rng = np.random.default_rng(21)
    R, V = 300, 9
    L = rng.integers(0, K + 1, size=R).astype(np.int32)
    qo = np.concatenate([[0], np.cumsum(L + 1)]).astype(np.int32)
    T = int(qo[-1])
    zt = rng.integers(-3, 3, size=(T, V)).astype(np.float32)     # many exact ties
    zd = rng.integers(-3, 3, size=(R, K, V)).astype(np.float32)
    x = rng.integers(0, V, size=(R, K)).astype(np.int32)
    for r in range(R):                                             # make some drafts right
        for k in range(K):
            if rng.random() < 0.6 and k < L[r]:
                x[r, k] = int(np.argmax(zt[qo[r] + k]))
    u0 = np.zeros((R, K), np.float32)
    res = accept_ref(zt, zd, x, L, qo, u0, np.zeros((R, K + 1), np.float32), 0.0)
    for r in range(R):
        a = 0
        while a < L[r]:
            row = zt[qo[r] + a]
            best = min(v for v in range(V) if row[v] == row.max())
            if x[r, a] != best:
                break
            a += 1
        row = zt[qo[r] + a]
        corr = min(v for v in range(V) if row[v] == row.max())
        assert res["accepted_len"][r] == a
        assert list(res["out_tokens"][r, :a + 1]) == list(x[r, :a]) + [corr]
        assert res["n_out"][r] == a + 1


def test_invariants_random():
    rng = np.random.default_rng(8)
    R, V = 200, 50
    L = rng.integers(0, K + 1, size=R).astype(np.int32)
    qo = np.concatenate([[0], np.cumsum(L + 1)]).astype(np.int32)
    zt = rng.normal(0, 2, size=(int(qo[-1]), V)).astype(np.float32)
    zd = rng.normal(0, 2, size=(R, K, V)).astype(np.float32)
    x = rng.integers(0, V, size=(R, K)).astype(np.int32)
    ua = rng.random((R, K)).astype(np.float32)
    ur = rng.random((R, K + 1)).astype(np.float32)
    for tau in (1.0, 0.7, 0.0):
        res = accept_ref(zt, zd, x, L, qo, ua, ur, tau)
        a = res["accepted_len"]
        assert np.all((a >= 0) & (a <= L))
        assert np.array_equal(res["n_out"], a + 1)
        for r in range(R):
            assert np.array_equal(res["out_tokens"][r, :a[r]], x[r, :a[r]])
            assert 0 <= res["out_tokens"][r, a[r]] < V
            assert np.all(res["out_tokens"][r, a[r] + 1:] == -1)


def test_flags_mark_threshold_cases():
    """A uniform planted exactly on p/q is flagged; one far from it is not."""
    z = logits_of([0.2, 0.3, 0.5])
    zq = logits_of([0.4, 0.3, 0.3])
    zt = np.tile(z, (K + 1, 1))
    zd = np.tile(zq, (K, 1))
    rng = np.random.default_rng(2)
    tr = build_trials(zt, zd, 1, 2, rng, 0)
    tr["draft_tokens"][:, 0] = 0                    # p/q = 0.5
    tr["u_acc"] = np.array([[0.5] * K, [0.9] * K], dtype=np.float32)
    res = accept_ref(tr["target_logits"], tr["draft_logits"], tr["draft_tokens"],
                     tr["verify_len"], tr["q_offsets"], tr["u_acc"], tr["u_res"], 1.0)
    assert res["flag_accept"][0] and not res["flag_accept"][1]


def test_three_token_joint_position_dependent():
    """Context-free but position-dependent p_pos, q_pos: run verify steps, each starting at the
    next unfilled position, until three tokens exist; the triple must follow p_1 x p_2 x p_3."""
    V, Lstep, npos = 3, 3, 3 + K + 1
    rng0 = np.random.default_rng(77)
    P = rng0.dirichlet(np.ones(V) * 2.0, size=npos)
    Q = rng0.dirichlet(np.ones(V) * 2.0, size=npos)
    zt_all = logits_of(P)
    zd_all = logits_of(Q)
    rng = np.random.default_rng(13)
    n, chunk = 400_000, 100_000
    counts = np.zeros(V ** 3, dtype=np.int64)
    for c0 in range(0, n, chunk):
        seqs = [[] for _ in range(chunk)]
        for step in range(3):
            for start in range(3):          # trials whose next position is start + 1
                ids = [t for t in range(chunk) if len(seqs[t]) == start]
                if not ids:
                    continue
                tr = build_trials(zt_all[start:start + K + 1], zd_all[start:start + K], Lstep,
                                  len(ids), rng, round_idx=7000 + 100 * step + 10 * start + c0 // chunk)
                res = _run(tr)
                for i, t in enumerate(ids):
                    seqs[t].extend(res["out_tokens"][i, :res["n_out"][i]].tolist())
        idx = np.array([s[0] * V * V + s[1] * V + s[2] for s in seqs])
        counts += np.bincount(idx, minlength=V ** 3)
    pe = [target_probs(zt_all[i]) for i in range(3)]
    joint = np.einsum("i,j,k->ijk", pe[0], pe[1], pe[2]).reshape(-1)
    _chi2_ok(counts, joint)


def test_zero_uniform_picks_first_positive_mass():
    """u_res = 0: the draw is the smallest index with positive mass (C(v) > 0), never a
    zero-probability token before it — for the bonus and for the residual."""
    zt = np.tile(logits_of([0.0, 0.0, 0.6, 0.4]), (K + 1, 1))
    zd = np.tile(logits_of([0.0, 0.0, 0.2, 0.8]), (K, 1))
    rng = np.random.default_rng(4)
    tr = build_trials(zt, zd, 2, 64, rng, round_idx=3)
    tr["u_res"] = np.zeros_like(tr["u_res"])
    tr["draft_tokens"][:, :] = 3                    # p/q = 0.5
    tr["u_acc"][:32] = 0.9                          # rejected at position 1 -> residual (0,0,.4,0)
    tr["u_acc"][32:] = 0.1                          # accepted twice -> bonus from p_3
    res = _run(tr)
    assert np.all(res["accepted_len"][:32] == 0) and np.all(res["out_tokens"][:32, 0] == 2)
    assert np.all(res["accepted_len"][32:] == 2) and np.all(res["out_tokens"][32:, 2] == 2)


def test_empty_residual_draws_from_target():
    """p == q with u = 1 rejects the first draft token and leaves max(0, p - q) = 0 everywhere;
    the correction is then drawn from p by the same inverse CDF (hand-computed cumulative
    boundaries 0.1, 0.3, 0.6 of p = (0.1, 0.2, 0.3, 0.4)), and over many trials it follows p."""
    p = [0.1, 0.2, 0.3, 0.4]
    z = logits_of(p)
    zt = np.tile(z, (K + 1, 1))
    zd = np.tile(z, (K, 1))
    rng = np.random.default_rng(17)
    tr = build_trials(zt, zd, 3, 200_000, rng, round_idx=4)
    tr["u_acc"] = np.array(tr["u_acc"], copy=True)
    tr["u_res"] = np.array(tr["u_res"], copy=True)
    tr["u_acc"][:, 0] = 1.0
    tr["u_res"][:4, 0] = [0.05, 0.15, 0.45, 0.95]
    res = _run(tr)
    assert np.all(res["accepted_len"] == 0)
    assert np.all(res["n_out"] == 1)
    assert res["out_tokens"][:4, 0].tolist() == [0, 1, 2, 3]
    assert np.all(res["out_tokens"][:, 1:] == -1)
    _chi2_ok(np.bincount(res["out_tokens"][:, 0], minlength=4), target_probs(z))
