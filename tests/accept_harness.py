"""Trial builders for distribution tests of the acceptance rule (test infrastructure).

A "trial" is one request whose block positions share given target / draft distributions.
Logits are log-probabilities (float32, -inf where the probability is 0); drafts are sampled from
q by inverse CDF with numpy; uniforms come from Philox.  Nothing here implements acceptance.
"""
from __future__ import annotations

import numpy as np

from workloads.philox import step_uniforms


def logits_of(prob) -> np.ndarray:
    prob = np.asarray(prob, dtype=np.float64)
    with np.errstate(divide="ignore"):
        return np.log(prob).astype(np.float32)


def target_probs(z_row) -> np.ndarray:
    """The distribution a logit row defines (float64), for expected counts."""
    z = np.asarray(z_row, dtype=np.float64)
    e = np.exp(z - z.max())
    return e / e.sum()


def sample_rows(prob_rows: np.ndarray, rng: np.random.Generator) -> np.ndarray:
    """One draw per row from prob_rows [..., V] by inverse CDF."""
    cdf = np.cumsum(prob_rows, axis=-1)
    u = rng.random(prob_rows.shape[:-1])[..., None] * cdf[..., -1:]
    idx = (cdf <= u).sum(axis=-1)
    return np.minimum(idx, prob_rows.shape[-1] - 1)


def build_trials(zt_rows, zd_rows, L: int, n: int, rng, round_idx: int, r_base: int = 0):
    """n identical-distribution requests, each verifying L drafts.

    zt_rows: float32 [K+1][V] target logits for positions 1..K+1; zd_rows: float32 [K][V].
    Returns a dict of host arrays in the library's layout.
    """
    zt_rows = np.asarray(zt_rows, dtype=np.float32)
    zd_rows = np.asarray(zd_rows, dtype=np.float32)
    K = zd_rows.shape[0]
    qd = np.stack([target_probs(zd_rows[k]) for k in range(K)])       # [K][V]
    draft_tokens = sample_rows(np.broadcast_to(qd, (n, K, qd.shape[-1])), rng).astype(np.int32)
    verify_len = np.full(n, L, dtype=np.int32)
    q_offsets = np.arange(n + 1, dtype=np.int32) * (L + 1)
    target = np.tile(zt_rows[:L + 1], (n, 1))                        # [n*(L+1)][V]
    draft = np.broadcast_to(zd_rows, (n, K, zd_rows.shape[-1]))
    ua, ur = step_uniforms(round_idx, r_base + n, K)
    return dict(target_logits=target, draft_logits=draft, draft_tokens=draft_tokens,
                verify_len=verify_len, q_offsets=q_offsets,
                u_acc=ua[r_base:], u_res=ur[r_base:])
