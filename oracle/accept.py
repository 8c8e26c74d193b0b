"""Oracle: exact acceptance rule, longest accepted prefix, residual / bonus resampling.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

What the pages fix:
  * [P2 §一] the target verifies the N draft tokens in one pass, keeps the verified ones and
    resamples after the first divergence; the output distribution provably equals the target
    model's.  [P3 "DSpark的神奇之处"] keep the leading run of correct guesses, and from the
    first wrong one the large model writes a correct token itself.  [P3 "成本与质量的考量"]
    the acceptance rule (rejection sampling) preserves the target distribution exactly.
    [P4] the target accepts the longest correct prefix.
  * Readings (the pages give no formula; this is the textbook rule that has those
    properties): with p = softmax(z_target / tau), q = softmax(z_draft / tau) at each block
    position, draft token x_k is accepted iff u_acc[k] < min(1, p_k(x_k) / q_k(x_k));
    a = number accepted before the first rejection.  If a < L the correction is drawn from
    the residual max(0, p_{a+1} - q_{a+1}) (normalised); if a == L (including L == 0) a bonus
    token is drawn from p_{L+1}.  Draws use the inverse CDF in vocabulary index order: the
    smallest v with C(v) > u_res[a] * C(V-1), C the inclusive running sum.  If the residual
    is empty in floating point the draw falls back to p_{a+1}.
  * Greedy verification (temperature <= 0): accept iff x_k == argmax z_target row (lowest
    index on ties); the correction / bonus is that argmax at row a.
  * Layout: target row q_offsets[r] + j holds position j+1 of request r (j = 0..L_r);
    draft_logits[r][k-1] and draft_tokens[r][k-1] hold position k.

Decisions within FLAG_ABS of a threshold — |u - min(1, p/q)| or |u*Z - C(v)| relative to Z
at either side of the chosen index — are flagged per request: a float32-exp implementation
may legitimately decide them the other way.

Parity: pinned by a chi-square goodness-of-fit of the emitted tokens against p (marginal of
the first token, and 3-token joints under stationary p, q), deterministic hand-built cases
(ratios 0 or >= 1), greedy == numpy.argmax, and invariants (0 <= a <= L, n_out = a + 1).
"""
from __future__ import annotations

import numpy as np

FLAG_ABS = 1e-6


def _softmax(z: np.ndarray, tau: float) -> np.ndarray:
    m = z.max(axis=-1, keepdims=True)
    e = np.exp((z - m) / tau)
    return e / e.sum(axis=-1, keepdims=True)


def accept_ref(target_logits, draft_logits, draft_tokens, verify_len, q_offsets,
               u_acc, u_res, temperature: float, chunk_bytes: int = 1 << 28) -> dict:
    """Verify every request's scheduled draft prefix.

    target_logits [T][V], draft_logits [R][K][V] (any float dtype; upcast exactly to float64),
    draft_tokens int [R][K], verify_len int [R], q_offsets int [R+1], u_acc float32 [R][K],
    u_res float32 [R][K+1].  Returns accepted_len [R], out_tokens [R][K+1] (-1 padded),
    n_out [R], flagged [R] and the two flag components.
    """
    target_logits = np.asarray(target_logits)
    draft_logits = np.asarray(draft_logits)
    x_all = np.asarray(draft_tokens, dtype=np.int64)
    Lall = np.asarray(verify_len, dtype=np.int64)
    q_off = np.asarray(q_offsets, dtype=np.int64)
    R, K = x_all.shape
    V = target_logits.shape[1]
    greedy = temperature <= 0
    if np.any(Lall < 0) or np.any(Lall > K):
        raise ValueError("verify_len must lie in [0, K]")

    accepted = np.zeros(R, dtype=np.int32)
    out = np.full((R, K + 1), -1, dtype=np.int32)
    flag_acc = np.zeros(R, dtype=bool)
    flag_smp = np.zeros(R, dtype=bool)
    per_req = 6 * (2 * K + 1) * V * 8
    step = max(1, chunk_bytes // per_req)
    kk = np.arange(K)

    for r0 in range(0, R, step):
        r1 = min(R, r0 + step)
        n = r1 - r0
        ar = np.arange(n)
        L = Lall[r0:r1]
        x = x_all[r0:r1]
        rows = q_off[r0:r1, None] + np.minimum(np.arange(K + 1)[None, :], L[:, None])
        zt = target_logits[rows].astype(np.float64)            # [n][K+1][V]
        valid = kk[None, :] < L[:, None]

        if greedy:
            amax = zt.argmax(axis=-1)                            # lowest index on ties
            ok = (x == amax[:, :K]) & valid
            a = np.cumprod(ok, axis=1).sum(axis=1)
            corr = amax[ar, a]
        else:
            tau = float(temperature)
            p = _softmax(zt, tau)
            q = _softmax(draft_logits[r0:r1].astype(np.float64), tau)   # [n][K][V]
            px = np.take_along_axis(p[:, :K], x[..., None], axis=-1)[..., 0]
            qx = np.take_along_axis(q, x[..., None], axis=-1)[..., 0]
            with np.errstate(divide="ignore", invalid="ignore"):
                ratio = np.where(qx > 0, px / np.where(qx > 0, qx, 1.0),
                                 np.where(px > 0, np.inf, 0.0))
            thr = np.minimum(1.0, ratio)
            u = np.asarray(u_acc[r0:r1], dtype=np.float64)
            ok = (u < thr) & valid
            a = np.cumprod(ok, axis=1).sum(axis=1)
            taken = (kk[None, :] <= a[:, None]) & valid          # accepts, then the rejection
            flag_acc[r0:r1] = np.any(taken & (np.abs(u - thr) < FLAG_ABS), axis=1)

            pa = p[ar, a]                                        # target row at position a+1
            qa = q[ar, np.minimum(a, K - 1)]
            residual = (a < L)[:, None]
            w = np.where(residual, np.maximum(0.0, pa - qa), pa)
            C = np.cumsum(w, axis=-1)
            empty = C[:, -1] <= 0
            if np.any(empty):
                C[empty] = np.cumsum(pa[empty], axis=-1)
            Z = C[:, -1]
            thr_s = np.asarray(u_res[r0:r1], dtype=np.float64)[ar, a] * Z
            corr = np.argmax(C > thr_s[:, None], axis=-1)
            c_hi = C[ar, corr]
            c_lo = np.where(corr > 0, C[ar, np.maximum(corr - 1, 0)], 0.0)
            flag_smp[r0:r1] = ((np.abs(thr_s - c_hi) < FLAG_ABS * Z)
                               | (np.abs(thr_s - c_lo) < FLAG_ABS * Z))

        accepted[r0:r1] = a
        xpad = np.concatenate([x, np.full((n, 1), -1)], axis=1)
        block = np.where(np.arange(K + 1)[None, :] < a[:, None], xpad, -1)
        block[ar, a] = corr
        out[r0:r1] = block

    return dict(accepted_len=accepted, out_tokens=out, n_out=accepted + 1,
                flagged=flag_acc | flag_smp, flag_accept=flag_acc, flag_sample=flag_smp)
