"""Synthetic Markov-head draft step — oracle (TEST INFRASTRUCTURE ONLY).

[P1] section "1. 半自回归生成": the drafter keeps a parallel backbone (one pass produces the
whole block) and adds a light sequential module that injects the prefix token by token; one
form of it is a Markov head that depends only on the previous token.  [P3] "成本与质量的考量":
the drafting is a small share of the compute.

Readings (listed in the design notes; the pages give no formulas and no trained weights exist):
  * block position k (1..K) of request r has logits z_k = B[r, k] + E[x_{k-1}] @ U: the
    backbone's block logits plus a previous-token transition term of rank d (E: [V][d],
    U: [d][V]); x_0 is the request's last emitted token;
  * the draft distribution is the one the verifier reads: z_k rounded to bfloat16;
  * sampling is the Gumbel-max trick, x_k = argmax_v z_k[v] / tau + g_v, g = -log(-log(u)),
    u from Philox4x32-10 (workloads/philox.py), key (seed, 0), counter
    (round, r, v // 4, 3 + 256 * (k - 1)), word v % 4, u = ((word >> 8) + 1/2) * 2^-24;
    tau <= 0 is greedy: the lowest index of the maximum of z_k.

Parity: draft logits equal after bfloat16 rounding (a float32 sum may round differently from
the float64 one only at a rounding boundary: tolerated in a tiny fraction of elements); tokens
equal unless flagged (the two best scores closer than FLAG_GAP).  Pinned by
tests/test_oracle_draft.py: a transition that forces x_k = x_{k-1} + 1 (closed form), greedy
with no transition equals the library argmax, and a chi-square test of the sampled token
against softmax(z / tau).
"""
from __future__ import annotations

import numpy as np

from workloads.philox import philox4x32

FLAG_GAP = 1e-3
STREAM_DRAFT_VOCAB = 3


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), returned as float64.

    One rounding of the float64 value: bfloat16 keeps 8 significant bits down to 2^-126 and a
    fixed quantum of 2^-133 below it (subnormals); a value at or past the midpoint between the
    largest finite bfloat16, (2 - 2^-7) * 2^127, and 2^128 becomes infinite.
    """
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    fin = np.isfinite(x)
    xf = x[fin]
    _, e = np.frexp(xf)                        # xf = m * 2^e, 1/2 <= |m| < 1
    q = np.ldexp(1.0, np.maximum(e, -125) - 8)  # the bfloat16 quantum at xf's binade
    r = np.round(xf / q) * q                   # exact scaling, round half to even
    r[np.abs(r) >= 2.0 ** 128] = np.inf * np.sign(r[np.abs(r) >= 2.0 ** 128])
    out[fin] = r
    return out


def gumbel_uniforms(round_idx: int, r: int, k: int, V: int, seed: int = 0) -> np.ndarray:
    """u[v] in (0, 1) for block position k (1-based) of request r."""
    nb = (V + 3) // 4
    ctr = np.empty((nb, 4), dtype=np.uint32)
    ctr[:, 0] = np.uint32(round_idx)
    ctr[:, 1] = np.uint32(r)
    ctr[:, 2] = np.arange(nb, dtype=np.uint32)
    ctr[:, 3] = np.uint32(STREAM_DRAFT_VOCAB + 256 * (k - 1))
    key = np.array([seed & 0xFFFFFFFF, 0], dtype=np.uint32)
    words = philox4x32(ctr, key).reshape(-1)[:V]
    return ((words >> np.uint32(8)).astype(np.float64) + 0.5) * 2.0 ** -24


def markov_draft_ref(block_logits, E, U, x0, tau: float, round_idx: int, seed: int = 0):
    """block_logits [R][K][V], E [V][d], U [d][V], x0 int [R].
    Returns (draft logits [R][K][V] float64 holding bf16 values, tokens int32 [R][K],
    flags bool [R][K])."""
    B = np.asarray(block_logits, dtype=np.float64)
    E = np.asarray(E, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    R, K, V = B.shape
    z_all = np.empty_like(B)
    tok = np.empty((R, K), dtype=np.int32)
    flags = np.zeros((R, K), dtype=bool)
    prev = np.asarray(x0, dtype=np.int64).copy()
    for k in range(1, K + 1):
        for r in range(R):
            z = bf16_round(B[r, k - 1] + E[prev[r]] @ U)
            z_all[r, k - 1] = z
            if tau > 0:
                u = gumbel_uniforms(round_idx, r, k, V, seed)
                s = z / tau - np.log(-np.log(u))
            else:
                s = z
            best = int(np.argmax(s))
            tok[r, k - 1] = best
            if tau > 0:
                top2 = np.partition(s, -2)[-2:]
                flags[r, k - 1] = (top2[1] - top2[0]) < FLAG_GAP
            prev[r] = best
    return z_all, tok, flags
