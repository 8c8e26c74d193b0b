"""Philox4x32-10 counter-based random numbers, written from its published definition.

Source: J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel Random Numbers:
As Easy as 1, 2, 3", SC'11, section 3 (the Philox S-box: two 32x32->64 multiplies per
round, key schedule bumped by the Weyl constants between rounds).

This module is an input generator: the acceptance uniforms of a verify step are drawn here
and handed, as plain arrays, to both the CUDA path and the CPU oracle.  It holds none of
the verification arithmetic.

Uniform convention: u = (x0 >> 8) * 2**-24, exact in float32 and float64, in [0, 1).
Counter layout for the uniforms of one verify step: (round, request, position, stream) with
stream 0 = draft sampling, 1 = acceptance tests, 2 = residual / bonus sampling.
"""
from __future__ import annotations

import numpy as np

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
_MASK32 = np.uint64(0xFFFFFFFF)

STREAM_DRAFT = 0
STREAM_ACCEPT = 1
STREAM_RESIDUAL = 2


def philox4x32(counter, key, rounds: int = 10) -> np.ndarray:
    """Apply the Philox4x32 bijection.

    counter: uint32 array [..., 4]; key: uint32 array [..., 2] (broadcast against counter).
    Returns uint32 [..., 4].
    """
    counter = np.asarray(counter, dtype=np.uint32)
    key = np.asarray(key, dtype=np.uint32)
    c0, c1, c2, c3 = (counter[..., i].astype(np.uint64) for i in range(4))
    k0 = key[..., 0].astype(np.uint64)
    k1 = key[..., 1].astype(np.uint64)
    m0 = np.uint64(PHILOX_M0)
    m1 = np.uint64(PHILOX_M1)
    for rnd in range(rounds):
        if rnd > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK32
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK32
        p0 = m0 * c0  # 32x32 -> 64 bit product, exact in uint64
        p1 = m1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def uniforms_from_words(x0: np.ndarray) -> np.ndarray:
    """Map 32-bit words to float32 uniforms in [0, 1) using their top 24 bits."""
    return ((np.asarray(x0, dtype=np.uint32) >> np.uint32(8)).astype(np.float64)
            * 2.0 ** -24).astype(np.float32)


def step_uniforms(round_idx: int, R: int, K: int, seed: int = 0):
    """Acceptance uniforms u_acc[R][K] and residual uniforms u_res[R][K+1] for one round."""
    key = np.array([seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF], dtype=np.uint32)

    def draw(n_pos: int, stream: int) -> np.ndarray:
        r = np.arange(R, dtype=np.uint32)[:, None]
        k = np.arange(n_pos, dtype=np.uint32)[None, :]
        ctr = np.empty((R, n_pos, 4), dtype=np.uint32)
        ctr[..., 0] = np.uint32(round_idx)
        ctr[..., 1] = r
        ctr[..., 2] = k
        ctr[..., 3] = np.uint32(stream)
        return uniforms_from_words(philox4x32(ctr, key)[..., 0])

    return draw(K, STREAM_ACCEPT), draw(K + 1, STREAM_RESIDUAL)
