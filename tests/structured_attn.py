"""Structured keys and values for attention checks whose expected output has a closed form.

Key dimension 0 of cache position s in physical page pg (KV head g) is 312 * kappa(pg, g, s),
kappa a pseudo-random bit; every other key dimension is 0, every verify token's own key has
dimension 0 = 312, and every query is e_0.  With scale 1/sqrt(128) a key with kappa = 1 scores
about 40 (log2 units) above one with kappa = 0, so each query averages the values of exactly
its selected keys (each other key weighs about 2^-40 as much).  Values carry codes of the
page, of the slot within the page and of the KV head; the verify tokens' own values are random
integers in [-8, 8].  Every value is a small multiple of 1/4, so the float32 sums a kernel forms
are exact and its only rounding is the final store.  A page read for the wrong position, a
dropped or repeated page, swapped d-halves, a wrong GQA head mapping, a misrouted split-KV
piece or a wrong causal range moves the output far outside that rounding.

Input synthesis and the closed form only: no attention arithmetic of either implementation
lives here.  Used on the CPU to pin the oracle and on the GPU for full-size parity.
"""
from __future__ import annotations

import numpy as np
import torch

KAPPA_SCORE = 312.0   # exact in bf16; 312 / sqrt(128) * log2(e) ~ 39.8


def kappa(pg, g, s):
    """Selection bit of cache slot s of physical page pg, KV head g (float64 0/1)."""
    h = (np.asarray(pg).astype(np.uint64) * np.uint64(2654435761)
         + np.asarray(g).astype(np.uint64) * np.uint64(40503)
         + np.asarray(s).astype(np.uint64) * np.uint64(9973)) & np.uint64(0xFFFFFFFF)
    return ((h >> np.uint64(7)) & np.uint64(1)).astype(np.float64)


def value_codes(pg, g, s):
    """Value of dimension class d % 3 = 0, 1, 2 at (pg, g, s) (broadcast shapes)."""
    pg, g, s = np.asarray(pg), np.asarray(g), np.asarray(s)
    pc = ((pg * 8 + g) * 37) % 17 - 8
    sc = (s % 16) - 8
    zero = 0 * pc + 0 * sc
    return ((pc + zero).astype(np.float64), (sc / 4.0 + zero).astype(np.float64),
            (((pc * sc) % 5) - 2 + zero).astype(np.float64))


def install_structured(inp, layer: int = 0, seed: int = 5):
    """Overwrite the KV cache (copy 0) and layer `layer`'s q, k_new, v_new of `inp` in place."""
    cache = inp.kv_caches[0]
    dev = cache.device
    P, _, Hkv, page, D = cache.shape
    g = np.arange(Hkv)[None, :, None]
    s = np.arange(page)[None, None, :]
    cls = (torch.arange(D, device=dev) % 3)[None, None, None, :]
    step = max(1, (1 << 26) // (Hkv * page * D))
    for p0 in range(0, P, step):
        p1 = min(P, p0 + step)
        pg = np.arange(p0, p1)[:, None, None]
        kap = torch.as_tensor(kappa(pg, g, s), dtype=torch.float32, device=dev)
        c0, c1, c2 = (torch.as_tensor(np.broadcast_to(c, (p1 - p0, Hkv, page)).copy(),
                                      dtype=torch.float32, device=dev)
                      for c in value_codes(pg, g, s))
        kblock = torch.zeros((p1 - p0, Hkv, page, D), device=dev)
        kblock[..., 0] = kap * KAPPA_SCORE
        vblock = torch.where(cls == 0, c0[..., None],
                             torch.where(cls == 1, c1[..., None], c2[..., None]))
        cache[p0:p1, 0] = kblock.to(cache.dtype)
        cache[p0:p1, 1] = vblock.to(cache.dtype)
    inp.q[layer].zero_()
    inp.q[layer][..., 0] = 1.0
    inp.k_new[layer].zero_()
    inp.k_new[layer][..., 0] = KAPPA_SCORE
    gen = torch.Generator(device=dev).manual_seed(seed)
    inp.v_new[layer].copy_(torch.randint(-8, 9, inp.v_new[layer].shape, generator=gen,
                                         device=dev).to(inp.v_new.dtype))


def structured_expected(inp, q_offsets, kv_len, layer: int = 0) -> np.ndarray:
    """Closed form [T][Hkv][D]: for verify token j of request r and KV head g, the mean of the
    values of r's cached keys with kappa = 1 and of r's verify tokens 0..j (every query head of
    the group gets it)."""
    cfg = inp.cfg
    page, Hkv, D = cfg.page_size, cfg.Hkv, cfg.D
    table = inp.block_table.cpu().numpy().astype(np.int64)
    vnew = inp.v_new[layer].float().cpu().numpy().astype(np.float64)   # [T_cap][Hkv][D]
    qo = np.asarray(q_offsets, dtype=np.int64)
    T = int(qo[-1])
    gg = np.broadcast_to(np.arange(Hkv)[:, None], (Hkv, page))
    ss = np.broadcast_to(np.arange(page)[None, :], (Hkv, page))
    cls = np.arange(D) % 3
    out = np.empty((T, Hkv, D))
    for r in range(cfg.R):
        n = int(kv_len[r])
        num = np.zeros((Hkv, 3))
        den = np.zeros(Hkv)
        for i in range(-(-n // page)):
            pg = np.full((Hkv, page), table[r, i])
            m = min(page, n - i * page)
            kap = kappa(pg, gg, ss)[:, :m]
            for c, code in enumerate(value_codes(pg, gg, ss)):
                num[:, c] += (kap * code[:, :m]).sum(axis=1)
            den += kap.sum(axis=1)
        run = num[:, cls].copy()                                   # [Hkv][D]
        for j, t in enumerate(range(int(qo[r]), int(qo[r + 1]))):  # token j sees tokens 0..j
            run += vnew[t]
            out[t] = run / (den + j + 1)[:, None]
    return out
