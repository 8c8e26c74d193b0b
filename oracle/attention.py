"""Oracle: flattened ragged GQA verify attention over a paged KV cache.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

What the pages fix and the readings taken:
  * [P1 engineering table, "内核利用率暴跌"] variable-length verification pads and unbalances
    standard decode kernels; DSpark flattens every verify token into an independent element
    and passes sequence membership and intra-sequence dependency through a marker tensor.
    [P2 §一] the target checks all draft tokens in one batched pass.
  * Readings (the pages give no attention formula): each verify token t = (r, pos) attends,
    per query head h, to its request's cached keys at positions 0..kv_len[r]-1 and to the
    request's own verify tokens at positions <= pos (causal); o = softmax(q.k^T * scale).v.
    Query heads g*G .. g*G+G-1 share KV head g.  Inputs are post-positional-encoding.
    The verify tokens' keys/values arrive in separate flat arrays k_new/v_new [T][Hkv][D]
    (row q_offsets[r] + j) and are not yet in the cache.
  * Cache layout kv_pages[page][0=K,1=V][Hkv][page_size][D]; block_table[r][i] is the
    physical page holding request r's positions i*page_size .. (i+1)*page_size - 1.

Two independent restatements: attn_ref_flat walks the flat token list through its markers;
attn_ref_dense pads every request into a dense masked batch.  Parity pins: flat == dense,
dense == torch scaled_dot_product_attention (float64, run as a library routine), and closed
forms with scale 0 (uniform weights over exactly the visible keys).
"""
from __future__ import annotations

import numpy as np


def _as64(a):
    return np.asarray(a, dtype=np.float64)


def gather_cache(kv_pages, block_table, r: int, g: int, n: int, page_size: int):
    """Keys and values of request r, KV head g, cache positions 0..n-1 -> ([n][D], [n][D])."""
    pos = np.arange(n)
    pages = np.asarray(block_table)[r, pos // page_size]
    slot = pos % page_size
    return kv_pages[pages, 0, g, slot, :], kv_pages[pages, 1, g, slot, :]


def attn_ref_flat(q, k_new, v_new, kv_pages, block_table, kv_len, markers, q_offsets,
                  scale: float, page_size: int, rows=None) -> np.ndarray:
    """Attention of every flattened verify token (or of the listed (t, h) rows only).

    q [T][Hq][D], k_new/v_new [T][Hkv][D], kv_pages [P][2][Hkv][page][D]; markers [T][2].
    Returns float64 [T][Hq][D] (rows not listed stay zero).
    """
    q, k_new, v_new, kv_pages = _as64(q), _as64(k_new), _as64(v_new), _as64(kv_pages)
    markers = np.asarray(markers)
    q_offsets = np.asarray(q_offsets)
    kv_len = np.asarray(kv_len)
    T, Hq, D = q.shape
    Hkv = k_new.shape[1]
    G = Hq // Hkv
    out = np.zeros((T, Hq, D), dtype=np.float64)
    if rows is None:
        rows = [(t, h) for t in range(T) for h in range(Hq)]
    for t, h in rows:
        r, pos = int(markers[t, 0]), int(markers[t, 1])
        n = int(kv_len[r])
        j = pos - n                      # index of this token within its request's block
        t0 = int(q_offsets[r])
        g = h // G
        Kc, Vc = gather_cache(kv_pages, block_table, r, g, n, page_size)
        Kall = np.concatenate([Kc, k_new[t0:t0 + j + 1, g]], axis=0)
        Vall = np.concatenate([Vc, v_new[t0:t0 + j + 1, g]], axis=0)
        s = (Kall @ q[t, h]) * scale
        w = np.exp(s - s.max())
        w = w / w.sum()
        out[t, h] = w @ Vall
    return out


def attn_ref_dense(q, k_new, v_new, kv_pages, block_table, kv_len, verify_len,
                   scale: float, page_size: int) -> np.ndarray:
    """Same attention computed request-padded: Q_max queries x (n_max + Q_max) keys per
    request with a -inf mask, one dense softmax(Q K^T) V per request, scattered back flat."""
    q, k_new, v_new, kv_pages = _as64(q), _as64(k_new), _as64(v_new), _as64(kv_pages)
    L = np.asarray(verify_len, dtype=np.int64)
    n = np.asarray(kv_len, dtype=np.int64)
    R = len(L)
    Hq, D = q.shape[1], q.shape[2]
    Hkv = k_new.shape[1]
    G = Hq // Hkv
    Qr = L + 1
    Qmax, nmax = int(Qr.max()), int(n.max())
    C = nmax + Qmax
    q_off = np.concatenate([[0], np.cumsum(Qr)])

    Qp = np.zeros((R, Qmax, Hq, D))
    Kp = np.zeros((R, C, Hkv, D))
    Vp = np.zeros((R, C, Hkv, D))
    mask = np.zeros((R, Qmax, C), dtype=bool)
    for r in range(R):
        a, b = q_off[r], q_off[r + 1]
        Qp[r, :Qr[r]] = q[a:b]
        for g in range(Hkv):
            Kc, Vc = gather_cache(kv_pages, block_table, r, g, int(n[r]), page_size)
            Kp[r, :n[r], g] = Kc
            Vp[r, :n[r], g] = Vc
        Kp[r, nmax:nmax + Qr[r]] = k_new[a:b]
        Vp[r, nmax:nmax + Qr[r]] = v_new[a:b]
        for j in range(Qr[r]):
            mask[r, j, :n[r]] = True
            mask[r, j, nmax:nmax + j + 1] = True

    Kh = np.repeat(Kp, G, axis=2)            # [R][C][Hq][D]: head h reads KV head h // G
    Vh = np.repeat(Vp, G, axis=2)
    scores = np.einsum("rjhd,rchd->rhjc", Qp, Kh) * scale
    scores = np.where(mask[:, None, :, :], scores, -np.inf)
    m = scores.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(scores - m)
    w = w / np.maximum(w.sum(axis=-1, keepdims=True), 1e-300)
    o = np.einsum("rhjc,rchd->rjhd", w, Vh)
    out = np.zeros((int(q_off[-1]), Hq, D))
    for r in range(R):
        out[q_off[r]:q_off[r + 1]] = o[r, :Qr[r]]
    return out
