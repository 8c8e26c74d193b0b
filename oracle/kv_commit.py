"""KV commit after acceptance — oracle (TEST INFRASTRUCTURE ONLY).

[P1] opening section (drafts the target confirms are adopted, "猜对了就采纳"; from the first
wrong one the target writes its own) and [P2] §一 (the verified tokens are kept): after the
accept step request r keeps its verify tokens j = 0 .. a_r — token 0 is the last emitted token
(position kv_len[r]), whose K/V this verify pass computed, then the a_r accepted drafts.  Their
K/V rows become part of the request's paged cache, at positions kv_len[r] + j, and the cache
length grows by a_r + 1.  Rejected drafts were only ever in k_new / v_new, so "rollback" writes
nothing.

Reading (listed in the design notes): the commit covers every layer given; a request whose
flattening (q_offsets), accepted length or block table is malformed is left untouched.

Parity: bit-exact (a copy).  Pinned by tests/test_oracle_kv_commit.py: attention over the
committed cache equals attention over the old cache plus the kept rows (the attention oracle's
own page gathering, an independent code path), bytes outside the written slots unchanged,
rejected rows absent, malformed requests skipped.
"""
from __future__ import annotations

import numpy as np


def kv_commit_ref(k_new, v_new, caches, block_table, kv_len, q_offsets, accepted_len, K: int,
                  T_cap: int):
    """k_new, v_new: [layers][T_cap][Hkv][D]; caches: [layers][P][2][Hkv][page][D] (any dtype,
    copied as is); block_table: int [R][max_pages]; kv_len, accepted_len: int [R];
    q_offsets: int [R + 1].  Returns (new caches, kv_len_out, skipped requests)."""
    caches = np.array(caches, copy=True)
    k_new, v_new = np.asarray(k_new), np.asarray(v_new)
    block_table = np.asarray(block_table)
    kv_len = np.asarray(kv_len, dtype=np.int64)
    qo = np.asarray(q_offsets, dtype=np.int64)
    acc = np.asarray(accepted_len, dtype=np.int64)
    layers, P, _, Hkv, page, D = caches.shape
    R, max_pages = block_table.shape
    out_len = kv_len.copy()
    skipped = []
    for r in range(R):
        t0, Q = int(qo[r]), int(qo[r + 1] - qo[r])
        n, a = int(kv_len[r]), int(acc[r])
        ok = 1 <= Q <= K + 1 and t0 >= 0 and t0 + Q <= T_cap and 0 <= a <= Q - 1 and n >= 0
        ok = ok and (n + a) // page < max_pages
        if ok:
            pages = [int(block_table[r, (n + j) // page]) for j in range(a + 1)]
            ok = all(0 <= pg < P for pg in pages)
        if not ok:
            skipped.append(r)
            continue
        for j in range(a + 1):
            pos = n + j
            pg, slot = int(block_table[r, pos // page]), pos % page
            caches[:, pg, 0, :, slot, :] = k_new[:, t0 + j]
            caches[:, pg, 1, :, slot, :] = v_new[:, t0 + j]
        out_len[r] = n + a + 1
    return caches, out_len.astype(np.int32), skipped
