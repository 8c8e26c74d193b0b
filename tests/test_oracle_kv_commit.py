"""Pins of the KV-commit oracle (oracle/kv_commit.py) against properties that do not go
through its own slot arithmetic.

The central pin uses the attention oracle (which gathers cache pages through the block table in
its own code): a fresh query attending over the committed cache must see exactly what it sees
when the kept rows are still verify tokens in front of it.
"""
import numpy as np
import pytest

from oracle.attention import attn_ref_flat
from oracle.kv_commit import kv_commit_ref

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _case(seed, R=4, Hkv=2, G=2, D=16, page=8, K=5, layers=2, P=None):
    rng = np.random.default_rng(seed)
    kv_len = rng.integers(0, 30, size=R)
    L = rng.integers(0, K + 1, size=R)
    acc = np.array([rng.integers(0, l + 1) for l in L])
    qo = np.concatenate([[0], np.cumsum(L + 1)]).astype(np.int64)
    T_cap = int(qo[-1]) + 3
    max_pages = (int(kv_len.max()) + K + 1) // page + 2
    P = P or R * max_pages + 3
    perm = rng.permutation(P)
    block_table = perm[: R * max_pages].reshape(R, max_pages)
    caches = rng.standard_normal((layers, P, 2, Hkv, page, D))
    k_new = rng.standard_normal((layers, T_cap, Hkv, D))
    v_new = rng.standard_normal((layers, T_cap, Hkv, D))
    return dict(rng=rng, R=R, Hkv=Hkv, G=G, D=D, page=page, K=K, layers=layers, kv_len=kv_len,
                L=L, acc=acc, qo=qo, T_cap=T_cap, block_table=block_table, caches=caches,
                k_new=k_new, v_new=v_new)


@pytest.mark.parametrize("seed", range(6))
def test_attention_over_committed_cache_equals_attention_over_kept_verify_rows(seed):
    c = _case(seed)
    new, kv_out, skipped = kv_commit_ref(c["k_new"], c["v_new"], c["caches"], c["block_table"],
                                         c["kv_len"], c["qo"], c["acc"], c["K"], c["T_cap"])
    assert skipped == []
    rng, R, Hkv, G, D = c["rng"], c["R"], c["Hkv"], c["G"], c["D"]
    Hq = Hkv * G
    scale = 1 / np.sqrt(D)
    for layer in range(c["layers"]):
        # next round: one fresh token per request at position kv_out[r]
        qf = rng.standard_normal((R, Hq, D))
        kf = rng.standard_normal((R, Hkv, D))
        vf = rng.standard_normal((R, Hkv, D))
        markers = np.stack([np.arange(R), kv_out], axis=1)
        got = attn_ref_flat(qf, kf, vf, new[layer], c["block_table"], kv_out, markers,
                            np.arange(R + 1), scale, c["page"])
        # same token as the last verify token after the kept rows, over the old cache
        for r in range(R):
            a, t0, n = int(c["acc"][r]), int(c["qo"][r]), int(c["kv_len"][r])
            kb = np.concatenate([c["k_new"][layer, t0:t0 + a + 1], kf[r:r + 1]], axis=0)
            vb = np.concatenate([c["v_new"][layer, t0:t0 + a + 1], vf[r:r + 1]], axis=0)
            qb = np.zeros((a + 2, Hq, D))
            qb[-1] = qf[r]
            mk = np.stack([np.full(a + 2, r), n + np.arange(a + 2)], axis=1)
            qo_b = np.zeros(R + 1, dtype=np.int64)
            qo_b[r + 1:] = a + 2
            want = attn_ref_flat(qb, kb, vb, c["caches"][layer], c["block_table"], c["kv_len"], mk,
                                 qo_b, scale, c["page"], rows=[(a + 1, h) for h in range(Hq)])
            np.testing.assert_allclose(got[r], want[a + 1], rtol=0, atol=1e-12)


def test_only_the_kept_slots_change_and_rejected_rows_never_appear():
    c = _case(11, R=6)
    new, kv_out, _ = kv_commit_ref(c["k_new"], c["v_new"], c["caches"], c["block_table"],
                                   c["kv_len"], c["qo"], c["acc"], c["K"], c["T_cap"])
    np.testing.assert_array_equal(kv_out, c["kv_len"] + c["acc"] + 1)
    changed = np.any(new != c["caches"], axis=(0, 2, 3, 5))       # [P][page]
    expect = np.zeros_like(changed)
    for r in range(c["R"]):
        for j in range(int(c["acc"][r]) + 1):
            pos = int(c["kv_len"][r]) + j
            expect[c["block_table"][r, pos // c["page"]], pos % c["page"]] = True
    np.testing.assert_array_equal(changed, expect)
    for r in range(c["R"]):
        t0, a, L = int(c["qo"][r]), int(c["acc"][r]), int(c["L"][r])
        for j in range(a + 1, L + 1):        # rejected drafts: rolled back by never being written
            assert not np.isin(c["k_new"][:, t0 + j], new).any()
            assert not np.isin(c["v_new"][:, t0 + j], new).any()


def test_each_layer_gets_its_own_rows():
    c = _case(3, layers=3)
    new, _, _ = kv_commit_ref(c["k_new"], c["v_new"], c["caches"], c["block_table"], c["kv_len"],
                              c["qo"], c["acc"], c["K"], c["T_cap"])
    r = 0
    pos = int(c["kv_len"][r])
    pg, slot = c["block_table"][r, pos // c["page"]], pos % c["page"]
    for layer in range(3):
        np.testing.assert_array_equal(new[layer, pg, 0, :, slot], c["k_new"][layer, c["qo"][r]])
        np.testing.assert_array_equal(new[layer, pg, 1, :, slot], c["v_new"][layer, c["qo"][r]])


def test_malformed_requests_are_skipped_untouched():
    c = _case(5, R=5)
    acc = c["acc"].copy()
    acc[1] = c["L"][1] + 1                   # more accepted than verified
    bt = c["block_table"].copy()
    n2 = int(c["kv_len"][2])
    bt[2, n2 // c["page"]] = 10 ** 6         # page outside the cache
    qo = c["qo"].copy()
    new, kv_out, skipped = kv_commit_ref(c["k_new"], c["v_new"], c["caches"], bt, c["kv_len"], qo,
                                         acc, c["K"], c["T_cap"])
    assert 1 in skipped and 2 in skipped
    for r in (1, 2):
        assert kv_out[r] == c["kv_len"][r]
    # requests 0, 3, 4 still committed
    for r in (0, 3, 4):
        assert kv_out[r] == c["kv_len"][r] + acc[r] + 1


def test_zero_accepted_commits_only_the_first_verify_token():
    c = _case(8, R=3)
    acc = np.zeros(3, dtype=np.int64)
    new, kv_out, _ = kv_commit_ref(c["k_new"], c["v_new"], c["caches"], c["block_table"],
                                   c["kv_len"], c["qo"], acc, c["K"], c["T_cap"])
    np.testing.assert_array_equal(kv_out, c["kv_len"] + 1)
    assert int(np.any(new != c["caches"], axis=(0, 2, 3, 5)).sum()) == 3
