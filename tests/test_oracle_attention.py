"""Pins for the attention oracle: two independent restatements, a library routine, closed forms."""
import numpy as np
import pytest
import torch

from oracle.attention import attn_ref_dense, attn_ref_flat
from oracle.schedule import flatten_ref
from workloads.generate import page_table


def _case(seed, R=5, Hq=4, Hkv=2, D=8, page=4, n_lo=0, n_hi=13, K=5):
    rng = np.random.default_rng(seed)
    kv = rng.integers(n_lo, n_hi + 1, size=R).astype(np.int32)
    L = rng.integers(0, K + 1, size=R).astype(np.int32)
    table, P = page_table(kv, page, rng)
    qo, mk = flatten_ref(L, kv)
    T = int(qo[-1])
    return dict(
        q=rng.standard_normal((T, Hq, D)), k_new=rng.standard_normal((T, Hkv, D)),
        v_new=rng.standard_normal((T, Hkv, D)),
        kv_pages=rng.standard_normal((P, 2, Hkv, page, D)), block_table=table,
        kv_len=kv, verify_len=L, q_offsets=qo, markers=mk, page=page)


def _flat(c, scale, rows=None):
    return attn_ref_flat(c["q"], c["k_new"], c["v_new"], c["kv_pages"], c["block_table"],
                         c["kv_len"], c["markers"], c["q_offsets"], scale, c["page"], rows)


def _dense(c, scale):
    return attn_ref_dense(c["q"], c["k_new"], c["v_new"], c["kv_pages"], c["block_table"],
                          c["kv_len"], c["verify_len"], scale, c["page"])


@pytest.mark.parametrize("seed", range(6))
def test_flat_equals_dense(seed):
    c = _case(seed)
    a, b = _flat(c, 0.37), _dense(c, 0.37)
    assert np.max(np.abs(a - b)) < 1e-12


def test_dense_equals_sdpa_library_routine():
    """The padded dense form against torch's scaled_dot_product_attention in float64."""
    c = _case(11, R=4, Hq=6, Hkv=3, D=16, page=8, n_lo=1, n_hi=30)
    scale = 0.25
    ours = _flat(c, scale)
    kv, L, qo = c["kv_len"], c["verify_len"], c["q_offsets"]
    G = 2
    for r in range(len(kv)):
        n, Q = int(kv[r]), int(L[r]) + 1
        pos = np.arange(n)
        pages = c["block_table"][r, pos // c["page"]]
        Kc = c["kv_pages"][pages, 0, :, pos % c["page"], :]       # [n][Hkv][D]
        Vc = c["kv_pages"][pages, 1, :, pos % c["page"], :]
        Kall = np.concatenate([Kc, c["k_new"][qo[r]:qo[r] + Q]], 0)
        Vall = np.concatenate([Vc, c["v_new"][qo[r]:qo[r] + Q]], 0)
        mask = np.zeros((Q, n + Q), dtype=bool)
        for j in range(Q):
            mask[j, :n + j + 1] = True
        qh = torch.tensor(c["q"][qo[r]:qo[r] + Q]).permute(1, 0, 2)             # [Hq][Q][D]
        kh = torch.tensor(np.repeat(Kall, G, axis=1)).permute(1, 0, 2)          # [Hq][n+Q][D]
        vh = torch.tensor(np.repeat(Vall, G, axis=1)).permute(1, 0, 2)
        o = torch.nn.functional.scaled_dot_product_attention(
            qh, kh, vh, attn_mask=torch.tensor(mask), scale=scale)
        assert np.max(np.abs(o.permute(1, 0, 2).numpy() - ours[qo[r]:qo[r] + Q])) < 1e-12


def test_uniform_weights_closed_form():
    """scale = 0 gives equal weights over exactly the visible keys.  Values encode the key:
    cache position p of request r carries p+1 (dim 0) and 100*r (dim 1); new token i carries
    -(i+1).  Token j of request r must average (sum_{p<n}(p+1) - sum_{i<=j}(i+1)) / (n+j+1)."""
    c = _case(3, R=6, Hq=2, Hkv=1, D=4, page=4, n_lo=0, n_hi=17)
    P, page = c["kv_pages"].shape[0], c["page"]
    kvp = np.zeros_like(c["kv_pages"])
    for r, n in enumerate(c["kv_len"]):
        for p in range(n):
            pg, sl = c["block_table"][r, p // page], p % page
            kvp[pg, 1, 0, sl, 0] = p + 1
            kvp[pg, 1, 0, sl, 1] = 100 * r
    c["kv_pages"] = kvp
    vn = np.zeros_like(c["v_new"])
    for r in range(len(c["kv_len"])):
        for i in range(c["verify_len"][r] + 1):
            vn[c["q_offsets"][r] + i, 0, 0] = -(i + 1)
    c["v_new"] = vn
    out = _flat(c, 0.0)
    for r, n in enumerate(c["kv_len"]):
        n = int(n)
        for j in range(c["verify_len"][r] + 1):
            t = c["q_offsets"][r] + j
            want0 = (n * (n + 1) / 2 - (j + 1) * (j + 2) / 2) / (n + j + 1)
            want1 = 100 * r * n / (n + j + 1)
            for h in range(2):
                assert abs(out[t, h, 0] - want0) < 1e-12
                assert abs(out[t, h, 1] - want1) < 1e-12


def test_single_visible_key_returns_its_value():
    c = _case(4, R=3, n_lo=0, n_hi=0)
    out = _flat(c, 1.0)
    for r in range(3):
        t = c["q_offsets"][r]                    # first verify token of an empty cache
        for h in range(4):
            assert np.array_equal(out[t, h], c["v_new"][t, h // 2])


def test_page_placement_does_not_matter():
    c = _case(7)
    a = _flat(c, 0.5)
    rng = np.random.default_rng(70)
    P = c["kv_pages"].shape[0]
    perm = rng.permutation(P)                    # move physical page i to slot perm[i]
    moved = np.empty_like(c["kv_pages"])
    moved[perm] = c["kv_pages"]
    table = np.where(c["block_table"] >= 0, perm[np.maximum(c["block_table"], 0)], -1)
    c2 = dict(c, kv_pages=moved, block_table=table)
    assert np.max(np.abs(_flat(c2, 0.5) - a)) == 0.0


def test_dominant_key():
    c = _case(8, R=2, Hq=2, Hkv=1, D=8, n_lo=5, n_hi=9)
    r, n = 1, int(c["kv_len"][1])
    t = c["q_offsets"][1]
    page = c["page"]
    pg, sl = c["block_table"][r, 2 // page], 2 % page
    c["kv_pages"][pg, 0, 0, sl] = 50.0 * c["q"][t, 0] / np.linalg.norm(c["q"][t, 0])
    out = _flat(c, 1.0, rows=[(t, 0)])
    assert np.max(np.abs(out[t, 0] - c["kv_pages"][pg, 1, 0, sl])) < 1e-6


def test_row_subset_matches_full():
    c = _case(9)
    full = _flat(c, 0.3)
    rows = [(0, 1), (3, 0), (int(c["q_offsets"][-1]) - 1, 3)]
    sub = _flat(c, 0.3, rows)
    for t, h in rows:
        assert np.array_equal(sub[t, h], full[t, h])


def test_structured_keys_select_and_average_exactly():
    """The closed form the full-size GPU checks use (tests/structured_attn.py): with keys that
    select cache slots by a pseudo-random bit and coded values, each query's output is the mean
    of the selected values and of its request's verify tokens up to itself.  The oracle must
    reproduce it on a workload shaped like the large ones (page 64, D 128, GQA 4, several pages
    per request, an empty cache, ragged last pages); the other keys weigh 2^-40 each."""
    import math

    from tests.structured_attn import install_structured, structured_expected
    from workloads.configs import QWEN3_4B
    from workloads.generate import build_step_inputs

    cfg = QWEN3_4B.with_(R=4, Hq=8, Hkv=2, kv_dist=("uniform", 0, 300), V=16, layers=1)
    inp = build_step_inputs(cfg, "cpu", seed=2, layers=1)
    inp.kv_len[0] = 0                                  # an empty cache: only the verify tokens
    install_structured(inp)
    kv = inp.kv_len.numpy().astype(np.int64)
    qo, mk = flatten_ref([5, 0, 3, 2], kv)
    T = int(qo[-1])
    f = lambda t: t.float().numpy().astype(np.float64)
    got = attn_ref_flat(f(inp.q[0, :T]), f(inp.k_new[0, :T]), f(inp.v_new[0, :T]),
                        f(inp.kv_caches[0]), inp.block_table.numpy(), kv, mk, qo,
                        1.0 / math.sqrt(cfg.D), cfg.page_size)
    ref = structured_expected(inp, qo, kv)             # [T][Hkv][D]
    want = np.repeat(ref, cfg.G, axis=1)               # query head h reads KV head h // G
    assert np.allclose(got, want, rtol=1e-9, atol=1e-9), np.abs(got - want).max()
    # the selection matters: the plain mean over every visible key (scale 0) is far from it
    uniform = attn_ref_flat(f(inp.q[0, :T]), f(inp.k_new[0, :T]), f(inp.v_new[0, :T]),
                            f(inp.kv_caches[0]), inp.block_table.numpy(), kv, mk, qo, 0.0,
                            cfg.page_size)
    assert np.abs(uniform - want).max() > 0.1
