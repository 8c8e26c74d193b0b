"""GPU Markov-head draft step against the oracle.

Weights are multiples of 1/16 in [-1, 1] (the input recipe of the synthetic head), so the rank-d
transition term is exact in float32 and float64 alike and both sides round the same logits to
bfloat16: draft logits must match exactly, tokens exactly except Gumbel near-ties the oracle
flags.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_support import binding, host

pytestmark = pytest.mark.gpu


def _inputs(R, K, V, d, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    B = (torch.randn((R, K, V), generator=g, device="cuda") * 3).to(torch.bfloat16)
    E = (torch.randint(-16, 17, (V, d), generator=g, device="cuda").float() / 16).to(torch.bfloat16)
    U = (torch.randint(-16, 17, (d, V), generator=g, device="cuda").float() / 16).to(torch.bfloat16)
    x0 = torch.randint(0, V, (R,), generator=g, device="cuda", dtype=torch.int32)
    return B, E, U, x0


def _run(B, E, U, x0, tau, rnd, seed=0):
    d = binding()
    R, K, V = B.shape
    out = torch.empty_like(B)
    tok = torch.empty((R, K), dtype=torch.int32, device="cuda")
    ws = torch.empty(d.dspark_markov_draft_workspace_bytes(R, V), dtype=torch.uint8, device="cuda")
    d.dspark_markov_draft(B, E, U, x0, tau, rnd, seed, out, tok, ws)
    torch.cuda.synchronize()
    return out, tok


@pytest.mark.parametrize("tau,R,V,dr", [(0.8, 16, 1000, 64), (0.0, 16, 1000, 64),
                                        (1.3, 70, 4096, 48), (0.0, 70, 4096, 16), (0.9, 3, 1000, 8)])
def test_draft_matches_oracle(tau, R, V, dr):
    K = 5
    B, E, U, x0 = _inputs(R, K, V, dr, seed=V + R)
    out, tok = _run(B, E, U, x0, tau, rnd=7)
    z, want_tok, flags = oracle.markov_draft_ref(host(B), host(E), host(U), host(x0), tau, 7)
    got_tok = host(tok)
    # a flagged (near-tie) position may take either candidate; everything after it in that
    # request then follows a different prefix, so compare only up to the first flag
    for r in range(R):
        for k in range(K):
            if flags[r, k]:
                break
            assert got_tok[r, k] == want_tok[r, k], (r, k)
            np.testing.assert_array_equal(host(out[r, k]), z[r, k])
    assert flags.mean() < 0.05
    assert binding().dspark_read_error() == 0


def test_draft_full_vocabulary_sampled():
    R, K, V, dr = 6, 5, 151936, 64
    B, E, U, x0 = _inputs(R, K, V, dr, seed=11)
    out, tok = _run(B, E, U, x0, 1.0, rnd=3, seed=5)
    z, want_tok, flags = oracle.markov_draft_ref(host(B), host(E), host(U), host(x0), 1.0, 3, 5)
    got = host(tok)
    for r in range(R):
        for k in range(K):
            if flags[r, k]:
                break
            assert got[r, k] == want_tok[r, k]
            np.testing.assert_array_equal(host(out[r, k]), z[r, k])


def test_bad_previous_token_sets_the_bit():
    B, E, U, x0 = _inputs(4, 2, 64, 8, seed=1)
    x0[1] = 64
    _run(B, E, U, x0, 0.0, rnd=0)
    assert binding().dspark_read_error() & (1 << 7)
