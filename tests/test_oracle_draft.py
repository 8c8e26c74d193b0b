"""Pins of the Markov-head draft oracle (oracle/draft.py)."""
import numpy as np
import torch
from scipy.stats import chisquare

from oracle.draft import bf16_round, gumbel_uniforms, markov_draft_ref


def test_bf16_rounding_matches_the_library_cast():
    # float32 inputs: the library's float32 -> bfloat16 cast is then a single rounding too
    rng = np.random.default_rng(0)
    x32 = np.concatenate([rng.normal(0, 10, size=10000), rng.normal(0, 1e-38, size=1000),
                          [0.0, -0.0, 3.38e38, -3.39e38, 1e-45]]).astype(np.float32)
    want = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(bf16_round(x32.astype(np.float64)), want)


def test_bf16_rounding_is_one_rounding_of_the_float64_value():
    e = 2.0 ** -8                                   # half a bfloat16 ulp at 1
    # just above the tie by less than a float32 ulp: a rounding through float32 would land on
    # the tie and go to the even neighbour 1; the float64 value rounds up
    assert bf16_round(np.array([1 + e + 2.0 ** -30]))[0] == 1 + 2 * e
    assert bf16_round(np.array([-(1 + e + 2.0 ** -30)]))[0] == -(1 + 2 * e)
    # exact ties go to the even neighbour
    assert bf16_round(np.array([1 + e]))[0] == 1.0
    assert bf16_round(np.array([1 + 3 * e]))[0] == 1 + 4 * e
    # subnormal quantum 2^-133: ties to even there too
    assert bf16_round(np.array([2.0 ** -134]))[0] == 0.0
    assert bf16_round(np.array([3 * 2.0 ** -134]))[0] == 2.0 ** -132
    # the largest finite value and overflow at the midpoint past it
    big = (2 - 2.0 ** -7) * 2.0 ** 127
    assert bf16_round(np.array([big]))[0] == big
    assert bf16_round(np.array([(2 - 2.0 ** -8) * 2.0 ** 127 - 2.0 ** 100]))[0] == big
    assert bf16_round(np.array([(2 - 2.0 ** -8) * 2.0 ** 127]))[0] == np.inf
    assert np.isnan(bf16_round(np.array([np.nan]))[0])
    assert bf16_round(np.array([-np.inf]))[0] == -np.inf


def test_forced_transition_walks_the_vocabulary():
    """E[x] = one-hot(x), U = 20 * shift: the transition favours x + 1 (mod V); with zero block
    logits and greedy sampling the draft is x0 + 1, x0 + 2, ... (closed form)."""
    V, R, K = 32, 3, 5
    E = np.eye(V)
    U = 20.0 * np.roll(np.eye(V), 1, axis=1)     # row x has its 20 at column x + 1
    x0 = np.array([0, 7, 30])
    _, tok, _ = markov_draft_ref(np.zeros((R, K, V)), E, U, x0, 0.0, round_idx=1)
    want = (x0[:, None] + np.arange(1, K + 1)[None, :]) % V
    np.testing.assert_array_equal(tok, want)


def test_greedy_without_transition_is_the_library_argmax():
    rng = np.random.default_rng(1)
    B = rng.normal(0, 3, size=(4, 5, 257))
    z, tok, _ = markov_draft_ref(B, np.zeros((257, 8)), np.zeros((8, 257)), np.zeros(4, int),
                                 0.0, round_idx=0)
    np.testing.assert_array_equal(tok, np.argmax(bf16_round(B), axis=-1))
    np.testing.assert_array_equal(z, bf16_round(B))


def test_uniforms_are_open_interval_and_distinct_per_counter():
    u = gumbel_uniforms(3, 5, 2, 1001)
    assert np.all((u > 0) & (u < 1)) and len(np.unique(u)) > 990
    assert not np.array_equal(u, gumbel_uniforms(3, 5, 3, 1001))
    assert not np.array_equal(u, gumbel_uniforms(4, 5, 2, 1001))


def test_sampled_token_follows_softmax_of_the_tempered_logits():
    V, tau = 6, 0.8
    z = np.array([0.5, -1.0, 2.0, 0.0, 1.0, -0.5])
    zb = bf16_round(z)
    p = np.exp(zb / tau - np.max(zb / tau))
    p /= p.sum()
    n = 20000
    counts = np.zeros(V)
    B = np.broadcast_to(z, (1, 1, V))
    for rnd in range(n):
        _, tok, _ = markov_draft_ref(B, np.zeros((V, 2)), np.zeros((2, V)), np.zeros(1, int),
                                     tau, round_idx=rnd)
        counts[tok[0, 0]] += 1
    assert chisquare(counts, p * n).pvalue > 0.01
