"""Pins of the oracle's embedding, LM head and sampling (oracle/vocab.py)."""

import math

import numpy as np

from oracle import vocab as V


def test_hash_matches_an_independent_implementation():
    """lowbias32 written twice (oracle, and the synthetic KV-cache filler, which
    does its 32-bit products in split halves): the same values."""
    from synthetic.kvfill import lowbias32 as other
    x = np.random.default_rng(0).integers(0, 2 ** 32, 5000, dtype=np.uint64)
    assert np.array_equal(V.lowbias32(x), np.array([other(int(t)) for t in x], dtype=np.uint64))
    # a hand-checked value of the published steps: H(0) = 0, H(1) != 1
    assert int(V.lowbias32(0)) == 0 and int(V.lowbias32(1)) != 1


def test_embedding_rows_are_the_normalised_table_rows():
    rng = np.random.default_rng(1)
    E = rng.standard_normal((50, 16))
    toks = np.array([3, 3, 49, 0])
    h = V.embed(E, toks)
    assert np.allclose(np.linalg.norm(h, axis=1), 1.0, atol=1e-15)
    for i, t in enumerate(toks):
        assert np.allclose(h[i], E[t] / math.sqrt(sum(x * x for x in E[t])), atol=1e-15)


def test_lm_head_brute_force():
    rng = np.random.default_rng(2)
    E = rng.standard_normal((7, 5))
    s = rng.uniform(1, 2, 7)
    h = rng.standard_normal((3, 5))
    z = V.lm_head(E, s, h)
    for i in range(3):
        for v in range(7):
            assert abs(z[i, v] - s[v] * sum(h[i, t] * E[v, t] for t in range(5))) < 1e-12


def test_greedy_is_argmax_with_the_lowest_index_on_ties():
    z = np.array([[0.1, 3.0, 3.0, -1.0], [5.0, 5.0, 5.0, 5.0]])
    assert list(V.sample(z, 0.0, 7, [0, 0])) == [1, 0]


def test_gumbel_max_samples_the_softmax():
    """Over many step counters the Gumbel-max draws follow softmax(z / T): a
    chi-square test on 6 tokens (and T -> 0 approaches greedy)."""
    z = np.array([1.0, 0.0, 2.0, -1.0, 0.5, 1.5])
    T = 0.8
    n = 20000
    toks = V.sample(np.tile(z, (n, 1)), T, 11, np.arange(n))
    counts = np.bincount(toks, minlength=6)
    p = np.exp(z / T) / np.exp(z / T).sum()
    chi2 = ((counts - n * p) ** 2 / (n * p)).sum()
    assert chi2 < 20.5                    # 5 degrees of freedom, p ~ 0.001
    cold = V.sample(np.tile(z, (200, 1)), 1e-3, 11, np.arange(200))
    assert np.all(cold == 2)


def test_draws_depend_on_seed_step_and_token():
    u = V.uniform(5, 3, np.arange(1000, dtype=np.uint64))
    assert np.all((u > 0) & (u < 1)) and abs(u.mean() - 0.5) < 0.05
    assert not np.array_equal(u, V.uniform(6, 3, np.arange(1000, dtype=np.uint64)))
    assert not np.array_equal(u, V.uniform(5, 4, np.arange(1000, dtype=np.uint64)))
