"""Pins for oracle.indexer: exact rational brute force on small cases, forced
ties, shortfall padding, and the fp32 chain's summation error bound."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import codecs, indexer


def _exact(code):
    v = float(codecs.e4m3_decode(np.uint8(code)))
    return Fraction(v)


def test_brute_force_exact_small_integers():
    # integer-valued keys and power-of-two scales keep the fp32 chain exact,
    # so the ranking must equal an exact rational sort
    rng = np.random.default_rng(10)
    ints = [c for c in range(256) if float(codecs.e4m3_decode(np.uint8(c))) in
            {0.0, 1.0, 2.0, 3.0, 4.0, -1.0, -2.0, -3.0, -4.0}]
    n, d = 300, 128
    keys = rng.choice(ints, size=(n, d)).astype(np.uint8)
    kscale = np.exp2(rng.integers(-3, 3, n)).astype(np.float32)
    q = rng.choice([-448.0, -224.0, 0.0, 224.0, 448.0], size=d).astype(np.float32)
    q[0] = 448.0                       # pins amax, so q / scale stays integral
    scores, qs = indexer.index_scores(q, keys, kscale)
    q8, _ = codecs.quantize_entry(q)
    exact = []
    for j in range(n):
        s = sum(_exact(q8[i]) * _exact(keys[j, i]) for i in range(d)) * Fraction(float(kscale[j]))
        assert Fraction(float(scores[j])) == s
        exact.append(s)
    for n_vis, k in [(300, 16), (300, 300), (100, 512), (0, 8)]:
        want = sorted(range(n_vis), key=lambda j: (-exact[j], j))[:k]
        got = indexer.topk(scores, n_vis, k)
        assert got[: len(want)].tolist() == want
        assert np.all(got[len(want):] == -1)


def test_ties_go_to_lowest_index():
    rng = np.random.default_rng(11)
    base = rng.integers(0, 0x7E, size=(5, 128)).astype(np.uint8)
    keys = np.repeat(base, 20, axis=0)            # every key appears 20 times
    perm = rng.permutation(100)
    keys = keys[perm]
    scores, _ = indexer.index_scores(rng.standard_normal(128), keys, np.ones(100, np.float32))
    got = indexer.topk(scores, 100, 30)
    # the 30 best are the best group(s), lowest indices first within a score
    s = scores[got]
    assert np.all(np.diff(s) <= 0)
    for i in range(1, 30):
        if s[i] == s[i - 1]:
            assert got[i] > got[i - 1]
    cut = s[-1]
    tied = np.nonzero(scores == cut)[0]
    n_above = int(np.sum(scores > cut))
    assert set(got.tolist()) == set(np.nonzero(scores > cut)[0].tolist()) | set(tied[: 30 - n_above].tolist())


def test_negative_zero_ranks_equal():
    scores = np.array([0.0, -0.0, 1.0, -0.0, 0.0], dtype=np.float32)
    assert indexer.topk(scores, 5, 5).tolist() == [2, 0, 1, 3, 4]


def test_fp32_chain_within_summation_bound():
    rng = np.random.default_rng(12)
    n = 2000
    keys = rng.integers(0, 0x7F, size=(n, 128)).astype(np.uint8)
    keys[keys == 0x7F] = 0
    q = rng.standard_normal(128).astype(np.float32)
    ks = rng.uniform(0.5, 2.0, n).astype(np.float32)
    scores, qs = indexer.index_scores(q, keys, ks)
    q8, _ = codecs.quantize_entry(q)
    qv = codecs.e4m3_decode(q8)
    kv = codecs.e4m3_decode(keys)
    prods = kv * qv[None, :]                       # exact in fp64
    exact = prods.sum(axis=1)                      # exact in fp64 (<= 43 bits)
    acc = scores.astype(np.float64) / ks.astype(np.float64)
    gamma = 127 * 2.0**-24 / (1 - 127 * 2.0**-24)
    bound = gamma * np.abs(prods).sum(axis=1) + np.abs(exact) * 2.0**-23
    assert np.all(np.abs(acc - exact) <= bound * 1.0001)


def test_reported_scores_include_query_scale():
    scores = np.array([3.0, 1.0, 2.0], dtype=np.float32)
    sel = np.array([0, 2, -1], dtype=np.int32)
    out = indexer.reported_scores(scores, np.float32(0.5), sel)
    assert out.tolist() == [1.5, 1.0, 0.0]


@pytest.mark.parametrize("n_vis,k", [(0, 4), (3, 4), (4, 4), (10, 4)])
def test_shortfall_padding(n_vis, k):
    s = np.arange(10, dtype=np.float32)
    got = indexer.topk(s, n_vis, k)
    m = min(n_vis, k)
    assert got[:m].tolist() == list(range(n_vis - 1, n_vis - 1 - m, -1))
    assert np.all(got[m:] == -1)


def test_fp4_keys_brute_force_exact_rational():
    # e2m1 keys (values k/2, integers up to 6) against integer-valued query
    # codes keep the fp32 chain exact: the scores equal an exact rational
    # dot product and the ranking an exact sort; a decode of the wrong format
    # (e4m3 instead of e2m1) or a dropped half-step would fail here
    rng = np.random.default_rng(17)
    n, d = 200, 128
    keys = rng.integers(0, 16, size=(n, d)).astype(np.uint8)
    kscale = np.exp2(rng.integers(-2, 3, n)).astype(np.float32)
    q = rng.choice([-448.0, -224.0, 0.0, 112.0, 448.0], size=d).astype(np.float32)
    q[0] = 448.0
    scores, qs = indexer.index_scores(q, keys, kscale, key_format="fp4")
    q8, _ = codecs.quantize_entry(q)
    vals = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
            Fraction(4), Fraction(6)]
    exact = []
    for j in range(n):
        s = Fraction(0)
        for i in range(d):
            c = int(keys[j, i])
            kv = -vals[c & 7] if c & 8 else vals[c & 7]
            s += _exact(q8[i]) * kv
        s *= Fraction(float(kscale[j]))
        assert Fraction(float(scores[j])) == s
        exact.append(s)
    want = sorted(range(n), key=lambda j: (-exact[j], j))[:64]
    assert indexer.topk(scores, n, 64)[:64].tolist() == want
