"""Pins for oracle.compressor: the hand-derived example, one-hot gates reducing
to token selection, uniform gates giving the mean, softmax shift invariance."""
import math
import os

import numpy as np

from oracle import codecs, compressor
from oracle.rope import rope_rotate

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _worked():
    rows = {}
    for line in open(os.path.join(GOLDEN, "compressor_worked.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            k, a, b = line.split()
            rows[k] = (float(a), float(b))
    return rows


def test_hand_derived_example():
    w = _worked()
    x = np.array([[1, 0], [0, 1], [2, 2], [-1, 3], [4, -2], [2, 6]], dtype=np.float32)
    gates = np.log(np.array([1, 2, 3, 4, 1, 1], dtype=np.float64)).astype(np.float32)
    gates[4:] = 0
    e = compressor.compress_prequant(x, gates, np.zeros(4), 4, rope_dim=0)
    assert e.shape == (2, 2)
    assert np.allclose(e[0], w["case1"], atol=1e-6)
    assert np.allclose(e[1], w["case3"], atol=1e-6)
    bias = np.log(np.array([1, 1, 1, 3.0]))
    e2 = compressor.compress_prequant(x[:4], np.zeros(4), bias, 4, rope_dim=0)
    assert np.allclose(e2[0], w["case2"], atol=1e-6)


def test_one_hot_gates_select_a_token():
    rng = np.random.default_rng(6)
    r, n = 4, 40
    x = codecs.bf16_round(rng.standard_normal((n, 512)).astype(np.float32))
    sel = rng.integers(0, r, n // r)
    gates = np.full(n, -1e30, dtype=np.float32)
    for g, s in enumerate(sel):
        gates[g * r + s] = 0.0
    e = compressor.compress_prequant(x, gates, np.zeros(r), r)
    picked = x[np.arange(n // r) * r + sel]
    want = rope_rotate(picked, np.arange(n // r) * r).astype(np.float32)
    assert np.array_equal(e, want)
    # selecting the group's first token reproduces the window copy of it
    first = np.zeros(n // r, dtype=int)
    gates = np.full(n, -1e30, dtype=np.float32)
    gates[np.arange(n // r) * r] = 0
    e = compressor.compress_prequant(x, gates, np.zeros(r), r)
    win = compressor.window_tokens(x[np.arange(n // r) * r + first], np.arange(n // r) * r)
    assert np.array_equal(e, win)


def test_uniform_gates_give_group_mean():
    rng = np.random.default_rng(7)
    for r in (4, 128):
        n = 3 * r + 5
        x = rng.standard_normal((n, 512)).astype(np.float32)
        e = compressor.compress_prequant(x, np.full(n, 0.7), np.zeros(r), r, rope_dim=0)
        for g in range(e.shape[0]):
            lo, hi = g * r, min(n, (g + 1) * r)
            assert np.allclose(e[g], x[lo:hi].astype(np.float64).mean(axis=0), atol=1e-6)


def test_gate_shift_invariance_and_weights_sum_to_one():
    rng = np.random.default_rng(8)
    a = rng.standard_normal(128)
    b = rng.normal(0, 0.5, 128)
    w = compressor.group_weights(a, b)
    assert math.isclose(w.sum(), 1.0, rel_tol=1e-14)
    assert np.allclose(w, compressor.group_weights(a + 123.0, b), rtol=1e-12)
    # bias enters per place in the group: permuting places changes weights
    assert not np.allclose(w, compressor.group_weights(a, b[::-1]))


def test_entry_count_and_partial_group():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((1024, 16)).astype(np.float32)
    g = rng.standard_normal(1024).astype(np.float32)
    assert compressor.compress_prequant(x, g, np.zeros(4), 4, rope_dim=0).shape[0] == 256
    assert compressor.compress_prequant(x, g, np.zeros(128), 128, n_tokens=1000, rope_dim=0).shape[0] == 8
    # a partial group equals the entry of the same tokens alone
    e = compressor.compress_prequant(x, g, np.zeros(128), 128, n_tokens=1000, rope_dim=0)
    alone = compressor.compress_prequant(x[896:1000], g[896:1000], np.zeros(128), 128, rope_dim=0)
    assert np.array_equal(e[7], alone[0])
