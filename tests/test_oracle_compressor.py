"""Pins for oracle.compressor: the hand-derived example, one-hot gates reducing
to token selection, uniform gates giving the mean, softmax shift invariance;
for the variants, the overlapping window reducing to the plain grouping when
the history is excluded and to the window mean / one token by brute force,
RMSNorm against torch's rms_norm and closed forms, per-channel gates reducing
to scalar gates and to scalar loops."""
import math
import os

import numpy as np

import synth
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


# ---- variants: overlapping c4a window, RMSNorm, per-channel gates


def test_overlap_with_excluded_history_is_the_plain_grouping():
    # bias -1e30 on the r tokens before the group makes their weights exactly 0,
    # so the overlapping entry equals the non-overlapping one with bias[r:]
    r = synth.rng(70)
    x = synth.normal(r, (37, 16))
    g = synth.normal(r, 37)
    b = synth.normal(r, 8, 0.5)
    b_ex = b.copy()
    b_ex[:4] = -1e30
    e_ov = compressor.compress_prequant(x, g, b_ex, 4, rope_dim=0, overlap=True)
    e_pl = compressor.compress_prequant(x, g, b[4:], 4, rope_dim=0)
    assert np.array_equal(e_ov, e_pl)


def test_overlap_brute_force_window_mean_and_one_hot():
    r = synth.rng(71)
    n, d = 23, 8
    x = synth.normal(r, (n, d))
    # uniform gates and zero bias: entry g is the mean of tokens [4g - 4, 4g + 4) that exist
    e = compressor.compress_prequant(x, np.zeros(n), np.zeros(8), 4, rope_dim=0, overlap=True)
    for g in range(e.shape[0]):
        toks = [t for t in range(4 * g - 4, 4 * g + 4) if 0 <= t < n]
        want = np.float32(sum(x[t].astype(np.float64) for t in toks) / len(toks))
        assert np.allclose(e[g], want, rtol=1e-6, atol=1e-7), g
    # one-hot gates picking a token of the previous group: the entry is that token
    gates = np.full(n, -1e30)
    gates[5] = 0.0                      # token 5 lies in entry 2's window [4, 12)
    e = compressor.compress_prequant(x, gates, np.zeros(8), 4, rope_dim=0, overlap=True)
    assert np.array_equal(e[2], x[5].astype(np.float32))


def test_rms_norm_against_torch_and_closed_forms():
    import torch
    r = synth.rng(72)
    v = synth.normal(r, (5, 64)).astype(np.float64)
    w = 1.0 + synth.normal(r, 64, 0.1)
    got = compressor.rms_norm(v, w, 1e-6)
    want = torch.nn.functional.rms_norm(torch.from_numpy(v), (64,), torch.from_numpy(w.astype(np.float64)),
                                        eps=1e-6).numpy()
    assert np.allclose(got, want, rtol=1e-12, atol=0)
    # a constant vector c: each element becomes c / sqrt(c^2 + eps) times the weight
    c = 3.0
    out = compressor.rms_norm(np.full(8, c), np.ones(8), 1e-6)
    assert np.allclose(out, c / np.sqrt(c * c + 1e-6), rtol=1e-15)


def test_norm_applies_before_rope():
    # RMSNorm (weights 1) keeps the vector's direction and RoPE keeps its norm:
    # the rope dims of the normed, rotated entry have the norm the pre-RoPE
    # normed vector has, and the other dims equal the normed vector
    r = synth.rng(73)
    x = synth.normal(r, (8, 512))
    g = synth.normal(r, 8)
    w = np.ones(512)
    e_n = compressor.compress_prequant(x, g, np.zeros(4), 4, norm_weight=w)
    e_raw = compressor.compress_prequant(x, g, np.zeros(4), 4, rope_dim=0).astype(np.float64)
    normed = compressor.rms_norm(e_raw, w)
    assert np.allclose(e_n[:, :448], normed[:, :448], rtol=1e-6, atol=1e-6)
    assert np.allclose(np.linalg.norm(e_n[:, 448:], axis=1), np.linalg.norm(normed[:, 448:], axis=1), rtol=1e-5)


def test_per_channel_gates_reduce_to_scalar_gates_and_brute_force():
    r = synth.rng(74)
    n, d = 13, 6
    x = synth.normal(r, (n, d))
    g = synth.normal(r, n)
    b = synth.normal(r, 4, 0.5)
    # the same logit on every channel: the scalar-gate entries, bit for bit
    same = np.repeat(g[:, None], d, axis=1)
    assert np.array_equal(compressor.compress_prequant(x, same, b, 4, rope_dim=0),
                          compressor.compress_prequant(x, g, b, 4, rope_dim=0))
    # independent channel logits: scalar loops
    gd = synth.normal(r, (n, d))
    e = compressor.compress_prequant(x, gd, b, 4, rope_dim=0)
    for gi in range(e.shape[0]):
        lo, hi = 4 * gi, min(4 * gi + 4, n)
        for c in range(d):
            z = [gd[t, c] + b[t - lo] for t in range(lo, hi)]
            m = max(z)
            u = [np.exp(v - m) for v in z]
            s = sum(u)
            want = sum(u[k] / s * float(x[lo + k, c]) for k in range(hi - lo))
            assert abs(float(e[gi, c]) - want) <= 1e-6 * max(1.0, abs(want)), (gi, c)


def test_qk_prepare_reduces_to_norm_and_rope():
    r = synth.rng(75)
    q = synth.normal(r, (3, 4, 512))
    k = synth.normal(r, (3, 512))
    pos = np.array([0, 17, 100000])
    w = 1.0 + synth.normal(r, 512, 0.1)
    qo, ko = compressor.qk_prepare(q, k, pos, w)
    # position 0: RoPE is the identity, so the result is the norm alone
    assert np.allclose(qo[0], compressor.rms_norm(q[0].astype(np.float64), w), rtol=1e-6, atol=1e-7)
    assert np.array_equal(ko[0], k[0].astype(np.float32))
    # RoPE keeps each rope pair's length and leaves the other dims alone
    nq = compressor.rms_norm(q[1].astype(np.float64), w)
    assert np.allclose(qo[1][:, :448], nq[:, :448], rtol=1e-6, atol=1e-7)
    a, b = qo[2][:, 448::2].astype(np.float64), qo[2][:, 449::2].astype(np.float64)
    nq2 = compressor.rms_norm(q[2].astype(np.float64), w)
    a0, b0 = nq2[:, 448::2], nq2[:, 449::2]
    assert np.allclose(a * a + b * b, a0 * a0 + b0 * b0, rtol=1e-5)
    # the K row is the window copy of the token (the compressor's window path)
    assert np.array_equal(ko[1], compressor.window_tokens(k[1][None], [17])[0])
    # no weights: RoPE only
    qo2, _ = compressor.qk_prepare(q, None, pos)
    assert np.array_equal(qo2[0], q[0].astype(np.float32))
