"""Pins for oracle.attention: window >= context is textbook full attention
(checked with torch's SDPA in fp64), brute force with scalar loops, page
permutation invariance, the relative-position invariance that inverse RoPE
brings, and the single-entry special case."""
import math

import numpy as np
import torch

from oracle import attention, codecs, paging
from oracle.rope import rope_rotate


def _paged(values_bits, dtype, perm=None, scales=None, spb=256):
    """Lay a sequence's logical rows into pages through a (permuted) table."""
    n, d = values_bits.shape
    nblk = -(-n // spb)
    bt, npages = paging.allocate_block_tables([nblk], perm)
    data = np.zeros((npages, spb, d), dtype=values_bits.dtype)
    sc = None if scales is None else np.zeros((npages, spb), dtype=np.float32)
    for j in range(n):
        data[bt[0, j // spb], j % spb] = values_bits[j]
        if sc is not None:
            sc[bt[0, j // spb], j % spb] = scales[j]
    return {"data": data, "scales": sc, "dtype": dtype, "block_table_row": bt[0]}


def test_full_window_is_textbook_attention():
    rng = np.random.default_rng(13)
    L, H, D = 200, 8, 512
    raw = rng.standard_normal((L, D)).astype(np.float32)
    keys = codecs.bf16_bits(rope_rotate(raw, np.arange(L)).astype(np.float32))
    win = _paged(keys, "bf16", perm=rng.permutation(1))
    main = _paged(np.zeros((0, D), np.uint8), "fp8", scales=np.zeros(0), spb=64)
    q = rng.standard_normal((H, D))
    out = attention.decode_one(q, main, win, L, 4, window_len=L, sm_scale=1 / math.sqrt(D))
    v = torch.from_numpy(codecs.bf16_to_f32(keys).astype(np.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], v[None, None].expand(1, H, L, D),
        v[None, None].expand(1, H, L, D), scale=1 / math.sqrt(D))[0, :, 0, :].numpy()
    ref = rope_rotate(ref, L - 1, inverse=True)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_brute_force_scalar_loops():
    rng = np.random.default_rng(14)
    H, D, n = 3, 16, 9
    q = rng.standard_normal((H, D))
    v = rng.standard_normal((n, D))
    out = attention.attend(q, v, 0.25, seq_len=1, rope_dim=0)
    for h in range(H):
        s = [0.25 * sum(q[h, d] * v[j, d] for d in range(D)) for j in range(n)]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = sum(e)
        for d in range(D):
            assert abs(out[h, d] - sum(e[j] * v[j, d] for j in range(n)) / z) < 1e-12


def test_single_entry_returns_it():
    rng = np.random.default_rng(15)
    v = rng.standard_normal((1, 512))
    q = rng.standard_normal((4, 512))
    out = attention.attend(q, v, 1.0, seq_len=1)
    assert np.allclose(out, np.repeat(v, 4, axis=0), atol=0)


def test_page_permutation_invariance():
    rng = np.random.default_rng(16)
    L, D = 3000, 512
    n_vis = paging.visible_entries(L, 128, 4)
    ent = rng.standard_normal((paging.entry_count(L, 4), D)).astype(np.float32)
    codes, sc = codecs.quantize_entry(ent)
    w = codecs.bf16_bits(rng.standard_normal((L, D)).astype(np.float32))
    q = rng.standard_normal((8, D))
    outs = []
    for seed in range(3):
        p = np.random.default_rng(seed)
        nb = -(-len(ent) // 64)
        main = _paged(codes, "fp8", perm=p.permutation(nb + 2), scales=sc, spb=64)
        win = _paged(w, "bf16", perm=p.permutation(-(-L // 256) + 1))
        outs.append(attention.decode_one(q, main, win, L, 4, 128, 1 / math.sqrt(D)))
    assert n_vis == 718
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_inverse_rope_removes_absolute_position():
    # K = V both carry RoPE at their own positions and q carries RoPE at the
    # query position; after the inverse RoPE at the query position the output
    # depends only on relative positions
    rng = np.random.default_rng(17)
    n, D = 50, 512
    x = rng.standard_normal((n, D))
    q0 = rng.standard_normal((4, D))
    pos = np.sort(rng.choice(1000, n, replace=False))
    L = 1001
    outs = []
    for shift in (0, 1, 12345, 700_000):
        v = rope_rotate(x, pos + shift)
        q = rope_rotate(q0, L - 1 + shift)
        outs.append(attention.attend(q, v, 1 / math.sqrt(D), seq_len=L + shift))
    for o in outs[1:]:
        assert np.allclose(o, outs[0], atol=1e-9)


def test_topk_restricts_the_set():
    rng = np.random.default_rng(18)
    D = 512
    L = 2048
    ent = rng.standard_normal((paging.entry_count(L, 4), D)).astype(np.float32)
    codes, sc = codecs.quantize_entry(ent)
    w = codecs.bf16_bits(rng.standard_normal((L, D)).astype(np.float32))
    main = _paged(codes, "fp8", scales=sc, spb=64)
    win = _paged(w, "bf16")
    q = rng.standard_normal((2, D))
    sel = np.array([5, 100, 3, -1, -1], dtype=np.int32)
    out = attention.decode_one(q, main, win, L, 4, 128, 0.1, topk_row=sel)
    vals = np.concatenate([codecs.dequantize_entry(codes[[3, 5, 100]], sc[[3, 5, 100]]),
                           codecs.bf16_to_f32(w[L - 128:]).astype(np.float64)])
    assert np.allclose(out, attention.attend(q, vals, 0.1, L), atol=1e-14)


def test_output_fp8_hand_worked_vector():
    # tests/golden/output_fp8_worked.txt: codes and scale derived by hand from
    # the e4m3 definition for a vector whose scale is exactly 2^-6
    import os
    rows, scale = [], None
    for line in open(os.path.join(os.path.dirname(__file__), "golden", "output_fp8_worked.txt")):
        f = line.split("#")[0].split()
        if not f:
            continue
        if f[0] == "scale":
            scale = float(f[1])
        else:
            rows.append((int(f[0]), float(f[1]), int(f[2], 16)))
    o = np.zeros((1, 512))
    for i, v, _ in rows:
        o[0, i] = v
    codes, sc = attention.output_fp8(o)
    assert sc[0] == scale
    for i, _, want in rows:
        assert codes[0, i] == want, (i, hex(codes[0, i]))
    assert np.all(codes[0, 7:] == 0)


def test_output_fp8_follows_the_fp32_rounding_of_the_output():
    # the quantiser sees the fp32 value of the fp64 output: an output 1 + 2^-40
    # quantises exactly like 1.0
    o = np.zeros((2, 512))
    o[0, 0], o[1, 0] = 1.0, 1.0 + 2.0 ** -40
    o[:, 1] = -3.0
    c, s = attention.output_fp8(o)
    assert np.array_equal(c[0], c[1]) and s[0] == s[1]
