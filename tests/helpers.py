"""Test-side builders: lay logical cache rows into paged pools (numpy for the
oracle, torch CUDA tensors for the library) and run the oracle per sequence.

Page layout uses oracle.paging (block tables, slots); values come from
synth draws, quantised or rounded by the oracle's codecs.
"""
import math

import numpy as np
import torch

import synth
from oracle import attention, codecs, compressor, indexer, paging


class NpPool:
    """A paged pool on the host: data [P, spb, D] (uint8 codes or uint16 bf16
    bits), scales [P, spb] fp32 or None, block table [B, max_blocks]."""

    def __init__(self, data, scales, bt, dtype):
        self.data, self.scales, self.bt, self.dtype = data, scales, bt, dtype

    def seq(self, b):
        return {"data": self.data, "scales": self.scales, "dtype": self.dtype,
                "block_table_row": self.bt[b]}

    def to_cuda(self):
        from paged_compressed_kv_b200 import PagedPool
        if self.dtype == "fp4":
            return PagedPool(data=torch.from_numpy(self.data).cuda(),
                             block_table=torch.from_numpy(self.bt).cuda(),
                             scales=torch.from_numpy(self.scales).cuda(), fp4=True)
        if self.dtype == "fp8":
            data = torch.from_numpy(self.data).cuda()
            sc = torch.from_numpy(self.scales).cuda()
        else:
            data = torch.from_numpy(self.data.view(np.int16)).view(torch.bfloat16).cuda()
            sc = None
        return PagedPool(data=data, block_table=torch.from_numpy(self.bt).cuda(), scales=sc)


def lay_out(rows_per_seq, spb, r, dtype, first_block=None, extra_pages=3, max_blocks=None,
            permute=True):
    """Pages for each sequence's logical rows.

    rows_per_seq: list of (values [n, D] uint8 / uint16, scales [n] or None),
    logical index 0 .. n-1; ``first_block[b]`` leaves blocks before it
    unmapped (-1), as a window pool does. Returns NpPool.
    """
    B = len(rows_per_seq)
    D = rows_per_seq[0][0].shape[1] if rows_per_seq else 1
    nblk = []
    for b, (vals, _) in enumerate(rows_per_seq):
        nb = -(-vals.shape[0] // spb)
        f = 0 if first_block is None else min(first_block[b], nb)
        nblk.append((f, nb))
    total = sum(nb - f for f, nb in nblk) + extra_pages
    perm = synth.permutation(r, total)      # drawn either way: same stream after
    if not permute:
        perm = np.arange(total)
    mb = max_blocks or max([nb for _, nb in nblk] + [1])
    bt = np.full((B, mb), -1, dtype=np.int32)
    vdt = rows_per_seq[0][0].dtype if rows_per_seq else np.uint8
    data = np.zeros((total, spb, D), dtype=vdt)
    scales = np.zeros((total, spb), dtype=np.float32) if dtype in ("fp8", "fp4") else None
    k = 0
    for b, (vals, sc) in enumerate(rows_per_seq):
        f, nb = nblk[b]
        for blk in range(f, nb):
            p = int(perm[k])
            k += 1
            bt[b, blk] = p
            lo, hi = blk * spb, min((blk + 1) * spb, vals.shape[0])
            data[p, : hi - lo] = vals[lo:hi]
            if scales is not None:
                scales[p, : hi - lo] = sc[lo:hi]
    return NpPool(data, scales, bt, dtype)


def entry_rows(r, n, dtype, std=0.5, dim=512):
    """n stored entries: N(0, std^2) values quantised (fp8) or rounded (bf16)."""
    x = synth.normal(r, (n, dim), std)
    if dtype == "fp8":
        return codecs.quantize_entry(x)
    return codecs.bf16_bits(x), None


def window_rows(r, L, W, dtype="bf16", dim=512):
    """Window rows at logical positions 0..L-1 (only [L-W, L) are filled)."""
    vals = np.zeros((L, dim), dtype=np.uint16 if dtype == "bf16" else np.uint8)
    w0 = max(0, L - W)
    x = synth.normal(r, (L - w0, dim))
    if dtype == "bf16":
        vals[w0:] = codecs.bf16_bits(x)
        return vals, None
    codes, sc = codecs.quantize_entry(x)
    full_sc = np.zeros(L, dtype=np.float32)
    vals[w0:] = codes
    full_sc[w0:] = sc
    return vals, full_sc


class DecodeCase:
    """A decode batch: caches on host and device, q, lengths."""

    def __init__(self, seed, lens, heads, ratio, main_dtype="fp8", window=128, win_dtype="bf16",
                 permute=True, q_std=1.0, entry_std=0.5, max_blocks_extra=0, entry_values=None):
        """entry_values(b, n) -> [n, 512] float values of sequence b's stored
        entries (quantised or rounded like the random ones); default random."""
        r = synth.rng(seed)
        self.lens = np.asarray(lens, dtype=np.int64)
        self.B, self.H, self.ratio, self.W = len(lens), heads, ratio, window
        spb = 256 // ratio
        if entry_values is None:
            ents = [entry_rows(r, paging.entry_count(L, ratio), main_dtype, entry_std) for L in lens]
        else:
            ents = []
            for b, L in enumerate(lens):
                x = np.asarray(entry_values(b, paging.entry_count(L, ratio)), dtype=np.float64)
                ents.append(codecs.quantize_entry(x) if main_dtype == "fp8" else (codecs.bf16_bits(x), None))
        self.main = lay_out(ents, spb, r, main_dtype, permute=permute,
                            max_blocks=max([-(-paging.entry_count(L, ratio) // spb) for L in lens] + [1]) + max_blocks_extra)
        wins = [window_rows(r, int(L), window, win_dtype) for L in lens]
        first = [max(0, int(L) - window) // 256 for L in lens]
        self.win = lay_out(wins, 256, r, win_dtype, first_block=first, permute=permute)
        self.q = synth.normal(r, (self.B, heads, 512), q_std)
        self.max_len = int(max(lens)) if len(lens) else 0

    def oracle(self, b, topk_row=None, sm_scale=None):
        sm = sm_scale or 1 / math.sqrt(512)
        return attention.decode_one(self.q[b].astype(np.float64), self.main.seq(b), self.win.seq(b),
                                    int(self.lens[b]), self.ratio, self.W, sm, topk_row=topk_row)


def bf16_of(x64):
    """fp64 -> bf16 value (as fp32) through fp32, round to nearest even."""
    return codecs.bf16_round(np.asarray(x64, dtype=np.float32))


def assert_close_bf16(got_bf16, ref64, what=""):
    """Tolerance of the decode path: against the oracle rounded to bf16,
    max|d| <= 1e-2 * max|ref| and sum|d| / sum|ref| <= 1e-3."""
    got = np.asarray(got_bf16, dtype=np.float64)
    ref = bf16_of(ref64).astype(np.float64)
    d = np.abs(got - ref)
    mx = np.abs(ref).max()
    assert d.max() <= 1e-2 * mx + 1e-30, f"{what}: max|d| {d.max():.3e} > 1e-2 * {mx:.3e}"
    rel = d.sum() / max(np.abs(ref).sum(), 1e-30)
    assert rel <= 1e-3, f"{what}: mean relative {rel:.3e} > 1e-3"
    return rel


def oracle_index(q_idx, pool, b, L, ratio, W, k):
    """Oracle top-k and reported scores of one sequence."""
    n_vis = paging.visible_entries(L, W, ratio)
    spb = pool.data.shape[1]
    codes = np.zeros((n_vis, pool.data.shape[2]), dtype=np.uint8)
    ks = np.zeros(n_vis, dtype=np.float32)
    for j in range(n_vis):
        p = pool.bt[b, j // spb]
        codes[j] = pool.data[p, j % spb]
        ks[j] = pool.scales[p, j % spb]
    if pool.dtype == "fp4":
        scores, qs = indexer.index_scores(q_idx, codecs.unpack_fp4(codes), ks, key_format="fp4")
    else:
        scores, qs = indexer.index_scores(q_idx, codes, ks)
    sel = indexer.topk(scores, n_vis, k)
    return sel, indexer.reported_scores(scores, qs, sel)


__all__ = ["NpPool", "lay_out", "entry_rows", "window_rows", "DecodeCase", "assert_close_bf16",
           "bf16_of", "oracle_index", "compressor"]
