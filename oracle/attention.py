"""Single-query decode attention over compressed entries plus the window.

TEST INFRASTRUCTURE (oracle).

P1 §2.1: keys and values are one shared vector per entry (K = V); the keys
carry RoPE, and after attention the output's rope dims are rotated back
(inverse RoPE) at the query position. c128a layers attend to all their
compressed entries; c4a layers attend to the entries the indexer picks
(P1 §2.2, §4.1). P1 §2.3: every layer also attends to the last 128 raw tokens,
kept uncompressed.

Readings adopted:
  * J = the visible entries (j < floor(max(0, L - W) / r)) or, when an index
    list is given, those of its indices that are >= 0, plus the window tokens
    [max(0, L - W), L);
  * s_hj = sm_scale * q_h . v_j, p = softmax over J, o_h = sum_j p_hj v_j,
    then the inverse RoPE at position L - 1 on the rope dims;
  * sm_scale = 1 / sqrt(D) unless given; no attention sink.
The result is this definition evaluated in fp64 on the exact values the cache
holds (dequantised entries, bf16 window tokens) and the exact query.
"""
import numpy as np

from . import codecs
from .rope import rope_rotate


def attend(q, values, sm_scale, seq_len, theta=1e6, rope_dim=64, rope_offset=448):
    """softmax(sm_scale q V^T) V for q [H, D], V [n, D], then inverse RoPE at
    position seq_len - 1. fp64 [H, D]. An empty V gives zeros.

    Follows P1 §2.1 (shared K=V entries, inverse RoPE on the output).
    """
    q = np.asarray(q, dtype=np.float64)
    v = np.asarray(values, dtype=np.float64)
    if v.shape[0] == 0:
        return np.zeros_like(q)
    s = sm_scale * (q @ v.T)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    o = p @ v
    return rope_rotate(o, seq_len - 1, theta, rope_dim, rope_offset, inverse=True)


def pool_values(data, scales, dtype, slots_per_page, page, slot):
    """Exact values (fp64 [D]) held in one slot of a paged pool.

    data: [num_pages, spb, D] uint8 codes (fp8) or uint16 bits (bf16);
    scales: [num_pages, spb] fp32 for fp8, None for bf16.

    Follows P1 §3.1.1 and §3.1.3 (paged pools, bf16 or fp8 with a per-entry scale).
    """
    if dtype == "fp8":
        return codecs.e4m3_decode(data[page, slot]) * np.float64(scales[page, slot])
    return codecs.bf16_to_f32(data[page, slot]).astype(np.float64)


def gather(data, scales, dtype, block_table_row, indices):
    """Values of logical indices through one block-table row, fp64 [n, D].

    Follows P1 §3.1.1 (logical index through the block table).
    """
    spb = data.shape[1]
    out = np.zeros((len(indices), data.shape[2]), dtype=np.float64)
    for i, j in enumerate(indices):
        page = int(block_table_row[j // spb])
        out[i] = pool_values(data, scales, dtype, spb, page, j % spb)
    return out


def decode_one(q, main, window, seq_len, ratio, window_len, sm_scale, topk_row=None,
               theta=1e6, rope_dim=64, rope_offset=448):
    """Attention output of one sequence, fp64 [H, D].

    main / window: dicts with keys data, scales, dtype, block_table_row.
    topk_row: optional int array of selected entry indices (-1 = none).

    Follows P1 §2.1, §2.2, §2.3 and §4.1 (entries or the selected set, plus the window).
    """
    n_vis = max(0, seq_len - window_len) // ratio
    if topk_row is None:
        ent = list(range(n_vis))
    else:
        ent = sorted(int(j) for j in topk_row if j >= 0)
    w0 = max(0, seq_len - window_len)
    wins = list(range(w0, seq_len))
    parts = []
    if ent:
        parts.append(gather(main["data"], main["scales"], main["dtype"], main["block_table_row"], ent))
    if wins:
        parts.append(gather(window["data"], window["scales"], window["dtype"], window["block_table_row"], wins))
    v = np.concatenate(parts, axis=0) if parts else np.zeros((0, q.shape[1]))
    return attend(q, v, sm_scale, seq_len, theta, rope_dim, rope_offset)


def output_fp8(o):
    """The attention output quantised to fp8-e4m3 per (sequence, head) vector.

    P1 §3.2.1 fuses the output's inverse RoPE with its fp8 quantisation (the
    next layer reads fp8). The pages fix neither the grouping nor the scale;
    this follows the cache entries' rule (codecs.quantize_entry) on each
    head's 512-vector: the fp64 output (after the inverse RoPE) is rounded to
    fp32, then amax, scale = amax / 448 (1 if amax == 0) and e4m3 codes of the
    per-element quotients. Returns (codes uint8 [..., D], scale fp32 [...]).
    """
    return codecs.quantize_entry(np.asarray(o, dtype=np.float32))
