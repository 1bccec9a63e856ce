"""c4a / c128a compression of raw tokens into shared K=V entries, and the
sliding-window copy of the raw tokens.

TEST INFRASTRUCTURE (oracle).

P1 §2.1: a c4a layer folds a group of raw tokens into one entry by a learned
weighted sum with a position bias (ratio 1/4); a c128a layer folds 128 raw
tokens into one entry. P1 §2.3: every layer also keeps the last 128 raw tokens
uncompressed (bf16 or fp8). P1 §3.1.2: the compressor keeps a rolling state of
the tokens of the group it has not finished.

Readings adopted (the pages are garbled or silent on these points):
  * a group is r = 4 (c4a) or r = 128 (c128a) consecutive raw tokens,
    non-overlapping: group g holds tokens [g*r, (g+1)*r);
  * the gate is one scalar logit a_t per raw token plus a learned bias
    bias[t - g*r] for its place in the group; weights w_t are the softmax of
    a_t + bias over the tokens of the group that exist so far;
  * entry g = sum_t w_t * x_t, then RoPE at position g*r (the group's first
    token) on the rope dims, then quantisation (fp8: per-entry absmax, see
    codecs.quantize_entry) or bf16 rounding;
  * a group that is not complete yet is stored too, normalised over the tokens
    it has, and rewritten as more tokens arrive (ceil(N/r) stored entries);
  * window token t = RoPE(x_t, t), stored bf16 (or quantised per token).

Variants (P1 §2.1, §3.1.2, §3.2.1), each optional:
  * overlapping window (c4a: "an 8-token overlapping state"): entry g folds the
    tokens [g*r - r, g*r + r) that exist, with a position bias of 2r values,
    bias[t - (g*r - r)]; the stride stays r, so there are still ceil(N/r)
    entries, and the RoPE position stays g*r;
  * RMSNorm in the compressor fusion (compressor -> RMSNorm -> RoPE -> insert):
    e <- e * w / sqrt(mean_d(e_d^2) + eps) with a per-dim weight w (eps 1e-6),
    after the weighted sum and before RoPE;
  * per-channel gates: one logit a_{t,d} per token and dim; the softmax over the
    entry's tokens is taken separately for every dim d, with the same position
    bias for all dims.

The oracle works on a sequence's whole token history, so it has no rolling
state: an append split into chunks must give exactly what one append gives.
Arithmetic is fp64; the value handed to the quantiser is that fp64 value
rounded once to fp32 (the "pre-quant" value).
"""
import numpy as np

from . import codecs
from .rope import rope_rotate


def group_weights(gates, bias):
    """Softmax over one group's tokens of gate + position bias (fp64).

    gates: [n] logits of the group's present tokens (n <= r);
    bias:  [r] position bias; token i of the group gets bias[i].

    Follows P1 §2.1 (learned, position-biased weights within a group).
    """
    z = np.asarray(gates, dtype=np.float64) + np.asarray(bias, dtype=np.float64)[: len(gates)]
    z = z - z.max()
    u = np.exp(z)
    return u / u.sum()


def entry_tokens(g, ratio, n, overlap=False):
    """The tokens [lo, hi) entry g folds, and the bias index of token lo.

    Without overlap: the group [g*r, (g+1)*r); with it: [g*r - r, g*r + r).
    Tokens that do not exist (t < 0 or t >= n) are left out; token t takes
    bias[t - start] where start = g*r (or g*r - r with overlap).

    Follows P1 §2.1 (groups of r tokens) and §3.1.2 (c4a's 8-token overlap).
    """
    start = g * ratio - (ratio if overlap else 0)
    lo, hi = max(0, start), min(g * ratio + ratio, n)
    return lo, hi, lo - start


def rms_norm(e, weight, eps=1e-6):
    """e * w / sqrt(mean_d(e_d^2) + eps) over the last axis (fp64).

    Follows P1 §3.2.1 (RMSNorm in the compressor fusion, before RoPE).
    """
    e = np.asarray(e, dtype=np.float64)
    ms = np.mean(e * e, axis=-1, keepdims=True)
    return e * np.asarray(weight, dtype=np.float64) / np.sqrt(ms + eps)


def compress_prequant(x, gates, bias, ratio, n_tokens=None, theta=1e6, rope_dim=64,
                      rope_offset=448, overlap=False, norm_weight=None, norm_eps=1e-6):
    """Pre-quantisation entries of one sequence, fp32 [ceil(N/r), D].

    x: raw tokens [N, D] (any float dtype; bf16 inputs are passed as their
    exact fp32 values); gates [N] (one logit per token) or [N, D] (per-channel
    gates); bias [r] (or [2r] with overlap). Only the first ``n_tokens`` tokens
    are used (default all). overlap: the 8-token c4a window; norm_weight: [D]
    RMSNorm weights (None: no norm).

    Follows P1 §2.1 (c4a / c128a folding), §3.1.2 (partial groups, the
    overlapping state) and §3.2.1 (RMSNorm before RoPE).
    """
    x = np.asarray(x, dtype=np.float64)
    gates = np.asarray(gates, dtype=np.float64)
    per_dim = gates.ndim == 2
    n = x.shape[0] if n_tokens is None else int(n_tokens)
    n_groups = -(-n // ratio)
    out = np.zeros((n_groups, x.shape[1]), dtype=np.float64)
    for g in range(n_groups):
        lo, hi, b0 = entry_tokens(g, ratio, n, overlap)
        b = np.asarray(bias, dtype=np.float64)[b0:b0 + hi - lo]
        if per_dim:
            # the softmax over the entry's tokens, separately for every dim
            z = gates[lo:hi] + b[:, None]
            z = z - z.max(axis=0, keepdims=True)
            u = np.exp(z)
            w = u / u.sum(axis=0, keepdims=True)
            out[g] = np.sum(w * x[lo:hi], axis=0)
        else:
            w = group_weights(gates[lo:hi], b)
            out[g] = w @ x[lo:hi]
    if n_groups and norm_weight is not None:
        out = rms_norm(out, norm_weight, norm_eps)
    if n_groups:
        out = rope_rotate(out, np.arange(n_groups) * ratio, theta, rope_dim, rope_offset)
    return out.astype(np.float32)


def store_entries(prequant, dtype):
    """What the cache holds for fp32 pre-quant entries.

    dtype "fp8": (codes uint8 [G, D], scale fp32 [G]);
    dtype "bf16": (bits uint16 [G, D], None).

    Follows P1 §2.1 and §3.1.3 (entries stored as fp8 or bf16).
    """
    if dtype == "fp8":
        return codecs.quantize_entry(prequant)
    return codecs.bf16_bits(prequant), None


def window_tokens(x, positions, theta=1e6, rope_dim=64, rope_offset=448):
    """Window copies: RoPE(x_t, t) in fp64, rounded to fp32 [n, D].

    Follows P1 §2.3 (the last 128 raw tokens, uncompressed).
    """
    return rope_rotate(np.asarray(x, dtype=np.float64), np.asarray(positions),
                       theta, rope_dim, rope_offset).astype(np.float32)


def qk_prepare(q, k_new, positions, norm_weight=None, norm_eps=1e-6, theta=1e6, rope_dim=64,
               rope_offset=448):
    """The inputs of one decode step before attention (P1 §3.2.1, the fused
    "Q norm + KV RoPE + K insert"): each query head's vector is RMS-normalised
    (when weights are given) and rotated by RoPE at its sequence's position; the
    new token's K = V row is rotated at the same position for the window.

    q [B, H, D], k_new [B, D] (or None), positions [B] -> (q_out fp32
    [B, H, D], k_out fp32 [B, D] or None); fp64 arithmetic rounded once.

    Follows P1 §3.2.1 (Q/K insertion fusion) with S38's RMSNorm and S5's RoPE.
    """
    q = np.asarray(q, dtype=np.float64)
    pos = np.asarray(positions).reshape(-1, 1)
    if norm_weight is not None:
        q = rms_norm(q, norm_weight, norm_eps)
    q_out = rope_rotate(q, pos, theta, rope_dim, rope_offset).astype(np.float32)
    k_out = None
    if k_new is not None:
        k_out = rope_rotate(np.asarray(k_new, dtype=np.float64), np.asarray(positions), theta, rope_dim,
                            rope_offset).astype(np.float32)
    return q_out, k_out
