"""Rotary position embedding on the rope dims, and its inverse.

TEST INFRASTRUCTURE (oracle).

P1 §2.1: the shared K=V vector carries RoPE; after attention an inverse RoPE
is applied to the output at the query position, which removes the absolute
position the shared value brought in. The model configuration fixes RoPE on the
last 64 of the 512 dims (offset 448) with theta = 1e6. The pages leave the pair
layout open; this oracle rotates interleaved pairs (offset + 2i, offset + 2i + 1)
for i = 0 .. rope_dim/2 - 1 by the angle pos * theta^(-2i / rope_dim).

All arithmetic is fp64.
"""
import numpy as np


def rope_angles(pos, theta, rope_dim):
    """Angles [..., rope_dim/2] for integer positions ``pos`` (fp64).

    Follows P1 §2.1 (keys carry RoPE).
    """
    i = np.arange(rope_dim // 2, dtype=np.float64)
    freq = np.power(np.float64(theta), -2.0 * i / rope_dim)
    return np.asarray(pos, dtype=np.float64)[..., None] * freq


def rope_rotate(x, pos, theta=1e6, rope_dim=64, rope_offset=448, inverse=False):
    """Rotate the rope dims of ``x`` [..., D] by +angle (or -angle if inverse).

    ``pos`` broadcasts against x's leading axes. Pair (a, b) becomes
    (a cos - b sin, a sin + b cos). Dims outside the rope range are unchanged.
    Returns a new fp64 array.

    Follows P1 §2.1 (RoPE on the keys, inverse RoPE on the output).
    """
    y = np.array(x, dtype=np.float64, copy=True)
    if rope_dim == 0:
        return y
    ang = rope_angles(pos, theta, rope_dim)
    if inverse:
        ang = -ang
    c, s = np.cos(ang), np.sin(ang)
    a = y[..., rope_offset:rope_offset + rope_dim:2].copy()
    b = y[..., rope_offset + 1:rope_offset + rope_dim:2].copy()
    y[..., rope_offset:rope_offset + rope_dim:2] = a * c - b * s
    y[..., rope_offset + 1:rope_offset + rope_dim:2] = a * s + b * c
    return y
