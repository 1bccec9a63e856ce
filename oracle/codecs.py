"""Number formats of the cache: bf16, fp8-e4m3 and the per-entry fp8 quantiser.

TEST INFRASTRUCTURE (oracle). Written from the format definitions, not from
any library's code.

P1 §2 and §3.1.3 store the cache as bf16 or as fp8 ("--kv-cache-dtype fp8",
one byte per element); the fp8 flavour is e4m3 and every entry carries one fp32
absmax scale. The pages do not fix rounding or the zero case, so this module
adopts: round-to-nearest-even, saturate to the largest finite value, scale =
amax / 448 computed in fp32, amax == 0 -> scale 1, element quotient x / scale
as an IEEE fp32 division.

OCP FP8 E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no
infinities, NaN only at S.1111.111, largest finite magnitude 448 = 1.75 * 2^8,
smallest subnormal 2^-9.
"""
import numpy as np

E4M3_MAX = 448.0


def f32(x):
    """Cast to float32 (IEEE round-to-nearest-even).

    Follows IEEE 754 binary32 rounding (the fp32 steps the pages leave to the implementation).
    """
    return np.asarray(x, dtype=np.float32)


# ---------------------------------------------------------------- bf16

def bf16_bits(x):
    """fp32 -> bf16 bit pattern (uint16), round to nearest, ties to even.

    bf16 keeps the top 16 bits of the fp32 pattern; the discarded low half
    decides the rounding. NaN stays a (quiet) NaN.

    Follows P1 §3.1.3 (bf16 cache storage); round to nearest even.
    """
    u = f32(x).view(np.uint32).astype(np.uint64)
    low = u & 0xFFFF
    top = u >> 16
    round_up = (low > 0x8000) | ((low == 0x8000) & ((top & 1) == 1))
    out = top + round_up.astype(np.uint64)
    nan = np.isnan(f32(x))
    out = np.where(nan, (top | 0x40), out)
    return out.astype(np.uint16)


def bf16_to_f32(bits):
    """bf16 bit pattern -> float32 (exact).

    Follows P1 §3.1.3 (bf16 cache storage).
    """
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def bf16_round(x):
    """Round fp32 values to the nearest bf16 value, returned as float32.

    Follows P1 §3.1.3 (bf16 cache storage); round to nearest even.
    """
    return bf16_to_f32(bf16_bits(x))


# ---------------------------------------------------------------- e4m3

def e4m3_decode(codes):
    """fp8-e4m3 byte -> float64 value (exact). NaN for S.1111.111.

    Follows P1 §3.1.3 (fp8 cache) and the OCP FP8 E4M3 format.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) == 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    sub = m * 2.0 ** -9                                   # e == 0: 0.mmm * 2^-6
    nrm = (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64))
    val = np.where(e == 0, sub, nrm)
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def e4m3_encode(x):
    """float32 -> fp8-e4m3 byte: round to nearest even, saturate to +-448.

    Magnitudes at or above 448 become 448 (code 0x7E); NaN becomes 0x7F; the
    sign bit is kept for zero results (-0.0 and negative underflow -> 0x80).
    The rounding is done on the exact fp64 value of the fp32 input: in the
    subnormal range the quantum is 2^-9; in binade [2^e, 2^(e+1)) it is
    2^(e-3).

    Follows P1 §3.1.3 (fp8 cache) and the OCP FP8 E4M3 format.
    """
    x = f32(x)
    a = np.abs(x.astype(np.float64))
    neg = np.signbit(x)
    mag = np.zeros(a.shape, dtype=np.int64)

    sub = a < 2.0 ** -6
    # subnormal range (quantum 2^-9); rint is round-half-even. A result of 8
    # is the smallest normal 2^-6, whose code is also 8.
    mag = np.where(sub, np.rint(np.where(sub, a, 0.0) * 2.0 ** 9).astype(np.int64), mag)

    nrm = (~sub) & (a < E4M3_MAX) & ~np.isnan(a)
    safe = np.where(nrm, a, 1.0)
    _, k = np.frexp(safe)                     # safe = f * 2^k, f in [0.5, 1)
    e = k - 1                                 # safe in [2^e, 2^(e+1))
    q = np.rint((safe / np.exp2(e.astype(np.float64)) - 1.0) * 8.0).astype(np.int64)
    carry = q == 8
    e = np.where(carry, e + 1, e)
    q = np.where(carry, 0, q)
    code_n = ((e + 7) << 3) | q
    mag = np.where(nrm, np.minimum(code_n, 0x7E), mag)

    mag = np.where(a >= E4M3_MAX, 0x7E, mag)
    out = np.where(neg, mag | 0x80, mag)
    out = np.where(np.isnan(a), 0x7F, out)
    return out.astype(np.uint8)


def quantize_entry(x):
    """Per-entry absmax fp8 quantisation of fp32 vectors (last axis = one entry).

    Steps, all in fp32: amax = max |x_d|; scale = amax / 448 (IEEE division),
    or 1 if amax == 0; code_d = e4m3(x_d / scale) with an IEEE division per
    element. Returns (codes uint8 [..., D], scale float32 [...]).
    Dequantised value of element d: float(code_d) * scale.

    Follows P1 §2 and §3.1.3 (fp8 entries, one fp32 absmax scale each).
    """
    x = f32(x)
    amax = np.max(np.abs(x), axis=-1)
    scale = np.where(amax == 0, np.float32(1.0), amax / np.float32(E4M3_MAX)).astype(np.float32)
    quot = (x / scale[..., None]).astype(np.float32)
    return e4m3_encode(quot), scale


def dequantize_entry(codes, scale):
    """fp8 codes and per-entry fp32 scale -> the values they stand for, in fp64.

    Value of element d = e4m3_decode(code_d) * scale, formed exactly in fp64
    (a 4-bit-mantissa code times a 24-bit scale needs at most 28 bits).

    Follows P1 §2 and §3.1.3 (fp8 entries, one fp32 absmax scale each).
    """
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[..., None]


# ---------------------------------------------------------------- e2m1 (fp4)
# OCP MX FP4 E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit, no
# infinities or NaN. Code magnitudes 0..7: 0, 0.5 (subnormal), 1, 1.5, 2, 3,
# 4, 6; the sign is bit 3. P1 §2 stores the c4a indexer keys in fp4 for its
# 9.62 GiB figure; the pages fix nothing else, so the keys are quantised like
# the fp8 entries: one fp32 absmax scale per key, scale = amax / 6.

E2M1_MAX = 6.0
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(codes):
    """fp4-e2m1 code (low 4 bits) -> float64 value (exact).

    Follows P1 §2 (fp4 indexer) and the OCP MX FP4 E2M1 format.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64) & 0xF
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.exp2((e - 1).astype(np.float64)))
    return np.where((c >> 3) == 1, -mag, mag)


def e2m1_encode(x):
    """float32 -> fp4-e2m1 code: round to nearest, ties to even, saturate to
    +-6; the sign bit is kept for zero results (-0 and negative underflow ->
    0x8). The rounding works on the exact value of the fp32 input: the
    representable magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6, and at a tie the
    code with the even mantissa bit (0, 1, 2, 4 and 0.5's neighbour 1) wins.

    Follows P1 §2 (fp4 indexer) and the OCP MX FP4 E2M1 format.
    """
    x = f32(x).astype(np.float64)
    a = np.abs(x)
    neg = np.signbit(x)
    # index of the largest representable magnitude <= a, and the next one up
    lo = np.searchsorted(E2M1_VALUES, a, side="right") - 1
    lo = np.clip(lo, 0, 7)
    hi = np.minimum(lo + 1, 7)
    vlo, vhi = E2M1_VALUES[lo], E2M1_VALUES[hi]
    up = (a - vlo) > (vhi - a)
    tie = (a - vlo) == (vhi - a)
    up = up | (tie & ((lo & 1) == 1))      # ties go to the even code (mantissa bit 0)
    mag = np.where(up & (hi != lo), hi, lo)
    mag = np.where(a >= E2M1_MAX, 7, mag)
    return (np.where(neg, mag | 0x8, mag)).astype(np.uint8)


def quantize_entry_fp4(x):
    """Per-key absmax fp4 quantisation of fp32 vectors (last axis = one key).

    amax = max |x_d| (fp32); scale = amax / 6 (IEEE fp32 division), 1 if
    amax == 0; code_d = e2m1(x_d / scale) with an IEEE division per element.
    Returns (codes uint8 [..., D], one code per byte, and scale fp32 [...]).

    Follows P1 §2 (fp4 indexer keys with a per-key scale, read like the fp8 entries).
    """
    x = f32(x)
    amax = np.max(np.abs(x), axis=-1)
    scale = np.where(amax == 0, np.float32(1.0), amax / np.float32(E2M1_MAX)).astype(np.float32)
    quot = (x / scale[..., None]).astype(np.float32)
    return e2m1_encode(quot), scale


def pack_fp4(codes):
    """Two fp4 codes per byte: dim 2i in the low nibble, dim 2i + 1 in the high
    nibble ([..., D] -> [..., D/2] uint8).

    Follows the storage layout of the fp4 indexer pool (one byte per two dims).
    """
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_fp4(packed):
    """Inverse of pack_fp4: [..., D/2] bytes -> [..., D] codes.

    Follows the storage layout of the fp4 indexer pool (one byte per two dims).
    """
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out
