"""Pins for oracle.codecs against the OCP FP8 spec points and torch's casts."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import codecs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _spec_points():
    pts = []
    for line in open(os.path.join(GOLDEN, "e4m3_spec_points.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        val, code = line.split()[:2]
        pts.append((float(val), int(code, 16)))
    return pts


@pytest.mark.parametrize("val,code", _spec_points())
def test_e4m3_spec_points(val, code):
    got = int(codecs.e4m3_encode(np.float32(val)))
    assert got == code, (val, hex(got), hex(code))


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = codecs.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert sorted(np.nonzero(nan)[0].tolist()) == [0x7F, 0xFF]


def test_e4m3_encode_matches_torch_below_saturation():
    # torch's cast rounds to nearest even and gives NaN from 464 up; below 464
    # it must agree with the oracle bit for bit.
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2**32, size=4_000_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) < 464.0)]
    # plus every e4m3 value, every midpoint between neighbours, and 1 ulp
    # either side of each midpoint (the rounding boundaries)
    vals = codecs.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2
    b = np.concatenate([vals, mids]).astype(np.float32)
    b = np.concatenate([b, np.nextafter(b, np.float32(0)), np.nextafter(b, np.float32(1e9))])
    b = np.concatenate([b, -b])
    # a dense sweep of all fp32 patterns between 2^-12 and 2^-5 (subnormal edge)
    lo, hi = np.float32(2.0**-12).view(np.uint32), np.float32(2.0**-5).view(np.uint32)
    sweep = np.arange(lo, hi, 7, dtype=np.uint32).view(np.float32)
    x = np.concatenate([x, b, sweep, -sweep]).astype(np.float32)
    ours = codecs.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(x[i]), hex(ours[i]), hex(ref[i])) for i in bad[:5]]


def test_e4m3_encode_saturates_from_464():
    x = np.array([464.0, 479.9, 480.0, 1e30, np.inf, -500.0], dtype=np.float32)
    assert codecs.e4m3_encode(x).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_bf16_matches_torch():
    rng = np.random.default_rng(2)
    bits = rng.integers(0, 2**32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[~np.isnan(x)]
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(codecs.bf16_bits(x), ref)
    assert np.array_equal(codecs.bf16_to_f32(ref), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_quantize_entry_error_bound_and_max_code():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((200, 512)).astype(np.float32) * rng.uniform(1e-3, 1e3, (200, 1)).astype(np.float32)
    codes, scale = codecs.quantize_entry(x)
    assert scale.dtype == np.float32
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(scale, (amax / np.float32(448.0)).astype(np.float32))
    # the largest-magnitude element lands on the largest code
    i = np.abs(x).argmax(axis=1)
    assert np.all((codes[np.arange(200), i] & 0x7F) == 0x7E)
    # every element is within half a quantum of its fp32 quotient: 2^-4
    # relative in the normal range, 2^-10 absolute (in units of scale) below it
    v = codecs.dequantize_entry(codes, scale)
    q = x.astype(np.float64) / scale[:, None].astype(np.float64)
    err = np.abs(v / scale[:, None] - q)
    bound = np.maximum(np.abs(q) * 2.0**-4, 2.0**-10) * (1 + 1e-6)
    assert np.all(err <= bound)


def test_quantize_entry_zero_vector():
    codes, scale = codecs.quantize_entry(np.zeros((2, 8), dtype=np.float32))
    assert np.all(scale == 1.0) and np.all(codes == 0)


def test_decode_known_values():
    assert codecs.e4m3_decode(np.uint8(0x7E)) == 448.0
    assert codecs.e4m3_decode(np.uint8(0x01)) == math.ldexp(1.0, -9)
    assert codecs.e4m3_decode(np.uint8(0xB8)) == -1.0


def _e2m1_points():
    import os
    codes, encs = [], []
    for line in open(os.path.join(os.path.dirname(__file__), "golden", "e2m1_spec_points.txt")):
        f = line.split("#")[0].split()
        if not f:
            continue
        if f[0] == "code":
            codes.append((int(f[1], 16), float(f[2])))
        else:
            encs.append((float(f[1]), int(f[2], 16)))
    return codes, encs


def test_e2m1_decode_all_sixteen_codes():
    codes, _ = _e2m1_points()
    assert len(codes) == 16
    for c, v in codes:
        got = codecs.e2m1_decode(np.array([c]))[0]
        assert got == v and np.signbit(got) == np.signbit(v), (hex(c), got, v)


def test_e2m1_encode_spec_points():
    _, encs = _e2m1_points()
    for x, c in encs:
        got = int(codecs.e2m1_encode(np.array([x], dtype=np.float32))[0])
        assert got == c, (x, hex(got), hex(c))


def test_e2m1_round_trip_and_nearest():
    # every code decodes to a value that encodes back to it (except -0 / +0,
    # which keep their sign), and on a dense grid the encoder's choice is
    # never farther than the other neighbour (the nearest value)
    for c in range(16):
        v = codecs.e2m1_decode(np.array([c]))[0]
        assert int(codecs.e2m1_encode(np.array([v], dtype=np.float32))[0]) == c
    x = np.linspace(-7, 7, 20001).astype(np.float32)
    dec = codecs.e2m1_decode(codecs.e2m1_encode(x))
    grid = np.concatenate([-codecs.E2M1_VALUES[::-1], codecs.E2M1_VALUES])
    best = np.min(np.abs(x[:, None].astype(np.float64) - grid[None, :]), axis=1)
    assert np.all(np.abs(np.clip(x, -6, 6) - dec) <= best + 1e-12)


def test_fp4_key_quantiser_bound_and_packing():
    rng = np.random.default_rng(31)
    x = rng.standard_normal((50, 128)).astype(np.float32)
    x[3] = 0.0
    codes, sc = codecs.quantize_entry_fp4(x)
    assert sc[3] == 1.0 and np.all(codes[3] == 0)
    amax = np.abs(x).max(axis=1)
    assert np.all(sc[np.arange(50) != 3] == (amax / np.float32(6.0)).astype(np.float32)[np.arange(50) != 3])
    dq = codecs.e2m1_decode(codes) * sc[:, None].astype(np.float64)
    # the largest e2m1 gap is 2 (between 4 and 6): error <= 1 * scale; below
    # 2 it is <= 0.25 * scale
    err = np.abs(dq - x)
    assert np.all(err <= sc[:, None] * 1.0 + 1e-12)
    small = np.abs(x / sc[:, None]) < 2
    assert np.all(err[small] <= sc[:, None].repeat(128, 1)[small] * 0.25 + 1e-12)
    assert np.array_equal(codecs.unpack_fp4(codecs.pack_fp4(codes)), codes)
    p = codecs.pack_fp4(np.array([[0x1, 0xF, 0x7, 0x8]], dtype=np.uint8))
    assert p.tolist() == [[0xF1, 0x87]]
