"""Pins for the oracle's small helpers: the ranges an append touches, the
values a paged pool holds and gathers in logical order, the stored form of an
entry, and the fp32 rounding step. Each is checked against brute force or a
fact of the number format, not against the helper's own formula."""
import numpy as np
import pytest

from oracle import attention, codecs, compressor, paging


@pytest.mark.parametrize("ratio", [1, 4, 128])
def test_touched_range_is_the_set_of_groups_the_new_tokens_fall_in(ratio):
    rng = np.random.default_rng(11)
    for _ in range(300):
        s = int(rng.integers(0, 2000))
        n = int(rng.integers(0, 700))
        first, end = paging.touched_range(s, n, ratio)
        groups = sorted({t // ratio for t in range(s, s + n)})
        assert list(range(first, end)) == groups


def test_gather_returns_logical_rows_through_a_permuted_table():
    # every stored row holds a value unique to (sequence, logical index), so a
    # wrong page, slot or order shows up as a wrong row
    rng = np.random.default_rng(12)
    spb, dim = 4, 8
    counts = [7, 3, 10]
    nblk = [-(-c // spb) for c in counts]
    bt, npages = paging.allocate_block_tables(nblk, rng.permutation(sum(nblk)))
    data = np.zeros((npages, spb, dim), dtype=np.uint16)
    for b, c in enumerate(counts):
        for j in range(c):
            page = bt[b, j // spb]
            data[page, j % spb] = codecs.bf16_bits(np.full(dim, 100.0 * b + j, dtype=np.float32))
    for b, c in enumerate(counts):
        idx = list(rng.permutation(c))
        got = attention.gather(data, None, "bf16", bt[b], idx)
        assert np.array_equal(got, np.repeat(np.array(idx, dtype=np.float64)[:, None] + 100.0 * b,
                                             dim, axis=1))


def test_pool_values_fp8_is_code_value_times_scale():
    # e4m3 0x38 is 1.0, 0x40 is 2.0, 0xC0 is -2.0 (sign bit); 0x01 is 2^-9
    data = np.array([[[0x38, 0x40, 0xC0, 0x01]]], dtype=np.uint8)
    scales = np.array([[0.25]], dtype=np.float32)
    got = attention.pool_values(data, scales, "fp8", 1, 0, 0)
    assert np.array_equal(got, np.array([0.25, 0.5, -0.5, 2.0**-11]))


def test_store_entries_keeps_bf16_exact_values_and_bounds_fp8_error():
    rng = np.random.default_rng(13)
    exact = codecs.bf16_round(rng.standard_normal((5, 64)).astype(np.float32))
    bits, none = compressor.store_entries(exact, "bf16")
    assert none is None and np.array_equal(codecs.bf16_to_f32(bits), exact)
    x = rng.standard_normal((5, 64)).astype(np.float32) * 3.0
    codes, scale = compressor.store_entries(x, "fp8")
    back = codecs.dequantize_entry(codes, scale)
    amax = np.abs(x).max(axis=1, keepdims=True)
    # half a step of e4m3 (3 mantissa bits) above the normal range, and half the
    # subnormal spacing 2^-9 of the scale unit below it
    bound = np.maximum(np.abs(x) * 2.0**-4, amax / 448 * 2.0**-10) * 1.0001
    assert np.all(np.abs(back - x) <= bound)
    assert np.all((codes & 0x7F) != 0x7F)  # never a NaN code (S.1111.111)


def test_f32_rounds_to_nearest_even():
    one = 1.0
    assert float(codecs.f32(one + 2.0**-24)) == 1.0                    # tie -> even (1.0)
    assert float(codecs.f32(one + 3 * 2.0**-24)) == 1.0 + 2.0**-22     # tie -> even (up)
    assert float(codecs.f32(one + 2.0**-23)) == 1.0 + 2.0**-23         # representable
    assert float(codecs.f32(2.0**-149)) == 2.0**-149                   # smallest subnormal
    assert float(codecs.f32(2.0**-151)) == 0.0                         # below half of it
