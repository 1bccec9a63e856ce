"""Pins for oracle.paging: the page's block arithmetic and brute-force slots."""
import os

import numpy as np
import pytest

from oracle import paging

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    out = {}
    for line in open(os.path.join(GOLDEN, "p1_footprint.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()[:2]
            out[k] = float(v)
    return out


G = _golden()


def test_slots_per_block_from_page():
    assert paging.LOGICAL_BLOCK_TOKENS == G["logical_block_tokens"]
    assert paging.slots_per_page(4) == G["c4a_slots_per_block"] == 64
    assert paging.slots_per_page(128) == G["c128a_slots_per_block"] == 2


def test_entry_counts_from_page_and_workload():
    assert paging.entry_count(1_000_000, 4) == G["c4a_entries_1M"]
    assert paging.entry_count(1_000_000, 128) == G["c128a_entries_1M"] == 7813
    assert paging.entry_count(1024, 4) == 256          # tiny c4a workload
    for n in [0, 1, 3, 4, 5, 127, 128, 129, 255, 256, 257]:
        for r in (4, 128):
            assert paging.entry_count(n, r) == -(-n // r) == int(np.ceil(n / r))
            if n % r == 0:
                assert paging.entry_count(n, r) == n // r


def test_visibility_and_window():
    assert paging.visible_entries(1024, 128, 4) == 224
    assert paging.visible_entries(1_000_000, 128, 128) == 7811
    assert paging.visible_entries(100, 128, 4) == 0
    assert paging.window_range(1024, 128) == (896, 1024)
    assert paging.window_range(50, 128) == (0, 50)
    # every visible group ends at or before the window start
    for L in range(0, 600, 7):
        for r in (4, 128):
            nv = paging.visible_entries(L, 128, r)
            w0, _ = paging.window_range(L, 128)
            assert nv * r <= w0 < (nv + 1) * r or w0 == 0


def test_identity_table_slot_is_index():
    bt, _ = paging.allocate_block_tables([5])
    for j in range(5 * 64):
        assert paging.slot_of(bt[0], j, 64) == j


def test_permuted_table_brute_force():
    rng = np.random.default_rng(4)
    nblk = [3, 1, 4, 2]
    perm = rng.permutation(sum(nblk))
    bt, npages = paging.allocate_block_tables(nblk, perm)
    # brute force: enumerate (page, slot) for each sequence's logical index
    seen = set()
    k = 0
    for b, n in enumerate(nblk):
        for blk in range(n):
            page = perm[k]
            k += 1
            for s in range(64):
                slot = paging.slot_of(bt[b], blk * 64 + s, 64)
                assert slot == page * 64 + s
                seen.add(slot)
    assert seen == set(range(npages * 64))


@pytest.mark.parametrize("ratio", [1, 4, 128])
def test_slot_mapping_touched_ranges(ratio):
    spb = 256 // ratio
    rng = np.random.default_rng(5)
    seq_start = np.array([0, 3, 4, 255, 256, 1000])
    n_new = np.array([0, 1, 9, 2, 300, 0])
    ends = seq_start + n_new
    nblk = [-(-int(e) // 256) + 1 for e in ends]
    bt, _ = paging.allocate_block_tables(nblk, rng.permutation(sum(nblk)))
    slots, cu = paging.slot_mapping(bt, seq_start, n_new, ratio, spb)
    for b in range(len(seq_start)):
        got = slots[cu[b]:cu[b + 1]]
        if n_new[b] == 0:
            assert got.size == 0
            continue
        first = seq_start[b] // ratio
        last = (ends[b] - 1) // ratio
        assert got.size == last - first + 1
        for i, j in enumerate(range(first, last + 1)):
            assert got[i] == bt[b, j // spb] * spb + j % spb
