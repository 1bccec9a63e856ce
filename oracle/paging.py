"""Logical blocks, block tables, slot mapping and entry counts.

TEST INFRASTRUCTURE (oracle).

P1 §3.1.1: every cache kind is allocated in one logical unit, a block of 256
raw tokens. A c4a block therefore holds 256/4 = 64 compressed entries, a c128a
block 256/128 = 2, a sliding-window block 256 raw tokens. P1 §3 (PagedAttention)
maps each sequence's logical blocks onto physical pages through a block table.
P1 §2.1: c4a keeps ceil(N/4) entries and c128a ceil(N/128) (1,000,000 tokens ->
7,813 entries).

Reading adopted where the pages are silent: one logical block is one physical
page of its cache kind (the page-size formula of P1 §3.1.3 read as
(256 / ratio) * bytes per entry); entry j of a sequence lives in slot
block_table[j // spb] * spb + j % spb of its pool, spb = 256 / ratio.
"""
import numpy as np

LOGICAL_BLOCK_TOKENS = 256


def slots_per_page(ratio):
    """Compressed entries (or raw tokens, ratio 1) per 256-token logical block.

    Follows P1 §3.1.1 (256-token logical blocks).
    """
    assert LOGICAL_BLOCK_TOKENS % ratio == 0
    return LOGICAL_BLOCK_TOKENS // ratio


def entry_count(n_tokens, ratio):
    """Entries stored after n_tokens raw tokens: ceil(n / ratio).

    The trailing partial group is stored too (normalised over the tokens it
    has) and rewritten as more tokens arrive.

    Follows P1 §2.1 (ceil(N/r) entries; 1,000,000 tokens -> 7,813 at r = 128).
    """
    return -(-int(n_tokens) // int(ratio))


def visible_entries(seq_len, window, ratio):
    """Entries attended besides the window: groups that end at or before the
    window's first token, floor(max(0, L - W) / ratio).

    Follows P1 §2.1 and §2.3 (compressed entries before the window).
    """
    return max(0, int(seq_len) - int(window)) // int(ratio)


def window_range(seq_len, window):
    """Raw-token positions [max(0, L - W), L) held by the sliding window.

    Follows P1 §2.3 (the last 128 raw tokens).
    """
    return max(0, int(seq_len) - int(window)), int(seq_len)


def slot_of(block_table_row, index, spb):
    """Physical slot of logical index ``index`` through one block-table row.

    Follows P1 §3.1.1 (logical block -> page through the block table).
    """
    page = int(block_table_row[index // spb])
    return page * spb + index % spb


def touched_range(seq_start, n_new, ratio):
    """Logical indices [first, end) whose content changes when tokens
    [seq_start, seq_start + n_new) are appended (empty if n_new == 0).

    Follows P1 §3.1.1 and §3.1.2 (the groups an append writes).
    """
    if n_new <= 0:
        return 0, 0
    first = int(seq_start) // int(ratio)
    end = entry_count(int(seq_start) + int(n_new), ratio)
    return first, end


def slot_mapping(block_table, seq_start, n_new, ratio, spb):
    """Slots of every touched logical index of every sequence, concatenated.

    Returns (slots int64 [sum of counts], cu int32 [B + 1]) where sequence b's
    slots are slots[cu[b]:cu[b+1]], in ascending logical index.

    Follows P1 §3.1.1 (slots of the entries an append writes).
    """
    slots, cu = [], [0]
    for b in range(len(seq_start)):
        first, end = touched_range(seq_start[b], n_new[b], ratio)
        for j in range(first, end):
            slots.append(slot_of(block_table[b], j, spb))
        cu.append(len(slots))
    return np.array(slots, dtype=np.int64), np.array(cu, dtype=np.int32)


def allocate_block_tables(n_blocks_per_seq, perm=None, max_blocks=None):
    """Give each sequence's logical blocks physical pages, in order of a free
    list ``perm`` (identity if None). Unused table entries are -1.

    Returns (block_table int32 [B, max_blocks], num_pages).

    Follows P1 §3 (PagedAttention block tables onto physical pages).
    """
    n_blocks_per_seq = [int(n) for n in n_blocks_per_seq]
    total = sum(n_blocks_per_seq)
    if perm is None:
        perm = np.arange(total)
    assert len(perm) >= total
    if max_blocks is None:
        max_blocks = max(n_blocks_per_seq + [1])
    bt = np.full((len(n_blocks_per_seq), max_blocks), -1, dtype=np.int32)
    k = 0
    for b, n in enumerate(n_blocks_per_seq):
        for j in range(n):
            bt[b, j] = perm[k]
            k += 1
    return bt, len(perm)
