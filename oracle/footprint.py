"""KV-cache bytes per sequence.

TEST INFRASTRUCTURE (oracle).

P1 §2 computes the cache of one 1,000,000-token sequence on the 61-layer model
(30 c4a layers, then 31 c128a layers): a c4a layer keeps 1,000,000 / 4 =
250,000 entries and a c128a layer about 1,000,000 / 128 = 7,813; with one
shared 5,120-element bf16 vector (10,240 bytes) per entry that is about
2.38 GiB per c4a layer and 0.075 GiB per c128a layer, 73.73 GiB in bf16 as the
page rounds it. It then states 9.62 GiB for fp8 entries with an fp4 indexer and
compares with 83.9 GiB for the previous model (an "8.7x" saving). The 9.62
comes from a division by an unexplained 7.66 that no formula on the page
produces, so it is not restated here; the tests only note it.

``kv_bytes`` is the general formula: per layer, ceil(N / r) entries of
(dim * bytes per element + scale bytes), plus for c4a layers ceil(N / 4)
indexer keys, plus the raw-token window, plus the compressor state.
"""

def layer_entries(n_tokens, ratio):
    """Stored entries of one layer: ceil(N / r).

    Follows P1 §2.1 and §2.2 (ceil(N/4) and ceil(N/128) entries per layer).
    """
    return -(-int(n_tokens) // int(ratio))


def kv_bytes(n_tokens, layer_ratios, dim, entry_elem_bytes, entry_scale_bytes=0,
             indexer_dim=0, indexer_elem_bytes=0.0, indexer_scale_bytes=0,
             window=0, window_elem_bytes=0, state_rows=False, state_elem_bytes=2):
    """Cache bytes of one sequence of n_tokens raw tokens.

    layer_ratios: one compression ratio per layer (4 = c4a, 128 = c128a);
    indexer keys are kept for the c4a (ratio 4) layers only; ``window`` raw
    tokens per layer; with ``state_rows`` each layer also holds r raw tokens
    (and one fp32 gate each) of compressor state.

    Follows P1 §2 (cache bytes per sequence).
    """
    total = 0.0
    for r in layer_ratios:
        total += layer_entries(n_tokens, r) * (dim * entry_elem_bytes + entry_scale_bytes)
        if r == 4 and indexer_dim:
            total += layer_entries(n_tokens, 4) * (indexer_dim * indexer_elem_bytes + indexer_scale_bytes)
        total += min(window, n_tokens) * dim * window_elem_bytes
        if state_rows:
            total += r * (dim * state_elem_bytes + 4)
    return total


def page_bf16_breakdown():
    """P1 §2's bf16 arithmetic with its own parameters, in GiB:
    (c4a per layer, c4a total, c128a per layer, c128a total, sum)."""
    gib = float(1 << 30)
    c4a = layer_entries(1_000_000, 4) * 5120 * 2 / gib
    c128a = layer_entries(1_000_000, 128) * 5120 * 2 / gib
    return c4a, 30 * c4a, c128a, 31 * c128a, 30 * c4a + 31 * c128a


def saving_ratio():
    """83.9 GiB (previous model) / 9.62 GiB, the page's "8.7x".

    Follows P1 §2.2 (the saving against the previous model).
    """
    return 83.9 / 9.62


def gib(nbytes):
    """Follows P1 §2 (the page quotes sizes in GiB)."""
    return nbytes / float(1 << 30)

