"""Indexer scores over c4a entries and the exact top-k.

TEST INFRASTRUCTURE (oracle).

P1 §2.2: c4a layers carry a smaller "indexer" KV cache whose job is to decide
which compressed entries a query reads, so that attention does not have to
scan all of them; the fp8 cache setting applies to it as well. P1 §4.1 calls
c4a attention over the selected entries sparse attention. The workload fixes a
128-dim fp8 key per c4a entry, a 128-dim query, dot-product scores, k = 512
and ties broken by the lowest entry index.

Readings adopted:
  * the query is quantised like an entry (codecs.quantize_entry): codes q8,
    scale qs;
  * score_j = (sum over d = 0..127, in ascending d, of q8[d] * k8_j[d],
    accumulated in fp32) * kscale_j, rounded to fp32. Each product of two
    e4m3 values is exact in fp32, so each step is one fp32 rounding of
    acc + product, which is what an fp32 fused multiply-add gives;
  * qs > 0 is common to all entries of a sequence, so it is left out of the
    ranking and multiplied into the reported score (score * qs, fp32);
  * entries eligible are j < n_vis (see paging.visible_entries); the result is
    the min(k, n_vis) best by (score descending, index ascending), padded
    with -1. -0.0 and +0.0 rank equal.
"""
import numpy as np

from . import codecs


def index_scores(q_idx, key_codes, key_scales, key_format="fp8"):
    """Ranking scores (fp32 [n]) of n keys against one fp32 query.

    key_codes [n, D]: one code per element, fp8-e4m3 (key_format "fp8") or
    fp4-e2m1 (key_format "fp4": P1 §2 keeps the c4a indexer in fp4 for its
    9.62 GiB figure). Each product of an e4m3 query value and an e4m3 or e2m1
    key value is exact in fp32, so the chain is the same in both formats.

    Follows P1 §2.2 (indexer cache scores the c4a entries).
    """
    q8, qs = codecs.quantize_entry(np.asarray(q_idx, dtype=np.float32))
    qv = codecs.e4m3_decode(q8).astype(np.float32)
    dec = codecs.e2m1_decode if key_format == "fp4" else codecs.e4m3_decode
    kv = dec(np.asarray(key_codes)).astype(np.float32)
    acc = np.zeros(kv.shape[0], dtype=np.float32)
    for d in range(kv.shape[1]):
        acc = (acc + qv[d] * kv[:, d]).astype(np.float32)
    score = (acc * np.asarray(key_scales, dtype=np.float32)).astype(np.float32)
    return score, np.float32(qs)


def topk(scores, n_vis, k):
    """Indices of the min(k, n_vis) best scores among the first n_vis, by
    (score descending, index ascending), padded with -1 to length k.

    Follows P1 §2.2 and §4.1 (the selected entries of sparse c4a attention).
    """
    s = np.asarray(scores[:n_vis], dtype=np.float64) + 0.0   # -0.0 -> +0.0
    idx = np.arange(n_vis)
    order = np.lexsort((idx, -s))          # last key is primary
    sel = order[: min(k, n_vis)]
    out = np.full(k, -1, dtype=np.int32)
    out[: len(sel)] = sel
    return out


def reported_scores(scores, qs, sel):
    """Scores written beside the indices: score * qs in fp32, 0 for padding.

    Follows P1 §2.2 (indexer scores).
    """
    out = np.zeros(len(sel), dtype=np.float32)
    valid = sel >= 0
    out[valid] = (np.asarray(scores, dtype=np.float32)[sel[valid]] * np.float32(qs)).astype(np.float32)
    return out
