"""The unified page pools (host library): page sizes per cache kind, the
bucket plan, and the fixed-size page allocator (P1 §3.1.3: every kind's pages
fall into a few buckets, each one pool of fixed-size pages; pages are then
handed out per kind with no compaction or migration)."""
import itertools
import os
import random
import threading

import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "p1_footprint.txt")


def _g():
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()[:2]
            out[k] = float(v)
    return out


def test_page_bytes_match_the_page():
    from paged_compressed_kv_b200 import v4kv
    g = _g()
    # the page's bf16 model (one 5120-element vector per entry, no scale)
    assert v4kv.v4kv_page_bytes(4, 5120, 16, 0) == g["c4a_page_bytes_bf16"]
    assert v4kv.v4kv_page_bytes(128, 5120, 16, 0) == g["c128a_page_bytes_bf16"]
    # this build's kinds: fp8 entries + 4-byte scale, fp8 / fp4 indexer keys,
    # raw bf16 window tokens (ratio 1)
    assert v4kv.v4kv_page_bytes(4, 512, 8, 4) == 64 * 516
    assert v4kv.v4kv_page_bytes(128, 512, 8, 4) == 2 * 516
    assert v4kv.v4kv_page_bytes(4, 128, 4, 4) == 64 * 68
    assert v4kv.v4kv_page_bytes(1, 512, 16, 0) == 256 * 1024
    assert v4kv.v4kv_page_bytes(3, 512, 8, 4) == 0  # 3 does not divide 256


def _brute_plan(sizes, k):
    """All splits of the ascending distinct sizes into <= k contiguous groups;
    the best by (largest bucket/kind ratio, sum of ratios)."""
    u = sorted(set(sizes))
    best = None
    for m in range(1, min(k, len(u)) + 1):
        for cuts in itertools.combinations(range(1, len(u)), m - 1):
            bounds = [0, *cuts, len(u)]
            worst, tot, top_of = 1.0, 0.0, {}
            for a, b in zip(bounds, bounds[1:]):
                top = u[b - 1]
                for s in u[a:b]:
                    worst = max(worst, top / s)
                    tot += top / s
                    top_of[s] = top
            key = (worst, tot)
            if best is None or key < best[0]:
                best = (key, top_of)
    return best[1]


@pytest.mark.parametrize("sizes", [
    [64 * 516, 2 * 516, 64 * 132, 64 * 68, 256 * 1024],        # this build's five kinds
    [655360, 20480, 655360, 64 * 132, 262144],                  # the page's bf16 model + others
    [100, 100, 100],
    [7, 3, 11, 5, 2, 13, 17],
])
def test_plan_is_the_best_split_and_keeps_equal_sizes_together(sizes):
    from paged_compressed_kv_b200 import v4kv
    bucket_of, bucket_bytes = v4kv.v4kv_plan_buckets(sizes, 3)
    assert len(bucket_bytes) == min(3, len(set(sizes)))
    assert bucket_bytes == sorted(bucket_bytes, reverse=True)   # bucket 0 = largest pages
    want = _brute_plan(sizes, 3)
    for s, b in zip(sizes, bucket_of):
        assert bucket_bytes[b] == want[s] and bucket_bytes[b] >= s
    for (s1, b1), (s2, b2) in itertools.combinations(zip(sizes, bucket_of), 2):
        if s1 == s2:
            assert b1 == b2


def test_alloc_free_semantics():
    from paged_compressed_kv_b200 import v4kv
    pools = v4kv.PagePools([4096, 1024], [5, 3])
    a = pools.alloc(0, 3)
    assert a == [0, 1, 2] and pools.free_pages(0) == 2
    with pytest.raises(v4kv.V4KVError) as e:
        pools.alloc(0, 3)                      # only 2 left: nothing taken
    assert e.value.status == v4kv.V4KV_ERR_UNSUPPORTED and pools.free_pages(0) == 2
    with pytest.raises(v4kv.V4KVError):
        pools.free(0, [1, 1])                  # listed twice: nothing freed
    with pytest.raises(v4kv.V4KVError):
        pools.free(0, [2, 4])                  # 4 was never allocated: nothing freed
    assert pools.free_pages(0) == 2
    pools.free(0, [1])
    assert pools.free_pages(0) == 3
    assert pools.alloc(0, 1) == [1]            # last freed, first reused
    assert pools.alloc(1, 3) == [0, 1, 2] and pools.free_pages(1) == 0
    with pytest.raises(v4kv.V4KVError):
        pools.alloc(2, 1)                      # no such bucket
    pools.close()


def test_random_workload_never_hands_out_a_page_twice():
    from paged_compressed_kv_b200 import v4kv
    r = random.Random(7)
    n = [200, 50, 900]
    pools = v4kv.PagePools([33024, 8448, 1032], n)
    held = [set(), set(), set()]
    for _ in range(3000):
        b = r.randrange(3)
        if held[b] and r.random() < 0.45:
            give = r.sample(sorted(held[b]), r.randint(1, len(held[b])))
            pools.free(b, give)
            held[b] -= set(give)
        else:
            k = r.randint(1, 20)
            if k <= n[b] - len(held[b]):
                got = pools.alloc(b, k)
                assert not (set(got) & held[b]) and len(set(got)) == k
                assert all(0 <= p < n[b] for p in got)
                held[b] |= set(got)
            else:
                with pytest.raises(v4kv.V4KVError):
                    pools.alloc(b, k)
        assert pools.free_pages(b) == n[b] - len(held[b])
    pools.close()


def test_threads_share_one_pool():
    from paged_compressed_kv_b200 import v4kv
    pools = v4kv.PagePools([4096], [4000])
    taken = [[] for _ in range(8)]

    def work(i):
        rr = random.Random(i)
        for _ in range(200):
            got = pools.alloc(0, rr.randint(1, 4))
            taken[i].extend(got)
            if rr.random() < 0.3:
                give = taken[i][-1:]
                pools.free(0, give)
                del taken[i][-1:]

    ts = [threading.Thread(target=work, args=(i,)) for i in range(8)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    flat = [p for t in taken for p in t]
    assert len(flat) == len(set(flat))
    assert pools.free_pages(0) == 4000 - len(flat)
    pools.close()
