"""Parity of v4kv_index_topk (through the C ABI) with the oracle: bit-exact
indices and reported scores, forced ties, shortfall padding."""
import numpy as np
import pytest
import torch

import synth
from oracle import codecs, paging
from tests.helpers import lay_out, oracle_index

pytestmark = pytest.mark.gpu


def build(seed, lens, dup_groups=0, dim=128, ratio=4, fp4=False):
    r = synth.rng(seed)
    rows = []
    for L in lens:
        n = paging.entry_count(L, ratio)
        x = synth.normal(r, (n, dim))
        if dup_groups and n:
            base = x[: dup_groups].copy()
            x = base[r.integers(0, dup_groups, n)]
        if fp4:
            codes, sc = codecs.quantize_entry_fp4(x)
            rows.append((codecs.pack_fp4(codes), sc))
        else:
            rows.append(codecs.quantize_entry(x))
    pool = lay_out(rows, 256 // ratio, r, "fp4" if fp4 else "fp8")
    q = synth.normal(r, (len(lens), dim))
    return pool, q


def run(pool, q, lens, k, ratio=4, W=128):
    from paged_compressed_kv_b200 import v4kv
    dev = torch.device("cuda")
    B = len(lens)
    max_len = int(max(lens))
    ws = v4kv.v4kv_workspace_size(v4kv.V4KV_OP_INDEX_TOPK, B, 1, max_len, ratio, W, k,
                                  v4kv.V4KV_FP8_E4M3, 128)
    workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
    topk = torch.empty(B, k, dtype=torch.int32, device=dev)
    score = torch.empty(B, k, dtype=torch.float32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    v4kv.v4kv_index_topk(torch.from_numpy(q).to(dev), pool.to_cuda(),
                         torch.tensor(lens, dtype=torch.int32, device=dev), max_len, ratio, W, k,
                         topk, workspace, score_out=score, dev_status=st)
    torch.cuda.synchronize()
    return topk.cpu().numpy(), score.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("k", [1, 16, 512, 2048])
def test_topk_bit_exact(k):
    lens = [0, 100, 128 + 4 * 300, 4096, 20000, 65536]
    pool, q = build(300 + k, lens)
    got, sc, st = run(pool, q, lens, k)
    assert st == 0
    for b, L in enumerate(lens):
        sel, rs = oracle_index(q[b], pool, b, L, 4, 128, k)
        assert np.array_equal(got[b], sel), f"seq {b}"
        assert np.array_equal(sc[b].view(np.uint32), rs.view(np.uint32)), f"seq {b}"


def test_forced_ties_lowest_index_wins():
    lens = [8000, 3000]
    pool, q = build(310, lens, dup_groups=7)
    got, sc, st = run(pool, q, lens, 512)
    assert st == 0
    for b, L in enumerate(lens):
        sel, rs = oracle_index(q[b], pool, b, L, 4, 128, 512)
        assert np.array_equal(got[b], sel)


def test_full_size_sampled():
    # the mixed-stack indexer shape: 128 sequences, L ~ U[1K, 256K], k = 512;
    # the oracle checks a sample of sequences
    r = synth.rng(synth.seed_for("mixed-61"))
    lens = synth.lengths_uniform(r, 128, 1024, 262144, 4)
    pool, q = build(311, lens.tolist())
    got, sc, st = run(pool, q, lens.tolist(), 512)
    assert st == 0
    for b in [0, int(np.argmax(lens)), int(np.argmin(lens)), 77]:
        sel, rs = oracle_index(q[b], pool, b, int(lens[b]), 4, 128, 512)
        assert np.array_equal(got[b], sel)
        assert np.array_equal(sc[b].view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("dim", [64, 256])
def test_other_key_widths(dim):
    # keys that are not 128 bytes take the generic scoring kernel
    lens = [300, 128 + 4 * 1000 + 3, 30000]
    pool, q = build(320 + dim, lens, dim=dim)
    got, sc, st = run(pool, q, lens, 512)
    assert st == 0
    for b, L in enumerate(lens):
        sel, rs = oracle_index(q[b], pool, b, L, 4, 128, 512)
        assert np.array_equal(got[b], sel), f"seq {b}"
        assert np.array_equal(sc[b].view(np.uint32), rs.view(np.uint32)), f"seq {b}"


def test_bad_page_is_flagged_and_scored_zero():
    # a block-table entry past the pool: the kernel flags it and scores the
    # block's entries 0, the same as an oracle pool whose block is all-zero codes
    from paged_compressed_kv_b200 import v4kv
    from tests.helpers import NpPool
    lens = [128 + 4 * 5000, 9000]
    pool, q = build(330, lens)
    P, spb, D = pool.data.shape
    zero = NpPool(np.concatenate([pool.data, np.zeros((1, spb, D), np.uint8)]),
                  np.concatenate([pool.scales, np.ones((1, spb), np.float32)]),
                  pool.bt.copy(), "fp8")
    zero.bt[0, 3] = P
    pool.bt[0, 3] = P  # past the end of the device pool
    got, sc, st = run(pool, q, lens, 512)
    assert st & v4kv.V4KV_DEV_BAD_PAGE
    for b, L in enumerate(lens):
        sel, rs = oracle_index(q[b], zero, b, L, 4, 128, 512)
        assert np.array_equal(got[b], sel), f"seq {b}"
        assert np.array_equal(sc[b].view(np.uint32), rs.view(np.uint32)), f"seq {b}"


@pytest.mark.parametrize("k", [16, 512])
def test_fp4_keys_bit_exact(k):
    # fp4-e2m1 keys with one fp32 scale each (two codes per byte): the
    # 128-dim keys take the TMA kernel on the pool seen as 128-byte rows of two
    # keys; indices and reported scores bit-exact against the oracle
    lens = [0, 100, 128 + 4 * 300, 4096, 20000, 65536]
    pool, q = build(340 + k, lens, fp4=True)
    assert pool.data.shape[2] == 64
    got, sc, st = run(pool, q, lens, k)
    assert st == 0
    for b, L in enumerate(lens):
        sel, rs = oracle_index(q[b], pool, b, L, 4, 128, k)
        assert np.array_equal(got[b], sel), f"seq {b}"
        assert np.array_equal(sc[b].view(np.uint32), rs.view(np.uint32)), f"seq {b}"


def test_fp4_keys_other_width_generic_kernel():
    # 256-dim fp4 keys (128 bytes) take the generic scoring kernel
    lens = [300, 128 + 4 * 1000 + 3, 30000]
    pool, q = build(350, lens, dim=256, fp4=True)
    got, sc, st = run(pool, q, lens, 512)
    assert st == 0
    for b, L in enumerate(lens):
        sel, rs = oracle_index(q[b], pool, b, L, 4, 128, 512)
        assert np.array_equal(got[b], sel), f"seq {b}"
        assert np.array_equal(sc[b].view(np.uint32), rs.view(np.uint32)), f"seq {b}"
