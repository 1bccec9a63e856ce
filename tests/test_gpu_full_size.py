"""Decode parity at full size, in the launch configuration bench.py times.

The caches, queries and lengths are the bench's own (bench.DecodeStep and
bench.MixedStep: seeded device draws). The library runs the decode call once
over the whole batch, exactly as the bench does. Then a few sampled sequences
(the shortest, the longest and two drawn at random) have their pages copied
to the host and are recomputed one by one by the oracle. The outputs must
meet the bf16 bar: max|d| <= 1e-2 * max|ref| and sum|d| / sum|ref| <= 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import bench
import synth
from helpers import assert_close_bf16
from oracle import attention

pytestmark = pytest.mark.gpu


def seq_pool(pool, b):
    """Sequence b's pages of a device pool, copied to the host in the oracle's
    form (a compact page array and the block-table row renumbered onto it)."""
    row = pool.block_table[b].cpu().numpy()
    used = row >= 0
    pages = torch.from_numpy(row[used].astype(np.int64)).to(pool.data.device)
    if pool.scales is not None:
        data = pool.data[pages].cpu().numpy()
        scales = pool.scales[pages].cpu().numpy()
        dtype = "fp8"
    else:
        data = pool.data[pages].view(torch.int16).cpu().numpy().view(np.uint16)
        scales = None
        dtype = "bf16"
    new_row = np.full_like(row, -1)
    new_row[used] = np.arange(int(used.sum()), dtype=row.dtype)
    return {"data": data, "scales": scales, "dtype": dtype, "block_table_row": new_row}


def sampled(lens, seed, n_random=2):
    r = synth.rng(seed)
    picks = {int(np.argmin(lens)), int(np.argmax(lens))}
    picks.update(int(v) for v in r.choice(len(lens), size=n_random, replace=False))
    return sorted(picks)


@pytest.mark.parametrize("workload", ["c4a-b64", "c128a-b32"])
def test_bench_workload_sampled(workload):
    dev = torch.device("cuda", 0)
    step = bench.DecodeStep(workload, dev)
    step.status.zero_()
    step.decode()
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    out = step.out.float().cpu().numpy()
    q = step.q.cpu().numpy()
    for b in sampled(step.lens, synth.seed_for(workload) + 17):
        L = int(step.lens[b])
        ref = attention.decode_one(q[b], seq_pool(step.main, b), seq_pool(step.win, b), L,
                                   step.ratio, bench.W, 1.0 / math.sqrt(bench.D))
        assert_close_bf16(out[b], ref, f"{workload} sequence {b} (L = {L})")


def test_mixed_c4a_layer_sampled():
    # one c4a layer of the 61-layer step at its batch of 128: the indexer's
    # top-512 selection, then the decode over the selected entries and the window
    dev = torch.device("cuda", 0)
    st = bench.MixedStep(dev, c4a_layers=1, c128a_layers=0)
    st.status.zero_()
    st.index(0)
    st.attend_c4a(0)
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0
    layer = st.c4a[0]
    out = st.out.float().cpu().numpy()
    q = layer["q"].cpu().numpy()
    topk = st.topk.cpu().numpy()
    for b in sampled(st.lens, synth.seed_for("mixed-61") + 17):
        L = int(st.lens[b])
        ref = attention.decode_one(q[b], seq_pool(layer["main"], b), seq_pool(layer["win"], b), L,
                                   4, bench.W, 1.0 / math.sqrt(bench.D), topk_row=topk[b])
        assert_close_bf16(out[b], ref, f"mixed c4a sequence {b} (L = {L})")


def test_two_stream_step_equals_the_serial_step():
    # P1 §3.2.2: a c4a layer's indexer runs on a second stream while its
    # compressor append runs on the first; attention waits for both. The
    # overlapped step must give exactly the serial step's outputs (every
    # layer's append is idempotent for a fixed token, so both orders start
    # from the same caches).
    dev = torch.device("cuda", 0)
    st = bench.MixedStep(dev, seqs=24, c4a_layers=3, c128a_layers=2)
    side = torch.cuda.Stream()

    def run(overlap):
        outs = []
        cur = torch.cuda.current_stream()
        for l in range(len(st.c4a)):
            L = st.c4a[l]
            if overlap:
                side.wait_stream(cur)
                with torch.cuda.stream(side):
                    st.index(l)
                st.append(L, 4)
                cur.wait_stream(side)
            else:
                st.append(L, 4)
                st.index(l)
            st.attend_c4a(l)
            outs.append((st.topk.clone(), st.out.clone()))
        for l in range(len(st.c128a)):
            st.append(st.c128a[l], 128)
            st.attend_c128a(l)
            outs.append((None, st.out.clone()))
        torch.cuda.synchronize()
        return outs

    serial = run(False)
    overlap = run(True)
    again = run(False)
    assert int(st.status.item()) == 0
    for (ta, oa), (tb, ob), (tc, oc) in zip(serial, overlap, again):
        if ta is not None:
            assert torch.equal(ta, tb) and torch.equal(ta, tc)
        assert torch.equal(oa.view(torch.int16), ob.view(torch.int16))
        assert torch.equal(oa.view(torch.int16), oc.view(torch.int16))
