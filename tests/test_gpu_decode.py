"""Parity of v4kv_decode_attention (through the C ABI) with the oracle."""
import math

import numpy as np
import pytest
import torch

import synth
from tests.helpers import DecodeCase, assert_close_bf16

pytestmark = pytest.mark.gpu


def run_decode(case, topk=None, q_dtype=torch.float32, sm_scale=None, k=None):
    from paged_compressed_kv_b200 import v4kv
    dev = torch.device("cuda")
    q = torch.from_numpy(case.q).to(dev)
    if q_dtype == torch.bfloat16:
        q = q.to(torch.bfloat16)
    main, win = case.main.to_cuda(), case.win.to_cuda()
    seq = torch.from_numpy(case.lens.astype(np.int32)).to(dev)
    out = torch.empty(case.B, case.H, 512, dtype=torch.bfloat16, device=dev)
    kk = 0 if topk is None else topk.shape[1]
    ws = v4kv.v4kv_workspace_size(v4kv.V4KV_OP_DECODE, case.B, case.H, case.max_len, case.ratio,
                                  case.W, kk, main.dtype_code)
    workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    tk = None if topk is None else torch.from_numpy(topk.astype(np.int32)).to(dev)
    v4kv.v4kv_decode_attention(q, main, win, seq, case.max_len, case.ratio, case.W, out, workspace,
                               topk=tk, sm_scale=sm_scale, dev_status=status)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), int(status.item())


def check_all(case, got, topk=None, seqs=None, q_round=None):
    for b in (range(case.B) if seqs is None else seqs):
        ref = case.oracle(b, None if topk is None else topk[b])
        assert_close_bf16(got[b], ref, f"seq {b} L={case.lens[b]}")


@pytest.mark.parametrize("heads", [8, 64])
def test_tiny_c4a_bf16_identity_table(heads):
    # 1 sequence, 1024 raw tokens, bf16 entries, identity table (64 heads: the
    # tensor-core path's bf16 entry tiles)
    case = DecodeCase(synth.seed_for("tiny-c4a"), [1024], heads, 4, main_dtype="bf16", permute=False)
    got, st = run_decode(case)
    assert st == 0
    check_all(case, got)


@pytest.mark.parametrize("heads", [1, 8, 16, 64])
def test_c4a_fp8_shuffled(heads):
    lens = [1, 2, 127, 128, 129, 255, 256, 257, 1023, 4096 + 3, 9000]
    case = DecodeCase(101 + heads, lens, heads, 4)
    got, st = run_decode(case)
    assert st == 0
    check_all(case, got)


def test_c128a_fp8_shuffled():
    lens = [131072 + 5, 200000, 128, 129, 1000, 300000]
    case = DecodeCase(202, lens, 64, 128)
    got, st = run_decode(case)
    assert st == 0
    check_all(case, got)


def test_bf16_query():
    case = DecodeCase(203, [5000, 7777], 64, 4)
    got, st = run_decode(case, q_dtype=torch.bfloat16)
    assert st == 0
    # the oracle sees the same bf16-rounded query
    case.q = torch.from_numpy(case.q).to(torch.bfloat16).float().numpy()
    check_all(case, got)


def test_topk_selection_with_padding_and_holes():
    r = synth.rng(204)
    lens = [6000, 3000, 200]
    case = DecodeCase(204, lens, 64, 4)
    k = 512
    topk = np.full((3, k), -1, dtype=np.int64)
    for b, L in enumerate(lens):
        nv = max(0, L - 128) // 4
        sel = r.permutation(nv)[: min(k, nv)]
        topk[b, : len(sel)] = sel
    topk[0, 7] = -1      # a hole in the middle
    got, st = run_decode(case, topk=topk)
    assert st == 0
    check_all(case, got, topk=topk)


@pytest.mark.parametrize("heads", [16, 64])
def test_window_covers_context_is_full_attention(heads):
    # W >= L: no entry is visible, attention runs over all raw tokens
    lens = [1, 17, 300, 1000]
    case = DecodeCase(205, lens, heads, 4, window=1024)
    got, st = run_decode(case)
    assert st == 0
    check_all(case, got)


def test_page_permutation_invariance_bitwise():
    lens = [5000, 12345, 700]
    a = DecodeCase(206, lens, 64, 4, permute=False)
    b = DecodeCase(206, lens, 64, 4, permute=True)
    ga, _ = run_decode(a)
    gb, _ = run_decode(b)
    assert np.array_equal(ga, gb)


@pytest.mark.parametrize("heads", [8, 64])
def test_empty_sequence_gives_zeros(heads):
    case = DecodeCase(207, [0, 500, 0], heads, 4)
    got, st = run_decode(case)
    assert st == 0
    assert np.all(got[0] == 0) and np.all(got[2] == 0)
    check_all(case, got, seqs=[1])


@pytest.mark.parametrize("heads", [8, 64])
def test_bad_page_is_flagged_not_read(heads):
    case = DecodeCase(208, [3000], heads, 4)
    case.main.bt[0, 2] = 10_000_000
    _, st = run_decode(case)
    assert st & 1


@pytest.mark.parametrize("heads", [8, 64])
def test_out_of_range_topk_index_is_flagged(heads):
    case = DecodeCase(209, [3000], heads, 4)
    topk = np.array([[1, 2, 100000, -1]], dtype=np.int64)
    _, st = run_decode(case, topk=topk)
    assert st & 4


@pytest.mark.parametrize("heads", [8, 64])
def test_sm_scale_argument(heads):
    case = DecodeCase(210, [2000], heads, 4)
    got, _ = run_decode(case, sm_scale=0.2)
    ref = case.oracle(0, sm_scale=0.2)
    assert_close_bf16(got[0], ref)


@pytest.mark.parametrize("heads", [8, 64])
def test_rising_scores_raise_the_reference(heads):
    # entries increasingly aligned with the query: the scores climb by about
    # 60 nats over the sequence, so the running reference maximum is raised
    # (and the partial output rescaled) many times along the way
    lens = [128 + 4 * 2500, 128 + 4 * 700]
    r = synth.rng(211)
    base = synth.normal(r, (len(lens), 512))

    def values(b, n):
        u = base[b] / np.linalg.norm(base[b])
        c = 60.0 * np.arange(n) / max(n - 1, 1)  # score of entry j is about c_j
        noise = synth.normal(r, (n, 512), 0.05)
        return (c[:, None] * math.sqrt(512) / np.linalg.norm(base[b])) * (u[None, :] + noise)

    case = DecodeCase(211, lens, heads, 4, entry_values=values)
    for b in range(len(lens)):
        case.q[b, :, :] = base[b]
    got, st = run_decode(case)
    assert st == 0
    check_all(case, got)


def test_many_short_sequences_per_block():
    # 300 sequences of 1 to 3 tiles: every sweep block opens several segments
    r = synth.rng(212)
    lens = r.integers(1, 700, 300).tolist()
    case = DecodeCase(212, lens, 64, 4)
    got, st = run_decode(case)
    assert st == 0
    check_all(case, got, seqs=list(range(0, 300, 7)))


@pytest.mark.parametrize("heads", [8, 64])
def test_fp8_window(heads):
    case = DecodeCase(213, [3000, 100], heads, 4, win_dtype="fp8")
    got, st = run_decode(case)
    assert st == 0
    check_all(case, got)


@pytest.mark.parametrize("heads", [8, 64])
def test_zero_and_negative_scale_entries(heads):
    # value = code * scale for any scale: a zero scale is a zero-valued entry
    # that still takes part in the softmax (score 0), a negative scale flips
    # the entry's sign; both head-count paths must agree with the oracle
    case = DecodeCase(214, [3000, 9000], heads, 4)
    r = synth.rng(215)
    sc = case.main.scales
    used = np.unique(case.main.bt[case.main.bt >= 0])
    for p in used[:: 3]:
        rows = r.choice(sc.shape[1], 8, replace=False)
        sc[p, rows[:4]] = 0.0
        sc[p, rows[4:]] = -sc[p, rows[4:]]
    got, st = run_decode(case)
    assert st == 0
    check_all(case, got)


def test_bf16_beyond_f16_range_is_flagged_on_the_tensor_core_path():
    # 64 heads convert bf16 window tokens to f16: a magnitude of 2^16 or more
    # cannot be represented there, so it is clamped and flagged
    # (V4KV_DEV_RANGE = 32); other head counts use the bf16 value exactly
    from oracle import codecs
    for heads in (8, 64):
        case = DecodeCase(216, [2000], heads, 4)
        L = 2000
        page = case.win.bt[0, (L - 3) // 256]
        row = case.win.data[page, (L - 3) % 256]
        row[:4] = codecs.bf16_bits(np.array([1e5, -7e4, 3e4, 65536.0], dtype=np.float32))
        got, st = run_decode(case)
        if heads == 64:
            assert st & 32
        else:
            assert st == 0
            check_all(case, got)


def test_fp8_window_then_bf16_entries_64_heads():
    # a segment whose window tiles (fp8) run in the pipelined path and whose
    # entry tiles (bf16) run one at a time, with several such segments per
    # sweep block and blocks starting in the middle of a sequence
    lens = [3000, 700, 128 * 4 + 129, 5000, 1]
    case = DecodeCase(217, lens, 64, 4, main_dtype="bf16", win_dtype="fp8", window=300)
    got, st = run_decode(case)
    assert st == 0
    check_all(case, got)


@pytest.mark.parametrize("heads", [64])
def test_long_window_fp8_many_segments(heads):
    # windows of several tiles, fp8 window and fp8 entries: consecutive fp8
    # segments across segment boundaries in one block
    r = synth.rng(218)
    lens = r.integers(1, 2500, 40).tolist()
    case = DecodeCase(218, lens, heads, 4, win_dtype="fp8", window=700)
    got, st = run_decode(case)
    assert st == 0
    check_all(case, got, seqs=list(range(0, 40, 3)))


@pytest.mark.parametrize("heads", [8, 64])
def test_fp8_output_epilogue(heads):
    # v4kv_decode_attention_fp8out: the merge epilogue quantises each
    # (sequence, head) output vector to e4m3 after the inverse RoPE. The fp32
    # values it hands to the quantiser meet the decode tolerance against the
    # oracle; codes and scales are bit-exact against the oracle's quantiser on
    # those same fp32 values; and the bf16 entry point's output is exactly
    # their bf16 rounding
    from oracle import attention, codecs
    from paged_compressed_kv_b200 import v4kv
    case = DecodeCase(219, [3000, 129, 9000, 0], heads, 4)
    dev = torch.device("cuda")
    q = torch.from_numpy(case.q).to(dev)
    main, win = case.main.to_cuda(), case.win.to_cuda()
    seq = torch.from_numpy(case.lens.astype(np.int32)).to(dev)
    ws = v4kv.v4kv_workspace_size(v4kv.V4KV_OP_DECODE, case.B, case.H, case.max_len, case.ratio,
                                  case.W, 0, main.dtype_code)
    workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    codes = torch.empty(case.B, case.H, 512, dtype=torch.uint8, device=dev)
    scales = torch.empty(case.B, case.H, dtype=torch.float32, device=dev)
    pre = torch.full((case.B, case.H, 512), float("nan"), dtype=torch.float32, device=dev)
    v4kv.v4kv_decode_attention_fp8out(q, main, win, seq, case.max_len, case.ratio, case.W, codes,
                                      scales, workspace, prequant_out=pre, dev_status=st)
    out = torch.empty(case.B, case.H, 512, dtype=torch.bfloat16, device=dev)
    v4kv.v4kv_decode_attention(q, main, win, seq, case.max_len, case.ratio, case.W, out, workspace,
                               dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    pre = pre.cpu().numpy()
    assert not np.isnan(pre).any()
    want_c, want_s = attention.output_fp8(pre)
    assert np.array_equal(codes.cpu().numpy(), want_c)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), want_s.view(np.uint32))
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), codecs.bf16_bits(pre))
    for b in range(case.B):
        ref = case.oracle(b)
        d = np.abs(pre[b].astype(np.float64) - ref)
        mx = np.abs(ref).max() if case.lens[b] else 0.0
        assert d.max() <= 1e-2 * mx + 1e-30
        if case.lens[b]:
            assert d.sum() / np.abs(ref).sum() <= 1e-3
        else:
            assert np.all(want_c[b] == 0) and np.all(scales.cpu().numpy()[b] == 1.0)


def test_whole_sequence_blocks_write_the_merge_result_bitwise():
    # When every sequence fits one sweep block at little cost (here 100
    # sequences of a top-256 selection plus the window), each block writes its
    # own sequence's output and the merge kernel skips the sequence. That output
    # must be, bit for bit, the bf16 rounding of the merge kernel's fp32 result
    # (the fp8-output entry point always merges and returns those fp32 values),
    # inverse RoPE included, and meet the tolerance against the oracle.
    from oracle import codecs
    from paged_compressed_kv_b200 import v4kv
    r = synth.rng(221)
    lens = r.integers(1200, 1600, 100).tolist()
    case = DecodeCase(221, lens, 64, 4)
    k = 256
    topk = np.full((case.B, k), -1, dtype=np.int64)
    for b, L in enumerate(lens):
        nv = max(0, L - 128) // 4
        topk[b, :] = r.permutation(nv)[:k]
    got, st = run_decode(case, topk=topk)
    assert st == 0
    dev = torch.device("cuda")
    q = torch.from_numpy(case.q).to(dev)
    main, win = case.main.to_cuda(), case.win.to_cuda()
    seq = torch.from_numpy(case.lens.astype(np.int32)).to(dev)
    tk = torch.from_numpy(topk.astype(np.int32)).to(dev)
    ws = v4kv.v4kv_workspace_size(v4kv.V4KV_OP_DECODE, case.B, case.H, case.max_len, case.ratio,
                                  case.W, k, main.dtype_code)
    workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    codes = torch.empty(case.B, case.H, 512, dtype=torch.uint8, device=dev)
    scales = torch.empty(case.B, case.H, dtype=torch.float32, device=dev)
    pre = torch.full((case.B, case.H, 512), float("nan"), dtype=torch.float32, device=dev)
    v4kv.v4kv_decode_attention_fp8out(q, main, win, seq, case.max_len, case.ratio, case.W, codes, scales,
                                      workspace, topk=tk, prequant_out=pre, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    pre = pre.cpu().numpy()
    got_bits = torch.from_numpy(got).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got_bits, codecs.bf16_bits(pre))
    check_all(case, got, topk=topk, seqs=list(range(0, case.B, 11)))


def test_whole_sequence_plan_with_wide_rope_and_empty_sequences():
    # The one-sequence-per-block plan when the output cannot be written by the
    # sweep (rope dims beyond the prep kernel's 32-pair cos/sin table): every
    # sequence then goes through the merge, which must not skip any. Empty
    # sequences in the batch own empty blocks and come out as zeros.
    from oracle import attention
    from paged_compressed_kv_b200 import Rope, v4kv
    r = synth.rng(222)
    lens = r.integers(1200, 1600, 100).tolist()
    for b in (3, 50, 99):
        lens[b] = 0
    case = DecodeCase(222, lens, 64, 4)
    k = 256
    topk = np.full((case.B, k), -1, dtype=np.int64)
    for b, L in enumerate(lens):
        nv = max(0, L - 128) // 4
        topk[b, : min(k, nv)] = r.permutation(nv)[:k]
    rope = Rope(rope_dim=128, rope_offset=384)
    dev = torch.device("cuda")
    q = torch.from_numpy(case.q).to(dev)
    main, win = case.main.to_cuda(), case.win.to_cuda()
    seq = torch.from_numpy(case.lens.astype(np.int32)).to(dev)
    out = torch.full((case.B, case.H, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    ws = v4kv.v4kv_workspace_size(v4kv.V4KV_OP_DECODE, case.B, case.H, case.max_len, case.ratio,
                                  case.W, k, main.dtype_code)
    workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    v4kv.v4kv_decode_attention(q, main, win, seq, case.max_len, case.ratio, case.W, out, workspace,
                               topk=torch.from_numpy(topk.astype(np.int32)).to(dev), rope=rope,
                               dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = out.float().cpu().numpy()
    assert not np.isnan(got).any()
    for b in (3, 50, 99):
        assert np.all(got[b] == 0)
    for b in range(0, case.B, 9):
        if lens[b] == 0:
            continue
        ref = attention.decode_one(case.q[b].astype(np.float64), case.main.seq(b), case.win.seq(b), lens[b],
                                   4, case.W, 1 / math.sqrt(512), topk_row=topk[b], rope_dim=128,
                                   rope_offset=384)
        assert_close_bf16(got[b], ref, f"seq {b} L={lens[b]}")
