"""Parity of v4kv_slot_mapping and v4kv_compress_append (through the C ABI)
with the oracle: slots bit-exact, pre-quant values within tolerance, fp8 bytes
and scales bit-exact on the kernel's own pre-quant values, window copies,
rolling state, and chunking invariance."""
import numpy as np
import pytest
import torch

import synth
from oracle import codecs, compressor, paging

pytestmark = pytest.mark.gpu

D = 512


class Appender:
    """Runs appends of per-sequence chunks through the library."""

    def __init__(self, seed, n_tokens, ratio, main_dtype="fp8", W=128, gates=None, dim=D,
                 rope=True, win_dtype="bf16", x=None, bias=None, overlap=False, per_channel=False,
                 norm=False):
        from paged_compressed_kv_b200 import PagedPool, Rope
        self.r = synth.rng(seed)
        self.n = [int(v) for v in n_tokens]
        self.B, self.ratio, self.W, self.dim = len(n_tokens), ratio, W, dim
        self.main_dtype, self.win_dtype = main_dtype, win_dtype
        # the last 64 dims carry RoPE (dims 448..511 at the model width)
        self.rope = Rope(rope_offset=dim - 64) if rope else Rope(rope_dim=0)
        self.x = [synth.normal(self.r, (N, dim)) for N in self.n]
        self.x = [codecs.bf16_round(v) for v in self.x]             # exact bf16 values
        if x is not None:
            self.x = [codecs.bf16_round(np.asarray(v, dtype=np.float32)) for v in x]
        self.overlap, self.per_channel = overlap, per_channel
        if gates is not None:
            self.g = gates
        elif per_channel:
            self.g = [synth.normal(self.r, (N, dim)) for N in self.n]
        else:
            self.g = [synth.normal(self.r, N) for N in self.n]
        self.bias = synth.normal(self.r, 2 * ratio if overlap else ratio, 0.5)
        self.norm_w = (1.0 + synth.normal(self.r, dim, 0.1)).astype(np.float32) if norm else None
        if bias is not None:
            self.bias = np.asarray(bias, dtype=np.float32)
        spb = 256 // ratio
        nblk = [-(-paging.entry_count(N, ratio) // spb) for N in self.n]
        self.bt, self.P = paging.allocate_block_tables(nblk, synth.permutation(self.r, sum(nblk) + 2))
        wblk = [-(-N // 256) for N in self.n]
        self.wbt, self.Pw = paging.allocate_block_tables(wblk, synth.permutation(self.r, sum(wblk) + 1))
        dev = torch.device("cuda")
        if main_dtype == "fp8":
            data = torch.zeros(self.P, spb, dim, dtype=torch.uint8, device=dev)
            sc = torch.zeros(self.P, spb, dtype=torch.float32, device=dev)
        else:
            data = torch.zeros(self.P, spb, dim, dtype=torch.bfloat16, device=dev)
            sc = None
        self.main = PagedPool(data=data, block_table=torch.from_numpy(self.bt).to(dev), scales=sc)
        if win_dtype == "fp8":
            self.win = PagedPool(data=torch.zeros(self.Pw, 256, dim, dtype=torch.uint8, device=dev),
                                 block_table=torch.from_numpy(self.wbt).to(dev),
                                 scales=torch.zeros(self.Pw, 256, dtype=torch.float32, device=dev))
        else:
            self.win = PagedPool(data=torch.zeros(self.Pw, 256, dim, dtype=torch.bfloat16, device=dev),
                                 block_table=torch.from_numpy(self.wbt).to(dev))
        rows = 2 * ratio if overlap else ratio
        self.state_x = torch.zeros(self.B, rows, dim, dtype=torch.bfloat16, device=dev)
        self.state_g = torch.zeros((self.B, rows, dim) if per_channel else (self.B, rows),
                                   dtype=torch.float32, device=dev)
        self.done = [0] * self.B
        self.prequant = [np.full((paging.entry_count(N, ratio), dim), np.nan, np.float32) for N in self.n]
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self._host = None

    def append(self, sizes, inline_slots=False):
        """One append call. inline_slots: no v4kv_slot_mapping call; the
        compressor derives the slots from the block table itself."""
        self._host = None  # the pools change
        from paged_compressed_kv_b200 import v4kv
        dev = torch.device("cuda")
        sizes = [min(int(s), N - d) for s, N, d in zip(sizes, self.n, self.done)]
        seq_start = np.array(self.done, dtype=np.int32)
        n_new = np.array(sizes, dtype=np.int32)
        cu = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
        xs = np.concatenate([self.x[b][self.done[b]:self.done[b] + sizes[b]] for b in range(self.B)])
        gs = np.concatenate([self.g[b][self.done[b]:self.done[b] + sizes[b]] for b in range(self.B)])
        cap = int(n_new.sum()) // self.ratio + 2 * self.B
        slots = torch.full((cap,), -7, dtype=torch.int64, device=dev)
        cu_e = torch.zeros(self.B + 1, dtype=torch.int32, device=dev)
        ss = torch.from_numpy(seq_start).to(dev)
        nn = torch.from_numpy(n_new).to(dev)
        want, want_cu = paging.slot_mapping(self.bt, seq_start, n_new, self.ratio, 256 // self.ratio)
        if inline_slots:
            slots = cu_e = None
        else:
            v4kv.v4kv_slot_mapping(self.main.block_table, ss, nn, self.ratio, self.P, slots, cu_e,
                                   dev_status=self.status)
            # slots must equal the oracle's slot mapping bit for bit
            got_cu = cu_e.cpu().numpy()
            assert np.array_equal(got_cu, want_cu)
            assert np.array_equal(slots[: len(want)].cpu().numpy(), want)
        pre = torch.full((max(1, len(want)), self.dim), np.nan, dtype=torch.float32, device=dev)
        v4kv.v4kv_compress_append(
            synth.bf16_tensor(xs).to(dev).reshape(-1, self.dim), torch.from_numpy(gs).to(dev),
            torch.from_numpy(cu).to(dev), ss, torch.from_numpy(self.bias).to(dev), self.ratio,
            self.state_x, self.state_g, self.main, slots, cu_e, window=self.win, window_len=self.W,
            rope=self.rope, prequant_out=pre, dev_status=self.status, overlap=self.overlap,
            gate_per_channel=self.per_channel,
            norm_weight=None if self.norm_w is None else torch.from_numpy(self.norm_w).to(dev))
        pre = pre.cpu().numpy()
        for b in range(self.B):
            first, end = paging.touched_range(self.done[b], sizes[b], self.ratio)
            self.prequant[b][first:end] = pre[want_cu[b]:want_cu[b + 1]]
            self.done[b] += sizes[b]
        assert int(self.status.item()) == 0

    def host_pools(self):
        """Host copies of the pools, taken once after the last append."""
        if self._host is None:
            main = self.main.data.view(torch.int16) if self.main_dtype == "bf16" else self.main.data
            win = self.win.data.view(torch.int16) if self.win_dtype == "bf16" else self.win.data
            self._host = {
                "main": main.cpu().numpy(),
                "main_scales": self.main.scales.cpu().numpy() if self.main.scales is not None else None,
                "win": win.cpu().numpy(),
                "win_scales": self.win.scales.cpu().numpy() if self.win.scales is not None else None,
            }
        return self._host

    def entries(self, b):
        """Stored entries of sequence b: (codes or bf16 bits [n, D], scales or None)."""
        spb = 256 // self.ratio
        n = paging.entry_count(self.n[b], self.ratio)
        h = self.host_pools()
        data, sc = h["main"], h["main_scales"]
        rows = np.stack([data[self.bt[b, j // spb], j % spb] for j in range(n)]) if n else data[:0, 0]
        scs = np.array([sc[self.bt[b, j // spb], j % spb] for j in range(n)]) if sc is not None else None
        return rows, scs

    def window_values(self, b):
        """Stored window rows of sequence b as fp32 (bf16 values, or fp8 codes x scale)."""
        N = self.n[b]
        ts = list(range(max(0, N - self.W), N))
        if not ts:
            return np.zeros((0, self.dim), np.float32)
        pages = [self.wbt[b, t // 256] for t in ts]
        h = self.host_pools()
        if self.win_dtype == "fp8":
            codes, sc = h["win"], h["win_scales"]
            return np.stack([codecs.dequantize_entry(codes[p, t % 256][None], sc[p, t % 256])[0]
                             for p, t in zip(pages, ts)])
        w = h["win"].view(np.uint16)
        return codecs.bf16_to_f32(np.stack([w[p, t % 256] for p, t in zip(pages, ts)]))


def check_against_oracle(ap):
    rope_dim = ap.rope.rope_dim
    for b in range(ap.B):
        N = ap.n[b]
        ref = compressor.compress_prequant(ap.x[b], ap.g[b], ap.bias, ap.ratio, rope_dim=rope_dim,
                                           rope_offset=ap.rope.rope_offset, overlap=ap.overlap,
                                           norm_weight=ap.norm_w)
        got = ap.prequant[b]
        assert not np.isnan(got).any()
        amax = np.abs(ref).max(axis=1, keepdims=True)
        assert np.all(np.abs(got - ref) <= 5e-5 * amax + 1e-30), f"seq {b}: pre-quant"
        rows, scs = ap.entries(b)
        if ap.main_dtype == "fp8":
            codes, sc = codecs.quantize_entry(got)
            assert np.array_equal(rows, codes), f"seq {b}: fp8 bytes"
            assert np.array_equal(scs.view(np.uint32), sc.view(np.uint32)), f"seq {b}: scales"
        else:
            assert np.array_equal(rows.view(np.uint16), codecs.bf16_bits(got)), f"seq {b}: bf16"
        # window: last W tokens RoPE'd at their own position, bf16 or fp8
        w0 = max(0, N - ap.W)
        wtok = compressor.window_tokens(ap.x[b][w0:], np.arange(w0, N), rope_dim=rope_dim,
                                        rope_offset=ap.rope.rope_offset)
        wgot = ap.window_values(b)
        if ap.win_dtype == "fp8":
            # e4m3: 3 mantissa bits (relative step 2^-3, so rounding error <= 2^-4),
            # subnormal spacing 2^-9 of the scale unit amax / 448
            amax = np.abs(wtok).max(axis=1, keepdims=True)
            bound = np.abs(wtok) * 2.0**-4 * 1.001 + amax / 448 * 2.0**-9 + 1e-30
            assert np.all(np.abs(wgot - wtok) <= bound), f"seq {b}: fp8 window"
        else:
            # bf16 rounding of the result, plus the fp32 rotation's own error: a*c - b*s
            # in fp32 is off by up to about 3 * 2^-24 * (|a| + |b|), which a near-total
            # cancellation turns into a large relative error
            wref = codecs.bf16_round(wtok)
            xmax = np.abs(ap.x[b][w0:]).max(axis=1, keepdims=True) if N else 0.0
            bound = np.abs(wref) * 2.0**-7 + xmax * 2.0**-20 + 1e-30
            assert np.all(np.abs(wgot - wref) <= bound), f"seq {b}: window"
        # state: the raw tokens and gates of the unfinished group (and, with
        # the overlapping window, of the group before it) at row t - base
        base = (N // ap.ratio) * ap.ratio - (ap.ratio if ap.overlap else 0)
        lo = max(0, base)
        st = ap.state_x[b, lo - base: N - base].float().cpu().numpy()
        assert np.array_equal(st, ap.x[b][lo:N]), f"seq {b}: state"
        sg = ap.state_g[b, lo - base: N - base].cpu().numpy()
        assert np.array_equal(sg, np.asarray(ap.g[b][lo:N], dtype=np.float32)), f"seq {b}: state gates"


@pytest.mark.parametrize("ratio", [4, 128])
@pytest.mark.parametrize("main_dtype", ["fp8", "bf16"])
def test_one_shot_append(ratio, main_dtype):
    ap = Appender(400 + ratio, [1, 3, 4, 5, 127, 128, 129, 1024, 3000], ratio, main_dtype)
    ap.append(ap.n)
    check_against_oracle(ap)


def test_tiny_c4a_workload():
    # one sequence of 1024 raw tokens, bf16 entries: 256 entries
    ap = Appender(synth.seed_for("tiny-c4a"), [1024], 4, "bf16")
    ap.append([1024])
    check_against_oracle(ap)
    assert ap.prequant[0].shape[0] == 256


@pytest.mark.parametrize("ratio", [4, 128])
def test_chunked_equals_one_shot_bitwise(ratio):
    n = [5000, 2049, 777, 9000]
    a = Appender(410, n, ratio)
    a.append(n)
    b = Appender(410, n, ratio)
    r = synth.rng(411)
    while any(d < N for d, N in zip(b.done, b.n)):
        b.append([int(r.integers(1, 700)) for _ in n])
    check_against_oracle(b)
    for s in range(len(n)):
        ra, sa = a.entries(s)
        rb, sb = b.entries(s)
        assert np.array_equal(ra, rb) and np.array_equal(sa, sb)
        assert np.array_equal(a.prequant[s].view(np.uint32), b.prequant[s].view(np.uint32))


@pytest.mark.parametrize("ratio", [4, 128])
def test_inline_slot_mapping_equals_explicit_bitwise(ratio):
    """The compressor without a slot mapping (slots from the block table, in
    the kernel) writes the same bytes, state and pre-quantisation values as
    with the v4kv_slot_mapping output, over random chunks (P1 §3.1.1)."""
    n = [5000, 2049, 777, 9000, 1]
    a = Appender(430, n, ratio)
    b = Appender(430, n, ratio)
    r = synth.rng(431)
    while any(d < N for d, N in zip(a.done, a.n)):
        sizes = [int(r.integers(0, 900)) for _ in n]
        a.append(sizes)
        b.append(sizes, inline_slots=True)
    check_against_oracle(b)
    for s in range(len(n)):
        ra, sa = a.entries(s)
        rb, sb = b.entries(s)
        assert np.array_equal(ra, rb) and np.array_equal(sa, sb)
        assert np.array_equal(a.prequant[s].view(np.uint32), b.prequant[s].view(np.uint32))
        assert np.array_equal(a.window_values(s), b.window_values(s))
    assert torch.equal(a.state_x, b.state_x) and torch.equal(a.state_g, b.state_g)


@pytest.mark.parametrize("ratio", [4, 128])
@pytest.mark.parametrize("batch", [31, 32, 33])
def test_batch_at_the_one_warp_table_limit(ratio, batch):
    """Batches of 31, 32 and 33 sequences, with the slot mapping passed and
    without: the kernel's per-call sequence tables are built by one warp up
    to 32 sequences (the entry total sits one past the last lane) and by the
    whole block above; every entry, the state and the window match the oracle."""
    r = synth.rng(470 + batch + ratio)
    n = [int(v) for v in r.integers(1, 700, batch)]
    for inline in (False, True):
        ap = Appender(471 + batch + ratio, n, ratio)
        while any(d < N for d, N in zip(ap.done, ap.n)):
            ap.append([int(v) for v in r.integers(0, 400, batch)], inline_slots=inline)
        check_against_oracle(ap)


def test_inline_slot_mapping_arguments():
    """Exactly one of slot_mapping / cu_entries missing is an argument error."""
    from paged_compressed_kv_b200 import v4kv
    ap = Appender(432, [10], 4)
    dev = torch.device("cuda")
    cu_e = torch.zeros(2, dtype=torch.int32, device=dev)
    with pytest.raises(ValueError):
        v4kv.v4kv_compress_append(
            torch.zeros(10, D, dtype=torch.bfloat16, device=dev), torch.zeros(10, device=dev),
            torch.tensor([0, 10], dtype=torch.int32, device=dev), torch.zeros(1, dtype=torch.int32, device=dev),
            torch.zeros(4, device=dev), 4, ap.state_x, ap.state_g, ap.main, None, cu_e)


def test_one_hot_gates_store_the_selected_token():
    r = synth.rng(420)
    n = [64, 130]
    gates = []
    for N in n:
        g = np.full(N, -1e30, dtype=np.float32)
        g[::4] = 0.0                       # the first token of every group
        gates.append(g)
    ap = Appender(421, n, 4, "bf16", gates=gates)
    ap.append(n)
    check_against_oracle(ap)
    for b, N in enumerate(n):
        rows, _ = ap.entries(b)
        # entry g == window-style copy of token 4g (RoPE at 4g), as bf16
        want = codecs.bf16_bits(compressor.window_tokens(ap.x[b][::4], np.arange(0, N, 4)))
        d = np.abs(codecs.bf16_to_f32(rows) - codecs.bf16_to_f32(want))
        assert np.all(d <= np.abs(codecs.bf16_to_f32(want)) * 2.0**-7 + 1e-30)


@pytest.mark.parametrize("ratio", [4, 128])
def test_full_size_random_chunks(ratio):
    # 8 sequences x 32K raw tokens appended in random chunks of 1..4096
    r = synth.rng(synth.seed_for("compressor") + ratio)
    n = [32768] * 8
    ap = Appender(synth.seed_for("compressor"), n, ratio)
    while any(d < N for d, N in zip(ap.done, ap.n)):
        ap.append([int(r.integers(1, 4097)) for _ in n])
    check_against_oracle(ap)


@pytest.mark.parametrize("ratio", [4, 128])
@pytest.mark.parametrize("dim", [128, 200, 1024])
def test_other_widths(ratio, dim):
    # one, ragged and four 256-dim spans per lane; two appends so the second
    # reads back the rolling state
    n = [1, 300, 1000, 129]
    ap = Appender(430 + dim + ratio, n, ratio, dim=dim)
    ap.append([v // 2 + 1 for v in n])
    ap.append(n)
    check_against_oracle(ap)


def test_fp8_window():
    n = [5, 128, 700, 2000]
    ap = Appender(440, n, 4, win_dtype="fp8")
    ap.append([v // 3 + 1 for v in n])
    ap.append(n)
    check_against_oracle(ap)


@pytest.mark.parametrize("ratio", [4, 128])
def test_more_sequences_than_cached_prefix_sums(ratio):
    # 1100 sequences (entry prefix sums do not fit the kernel's shared copy),
    # several with no new tokens in a call
    r = synth.rng(450 + ratio)
    n = [int(v) for v in r.integers(0, 300, 1100)]
    ap = Appender(451 + ratio, n, ratio)
    ap.append([int(v) for v in r.integers(0, 150, 1100)])
    ap.append(n)
    check_against_oracle(ap)


def test_slot_mapping_flags_bad_pages_and_overflow():
    from paged_compressed_kv_b200 import v4kv
    dev = torch.device("cuda")
    bt = torch.tensor([[0, 5, -1, 2]], dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    slots = torch.zeros(300, dtype=torch.int64, device=dev)
    cu = torch.zeros(2, dtype=torch.int32, device=dev)
    ss = torch.tensor([0], dtype=torch.int32, device=dev)
    nn = torch.tensor([1000], dtype=torch.int32, device=dev)
    v4kv.v4kv_slot_mapping(bt, ss, nn, 4, 3, slots, cu, dev_status=st)
    torch.cuda.synchronize()
    s = slots.cpu().numpy()
    assert cu.cpu().tolist() == [0, 250]
    assert np.array_equal(s[:64], np.arange(64))
    assert np.all(s[64:192] == -1)              # page 5 >= num_pages, and a -1 block
    assert np.array_equal(s[192:250], 2 * 64 + np.arange(58))
    assert int(st.item()) & 1
    st.zero_()
    small = torch.zeros(10, dtype=torch.int64, device=dev)
    v4kv.v4kv_slot_mapping(bt, ss, nn, 4, 3, small, None, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & 8


# Crafted quantiser inputs (scale 1 when amax = 448, so each quotient is the
# value itself). Expected e4m3 codes are worked by hand from the OCP FP8 E4M3
# definition (bias 7, 3 mantissa bits, subnormal quantum 2^-9, largest 448):
#   448 -> 0x7E; 1.0625 (midway 1.0 | 1.125) -> 1.0 = 0x38 (even mantissa);
#   1.1875 (midway 1.125 | 1.25) -> 1.25 = 0x3A; 1.0703125 -> 1.125 = 0x39;
#   -1.0625 -> 0xB8; 2^-8 -> 2 * 2^-9 = 0x02; 3 * 2^-10 (midway 1 | 2 quanta)
#   -> 0x02; 2^-10 (midway 0 | 1 quantum) -> 0x00; -2^-11 -> -0 = 0x80;
#   2^-9 -> 0x01; 5 * 2^-10 (midway 2 | 3 quanta) -> 0x02; 240 = 1.875 * 2^7
#   -> 0x77; 232 (midway 224 | 240) -> 224 = 0x76; -0.0 -> 0x80 (or 0x00 when the
#   fp32 group sum has returned +0, see below).
CRAFTED = [(448.0, 0x7E), (1.0625, 0x38), (1.1875, 0x3A), (1.0703125, 0x39), (-1.0625, 0xB8),
           (2.0 ** -8, 0x02), (3 * 2.0 ** -10, 0x02), (2.0 ** -10, 0x00), (-(2.0 ** -11), 0x80),
           (2.0 ** -9, 0x01), (5 * 2.0 ** -10, 0x02), (240.0, 0x77), (232.0, 0x76)]


def test_quantiser_edge_cases_through_the_compressor():
    # one-hot gates (the group's first token has logit 0, the others -1e30),
    # zero position bias and no RoPE make every entry exactly its group's first
    # token, so the quantiser sees chosen values: e4m3 ties to even, subnormal
    # quotients, -0 and negative underflow, an all-zero entry (scale 1), an
    # entry whose fp32 scale is itself subnormal (amax 2^-120), and a scale that
    # is not a power of two
    r = synth.rng(460)
    n_groups = 6
    N = 4 * n_groups
    x = np.zeros((N, D), dtype=np.float32)
    e0 = synth.normal(r, D, 8.0)
    for i, (v, _) in enumerate(CRAFTED):
        e0[i] = v
    e0[len(CRAFTED)] = -0.0
    e0[len(CRAFTED) + 1:] = np.clip(e0[len(CRAFTED) + 1:], -447.0, 447.0)
    x[0] = e0                                           # entry 0: amax 448, scale 1
    # entry 1 stays all zero
    x[8] = synth.normal(r, D, 30.0)                     # entry 2: a general scale
    x[8, 7] = 100.0
    x[12] = np.where(r.random(D) < 0.5, -1.0, 1.0) * 2.0 ** -120 * r.integers(1, 5, D)  # entry 3
    x[16] = -np.abs(synth.normal(r, D, 1e-3))           # entry 4: all negative, small,
    x[16, :8] = -1e-12 * np.arange(1, 9)                # eight of them far below the quantum
    x[20] = synth.normal(r, D, 1.0)                     # entry 5
    x[20, 3] = -0.0
    gates = np.full(N, -1e30, dtype=np.float32)
    gates[::4] = 0.0
    ap = Appender(461, [N], 4, "fp8", gates=[gates], rope=False, x=[x], bias=np.zeros(4))
    ap.append([N])
    tok = codecs.bf16_round(x[::4])                     # the exact token values
    pre = ap.prequant[0]
    assert np.array_equal(pre, tok)                     # -0 == +0 here
    rows, scs = ap.entries(0)
    # bytes and scales: bit-exact against the oracle's quantiser on the
    # kernel's own pre-quant values ...
    codes, sc = codecs.quantize_entry(pre)
    assert np.array_equal(rows, codes)
    assert np.array_equal(scs.view(np.uint32), sc.view(np.uint32))
    # ... and on the chosen tokens, except that a -0 token may reach the
    # quantiser as +0 (the fp32 group sum starts from +0)
    codes_t, sc_t = codecs.quantize_entry(tok)
    negzero = (tok == 0) & np.signbit(tok)
    assert np.array_equal(rows[~negzero], codes_t[~negzero])
    assert np.all(np.isin(rows[negzero], [0x00, 0x80]))
    assert np.array_equal(scs.view(np.uint32), sc_t.view(np.uint32))
    # the hand-worked codes of entry 0 (scale exactly 1)
    assert scs[0] == 1.0
    for i, (_, want) in enumerate(CRAFTED):
        assert rows[0, i] == want, (i, CRAFTED[i], hex(rows[0, i]))
    # the all-zero entry: scale 1, every code 0
    assert scs[1] == 1.0 and np.all(rows[1] == 0)
    # the tiny entry's scale is an fp32 subnormal, computed as amax / 448
    assert 0 < scs[3] < np.finfo(np.float32).tiny
    # negative underflow keeps the sign: 0x80, never 0x00, in the all-negative entry
    q4 = (x[16] / scs[4]).astype(np.float32)
    under = np.abs(q4) < 2.0 ** -10
    assert under.sum() >= 8
    assert np.all(rows[4][under] == 0x80)


VARIANTS = [
    (4, dict(overlap=True)),
    (4, dict(per_channel=True)),
    (128, dict(per_channel=True)),
    (4, dict(norm=True)),
    (128, dict(norm=True)),
    (4, dict(overlap=True, per_channel=True, norm=True)),
]


@pytest.mark.parametrize("ratio,opts", VARIANTS)
def test_variants_match_oracle_and_chunking(ratio, opts):
    """The compressor variants (P1 §2.1, §3.1.2, §3.2.1): the overlapping c4a
    window, per-channel gates, RMSNorm before RoPE. Random chunks against the
    oracle (pre-quantisation values, fp8 bytes on the GPU's own values,
    window, state), and chunked appends bitwise equal to one-shot ones."""
    n = [3000, 517, 5, 1200, 257] if ratio == 4 else [3000, 517, 5, 1200, 300]
    a = Appender(440 + ratio, n, ratio, **opts)
    a.append(n)
    b = Appender(440 + ratio, n, ratio, **opts)
    r = synth.rng(441)
    while any(d < N for d, N in zip(b.done, b.n)):
        b.append([int(r.integers(0, 700)) for _ in n])
    check_against_oracle(a)
    check_against_oracle(b)
    for s in range(len(n)):
        ra, sa = a.entries(s)
        rb, sb = b.entries(s)
        assert np.array_equal(ra, rb) and np.array_equal(sa, sb)
        assert np.array_equal(a.prequant[s].view(np.uint32), b.prequant[s].view(np.uint32))


@pytest.mark.parametrize("dim", [200, 1024])
@pytest.mark.parametrize("opts", [dict(overlap=True), dict(overlap=True, per_channel=True, norm=True)])
def test_c4a_variants_at_other_widths(dim, opts):
    """The c4a variant kernel at a ragged width (one partial chunk row per
    lane) and at 1024 dims (four chunk rows per lane): random chunks against
    the oracle, reading back the rolling state of the overlapping window."""
    n = [700, 129, 5, 300]
    ap = Appender(480 + dim, n, 4, dim=dim, **opts)
    r = synth.rng(481 + dim)
    while any(d < N for d, N in zip(ap.done, ap.n)):
        ap.append([int(r.integers(0, 260)) for _ in n])
    check_against_oracle(ap)


def test_variant_arguments():
    """The overlapping window is c4a's only; odd option values are rejected."""
    from paged_compressed_kv_b200 import v4kv
    ap = Appender(450, [10], 128)
    dev = torch.device("cuda")
    with pytest.raises(v4kv.V4KVError):
        v4kv.v4kv_compress_append(
            torch.zeros(10, D, dtype=torch.bfloat16, device=dev), torch.zeros(10, device=dev),
            torch.tensor([0, 10], dtype=torch.int32, device=dev), torch.zeros(1, dtype=torch.int32, device=dev),
            torch.zeros(256, device=dev), 128, ap.state_x, ap.state_g, ap.main, None, None, overlap=True)


def test_qk_prepare_matches_oracle_and_the_compressor_window_row():
    """v4kv_qk_prepare (P1 §3.2.1 Q/K insertion fusion): per-head RMSNorm and
    RoPE of q against the oracle; the new K row in the window is bitwise the
    row the compressor writes for the same token."""
    from paged_compressed_kv_b200 import PagedPool, Rope, v4kv
    dev = torch.device("cuda")
    r = synth.rng(460)
    B, H = 5, 64
    q = synth.normal(r, (B, H, D))
    kx = codecs.bf16_round(synth.normal(r, (B, D)))
    pos = np.array([0, 1, 255, 256 + 77, 100000], dtype=np.int32)
    w = (1.0 + synth.normal(r, D, 0.1)).astype(np.float32)
    wblk = [int(p // 256) + 1 for p in pos]
    wbt, Pw = paging.allocate_block_tables(wblk, synth.permutation(r, sum(wblk) + 1))
    win = PagedPool(data=torch.zeros(Pw, 256, D, dtype=torch.bfloat16, device=dev),
                    block_table=torch.from_numpy(wbt).to(dev))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    q_out = torch.empty(B, H, D, dtype=torch.float32, device=dev)
    v4kv.v4kv_qk_prepare(torch.from_numpy(q).to(dev), torch.from_numpy(pos).to(dev), q_out,
                         q_norm_weight=torch.from_numpy(w).to(dev), k_new=synth.bf16_tensor(kx).to(dev),
                         window=win, dev_status=st)
    qo_ref, ko_ref = compressor.qk_prepare(q, kx, pos, w)
    got = q_out.cpu().numpy()
    amax = np.abs(qo_ref).max(axis=2, keepdims=True)
    assert np.all(np.abs(got - qo_ref) <= 1e-5 * amax), float(np.abs(got - qo_ref).max())
    assert int(st.item()) == 0
    # the same token appended alone through the compressor (its window row)
    win2 = PagedPool(data=torch.zeros(Pw, 256, D, dtype=torch.bfloat16, device=dev),
                     block_table=torch.from_numpy(wbt).to(dev))
    # (its entries all land on one scratch page: only the window is compared)
    main = PagedPool(data=torch.zeros(1, 64, D, dtype=torch.uint8, device=dev),
                     block_table=torch.zeros(B, 400, dtype=torch.int32, device=dev),
                     scales=torch.zeros(1, 64, dtype=torch.float32, device=dev))
    v4kv.v4kv_compress_append(
        synth.bf16_tensor(kx).to(dev), torch.zeros(B, device=dev),
        torch.arange(B + 1, dtype=torch.int32, device=dev), torch.from_numpy(pos).to(dev),
        torch.zeros(4, device=dev), 4, torch.zeros(B, 4, D, dtype=torch.bfloat16, device=dev),
        torch.zeros(B, 4, device=dev), main, None, None, window=win2, window_len=128, dev_status=st)
    a1 = win.data.view(torch.int16).cpu().numpy()
    a2 = win2.data.view(torch.int16).cpu().numpy()
    for b in range(B):
        p = int(pos[b])
        pg = wbt[b, p // 256]
        assert np.array_equal(a1[pg, p % 256], a2[pg, p % 256]), b
        ref = codecs.bf16_bits(ko_ref[b:b + 1])[0].view(np.int16)
        xmax = float(np.abs(kx[b]).max())
        d = np.abs(codecs.bf16_to_f32(a1[pg, p % 256].view(np.uint16)) - codecs.bf16_to_f32(ref.view(np.uint16)))
        assert np.all(d <= np.abs(ko_ref[b]) * 2.0**-7 + xmax * 2.0**-20 + 1e-30)
    # bf16 output and no norm: RoPE only
    q_bf = torch.empty(B, H, D, dtype=torch.bfloat16, device=dev)
    v4kv.v4kv_qk_prepare(torch.from_numpy(q).to(dev), torch.from_numpy(pos).to(dev), q_bf, dev_status=st)
    qo2, _ = compressor.qk_prepare(q, None, pos)
    got2 = q_bf.float().cpu().numpy()
    assert np.all(np.abs(got2 - qo2) <= np.abs(qo2) * 2.0**-7 + np.abs(q).max(axis=2, keepdims=True) * 2.0**-20)
