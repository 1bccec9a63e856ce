"""Benchmark of the decode step over a paged, compressed fp8 KV cache.

Default workload (one GPU): c4a decode, batch 64, context lengths uniform on
[4K, 64K], 64 query heads, shared KV dim 512 stored as fp8-e4m3 with one fp32
scale per entry, 128-token bf16 window, physical pages randomly permuted.
One step = the whole hot path for one new token per sequence:
v4kv_compress_append (1 token each; the slots come from the block tables
inside the compressor) -> v4kv_decode_attention (all visible entries +
window). Inputs are synthetic
(seeded device draws) and resident in HBM; L2 is flushed between steps.

The default run (N = 1) also measures the other workloads and adds them to
the same JSON line under "configs": the c128a decode (batch 32, context
log-uniform [128K, 1M]), the compressor write path (8 x 32K tokens in random
chunks, ratios 4 and 128) and the 61-layer mixed decode step (30 c4a layers
with the indexer's top-512 + 31 c128a layers, batch 128, context U[1K, 256K]).
Each sub-record carries its time, algorithmic bytes, GB/s, fraction of the
HBM peak and the SM clocks sampled while it ran.

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME]

Workloads: c4a-b64 (default, above); c128a-b32; tiny-c4a (1 sequence of 1024
tokens, 8 heads); compressor; mixed-61.
    python bench.py --impl reference ...   # the CPU oracle on host cores

Prints one JSON line (rank 0).
"""
import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decode-attention tokens/s and achieved HBM GB/s (% of B200 peak), fp8 paged KV"
D = 512
W = 128
HEADS = 64
L2_BYTES = 126e6
DTYPE = "f16"   # the tensor cores' operand type (fp8 codes convert to f16 exactly)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def l2_note(alg_bytes):
    rel = "exceed" if alg_bytes > L2_BYTES else "are smaller than"
    return (f"L2 flushed between steps (256 MB write); the step's algorithmic bytes "
            f"({alg_bytes / 1e6:.0f} MB) {rel} L2 (126 MB)")


# ------------------------------------------------------------------ workloads

def decode_workload(name, seqs=0):
    c = _decode_workload(name)
    if seqs:
        c["lens"] = c["lens"][:seqs]
    return c


def _decode_workload(name):
    r = synth.rng(synth.seed_for(name))
    if name == "c4a-b64":
        lens = synth.lengths_uniform(r, 64, 4096, 65536, 4)
        return dict(name="c4a decode, batch 64, context U[4K, 64K], 64 heads, fp8-e4m3 KV dim 512 "
                         "+ fp32 per-entry scale, 128-token bf16 window, shuffled pages",
                    lens=lens, ratio=4, r=r)
    if name == "c128a-b32":
        lens = synth.lengths_loguniform(r, 32, 131072, 1_000_000)
        return dict(name="c128a decode, batch 32, context log-uniform [128K, 1M], 64 heads, fp8-e4m3 "
                         "KV dim 512 + fp32 per-entry scale, 128-token bf16 window, shuffled pages",
                    lens=lens, ratio=128, r=r)
    if name == "tiny-c4a":
        return dict(name="tiny c4a decode, 1 sequence, context 1024, 8 heads", lens=np.array([1024]),
                    ratio=4, r=r, heads=8)
    raise ValueError(name)


def decode_inputs(workload, device, seed_offset=0, seqs=0):
    """Device-resident caches and per-step inputs of one decode workload, as
    plain torch tensors (seeded draws only; nothing here calls the library)."""
    c = decode_workload(workload, seqs)
    lens = c["lens"].astype(np.int64)
    ratio = c["ratio"]
    H = c.get("heads", HEADS)
    B = len(lens)
    r = c["r"]
    g = synth.device_generator(synth.seed_for(workload) + 7919 * seed_offset, device)
    spb = 256 // ratio
    n_ent = [-(-int(L) // ratio) for L in lens]
    nblk = [-(-n // spb) for n in n_ent]
    P = int(sum(nblk))
    perm = synth.permutation(r, P)
    bt = np.full((B, max(nblk)), -1, dtype=np.int32)
    k = 0
    for b, nb in enumerate(nblk):
        bt[b, :nb] = perm[k:k + nb]
        k += nb
    data = torch.empty(P, spb, D, dtype=torch.uint8, device=device)
    synth.fill_fp8_codes(data, g)
    scales = torch.empty(P, spb, dtype=torch.float32, device=device)
    synth.fill_uniform(scales, g, 0.5 / 112, 1.5 / 112)
    # window: pages only for the blocks holding tokens [L - W, L)
    wfirst = [max(0, int(L) - W) // 256 for L in lens]
    wlast = [(int(L) - 1) // 256 for L in lens]
    Pw = int(sum(l - f + 1 for f, l in zip(wfirst, wlast)))
    wperm = synth.permutation(r, Pw)
    wbt = np.full((B, max(wlast) + 1), -1, dtype=np.int32)
    k = 0
    for b in range(B):
        for blk in range(wfirst[b], wlast[b] + 1):
            wbt[b, blk] = wperm[k]
            k += 1
    wdata = torch.empty(Pw, 256, D, dtype=torch.bfloat16, device=device)
    synth.fill_normal_bf16(wdata, g)
    return dict(
        name=c["name"], lens=lens, ratio=ratio, H=H, B=B, P=P,
        data=data, scales=scales, bt=torch.from_numpy(bt).to(device),
        wdata=wdata, wbt=torch.from_numpy(wbt).to(device),
        # per-step inputs: the new token at position L - 1, then decode at L
        q=torch.randn(B, H, D, generator=g, device=device),
        x=torch.randn(B, D, generator=g, device=device).to(torch.bfloat16),
        gate=torch.randn(B, generator=g, device=device),
        bias=torch.randn(ratio, generator=g, device=device) * 0.5,
        state_x=torch.randn(B, ratio, D, generator=g, device=device).to(torch.bfloat16),
        state_g=torch.randn(B, ratio, generator=g, device=device),
    )


def decode_algorithmic_bytes(lens, ratio, H):
    """KV, scales, window, q, output and block-table bytes one decode call must touch."""
    tot = 0
    for L in lens:
        L = int(L)
        n_vis = max(0, L - W) // ratio
        tot += n_vis * (D + 4) + min(L, W) * D * 2 + H * D * 4 + H * D * 2
        tot += 4 * (-(-L // 256))
    return tot


class DecodeStep:
    """A decode workload wrapped for the library: pools, step buffers, workspace."""

    def __init__(self, workload, device, seed_offset=0, seqs=0):
        from paged_compressed_kv_b200 import PagedPool, v4kv
        inp = decode_inputs(workload, device, seed_offset, seqs)
        self.v4kv = v4kv
        self.name, self.lens, self.ratio = inp["name"], inp["lens"], inp["ratio"]
        self.H, self.B, self.P = inp["H"], inp["B"], inp["P"]
        self.main = PagedPool(data=inp["data"], block_table=inp["bt"], scales=inp["scales"])
        self.win = PagedPool(data=inp["wdata"], block_table=inp["wbt"])
        self.q, self.x, self.gate, self.bias = inp["q"], inp["x"], inp["gate"], inp["bias"]
        self.state_x, self.state_g = inp["state_x"], inp["state_g"]
        self.seq_start = torch.from_numpy((self.lens - 1).astype(np.int32)).to(device)
        self.n_new = torch.ones(self.B, dtype=torch.int32, device=device)
        self.cu_seqlens = torch.arange(self.B + 1, dtype=torch.int32, device=device)
        self.seq_lens = torch.from_numpy(self.lens.astype(np.int32)).to(device)
        self.out = torch.empty(self.B, self.H, D, dtype=torch.bfloat16, device=device)
        self.max_len = int(self.lens.max())
        ws = v4kv.v4kv_workspace_size(v4kv.V4KV_OP_DECODE, self.B, self.H, self.max_len, self.ratio,
                                      W, 0, v4kv.V4KV_FP8_E4M3)
        self.workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def launches_per_step(self):
        # compressor 1 (slots, entries, window rows and state in one launch),
        # decode 3 for 64 heads (query prep, sweep, merge) or 2 otherwise
        return 4 if self.H == 64 else 3

    def append(self, stream=None, inp=None):
        # the compressor derives the new token's slot from the block table
        x, gate, seq_start = (self.x, self.gate, self.seq_start) if inp is None else \
            (inp["x"], inp["gate"], inp["seq_start"])
        self.v4kv.v4kv_compress_append(x, gate, self.cu_seqlens, seq_start, self.bias,
                                       self.ratio, self.state_x, self.state_g, self.main, None, None,
                                       window=self.win, window_len=W, dev_status=self.status,
                                       stream=stream)

    def decode(self, stream=None, q=None, out=None, seq_lens=None):
        self.v4kv.v4kv_decode_attention(self.q if q is None else q, self.main, self.win,
                                        self.seq_lens if seq_lens is None else seq_lens,
                                        self.max_len, self.ratio, W,
                                        self.out if out is None else out, self.workspace,
                                        dev_status=self.status, stream=stream)

    def algorithmic_bytes(self):
        return decode_algorithmic_bytes(self.lens, self.ratio, self.H)

    def h2d_bytes(self):
        return (self.q.numel() * 4 + self.x.numel() * 2 + self.gate.numel() * 4 +
                self.seq_start.numel() * 4 + self.n_new.numel() * 4 + self.seq_lens.numel() * 4)

    def d2h_bytes(self):
        return self.out.numel() * 2


# ------------------------------------------------------------------ helpers

class ClockSampler:
    """nvidia-smi clock / throttle samples (every 50 ms) while the benchmark
    runs; summary(t0, t1) keeps the samples taken inside [t0, t1] (wall
    clock, time.time()), widened to the nearest sample on each side."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.rows = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in out.splitlines():
            f = [x.strip() for x in l.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(f[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + f[0].split(".")[1]) if "." in f[0] else 0.0
                sm, mx = float(f[2]), float(f[3])
            except (ValueError, IndexError):
                continue
            reasons = {n for n, v in zip(names, f[6:10]) if v.lower() == "active"}
            self.rows.append((ts, sm, mx, reasons))

    def summary(self, t0=None, t1=None):
        rows = self.rows
        if t0 is not None and rows:
            inside = [x for x in rows if t0 <= x[0] <= t1]
            before = [x for x in rows if x[0] < t0][-1:]
            after = [x for x in rows if x[0] > t1][:1]
            rows = before + inside + after
        if not rows:
            return None
        reasons = set()
        for x in rows:
            reasons |= x[3]
        return {"sm_mhz": float(np.median([x[1] for x in rows])),
                "sm_max_mhz": max(x[2] for x in rows), "reasons": sorted(reasons),
                "samples": len(rows)}


def max_over_ranks(values, device, world):
    """Element-wise maximum of per-rank timings over all ranks (every rank gets it)."""
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t]


def job_rates(batch_per_rank, world, t_step_ms, t_e2e_ms):
    """Whole-job tokens/s: every rank decodes its own batch (weak scaling), and the
    job takes as long as its slowest rank."""
    tokens = batch_per_rank * world
    return tokens / (t_step_ms * 1e-3), tokens / (t_e2e_ms * 1e-3)


def l2_flush(buf):
    buf.add_(1)


def source_digest(paths):
    h = hashlib.sha256()
    for p in paths:
        h.update(open(os.path.join(ROOT, p), "rb").read())
    return h.hexdigest()[:16]


SWEEP_SOURCES = ["paged_compressed_kv_b200/csrc/decode_tc.cu", "paged_compressed_kv_b200/csrc/tc.cuh"]


def sweep_traffic(workload):
    """DRAM bytes (read + write) of one sweep launch on this workload, from the
    committed ncu summary (profiles/decode_tc_traffic.txt), only when that
    capture was taken on the current sweep source; else None."""
    p = os.path.join(ROOT, "profiles", "decode_tc_traffic.txt")
    if not os.path.exists(p):
        return None
    digest = source_digest(SWEEP_SOURCES)
    for line in open(p):
        f = line.split()
        if len(f) >= 4 and f[0] == "traffic" and f[1] == workload and f[3] == digest:
            return float(f[2])
    return None


# ------------------------------------------------------------------ the oracle on host cores

SAMPLE_SEQS = 48   # fixed sample of whole sequences both CPU legs time


def oracle_host_pools(inp):
    """Host copies of one workload's caches (outside any timed region)."""
    return dict(
        main={"data": inp["data"].cpu().numpy(), "scales": inp["scales"].cpu().numpy(), "dtype": "fp8"},
        win={"data": inp["wdata"].view(torch.int16).cpu().numpy().view(np.uint16), "scales": None,
             "dtype": "bf16"},
        bt=inp["bt"].cpu().numpy(), wbt=inp["wbt"].cpu().numpy(),
        q=inp["q"].cpu().numpy().astype(np.float64), lens=inp["lens"], ratio=inp["ratio"])


def oracle_sample_order(B):
    """The sequences both CPU legs time, in order: a fixed seeded permutation."""
    return np.random.default_rng(0).permutation(B)[:min(SAMPLE_SEQS, B)]


def oracle_time(host, seqs):
    """Run the oracle on the given sequences; (wall s, process CPU s)."""
    from oracle import attention
    w0, c0 = time.perf_counter(), time.process_time()
    for b in seqs:
        m = dict(host["main"], block_table_row=host["bt"][b])
        w = dict(host["win"], block_table_row=host["wbt"][b])
        attention.decode_one(host["q"][b], m, w, int(host["lens"][b]), host["ratio"], W, 1 / math.sqrt(D))
    return time.perf_counter() - w0, time.process_time() - c0


def threads_available():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(inp):
    """The oracle as it stands on the host cores: the fixed sample once with the
    BLAS threads it has, and its first 8 sequences again on one thread."""
    host = oracle_host_pools(inp)
    order = oracle_sample_order(inp["B"])
    wall, cpu = oracle_time(host, order)
    one = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            w1, _ = oracle_time(host, order[:8])
        one = 8 / w1
    except Exception:
        pass
    return {"value": len(order) / wall, "unit": "tokens/s", "cores": round(cpu / wall, 2),
            "kind": "oracle", "threads_available": threads_available(),
            "value_1thread": one,
            "sample": f"{len(order)} whole sequences of the same workload (fixed seeded choice; fp64 "
                      f"numpy oracle, pages gathered on the host), {wall:.1f} s wall; 'cores' = "
                      f"process CPU time / wall time; value_1thread = its first 8 sequences with "
                      f"BLAS limited to one thread"}


# ------------------------------------------------------------------ arms

def time_events(fn, steps, flush, stream):
    """Median ms of fn() over `steps` runs, L2 flushed between runs."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        ev[i][0].record(stream)
        fn()
        ev[i][1].record(stream)
        l2_flush(flush)
    torch.cuda.synchronize()
    return float(np.median([a.elapsed_time(b) for a, b in ev]))


def run_ours(args, rank, world, device, clk):
    peak, peak_kind = load_peaks()
    step = DecodeStep(args.workload, device, seed_offset=rank, seqs=args.seqs)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    for _ in range(args.warmup):
        step.append()
        step.decode()
        l2_flush(flush)
    torch.cuda.synchronize()
    if step.status.item() != 0:
        raise RuntimeError(f"device status {step.status.item()}")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for i in range(args.steps):
        s0, s1, s2 = ev[i]
        s0.record(stream)
        step.append()
        s1.record(stream)
        step.decode()
        s2.record(stream)
        l2_flush(flush)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    step_ms = [a.elapsed_time(c) for a, _, c in ev]
    dec_ms = [b.elapsed_time(c) for _, b, c in ev]
    t_step = float(np.median(step_ms))
    t_dec = float(np.median(dec_ms))
    t_step, t_dec = max_over_ranks([t_step, t_dec], device, world)

    # End to end through the public API with host buffers (pinned), copies timed:
    # every step copies its inputs host -> device and its output back. Steps are
    # pipelined as a serving loop would run them: step i + 1's inputs travel on a
    # copy stream while step i computes, and step i's output returns on a third
    # stream, with two sets of device inputs and outputs. The K steps' total time
    # / K is the per-step figure; the caches a step reads (over 300 MB) exceed L2,
    # so no flush runs between them.
    names = ("q", "x", "gate", "seq_start", "n_new", "seq_lens")
    host_in = {n: getattr(step, n).cpu().pin_memory() for n in names}
    dev_in = [{n: getattr(step, n).clone() for n in names} for _ in range(2)]
    dev_out = [torch.empty_like(step.out) for _ in range(2)]
    host_out = [torch.empty(step.out.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    s_h2d, s_d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
    done = [torch.cuda.Event() for _ in range(2)]     # compute of the set finished
    landed = [torch.cuda.Event() for _ in range(2)]   # inputs of the set copied
    back = [torch.cuda.Event() for _ in range(2)]     # output of the set copied back

    def e2e_steps(n):
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(done[j])
                for nm in names:
                    dev_in[j][nm].copy_(host_in[nm], non_blocking=True)
                landed[j].record(s_h2d)
            stream.wait_event(landed[j])
            if i >= 2:
                stream.wait_event(back[j])
            step.append(stream=stream, inp=dev_in[j])
            step.decode(stream=stream, q=dev_in[j]["q"], out=dev_out[j], seq_lens=dev_in[j]["seq_lens"])
            done[j].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(done[j])
                host_out[j].copy_(dev_out[j], non_blocking=True)
                back[j].record(s_d2h)
        stream.wait_stream(s_d2h)
        stream.wait_stream(s_h2d)

    e2e_steps(args.warmup)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_h2d.wait_stream(stream)
    s_d2h.wait_stream(stream)
    e2e_steps(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    t_e2e = e0.elapsed_time(e1) / args.steps
    (t_e2e,) = max_over_ranks([t_e2e], device, world)
    if step.status.item() != 0:
        raise RuntimeError(f"device status {step.status.item()}")
    if not torch.equal(host_out[(args.steps - 1) % 2], dev_out[(args.steps - 1) % 2].cpu()):
        raise RuntimeError("end-to-end output copy mismatch")

    rate, rate_e2e = job_rates(step.B, world, t_step, t_e2e)
    alg = step.algorithmic_bytes()
    achieved = alg / (t_dec * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": rate,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPE,
        "data": "synthetic (seeded device draws: fp8 codes, fp32 scales, bf16 window, fp32 q)",
        "config": {"workload": step.name, "batch": step.B, "heads": step.H, "dim": D,
                   "ratio": step.ratio, "window": W, "parallelism": f"replicas x{world}",
                   "l2": l2_note(alg), "decode_ms": t_dec, "hbm_gbs": achieved,
                   "timing": f"median of {args.steps} steps (CUDA events)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": sweep_traffic(args.workload) if not args.seqs else None,
                     "kernel": "v4kv_decode_attention (query prep + sweep + merge)",
                     "algorithmic_bytes": alg, "peak_source": peak_kind},
        "e2e": {"value": rate_e2e, "unit": "tokens/s",
                "h2d_bytes_per_step": step.h2d_bytes(), "d2h_bytes_per_step": step.d2h_bytes(),
                "timing": f"{args.steps} steps pipelined over three streams (inputs in, compute, "
                          f"output out), total / steps; the caches read per step exceed L2"},
        "gpu_launches": step.launches_per_step() * args.steps,
    }
    line["_window"] = (t_wall0, t_wall1)
    return line, step


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step times a bounded sample of the
    same fixed sequence sample the cpu_baseline leg times. Inputs are the same
    seeded device draws as the library's arm; the library itself is not loaded."""
    if rank != 0:
        return None
    torch.set_grad_enabled(False)
    if not torch.cuda.is_available():
        return {"impl": "reference", "unavailable": "needs a CUDA device to draw the workload's caches"}
    dev = torch.device("cuda", 0)
    inp = decode_inputs(args.workload, dev, seqs=args.seqs)
    host = oracle_host_pools(inp)
    del inp["data"], inp["wdata"]
    order = oracle_sample_order(inp["B"])
    per = max(1, int(args.ref_seqs))
    cur = 0

    def next_seqs():
        nonlocal cur
        s = [order[(cur + i) % len(order)] for i in range(per)]
        cur += per
        return s

    for _ in range(args.warmup):
        oracle_time(host, next_seqs()[:1])
    cur = 0
    walls, cpus = [], []
    for _ in range(args.steps):
        w, c = oracle_time(host, next_seqs())
        walls.append(w)
        cpus.append(c)
    value = per * args.steps / float(np.sum(walls))
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * float(np.median(walls)), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded device draws)",
        "config": {"workload": inp["name"], "batch": inp["B"], "heads": inp["H"], "dim": D,
                   "ratio": inp["ratio"], "window": W, "parallelism": "cpu oracle, rank 0"},
        "cpu_baseline": {"value": value, "unit": "tokens/s",
                         "cores": round(float(np.sum(cpus)) / float(np.sum(walls)), 2),
                         "threads_available": threads_available(), "kind": "oracle",
                         "sample": f"{per} whole sequences per step, cycling through the fixed "
                                   f"{len(order)}-sequence sample the cpu_baseline leg times"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ other workloads

class CompressStep:
    """Compressor write path: 8 sequences x 32K raw bf16 tokens appended in
    random chunks of 1..4096 (one chunk per sequence per call), ratio 4 or 128,
    fp8 entries into shuffled pages, window copies of each chunk's last 128."""

    def __init__(self, device, ratio, seqs=8, tokens=32768, overlap=False, norm=False):
        from paged_compressed_kv_b200 import PagedPool, v4kv
        self.v4kv, self.ratio, self.B, self.N = v4kv, ratio, seqs, tokens
        self.overlap = overlap
        r = synth.rng(synth.seed_for("compressor") + ratio)
        g = synth.device_generator(synth.seed_for("compressor") + ratio, device)
        self.chunks = [synth.chunk_sizes(r, tokens) for _ in range(seqs)]
        self.calls = max(len(c) for c in self.chunks)
        spb = 256 // ratio
        nblk = -(-(-(-tokens // ratio)) // spb)
        P = nblk * seqs
        perm = synth.permutation(r, P)
        bt = perm.reshape(seqs, nblk).astype(np.int32)
        self.P = P
        self.main = PagedPool(data=torch.zeros(P, spb, D, dtype=torch.uint8, device=device),
                              block_table=torch.from_numpy(bt).to(device),
                              scales=torch.zeros(P, spb, dtype=torch.float32, device=device))
        wblk = -(-tokens // 256)
        wperm = synth.permutation(r, wblk * seqs).reshape(seqs, wblk).astype(np.int32)
        self.win = PagedPool(data=torch.zeros(wblk * seqs, 256, D, dtype=torch.bfloat16, device=device),
                             block_table=torch.from_numpy(wperm).to(device))
        self.x = torch.empty(seqs * tokens, D, dtype=torch.bfloat16, device=device)
        synth.fill_normal_bf16(self.x, g)
        self.gate = torch.randn(seqs * tokens, generator=g, device=device)
        self.bias = torch.randn(2 * ratio if overlap else ratio, generator=g, device=device) * 0.5
        rows = 2 * ratio if overlap else ratio
        self.state_x = torch.zeros(seqs, rows, D, dtype=torch.bfloat16, device=device)
        self.state_g = torch.zeros(seqs, rows, dtype=torch.float32, device=device)
        self.norm_w = (1.0 + 0.1 * torch.randn(D, generator=g, device=device)) if norm else None
        # per call: chunk rows gathered contiguously (inputs resident before timing)
        self.call_inputs = []
        done = [0] * seqs
        for c in range(self.calls):
            sizes = [self.chunks[b][c] if c < len(self.chunks[b]) else 0 for b in range(seqs)]
            rows = torch.cat([torch.arange(b * tokens + done[b], b * tokens + done[b] + sizes[b],
                                           device=device) for b in range(seqs)])
            cu = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device=device)
            ss = torch.tensor(done, dtype=torch.int32, device=device)
            nn = torch.tensor(sizes, dtype=torch.int32, device=device)
            self.call_inputs.append(dict(x=self.x[rows].contiguous(), gate=self.gate[rows].contiguous(),
                                         cu=cu, ss=ss, nn=nn, n=int(sum(sizes)),
                                         starts=np.array(done), sizes=np.array(sizes)))
            for b in range(seqs):
                done[b] += sizes[b]
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def call(self, c):
        """One append: the compressor derives the slots from the block table
        itself (no slot mapping argument, one launch)."""
        v, ci = self.v4kv, self.call_inputs[c]
        v.v4kv_compress_append(ci["x"], ci["gate"], ci["cu"], ci["ss"], self.bias, self.ratio,
                               self.state_x, self.state_g, self.main, None, None,
                               window=self.win, window_len=W, dev_status=self.status,
                               overlap=self.overlap, norm_weight=self.norm_w)

    def algorithmic_bytes(self, c):
        ci = self.call_inputs[c]
        n = ci["n"]
        touched = sum((-(-(int(s0) + int(m)) // self.ratio)) - int(s0) // self.ratio
                      for s0, m in zip(ci["starts"], ci["sizes"]) if m)
        win = sum(min(int(m), W) for m in ci["sizes"])
        rows = 2 * self.ratio if self.overlap else self.ratio
        return n * (D * 2 + 4) + touched * (D + 4) + win * D * 2 + self.B * rows * (D * 2 + 4)


def run_compress(args, device, clk):
    peak, _ = load_peaks()
    out = {}
    # the plain compressor for both ratios, then c4a with the overlapping
    # 8-token window and RMSNorm (the variant kernel)
    for key, ratio, var in (("r4", 4, {}), ("r128", 128, {}),
                            ("r4_overlap_norm", 4, dict(overlap=True, norm=True))):
        st = CompressStep(device, ratio, **var)
        for c in range(st.calls):  # warm-up pass (also fills the cache once)
            st.call(c)
        torch.cuda.synchronize()
        # eager: each call timed on its own, Python enqueue included
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(st.calls)]
        for c in range(st.calls):
            ev[c][0].record()
            st.call(c)
            ev[c][1].record()
        torch.cuda.synchronize()
        ms_eager = sum(a.elapsed_time(b) for a, b in ev)
        # the same calls captured once into a CUDA graph and replayed
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                for c in range(st.calls):
                    st.call(c)
        torch.cuda.synchronize()
        for _ in range(3):
            graph.replay()
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        reps, ms_g = max(5, args.steps), []
        torch.cuda.synchronize()
        t0 = time.time()
        for _ in range(reps):
            flush.fill_(1)  # inputs of one pass (~300 MB) exceed L2 anyway
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            ms_g.append(e0.elapsed_time(e1))
        t1 = time.time()
        del graph
        ms = float(np.median(ms_g))
        byts = sum(st.algorithmic_bytes(c) for c in range(st.calls))
        out[key] = {"calls": st.calls, "tokens": st.B * st.N, "ms": ms,
                            "algorithmic_bytes": byts,
                            "tokens_per_s": st.B * st.N / (ms * 1e-3),
                            "gbs": byts / (ms * 1e-3) / 1e9, "frac": byts / (ms * 1e-3) / 1e9 / peak,
                            "ms_eager": ms_eager,
                            "gbs_eager": byts / (ms_eager * 1e-3) / 1e9,
                            "status": int(st.status.item()),
                            "launches": st.calls, "_window": (t0, t1)}
        del st
        torch.cuda.empty_cache()
    return {"config": "compressor write path, 8 x 32K raw bf16 tokens, random chunks 1..4096, fp8 "
                      "entries, shuffled pages, slots from the block tables inside the compressor; "
                      "ms = one CUDA-graph replay of all calls (median), ms_eager = the calls launched "
                      "one by one from Python", "results": out}


class MixedStep:
    """61-layer mixed decode step: 30 c4a layers (indexer top-512 over fp8 keys
    of dim 128, then attention over the selected entries + window) and 31 c128a
    layers (attention over all visible entries + window); batch 128, context
    U[1K, 256K], 64 heads, fp8 KV dim 512. Every layer has its own caches."""

    def __init__(self, device, seqs=128, c4a_layers=30, c128a_layers=31, k=512):
        from paged_compressed_kv_b200 import PagedPool, v4kv
        self.v4kv, self.k = v4kv, k
        r = synth.rng(synth.seed_for("mixed-61"))
        self.lens = synth.lengths_uniform(r, seqs, 1024, 262144, 4)
        self.B = seqs
        g = synth.device_generator(synth.seed_for("mixed-61"), device)
        self.max_len = int(self.lens.max())
        self.seq_lens = torch.from_numpy(self.lens.astype(np.int32)).to(device)

        def pool(ratio, dim):
            spb = 256 // ratio
            nblk = [-(-(-(-int(L) // ratio)) // spb) for L in self.lens]
            P = int(sum(nblk))
            perm = synth.permutation(r, P)
            bt = np.full((seqs, max(nblk)), -1, dtype=np.int32)
            kk = 0
            for b, nb in enumerate(nblk):
                bt[b, :nb] = perm[kk:kk + nb]
                kk += nb
            data = torch.empty(P, spb, dim, dtype=torch.uint8, device=device)
            synth.fill_fp8_codes(data, g)
            sc = torch.empty(P, spb, dtype=torch.float32, device=device)
            synth.fill_uniform(sc, g, 0.5 / 112, 1.5 / 112)
            return PagedPool(data=data, block_table=torch.from_numpy(bt).to(device), scales=sc)

        def window():
            wf = [max(0, int(L) - W) // 256 for L in self.lens]
            wl = [(int(L) - 1) // 256 for L in self.lens]
            Pw = int(sum(l - f + 1 for f, l in zip(wf, wl)))
            wperm = synth.permutation(r, Pw)
            wbt = np.full((seqs, max(wl) + 1), -1, dtype=np.int32)
            kk = 0
            for b in range(seqs):
                for blk in range(wf[b], wl[b] + 1):
                    wbt[b, blk] = wperm[kk]
                    kk += 1
            wd = torch.empty(Pw, 256, D, dtype=torch.bfloat16, device=device)
            synth.fill_normal_bf16(wd, g)
            return PagedPool(data=wd, block_table=torch.from_numpy(wbt).to(device))

        def append_inputs(ratio, P):
            # the new token of every sequence (position L - 1) and the
            # compressor state of its unfinished group
            return dict(x=torch.randn(seqs, D, generator=g, device=device).to(torch.bfloat16),
                        gate=torch.randn(seqs, generator=g, device=device),
                        bias=torch.randn(ratio, generator=g, device=device) * 0.5,
                        sx=torch.randn(seqs, ratio, D, generator=g, device=device).to(torch.bfloat16),
                        sg=torch.randn(seqs, ratio, generator=g, device=device), P=P)

        self.c4a = []
        for _ in range(c4a_layers):
            main = pool(4, D)
            self.c4a.append(dict(main=main, idx=pool(4, 128), win=window(),
                                 q=torch.randn(seqs, HEADS, D, generator=g, device=device),
                                 qi=torch.randn(seqs, 128, generator=g, device=device),
                                 ap=append_inputs(4, main.data.shape[0])))
        self.c128a = []
        for _ in range(c128a_layers):
            main = pool(128, D)
            self.c128a.append(dict(main=main, win=window(),
                                   q=torch.randn(seqs, HEADS, D, generator=g, device=device),
                                   ap=append_inputs(128, main.data.shape[0])))
        self.seq_start = torch.from_numpy((self.lens - 1).astype(np.int32)).to(device)
        self.n_new = torch.ones(seqs, dtype=torch.int32, device=device)
        self.cu_seqlens = torch.arange(seqs + 1, dtype=torch.int32, device=device)
        self.topk = torch.empty(seqs, k, dtype=torch.int32, device=device)
        self.out = torch.empty(seqs, HEADS, D, dtype=torch.bfloat16, device=device)
        v = v4kv
        wsa = v.v4kv_workspace_size(v.V4KV_OP_DECODE, seqs, HEADS, self.max_len, 4, W, k, v.V4KV_FP8_E4M3)
        wsb = v.v4kv_workspace_size(v.V4KV_OP_DECODE, seqs, HEADS, self.max_len, 128, W, 0, v.V4KV_FP8_E4M3)
        wsi = v.v4kv_workspace_size(v.V4KV_OP_INDEX_TOPK, seqs, 1, self.max_len, 4, W, k, v.V4KV_FP8_E4M3, 128)
        self.ws = torch.empty(max(wsa, wsb, wsi, 256), dtype=torch.uint8, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def append(self, L, ratio, stream=None):
        """One new token per sequence into layer L's cache: the compressor
        (entry of the token's group, window row, state), slots derived from
        the block table inside it."""
        a, v = L["ap"], self.v4kv
        v.v4kv_compress_append(a["x"], a["gate"], self.cu_seqlens, self.seq_start, a["bias"], ratio,
                               a["sx"], a["sg"], L["main"], None, None, window=L["win"],
                               window_len=W, dev_status=self.status, stream=stream)

    def full_step(self, overlap, side=None):
        """The 61-layer decode step with each layer's append. With `overlap`,
        a c4a layer's indexer runs on the side stream while its compressor
        append runs on the current stream (P1 §3.2.2: indexer and main-KV
        compression / window insertion are independent after the
        projections); attention waits for both."""
        cur = torch.cuda.current_stream()
        for l in range(len(self.c4a)):
            L = self.c4a[l]
            if overlap:
                side.wait_stream(cur)
                with torch.cuda.stream(side):
                    self.index(l)
                self.append(L, 4)
                cur.wait_stream(side)
            else:
                self.append(L, 4)
                self.index(l)
            self.attend_c4a(l)
        for l in range(len(self.c128a)):
            self.append(self.c128a[l], 128)
            self.attend_c128a(l)

    def index(self, l):
        L = self.c4a[l]
        self.v4kv.v4kv_index_topk(L["qi"], L["idx"], self.seq_lens, self.max_len, 4, W, self.k, self.topk,
                                  self.ws, dev_status=self.status)

    def attend_c4a(self, l):
        L = self.c4a[l]
        self.v4kv.v4kv_decode_attention(L["q"], L["main"], L["win"], self.seq_lens, self.max_len, 4, W,
                                        self.out, self.ws, topk=self.topk, dev_status=self.status)

    def attend_c128a(self, l):
        L = self.c128a[l]
        self.v4kv.v4kv_decode_attention(L["q"], L["main"], L["win"], self.seq_lens, self.max_len, 128, W,
                                        self.out, self.ws, dev_status=self.status)

    def bytes(self):
        nv4 = np.maximum(0, self.lens - W) // 4
        nv128 = np.maximum(0, self.lens - W) // 128
        win = np.minimum(self.lens, W) * D * 2
        qo = HEADS * D * 4 + HEADS * D * 2
        idx = int(np.sum(nv4 * (128 + 4) + 128 * 4 + self.k * 4))
        att4 = int(np.sum(np.minimum(nv4, self.k) * (D + 4) + win + qo))
        att128 = int(np.sum(nv128 * (D + 4) + win + qo))
        return idx, att4, att128


def run_mixed(args, device, clk, layers=0, seqs=0):
    peak, _ = load_peaks()
    kw = {}
    if seqs:
        kw["seqs"] = seqs
    if layers:
        kw["c4a_layers"] = min(30, layers)
        kw["c128a_layers"] = min(31, layers)
    st = MixedStep(device, **kw)
    nl4, nl128 = len(st.c4a), len(st.c128a)

    def whole_step():
        for l in range(nl4):
            st.index(l)
            st.attend_c4a(l)
        for l in range(nl128):
            st.attend_c128a(l)

    side_stream = torch.cuda.Stream()
    parts = {"step": whole_step,
             "idx": lambda: [st.index(l) for l in range(nl4)],
             "att4": lambda: [st.attend_c4a(l) for l in range(nl4)],
             "att128": lambda: [st.attend_c128a(l) for l in range(nl128)],
             "full_serial": lambda: st.full_step(False),
             "full_overlap": lambda: st.full_step(True, side_stream)}
    for _ in range(args.warmup):
        whole_step()
    st.full_step(False)
    st.full_step(True, side_stream)
    torch.cuda.synchronize()
    # each part is captured once into a CUDA graph and replayed, so the times
    # are the device's, without the Python enqueue of ~150 calls per step
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graphs = {}
    with torch.cuda.stream(side):
        for name, fn in parts.items():
            graphs[name] = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graphs[name], stream=side):
                fn()
    torch.cuda.synchronize()
    tot, win = {}, {}
    for name, gr in graphs.items():
        gr.replay()
        gr.replay()
        ms = []
        torch.cuda.synchronize()
        t0 = time.time()
        for _ in range(args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            gr.replay()
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        win[name] = (t0, time.time())
        tot[name] = float(np.median(ms))
    graphs.clear()
    idx_b, a4_b, a128_b = st.bytes()
    step_ms = tot["step"]

    def rec(ms_layer, byts, key):
        gbs = byts / (ms_layer * 1e-3) / 1e9
        return {"ms_per_layer": ms_layer, "algorithmic_bytes_per_layer": byts, "gbs": gbs,
                "frac": gbs / peak, "_window": win[key]}

    step_bytes = nl4 * (idx_b + a4_b) + nl128 * a128_b
    res = {"step_ms": step_ms, "parts_ms_sum": tot["idx"] + tot["att4"] + tot["att128"],
           "tokens_per_s": st.B / (step_ms * 1e-3), "algorithmic_bytes": step_bytes,
           "indexer": rec(tot["idx"] / nl4, idx_b, "idx"),
           "c4a_attention": rec(tot["att4"] / nl4, a4_b, "att4"),
           "c128a_attention": rec(tot["att128"] / nl128, a128_b, "att128"),
           "step_gbs": step_bytes / (step_ms * 1e-3) / 1e9,
           "status": int(st.status.item()), "_window": win["step"]}
    res["step_frac"] = res["step_gbs"] / peak
    # the same step with every layer's append (one token per sequence), its
    # c4a indexers serialised or overlapped with the appends on a second stream
    res["full_step_serial_ms"] = tot["full_serial"]
    res["full_step_overlap_ms"] = tot["full_overlap"]
    res["overlap_saving"] = 1.0 - tot["full_overlap"] / tot["full_serial"]
    name = (f"{nl4 + nl128}-layer mixed step ({nl4} c4a with indexer top-512 + {nl128} c128a), "
            f"batch {st.B}, context U[1K, 256K], 64 heads, fp8 KV; CUDA-graph replays, median of "
            f"{args.steps}")
    del st
    torch.cuda.empty_cache()
    return {"config": name, "results": res}


def run_decode_only(args, device, workload, clk):
    """Decode call alone (v4kv_decode_attention) on one workload: median of
    `steps` calls with L2 flushed between them."""
    peak, _ = load_peaks()
    step = DecodeStep(workload, device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        step.decode()
        l2_flush(flush)
    torch.cuda.synchronize()
    t0 = time.time()
    ms = time_events(step.decode, max(args.steps, 20), flush, stream)
    t1 = time.time()
    alg = step.algorithmic_bytes()
    gbs = alg / (ms * 1e-3) / 1e9
    st = int(step.status.item())
    res = {"workload": step.name, "decode_ms": ms, "tokens_per_s": step.B / (ms * 1e-3),
           "algorithmic_bytes": alg, "gbs": gbs, "frac": gbs / peak, "l2": l2_note(alg),
           "traffic": sweep_traffic(workload), "status": st, "_window": (t0, t1)}
    del step
    torch.cuda.empty_cache()
    return res


def finish_clocks(d, clk):
    """Replace the wall-clock windows recorded in a result tree by clock summaries."""
    if isinstance(d, dict):
        if "_window" in d:
            w = d.pop("_window")
            if "clocks" not in d:
                d["clocks"] = clk.summary(*w)
        for v in d.values():
            finish_clocks(v, clk)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="c4a-b64",
                    choices=["c4a-b64", "c128a-b32", "tiny-c4a", "compressor", "mixed-61"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-seqs", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads' sub-records (headline line only)")
    ap.add_argument("--layers", type=int, default=0,
                    help="mixed-61: c4a and c128a layers each (small cases for profiler captures)")
    ap.add_argument("--seqs", type=int, default=0,
                    help="keep only the first n sequences (small cases for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if args.workload in ("compressor", "mixed-61") and world == 1:
        with ClockSampler(device.index) as clk:
            res = (run_compress(args, device, clk) if args.workload == "compressor"
                   else run_mixed(args, device, clk, args.layers, args.seqs))
        finish_clocks(res, clk)
        print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        with ClockSampler(device.index) as clk:
            line, step = run_ours(args, rank, world, device, clk)
            extra = None
            if rank == 0 and world == 1 and not args.no_configs and not args.seqs \
                    and args.workload == "c4a-b64":
                del step
                torch.cuda.empty_cache()
                extra = {
                    "c128a-b32": run_decode_only(args, device, "c128a-b32", clk),
                    "compressor": run_compress(args, device, clk),
                    "mixed-61": run_mixed(args, device, clk),
                }
        line["clocks"] = clk.summary(*line.pop("_window"))
        if extra is not None:
            finish_clocks(extra, clk)
            line["configs"] = extra
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            inp = decode_inputs(args.workload, device, seqs=args.seqs)
            line["cpu_baseline"] = cpu_baseline(inp)
            del inp
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
