"""Seeded synthetic inputs shared by the tests, the oracle runs and bench.py.

This module draws random numbers and nothing else: lengths, page
permutations, raw tokens, gates, queries, and (for caches too large to build
on the host) random fp8 codes, scales and bf16 tokens drawn directly on the
device. It holds none of the method's arithmetic (no compression, no
quantiser, no paging, no attention); tests that need a cache exactly as the
method would store it build it with the oracle.

Workload shapes follow the page's serving setting (P1 = "DeepSeek-V4 Serving:
KV cache and vLLM", wmrh.cn/news/47220): shared KV dim 512 with RoPE on the
last 64 dims, 64 query heads, 128-token window, c4a / c128a ratios 4 / 128,
indexer dim 128, top-k 512.
"""
import numpy as np
import torch

SEED_BASE = 20260000

# one seed per named workload (fixed numbers, so stored inputs never change)
WORKLOAD_SEEDS = {"tiny-c4a": 0, "c4a-b64": 1, "c128a-b32": 2, "compressor": 3, "mixed-61": 4}


def seed_for(workload):
    return SEED_BASE + WORKLOAD_SEEDS[workload]


def rng(seed):
    return np.random.default_rng(seed)


def lengths_uniform(r, n, lo, hi, multiple=1):
    """n lengths uniform on [lo, hi], rounded down to a multiple."""
    x = r.integers(lo, hi + 1, size=n)
    return (x // multiple * multiple).astype(np.int64)


def lengths_loguniform(r, n, lo, hi, multiple=1):
    """n lengths log-uniform on [lo, hi], rounded down to a multiple."""
    x = np.exp(r.uniform(np.log(lo), np.log(hi), size=n)).astype(np.int64)
    x = np.clip(x, lo, hi)
    return (x // multiple * multiple).astype(np.int64)


def chunk_sizes(r, total, lo=1, hi=4096):
    """Split `total` into chunks with sizes uniform on [lo, hi] (last one cut)."""
    out = []
    left = int(total)
    while left > 0:
        c = int(min(left, r.integers(lo, hi + 1)))
        out.append(c)
        left -= c
    return out


def permutation(r, n):
    return r.permutation(n).astype(np.int64)


def normal(r, shape, std=1.0):
    return (r.standard_normal(shape) * std).astype(np.float32)


def bf16_tensor(x):
    """fp32 numpy array -> torch bfloat16 tensor (torch's round-to-nearest-even)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


# ---------------------------------------------------------------- device draws
# For caches of tens of GB: codes, scales and tokens are drawn with torch's
# device generator in chunks. fp8 codes come from torch's own fp8 cast of a
# scaled normal draw; they are random inputs, not quantised method outputs.

def device_generator(seed, device="cuda"):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def fill_fp8_codes(t, gen, spread=112.0, chunk=1 << 28):
    """Fill uint8 tensor `t` with e4m3 codes of N(0, spread^2) draws (|x| <= 448)."""
    flat = t.view(-1)
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        x = torch.randn(n, generator=gen, device=t.device, dtype=torch.float32)
        x.mul_(spread).clamp_(-448.0, 448.0)
        flat[i:i + n].copy_(x.to(torch.float8_e4m3fn).view(torch.uint8))
    return t


def fill_uniform(t, gen, lo, hi, chunk=1 << 28):
    """Fill a float tensor with U[lo, hi) draws."""
    flat = t.view(-1)
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        x = torch.rand(n, generator=gen, device=t.device, dtype=torch.float32)
        flat[i:i + n].copy_(x.mul_(hi - lo).add_(lo))
    return t


def fill_normal_bf16(t, gen, std=1.0, chunk=1 << 28):
    """Fill a bfloat16 tensor with N(0, std^2) draws."""
    flat = t.view(-1)
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        x = torch.randn(n, generator=gen, device=t.device, dtype=torch.float32)
        flat[i:i + n].copy_(x.mul_(std).to(torch.bfloat16))
    return t
