"""Python binding of the v4kv C ABI (``include/v4kv.h``).

Argument marshalling only: every function here checks tensor placement and
dtypes, converts torch tensors to raw pointers and calls the function of the
same name in ``libv4kv.so``. No computation happens in Python and there is no
fallback: if the shared library is missing, importing this module raises.
"""
import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libv4kv.so")

V4KV_OK = 0
V4KV_ERR_INVALID_ARG = 1
V4KV_ERR_UNSUPPORTED = 2
V4KV_ERR_CUDA = 3
V4KV_DEV_BAD_PAGE = 1
V4KV_DEV_BAD_SLOT = 2
V4KV_DEV_BAD_INDEX = 4
V4KV_DEV_OVERFLOW = 8
V4KV_DEV_TIMEOUT = 16
V4KV_DEV_RANGE = 32
V4KV_BF16 = 0
V4KV_FP8_E4M3 = 1
V4KV_FP32 = 2
V4KV_FP4_E2M1 = 3
V4KV_OP_INDEX_TOPK = 1
V4KV_OP_DECODE = 2

EXPORTED = [
    "v4kv_status_string", "v4kv_version", "v4kv_slot_mapping", "v4kv_compress_append",
    "v4kv_compress_append_ex", "v4kv_qk_prepare",
    "v4kv_index_topk", "v4kv_decode_attention", "v4kv_workspace_size", "v4kv_kv_footprint_bytes",
    "v4kv_decode_attention_noalloc", "v4kv_decode_attention_fp8out",
    "v4kv_page_bytes", "v4kv_plan_buckets", "v4kv_page_pools_create", "v4kv_page_pools_destroy",
    "v4kv_page_alloc", "v4kv_page_free", "v4kv_pages_free",
]

V4KV_NOALLOC_SCRATCH_BYTES = 32 << 20


class V4KVError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: {status} ({_lib.v4kv_status_string(status).decode()})")
        self.status = status


class _Paged(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("num_pages", ctypes.c_int32), ("slots_per_page", ctypes.c_int32),
                ("dim", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("block_table", ctypes.c_void_p), ("max_blocks", ctypes.c_int32)]


class _Rope(ctypes.Structure):
    _fields_ = [("theta", ctypes.c_double), ("rope_dim", ctypes.c_int32),
                ("rope_offset", ctypes.c_int32)]


class _CompressOpts(ctypes.Structure):
    _fields_ = [("overlap", ctypes.c_int32), ("gate_per_channel", ctypes.c_int32),
                ("norm_weight", ctypes.c_void_p), ("norm_eps", ctypes.c_float)]


class _Footprint(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("layer_ratios", ctypes.POINTER(ctypes.c_int32)),
                ("dim", ctypes.c_int32), ("entry_bits", ctypes.c_int32),
                ("entry_scale_bytes", ctypes.c_int32), ("indexer_dim", ctypes.c_int32),
                ("indexer_bits", ctypes.c_int32), ("indexer_scale_bytes", ctypes.c_int32),
                ("window", ctypes.c_int32), ("window_bits", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libv4kv.so not built at {LIB_PATH}: run python -m paged_compressed_kv_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, F32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "v4kv_status_string": (ctypes.c_char_p, [I32]),
        "v4kv_version": (I32, []),
        "v4kv_slot_mapping": (I32, [P, I32, I32, P, P, I32, I32, I32, P, P, I64, P, P]),
        "v4kv_compress_append": (I32, [P, P, P, P, I32, I32, P, I32, _Rope, P, P,
                                       ctypes.POINTER(_Paged), P, P, ctypes.POINTER(_Paged), I32,
                                       P, P, P]),
        "v4kv_compress_append_ex": (I32, [P, P, P, P, I32, I32, P, I32, _Rope, P, P,
                                          ctypes.POINTER(_Paged), P, P, ctypes.POINTER(_Paged), I32,
                                          P, ctypes.POINTER(_CompressOpts), P, P]),
        "v4kv_qk_prepare": (I32, [P, I32, I32, I32, P, F32, P, _Rope, P, I32, P,
                                  ctypes.POINTER(_Paged), P, P]),
        "v4kv_index_topk": (I32, [P, ctypes.POINTER(_Paged), P, I32, I32, I32, I32, I32, P, P, P,
                                  SZ, P, P]),
        "v4kv_decode_attention": (I32, [P, I32, I32, I32, ctypes.POINTER(_Paged),
                                        ctypes.POINTER(_Paged), P, I32, I32, I32, P, I32, F32,
                                        _Rope, P, P, SZ, P, P]),
        "v4kv_decode_attention_noalloc": (I32, [P, I32, I32, I32, ctypes.POINTER(_Paged),
                                                ctypes.POINTER(_Paged), P, I32, I32, I32, P, I32,
                                                F32, _Rope, P, P, P]),
        "v4kv_decode_attention_fp8out": (I32, [P, I32, I32, I32, ctypes.POINTER(_Paged),
                                               ctypes.POINTER(_Paged), P, I32, I32, I32, P, I32,
                                               F32, _Rope, P, P, P, P, SZ, P, P]),
        "v4kv_workspace_size": (I32, [I32, I32, I32, I32, I32, I32, I32, I32, I32,
                                      ctypes.POINTER(SZ)]),
        "v4kv_kv_footprint_bytes": (ctypes.c_uint64, [ctypes.c_uint64, ctypes.POINTER(_Footprint)]),
        "v4kv_page_bytes": (ctypes.c_uint64, [I32, I32, I32, I32]),
        "v4kv_plan_buckets": (I32, [I32, P, I32, P, P, P]),
        "v4kv_page_pools_create": (I32, [I32, P, P, ctypes.POINTER(ctypes.c_void_p)]),
        "v4kv_page_pools_destroy": (None, [P]),
        "v4kv_page_alloc": (I32, [P, I32, I32, P]),
        "v4kv_page_free": (I32, [P, I32, I32, P]),
        "v4kv_pages_free": (I64, [P, I32]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


@dataclass
class Rope:
    theta: float = 1e6
    rope_dim: int = 64
    rope_offset: int = 448

    def c(self):
        return _Rope(self.theta, self.rope_dim, self.rope_offset)


@dataclass
class PagedPool:
    """One paged pool: data [num_pages, slots_per_page, dim] (uint8 fp8 codes or
    bfloat16), scales [num_pages, slots_per_page] fp32 (fp8 only) and the block
    table [batch, max_blocks] int32, all on the same CUDA device."""
    data: torch.Tensor
    block_table: torch.Tensor
    scales: Optional[torch.Tensor] = None
    fp4: bool = False  # uint8 data holds packed fp4-e2m1 pairs (indexer pools)

    @property
    def dtype_code(self):
        if self.fp4:
            return V4KV_FP4_E2M1
        return V4KV_FP8_E4M3 if self.data.dtype == torch.uint8 else V4KV_BF16

    @property
    def dim(self):
        return self.data.shape[2] * (2 if self.fp4 else 1)

    def c(self):
        d = self.data
        _need(d, (torch.uint8, torch.bfloat16, torch.int16), "pool data", ndim=3)
        _need(self.block_table, (torch.int32,), "block_table", ndim=2)
        if self.dtype_code in (V4KV_FP8_E4M3, V4KV_FP4_E2M1):
            _need(self.scales, (torch.float32,), "scales", ndim=2)
        return _Paged(d.data_ptr(), _ptr(self.scales), d.shape[0], d.shape[1], self.dim,
                      self.dtype_code, self.block_table.data_ptr(), self.block_table.shape[1])


def _need(t, dtypes, what, ndim=None):
    if t is None:
        raise ValueError(f"{what} is required")
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise ValueError(f"{what} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{what} must have {ndim} dims")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _check(fn, st):
    if st != V4KV_OK:
        raise V4KVError(fn, st)


def v4kv_version():
    return _lib.v4kv_version()


def v4kv_status_string(status):
    return _lib.v4kv_status_string(status).decode()


def v4kv_slot_mapping(block_table, seq_start, n_new, ratio, num_pages, slot_out, cu_out=None,
                      dev_status=None, stream=None):
    _need(block_table, (torch.int32,), "block_table", ndim=2)
    _need(seq_start, (torch.int32,), "seq_start")
    _need(n_new, (torch.int32,), "n_new")
    _need(slot_out, (torch.int64,), "slot_out")
    if cu_out is not None:
        _need(cu_out, (torch.int32,), "cu_out")
    st = _lib.v4kv_slot_mapping(block_table.data_ptr(), block_table.shape[1], block_table.shape[0],
                                seq_start.data_ptr(), n_new.data_ptr(), ratio, 256 // ratio,
                                num_pages, _ptr(cu_out), slot_out.data_ptr(), slot_out.numel(),
                                _ptr(dev_status), _stream(stream))
    _check("v4kv_slot_mapping", st)


def v4kv_compress_append(x, gate, cu_seqlens, seq_start, pos_bias, ratio, state_x, state_gate,
                         main, slot_mapping, cu_entries, window=None, window_len=128,
                         rope=None, prequant_out=None, dev_status=None, stream=None,
                         overlap=False, gate_per_channel=False, norm_weight=None, norm_eps=0.0):
    """v4kv_compress_append; with any of overlap, gate_per_channel, norm_weight
    set, v4kv_compress_append_ex with those options."""
    _need(x, (torch.bfloat16,), "x", ndim=2)
    _need(gate, (torch.float32,), "gate")
    _need(cu_seqlens, (torch.int32,), "cu_seqlens")
    _need(seq_start, (torch.int32,), "seq_start")
    _need(pos_bias, (torch.float32,), "pos_bias")
    _need(state_x, (torch.bfloat16,), "state_x", ndim=3)
    _need(state_gate, (torch.float32,), "state_gate", ndim=3 if gate_per_channel else 2)
    if norm_weight is not None:
        _need(norm_weight, (torch.float32,), "norm_weight")
    if (slot_mapping is None) != (cu_entries is None):
        raise ValueError("slot_mapping and cu_entries: both or neither")
    if slot_mapping is not None:
        _need(slot_mapping, (torch.int64,), "slot_mapping")
        _need(cu_entries, (torch.int32,), "cu_entries")
    rope = rope or Rope()
    mc = main.c()
    wc = window.c() if window is not None else None
    args = (x.data_ptr(), gate.data_ptr(), cu_seqlens.data_ptr(), seq_start.data_ptr(),
            seq_start.numel(), x.shape[0], pos_bias.data_ptr(), ratio, rope.c(), state_x.data_ptr(),
            state_gate.data_ptr(), ctypes.byref(mc), _ptr(slot_mapping), _ptr(cu_entries),
            ctypes.byref(wc) if wc is not None else None, window_len, _ptr(prequant_out))
    if overlap or gate_per_channel or norm_weight is not None:
        opts = _CompressOpts(int(bool(overlap)), int(bool(gate_per_channel)), _ptr(norm_weight),
                             float(norm_eps))
        st = _lib.v4kv_compress_append_ex(*args, ctypes.byref(opts), _ptr(dev_status), _stream(stream))
        _check("v4kv_compress_append_ex", st)
    else:
        st = _lib.v4kv_compress_append(*args, _ptr(dev_status), _stream(stream))
        _check("v4kv_compress_append", st)


def v4kv_qk_prepare(q_in, positions, q_out, q_norm_weight=None, q_norm_eps=0.0, k_new=None, window=None,
                    rope=None, dev_status=None, stream=None):
    """Per-head RMSNorm (optional) and RoPE of q at each sequence's position,
    and the new K row rotated into the window pool, in one launch."""
    _need(q_in, (torch.float32,), "q_in", ndim=3)
    _need(positions, (torch.int32,), "positions")
    _need(q_out, (torch.float32, torch.bfloat16), "q_out", ndim=3)
    if q_out.shape != q_in.shape:
        raise ValueError("q_out must have q_in's shape")
    if q_norm_weight is not None:
        _need(q_norm_weight, (torch.float32,), "q_norm_weight")
    if k_new is not None:
        _need(k_new, (torch.bfloat16,), "k_new", ndim=2)
    rope = rope or Rope()
    wc = window.c() if window is not None else None
    B, H, dim = q_in.shape
    st = _lib.v4kv_qk_prepare(q_in.data_ptr(), B, H, dim, _ptr(q_norm_weight), float(q_norm_eps),
                              positions.data_ptr(), rope.c(), q_out.data_ptr(),
                              V4KV_BF16 if q_out.dtype == torch.bfloat16 else V4KV_FP32, _ptr(k_new),
                              ctypes.byref(wc) if wc is not None else None, _ptr(dev_status),
                              _stream(stream))
    _check("v4kv_qk_prepare", st)


def v4kv_workspace_size(op, batch, heads, max_seq_len, ratio, window_len, k, main_dtype, dim=512):
    out = ctypes.c_size_t(0)
    st = _lib.v4kv_workspace_size(op, batch, heads, max_seq_len, ratio, window_len, k, main_dtype,
                                  dim, ctypes.byref(out))
    _check("v4kv_workspace_size", st)
    return out.value


def v4kv_index_topk(q_idx, idx_cache, seq_lens, max_seq_len, ratio, window_len, k, topk_out,
                    workspace, score_out=None, dev_status=None, stream=None):
    _need(q_idx, (torch.float32,), "q_idx", ndim=2)
    _need(seq_lens, (torch.int32,), "seq_lens")
    _need(topk_out, (torch.int32,), "topk_out", ndim=2)
    _need(workspace, (torch.uint8,), "workspace")
    c = idx_cache.c()
    st = _lib.v4kv_index_topk(q_idx.data_ptr(), ctypes.byref(c), seq_lens.data_ptr(),
                              q_idx.shape[0], max_seq_len, ratio, window_len, k,
                              topk_out.data_ptr(), _ptr(score_out), workspace.data_ptr(),
                              workspace.numel(), _ptr(dev_status), _stream(stream))
    _check("v4kv_index_topk", st)


def v4kv_decode_attention(q, main, window, seq_lens, max_seq_len, ratio, window_len, out,
                          workspace, topk=None, sm_scale=None, rope=None, dev_status=None,
                          stream=None):
    _need(q, (torch.float32, torch.bfloat16), "q", ndim=3)
    _need(seq_lens, (torch.int32,), "seq_lens")
    _need(out, (torch.bfloat16,), "out", ndim=3)
    _need(workspace, (torch.uint8,), "workspace")
    if topk is not None:
        _need(topk, (torch.int32,), "topk", ndim=2)
    rope = rope or Rope()
    if sm_scale is None:
        sm_scale = 0.0  # the library's default, 1/sqrt(512)
    mc, wc = main.c(), window.c()
    st = _lib.v4kv_decode_attention(
        q.data_ptr(), V4KV_FP32 if q.dtype == torch.float32 else V4KV_BF16, q.shape[0], q.shape[1],
        ctypes.byref(mc), ctypes.byref(wc), seq_lens.data_ptr(), max_seq_len, ratio, window_len,
        _ptr(topk), topk.shape[1] if topk is not None else 0, sm_scale, rope.c(), out.data_ptr(),
        workspace.data_ptr(), workspace.numel(), _ptr(dev_status), _stream(stream))
    _check("v4kv_decode_attention", st)


def v4kv_decode_attention_fp8out(q, main, window, seq_lens, max_seq_len, ratio, window_len,
                                 out_codes, out_scales, workspace, topk=None, sm_scale=None,
                                 rope=None, prequant_out=None, dev_status=None, stream=None):
    """v4kv_decode_attention with the output quantised to e4m3 per (sequence,
    head) vector: out_codes uint8 [B, H, 512], out_scales fp32 [B, H]."""
    _need(q, (torch.float32, torch.bfloat16), "q", ndim=3)
    _need(seq_lens, (torch.int32,), "seq_lens")
    _need(out_codes, (torch.uint8,), "out_codes", ndim=3)
    _need(out_scales, (torch.float32,), "out_scales", ndim=2)
    _need(workspace, (torch.uint8,), "workspace")
    if topk is not None:
        _need(topk, (torch.int32,), "topk", ndim=2)
    if prequant_out is not None:
        _need(prequant_out, (torch.float32,), "prequant_out", ndim=3)
    rope = rope or Rope()
    if sm_scale is None:
        sm_scale = 0.0  # the library's default, 1/sqrt(512)
    mc, wc = main.c(), window.c()
    st = _lib.v4kv_decode_attention_fp8out(
        q.data_ptr(), V4KV_FP32 if q.dtype == torch.float32 else V4KV_BF16, q.shape[0], q.shape[1],
        ctypes.byref(mc), ctypes.byref(wc), seq_lens.data_ptr(), max_seq_len, ratio, window_len,
        _ptr(topk), topk.shape[1] if topk is not None else 0, sm_scale, rope.c(),
        out_codes.data_ptr(), out_scales.data_ptr(), _ptr(prequant_out), workspace.data_ptr(),
        workspace.numel(), _ptr(dev_status), _stream(stream))
    _check("v4kv_decode_attention_fp8out", st)


def v4kv_decode_attention_noalloc(q, main, window, seq_lens, max_seq_len, ratio, window_len, out,
                                  topk=None, sm_scale=None, rope=None, dev_status=None,
                                  stream=None):
    """v4kv_decode_attention without a workspace: for callers that cannot
    allocate device memory. The library's fixed device scratch array
    (V4KV_NOALLOC_SCRATCH_BYTES, shared by all calls on a device) holds the
    partial results; sizes needing more scratch are rejected. Overlapping
    calls on one device race on that scratch."""
    _need(q, (torch.float32, torch.bfloat16), "q", ndim=3)
    _need(seq_lens, (torch.int32,), "seq_lens")
    _need(out, (torch.bfloat16,), "out", ndim=3)
    if topk is not None:
        _need(topk, (torch.int32,), "topk", ndim=2)
    rope = rope or Rope()
    if sm_scale is None:
        sm_scale = 0.0  # the library's default, 1/sqrt(512)
    mc, wc = main.c(), window.c()
    st = _lib.v4kv_decode_attention_noalloc(
        q.data_ptr(), V4KV_FP32 if q.dtype == torch.float32 else V4KV_BF16, q.shape[0], q.shape[1],
        ctypes.byref(mc), ctypes.byref(wc), seq_lens.data_ptr(), max_seq_len, ratio, window_len,
        _ptr(topk), topk.shape[1] if topk is not None else 0, sm_scale, rope.c(), out.data_ptr(),
        _ptr(dev_status), _stream(stream))
    _check("v4kv_decode_attention_noalloc", st)


def v4kv_kv_footprint_bytes(n_tokens, layer_ratios, dim, entry_bits, entry_scale_bytes=0,
                            indexer_dim=0, indexer_bits=0, indexer_scale_bytes=0, window=0,
                            window_bits=0):
    arr = (ctypes.c_int32 * len(layer_ratios))(*layer_ratios)
    cfg = _Footprint(len(layer_ratios), arr, dim, entry_bits, entry_scale_bytes, indexer_dim,
                     indexer_bits, indexer_scale_bytes, window, window_bits)
    return int(_lib.v4kv_kv_footprint_bytes(n_tokens, ctypes.byref(cfg)))


# ------------------------------------------------------------------ page pools (host)

def v4kv_page_bytes(ratio, dim, elem_bits, scale_bytes=0):
    return int(_lib.v4kv_page_bytes(ratio, dim, elem_bits, scale_bytes))


def v4kv_plan_buckets(page_bytes, max_buckets=3):
    """Group page sizes into at most max_buckets buckets; returns
    (bucket_of per kind, bucket page bytes)."""
    n = len(page_bytes)
    pb = (ctypes.c_uint64 * n)(*page_bytes)
    bo = (ctypes.c_int32 * n)()
    bb = (ctypes.c_uint64 * max(1, max_buckets))()
    nb = ctypes.c_int32(0)
    _check("v4kv_plan_buckets", _lib.v4kv_plan_buckets(n, pb, max_buckets, bo, bb, ctypes.byref(nb)))
    return list(bo), list(bb)[: nb.value]


class PagePools:
    """Host-side fixed-size page pools of the planned buckets."""

    def __init__(self, bucket_bytes, pages_per_bucket):
        n = len(bucket_bytes)
        h = ctypes.c_void_p()
        _check("v4kv_page_pools_create", _lib.v4kv_page_pools_create(
            n, (ctypes.c_uint64 * n)(*bucket_bytes), (ctypes.c_int32 * n)(*pages_per_bucket),
            ctypes.byref(h)))
        self._h = h

    def alloc(self, bucket, n):
        out = (ctypes.c_int32 * max(1, n))()
        _check("v4kv_page_alloc", _lib.v4kv_page_alloc(self._h, bucket, n, out))
        return list(out)[:n]

    def free(self, bucket, pages):
        arr = (ctypes.c_int32 * max(1, len(pages)))(*pages)
        _check("v4kv_page_free", _lib.v4kv_page_free(self._h, bucket, len(pages), arr))

    def free_pages(self, bucket):
        return int(_lib.v4kv_pages_free(self._h, bucket))

    def close(self):
        if self._h:
            _lib.v4kv_page_pools_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()
