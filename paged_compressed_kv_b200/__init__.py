"""v4kv: decode attention over a paged, compressed KV cache on B200 (sm_100a).

The product is the C-ABI shared library ``libv4kv.so`` (header
``include/v4kv.h``); ``paged_compressed_kv_b200.v4kv`` is its Python binding.
"""
from .v4kv import (  # noqa: F401
    EXPORTED, LIB_PATH, PagedPool, Rope, V4KVError, v4kv_compress_append,
    v4kv_decode_attention, v4kv_index_topk, v4kv_kv_footprint_bytes, v4kv_slot_mapping,
    v4kv_status_string, v4kv_version, v4kv_workspace_size,
)
