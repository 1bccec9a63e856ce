"""v4kv: decode attention over a paged, compressed KV cache on B200 (sm_100a).

The product is the C-ABI shared library ``libv4kv.so`` (header
``include/v4kv.h``); ``paged_compressed_kv_b200.v4kv`` is its Python binding.
Attributes of the binding are re-exported here on first use, so that the
build step (``paged_compressed_kv_b200.build``) imports without the library.
"""

_EXPORTS = {
    "EXPORTED", "LIB_PATH", "PagedPool", "PagePools", "v4kv_page_bytes", "v4kv_plan_buckets", "Rope", "V4KVError", "v4kv_compress_append",
    "v4kv_decode_attention", "v4kv_decode_attention_fp8out", "v4kv_decode_attention_noalloc", "v4kv_index_topk",
    "v4kv_kv_footprint_bytes", "v4kv_slot_mapping", "v4kv_status_string", "v4kv_version",
    "v4kv_workspace_size", "v4kv_qk_prepare",
}


def __getattr__(name):
    if name in _EXPORTS:
        from . import v4kv
        return getattr(v4kv, name)
    raise AttributeError(name)
