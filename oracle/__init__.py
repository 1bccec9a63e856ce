"""CPU oracle for the paged, compressed KV-cache decode path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The product path (``paged_compressed_kv_b200``) never imports it and
shares no code with it: no kernels, headers, helpers, tables or constants.

It is a plain, slow, obviously-correct restatement of what the method computes,
written from the source page

    P1 = "DeepSeek-V4 Serving: KV cache and vLLM" (wmrh.cn/news/47220)

whose sections are cited as "P1 §2.1" etc. Floating point is fp64 unless the
step itself is an encoding whose precision is part of its definition (the fp8
and bf16 codecs, the per-entry quantiser and the indexer's fp32 score), in
which case the precision is stated in the function.

Modules
-------
codecs      bf16 and fp8-e4m3 (OCP FP8) encode/decode; per-entry absmax quantiser
rope        rotary position embedding on the rope dims, and its inverse
paging      256-token logical blocks, block tables, slot mapping, entry counts
compressor  c4a / c128a softmax-gated compression of raw tokens into entries
indexer     fp8 indexer scores and the exact top-k (ties -> lowest index)
attention   single-query decode attention over compressed entries + window
footprint   KV-cache bytes per sequence

Pins: every function is checked in ``tests/test_oracle_*.py`` against facts the
pages or mathematics fix (closed forms, library routines, invariants, brute
force, hand-derived worked examples under ``tests/golden/``); nothing there
compares the oracle with itself.
"""
