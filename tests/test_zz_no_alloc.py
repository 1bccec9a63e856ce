"""v4kv_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (for example code running inside another framework's
memory pool, or a serving thread that must not synchronise or lock an
allocator per request). Instead of a caller-provided workspace it uses the
library's fixed device scratch array.

Checked through the C ABI against v4kv_decode_attention (with a workspace) on
two calls in a row with different shapes, so a second call that reused stale
scratch contents would show. This file is collected last so that a run that
stops at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from tests.helpers import DecodeCase

pytestmark = pytest.mark.gpu


def _both(case):
    from paged_compressed_kv_b200 import v4kv
    dev = torch.device("cuda")
    q = torch.from_numpy(case.q).to(dev)
    main, win = case.main.to_cuda(), case.win.to_cuda()
    seq = torch.from_numpy(case.lens.astype(np.int32)).to(dev)
    ref = torch.empty(case.B, case.H, 512, dtype=torch.bfloat16, device=dev)
    got = torch.full_like(ref, float("nan"))
    ws = v4kv.v4kv_workspace_size(v4kv.V4KV_OP_DECODE, case.B, case.H, case.max_len, case.ratio,
                                  case.W, 0, main.dtype_code)
    workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    v4kv.v4kv_decode_attention(q, main, win, seq, case.max_len, case.ratio, case.W, ref, workspace,
                               dev_status=st)
    v4kv.v4kv_decode_attention_noalloc(q, main, win, seq, case.max_len, case.ratio, case.W, got,
                                       dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return got.float().cpu().numpy().astype(np.float64), ref.float().cpu().numpy().astype(np.float64)


def _close(got, ref):
    # the decode tolerance: max|d| <= 1e-2 max|ref|, sum|d| / sum|ref| <= 1e-3
    d = np.abs(got - ref)
    assert d.max() <= 1e-2 * np.abs(ref).max()
    assert d.sum() / np.abs(ref).sum() <= 1e-3


def test_noalloc_matches_workspace_entry_point_twice():
    first = DecodeCase(601, [9000, 300, 4100], 64, 4)
    second = DecodeCase(602, [200000, 131072 + 5], 8, 128)
    for case in (first, second):
        got, ref = _both(case)
        assert not np.isnan(got).any()
        _close(got, ref)


def test_noalloc_rejects_sizes_beyond_the_scratch():
    from paged_compressed_kv_b200 import v4kv
    dev = torch.device("cuda")
    case = DecodeCase(603, [1000], 8, 4)
    main, win = case.main.to_cuda(), case.win.to_cuda()
    big_batch = 4096
    need = v4kv.v4kv_workspace_size(v4kv.V4KV_OP_DECODE, big_batch, 128, 1_000_000, 4, 128, 0,
                                    main.dtype_code)
    assert need > v4kv.V4KV_NOALLOC_SCRATCH_BYTES
    q = torch.zeros(big_batch, 128, 512, dtype=torch.float32, device=dev)
    out = torch.empty(big_batch, 128, 512, dtype=torch.bfloat16, device=dev)
    seq = torch.zeros(big_batch, dtype=torch.int32, device=dev)
    with pytest.raises(v4kv.V4KVError) as e:
        v4kv.v4kv_decode_attention_noalloc(q, main, win, seq, 1_000_000, 4, 128, out)
    assert e.value.status == v4kv.V4KV_ERR_INVALID_ARG


def test_noalloc_call_allocates_nothing_under_graph_capture():
    # The defining property: the call allocates no device memory. During a
    # CUDA-graph capture in global mode any device allocation in the process
    # fails the capture, so a warm call that captures cleanly allocates
    # nothing; its replay must give the warm call's output bit for bit.
    from paged_compressed_kv_b200 import v4kv
    dev = torch.device("cuda")
    case = DecodeCase(604, [5000, 700, 12000], 64, 4)
    q = torch.from_numpy(case.q).to(dev)
    main, win = case.main.to_cuda(), case.win.to_cuda()
    seq = torch.from_numpy(case.lens.astype(np.int32)).to(dev)
    warm = torch.empty(case.B, case.H, 512, dtype=torch.bfloat16, device=dev)
    got = torch.full_like(warm, float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    v4kv.v4kv_decode_attention_noalloc(q, main, win, seq, case.max_len, case.ratio, case.W, warm,
                                       dev_status=st)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side, capture_error_mode="global"):
            v4kv.v4kv_decode_attention_noalloc(q, main, win, seq, case.max_len, case.ratio, case.W, got,
                                               dev_status=st)
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(got.view(torch.int16), warm.view(torch.int16))
