"""The CSR build that allocates nothing (e3_csr_build_static).

Some callers cannot allocate device memory when they build a graph: code inside a CUDA stream
capture, a host program whose device memory all belongs to its own pool, or a loop that must not
pay the device synchronisation of cudaMalloc.  For them the library keeps the sort scratch in a
fixed device array.  This test calls that entry point through the C ABI and checks that it gives
the same index arrays as e3_csr_build (bit for bit, as every CSR test here), twice in a row on
different graphs, so that whatever the first call left in the shared array cannot leak into the
second result.  It lives in a file of its own that pytest collects last.
"""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _static_build(e3b, n, src, dst):
    E = src.shape[0]
    dev = src.device
    perm_dst = torch.full((E,), -7, dtype=torch.int32, device=dev)
    perm_src = torch.full((E,), -7, dtype=torch.int32, device=dev)
    rp_dst = torch.full((n + 1,), -7, dtype=torch.int32, device=dev)
    rp_src = torch.full((n + 1,), -7, dtype=torch.int32, device=dev)
    st = e3b.lib.e3_csr_build_static(n, E, e3b._ptr(src), e3b._ptr(dst), e3b._ptr(perm_dst), e3b._ptr(rp_dst),
                                     e3b._ptr(perm_src), e3b._ptr(rp_src), e3b._stream())
    assert st == e3b.E3_OK, e3b.lib.e3_last_error().decode()
    return perm_dst, rp_dst, perm_src, rp_src


def test_static_csr_matches_workspace_csr_two_calls():
    assert torch.cuda.is_available()
    from mlip_message_passing_b200 import e3b, workloads as W
    dev = torch.device("cuda", 0)
    g = W.graph_inputs(3000, 4, 0, 0, 0, seed=2)           # the water-box graph (~156k edges)
    rng = np.random.default_rng(11)
    n2, e2 = 70000, 90000                                     # a second, differently shaped graph
    cases = [(3000, g["src"], g["dst"]),
             (n2, rng.integers(0, n2, e2).astype(np.int32), rng.integers(0, n2, e2).astype(np.int32))]
    for n, src_h, dst_h in cases:
        src = torch.as_tensor(src_h, device=dev)
        dst = torch.as_tensor(dst_h, device=dev)
        ref = e3b.csr_build(n, src, dst)
        got = _static_build(e3b, n, src, dst)
        e3b.device_status()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


def test_static_csr_rejects_too_many_edges():
    from mlip_message_passing_b200 import e3b
    limit = 1 << 20
    st = e3b.lib.e3_csr_build_static(10, limit + 1, None, None, None, None, None, None, None)
    assert st == e3b.E3_ERR_SHAPE
    assert "limit" in e3b.lib.e3_last_error().decode()


def test_static_csr_runs_inside_a_stream_capture():
    """The reason the entry point exists: an ordinary call changes torch's allocated device memory by
    nothing, and a call recorded into a CUDA graph (stream capture fails on any allocation or
    synchronisation inside it) and replayed gives the workspace build's arrays."""
    from mlip_message_passing_b200 import e3b
    dev = torch.device("cuda", 0)
    rng = np.random.default_rng(5)
    n, e = 5000, 60000
    src = torch.as_tensor(rng.integers(0, n, e).astype(np.int32), device=dev)
    dst = torch.as_tensor(rng.integers(0, n, e).astype(np.int32), device=dev)
    ref = e3b.csr_build(n, src, dst)
    _static_build(e3b, n, src, dst)                           # warm-up: device state set up once
    torch.cuda.synchronize()
    bufs = [torch.full((e,), -7, dtype=torch.int32, device=dev), torch.full((n + 1,), -7, dtype=torch.int32, device=dev),
            torch.full((e,), -7, dtype=torch.int32, device=dev), torch.full((n + 1,), -7, dtype=torch.int32, device=dev)]
    # an ordinary call into preallocated outputs leaves torch's allocated device memory unchanged
    before = torch.cuda.memory_allocated(dev)
    st = e3b.lib.e3_csr_build_static(n, e, e3b._ptr(src), e3b._ptr(dst), e3b._ptr(bufs[0]), e3b._ptr(bufs[1]),
                                     e3b._ptr(bufs[2]), e3b._ptr(bufs[3]), e3b._stream())
    torch.cuda.synchronize()
    assert st == e3b.E3_OK and torch.cuda.memory_allocated(dev) == before
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        st = e3b.lib.e3_csr_build_static(n, e, e3b._ptr(src), e3b._ptr(dst), e3b._ptr(bufs[0]), e3b._ptr(bufs[1]),
                                         e3b._ptr(bufs[2]), e3b._ptr(bufs[3]), e3b._stream())
    assert st == e3b.E3_OK, e3b.lib.e3_last_error().decode()
    for b in bufs:
        b.fill_(-7)
    graph.replay()
    torch.cuda.synchronize()
    e3b.device_status()
    for got, want in zip(bufs, ref):
        assert torch.equal(got, want)
    del graph
