"""Failure detection without a GPU fault.

Every wait in the convolution kernels is bounded: a copy completion, a path group waiting for
the previous group of its sender, a row segment waiting for the earlier segments of its row.
Here a test hook withholds the first work item of a launch (its ticket is never drawn), so the
items that wait for it can only give up.  With a wait limit of a few milliseconds the launch must
return promptly, report E3_ERR_TIMEOUT through the device status word, and leave the context
usable: the next ordinary launch gives the oracle's result.  Nothing faults, traps or hangs: the
withheld item simply never runs, and every wait ends by its time limit."""

import math
import time

import numpy as np
import pytest
import torch

import oracle
from mlip_message_passing_b200 import workloads as W
from tests.conftest import rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def e3b():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from mlip_message_passing_b200 import e3b
    return e3b


def hub_graph(n=300, e=9000, hub=700, seed=31):
    """Random edges plus a hub at node 0 with `hub` in-edges and `hub` out-edges, so that node 0's
    rows are cut into several segments and work item 0 (group 0, row 0, segment 0) has waiters
    in both directions."""
    rng = np.random.default_rng(seed)
    src = rng.integers(1, n, e)
    dst = rng.integers(1, n, e)
    keep = src != dst
    src, dst = src[keep], dst[keep]
    others = rng.integers(1, n, hub)
    src = np.concatenate([src, others, np.zeros(hub, np.int64)]).astype(np.int32)
    dst = np.concatenate([dst, np.zeros(hub, np.int64), rng.integers(1, n, hub)]).astype(np.int32)
    vec = rng.standard_normal((src.shape[0], 3))
    return src, dst, vec


def test_withheld_work_item_times_out_and_context_survives(e3b):
    n, mul, lx, ly, lo = 300, 64, 2, 3, 2
    src, dst, vec = hub_graph(n)
    rng = np.random.default_rng(32)
    x = rng.standard_normal((n, mul * (lx + 1) ** 2)).astype(np.float32)
    p = e3b.Plan(W.irreps_str(mul, lx), W.sh_irreps(ly), lmax_out=lo)
    w = rng.standard_normal((src.shape[0], p.weight_numel)).astype(np.float32)
    go = rng.standard_normal((n, p.dim_out)).astype(np.float32)
    dev = "cuda"
    graph = e3b.Graph(n, torch.as_tensor(src, device=dev), torch.as_tensor(dst, device=dev))
    vr = graph.to_receiver_order(torch.as_tensor(vec.astype(np.float32), device=dev))
    wr = graph.to_receiver_order(torch.as_tensor(w, device=dev))
    xt, gt = torch.as_tensor(x, device=dev), torch.as_tensor(go, device=dev)
    s = 1 / math.sqrt(52)
    e3b.device_status()  # nothing pending
    assert e3b.lib.e3_set_test_knobs(5_000_000, 1) == e3b.E3_OK  # 5 ms limit, ticket 0 withheld
    try:
        for call in ("forward", "backward"):
            t0 = time.perf_counter()
            if call == "forward":
                e3b.conv_forward(p, graph, xt, wr, edge_vec=vr, out_scale=s)
            else:
                e3b.conv_backward(p, graph, xt, wr, gt, edge_vec=vr, out_scale=s)
            with pytest.raises(e3b.E3Error) as err:
                e3b.device_status()
            elapsed = time.perf_counter() - t0
            assert err.value.status == e3b.E3_ERR_TIMEOUT, call
            # the default limit is one second; the knob's few milliseconds must be what ended it
            assert elapsed < 0.5, (call, elapsed)
    finally:
        assert e3b.lib.e3_set_test_knobs(0, 0) == e3b.E3_OK
    e3b.device_status()  # cleared by the read above
    # the context is intact: ordinary launches give the oracle's results
    q = oracle.make_plan(W.irreps_str(mul, lx), W.sh_irreps(ly), lmax_out=lo)
    Y = oracle.real_sh_all(ly, vec.astype(np.float32).astype(np.float64))
    out = e3b.conv_forward(p, graph, xt, wr, edge_vec=vr, out_scale=s)
    gx, gy, gw = e3b.conv_backward(p, graph, xt, wr, gt, edge_vec=vr, out_scale=s)
    e3b.device_status()
    perm = graph.perm_dst.cpu().numpy()
    ref = oracle.conv_forward(q, n, src, dst, x, Y, w, s)
    rx, ry, rw = oracle.conv_backward(q, n, src, dst, x, Y, w, go, s)
    assert rel_err(out.cpu().numpy(), ref) <= 1e-5
    assert rel_err(gx.cpu().numpy(), rx) <= 1e-5
    assert rel_err(gy.cpu().numpy(), ry[perm]) <= 1e-5
    assert rel_err(gw.cpu().numpy(), rw[perm]) <= 1e-5
