"""Parity of the uuu tensor product (one weight per path and channel, every channel index tied;
e3nn course, lesson 03b) with the float64 oracle, through the C ABI: forward and backward for each
compiled path set, ragged and odd channel counts, shared weights, the full-size workload on sampled
rows, and the calls the mode has no kernels for."""

import numpy as np
import pytest
import torch

import oracle
from mlip_message_passing_b200 import workloads as W
from tests.conftest import rel_err

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-5, torch.float64: 1e-12}
NP = {torch.float32: np.float32, torch.float64: np.float64}
DEV = "cuda"


@pytest.fixture(scope="module")
def e3b():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from mlip_message_passing_b200 import e3b
    return e3b


def t(a):
    return torch.as_tensor(np.ascontiguousarray(a)).to(DEV)


def h(x):
    return x.detach().cpu().numpy().astype(np.float64)


def plans(e3b, mul, lx, ly, lo, dtype, shared=False):
    a, b = W.irreps_str(mul, lx), W.irreps_str(mul, ly)
    return (e3b.Plan(a, b, lmax_out=lo, dtype=dtype, mode="uuu", shared_weights=shared),
            oracle.make_plan(a, b, lmax_out=lo, mode="uuu", shared_weights=shared))


@pytest.mark.parametrize("dtype", [torch.float32, torch.float64])
@pytest.mark.parametrize("mul,lx,ly,lo,B", [(8, 1, 1, 2, 37), (5, 1, 2, 2, 64), (16, 2, 3, 2, 33),
                                            (3, 3, 3, 3, 45), (128, 3, 3, 3, 7), (32, 2, 3, 2, 9),
                                            (64, 1, 2, 2, 5)])
def test_uuu_forward_backward(e3b, dtype, mul, lx, ly, lo, B):
    p, q = plans(e3b, mul, lx, ly, lo, dtype)
    assert p.weight_numel == q.weight_numel and p.dim_in2 == q.irreps_in2.dim and p.dim_out == q.irreps_out.dim
    np.testing.assert_allclose(p.alphas, q.alphas, rtol=1e-15)
    d = W.channel_inputs(B, mul, lx, ly, lo, seed=B + mul, dtype=NP[dtype])
    out = e3b.tp_forward(p, t(d["x"]), t(d["y"]), t(d["w"]))
    ref = oracle.tp_forward(q, d["x"], d["y"], d["w"])
    assert rel_err(h(out), ref) <= TOL[dtype]
    g = np.random.default_rng(B).standard_normal(ref.shape).astype(NP[dtype])
    res = e3b.tp_backward(p, t(d["x"]), t(d["y"]), t(d["w"]), t(g))
    for got, want in zip(res, oracle.tp_backward(q, d["x"], d["y"], d["w"], g)):
        assert rel_err(h(got), want) <= TOL[dtype]


def test_uuu_optional_gradients_and_empty_batch(e3b):
    p, q = plans(e3b, 4, 2, 3, 2, torch.float32)
    d = W.channel_inputs(20, 4, 2, 3, 2, seed=1)
    g = np.random.default_rng(2).standard_normal((20, q.irreps_out.dim)).astype(np.float32)
    rx, ry, rw = oracle.tp_backward(q, d["x"], d["y"], d["w"], g)
    gx, gy, gw = e3b.tp_backward(p, t(d["x"]), t(d["y"]), t(d["w"]), t(g), need_x=False, need_y=True, need_w=False)
    assert gx is None and gw is None and rel_err(h(gy), ry) <= 1e-5
    gx, gy, gw = e3b.tp_backward(p, t(d["x"]), t(d["y"]), t(d["w"]), t(g), need_x=False, need_y=False, need_w=True)
    assert rel_err(h(gw), rw) <= 1e-5
    z = torch.zeros
    out = e3b.tp_forward(p, z((0, p.dim_in1), device=DEV), z((0, p.dim_in2), device=DEV), z((0, p.weight_numel), device=DEV))
    assert out.shape == (0, p.dim_out)


def test_uuu_shared_weights(e3b):
    p, q = plans(e3b, 8, 1, 2, 2, torch.float32, shared=True)
    d = W.channel_inputs(50, 8, 1, 2, 2, seed=3)
    w = d["w"][0]
    assert rel_err(h(e3b.tp_forward(p, t(d["x"]), t(d["y"]), t(w))), oracle.tp_forward(q, d["x"], d["y"], w)) <= 1e-5


def test_uuu_full_size_sampled(e3b):
    """The channelwise workload at full size (32768 samples, 128 channels, degrees 0..3) in the
    launch the benchmark times; 64 sampled rows against the oracle."""
    cfg = W.CONFIGS["tp_uuu"]
    mul, lx, ly, lo = cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"]
    p, q = plans(e3b, mul, lx, ly, lo, torch.float32)
    d = W.channel_inputs(cfg["B"], mul, lx, ly, lo, cfg["seed"])
    x, y, w = t(d["x"]), t(d["y"]), t(d["w"])
    out = e3b.tp_forward(p, x, y, w)
    rows = np.random.default_rng(0).choice(cfg["B"], 64, replace=False)
    rows[-1] = cfg["B"] - 1
    ref = oracle.tp_forward(q, d["x"][rows], d["y"][rows], d["w"][rows])
    assert rel_err(h(out[torch.as_tensor(rows, device=DEV)]), ref) <= 1e-5
    g = np.random.default_rng(1).standard_normal((cfg["B"], q.irreps_out.dim)).astype(np.float32)
    res = e3b.tp_backward(p, x, y, w, t(g))
    want = oracle.tp_backward(q, d["x"][rows], d["y"][rows], d["w"][rows], g[rows])
    for got, r in zip(res, want):
        assert rel_err(h(got[torch.as_tensor(rows, device=DEV)]), r) <= 1e-5


def test_uuu_layouts_and_convolution_unsupported(e3b):
    with pytest.raises(e3b.E3Error, match="UNSUPPORTED"):
        e3b.Plan("8x0e+8x1o", "1x0e+1x1o", lmax_out=1, mode="uuu")  # y with one channel
    p = e3b.Plan("8x0e+8x1o", "8x0e+8x1o", lmax_out=2, mode="uuu")
    with pytest.raises(e3b.E3Error, match="UNSUPPORTED"):
        e3b.conv_workspace(p, 10, 20, DEV)
