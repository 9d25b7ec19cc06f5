"""Parity of the fully connected (uvw) tensor product with shared weights (e3nn course, lesson 03b:
every channel of x and y feeds every output channel) with the float64 oracle, through the C ABI:
the forward and grad_x run on the tcgen05 tensor cores (three tf32 passes), grad_w and grad_y on the
CUDA cores.  Tolerance: the float32 bar of the other kernels, 1e-5 in the infinity-norm relative
error (the three-pass product keeps every term to about 2^-21 of its size)."""

import numpy as np
import pytest
import torch

import oracle
from mlip_message_passing_b200 import workloads as W
from tests.conftest import rel_err

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def e3b():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from mlip_message_passing_b200 import e3b
    return e3b


@pytest.fixture(autouse=True)
def no_device_error(e3b):
    # every bounded wait of the tensor-core kernel that gives up records E3_ERR_TIMEOUT
    yield
    e3b.device_status()


def t(a):
    return torch.as_tensor(np.ascontiguousarray(a)).to(DEV)


def h(x):
    return x.detach().cpu().numpy().astype(np.float64)


def fc_instructions(ir1, ir2, irout):
    """Every (i1, i2, i_out) allowed by the triangle and parity rules, in that loop order."""
    a, b, c = oracle.parse_irreps(ir1), oracle.parse_irreps(ir2), oracle.parse_irreps(irout)
    return [(i1, i2, io) for i1, x in enumerate(a) for i2, y in enumerate(b) for io, z in enumerate(c)
            if abs(x.l - y.l) <= z.l <= x.l + y.l and z.p == x.p * y.p]


def plans(e3b, ir1, ir2, irout):
    ins = fc_instructions(ir1, ir2, irout)
    return (e3b.Plan(ir1, ir2, irout, mode="uvw", shared_weights=True),
            oracle.make_plan(ir1, ir2, irout, instructions=ins, mode="uvw", shared_weights=True))


def inputs(p, B, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, p.dim_in1)).astype(np.float32)
    y = rng.standard_normal((B, p.dim_in2)).astype(np.float32)
    w = rng.standard_normal(p.weight_numel).astype(np.float32)
    return x, y, w


CASES = [
    ("32x0e+32x1o", "1x0e+1x1o", "32x0e+32x1o+32x1e+32x2e", 37),
    ("64x0e+64x1o+64x2e", "1x0e+1x1o+1x2e+1x3o", "32x0e+32x1o+32x2e+32x3o", 61),
    ("128x0e+128x1o+128x2e+128x3o", "1x0e+1x1o+1x2e+1x3o", "128x0e+128x1o+128x1e+128x2e+128x2o+128x3o+128x3e", 45),
    ("96x0e+96x1o", "1x0e+1x1o+1x2e", "64x1o+64x0e+64x2e", 130),
]


@pytest.mark.parametrize("ir1,ir2,irout,B", CASES)
def test_uvw_forward_backward(e3b, ir1, ir2, irout, B):
    p, q = plans(e3b, ir1, ir2, irout)
    assert p.weight_numel == q.weight_numel and p.dim_out == q.irreps_out.dim and p.n_paths == q.n_paths
    np.testing.assert_allclose(p.alphas, q.alphas, rtol=1e-15)
    x, y, w = inputs(p, B, seed=B)
    out = e3b.tp_forward(p, t(x), t(y), t(w))
    ref = oracle.tp_forward(q, x, y, w)
    assert rel_err(h(out), ref) <= 1e-5
    g = np.random.default_rng(B + 1).standard_normal(ref.shape).astype(np.float32)
    gx, gy, gw = e3b.tp_backward(p, t(x), t(y), t(w), t(g))
    rx, ry, rw = oracle.tp_backward(q, x, y, w, g)
    assert rel_err(h(gx), rx) <= 1e-5
    assert rel_err(h(gy), ry) <= 1e-5
    assert rel_err(h(gw), rw) <= 1e-5


def test_uvw_output_block_without_paths_is_zero(e3b):
    # 0e x (0e + 1o) reaches no 2e output: that block of the output is zero
    ir1, ir2, irout = "32x0e", "1x0e+1x1o", "32x0e+32x2e+32x1o"
    p, q = plans(e3b, ir1, ir2, irout)
    x, y, w = inputs(p, 50, seed=3)
    out = torch.full((50, p.dim_out), float("nan"), device=DEV)
    e3b.tp_forward(p, t(x), t(y), t(w), out=out)
    assert rel_err(h(out), oracle.tp_forward(q, x, y, w)) <= 1e-5
    assert float(out[:, 32:32 + 160].abs().max()) == 0.0


def test_uvw_ragged_batches(e3b):
    ir1, ir2, irout = "32x0e+32x1o+32x2e", "1x0e+1x1o+1x2e", "32x0e+32x1o+32x2e"
    p, q = plans(e3b, ir1, ir2, irout)
    for B in (1, 5, 25, 26, 127, 129):
        x, y, w = inputs(p, B, seed=B)
        assert rel_err(h(e3b.tp_forward(p, t(x), t(y), t(w))), oracle.tp_forward(q, x, y, w)) <= 1e-5
        g = np.random.default_rng(B).standard_normal((B, p.dim_out)).astype(np.float32)
        res = e3b.tp_backward(p, t(x), t(y), t(w), t(g))
        for got, want in zip(res, oracle.tp_backward(q, x, y, w, g)):
            assert rel_err(h(got), want) <= 1e-5


def test_uvw_full_size_sampled(e3b):
    """The fully connected workload at full size (65536 samples, 128 channels in and out, degrees
    0..3) in the launch the benchmark times; sampled rows against the oracle, and grad_w against
    the oracle on a sub-batch (it sums over every sample)."""
    cfg = W.CONFIGS["tp_uvw"]
    ir1, ir2, irout = W.irreps_str(cfg["mul"], cfg["lx"]), W.sh_irreps(cfg["ly"]), cfg["irreps_out"]
    p, q = plans(e3b, ir1, ir2, irout)
    d = W.uvw_inputs(cfg["B"], p.dim_in1, p.dim_in2, p.weight_numel, cfg["seed"])
    x, y, w = t(d["x"]), t(d["y"]), t(d["w"])
    out = e3b.tp_forward(p, x, y, w)
    rows = np.random.default_rng(0).choice(cfg["B"], 48, replace=False)
    rows[-1] = cfg["B"] - 1
    ridx = torch.as_tensor(rows, device=DEV)
    assert rel_err(h(out[ridx]), oracle.tp_forward(q, d["x"][rows], d["y"][rows], d["w"])) <= 1e-5
    g = np.random.default_rng(1).standard_normal((cfg["B"], p.dim_out)).astype(np.float32)
    gx, gy, _ = e3b.tp_backward(p, x, y, w, t(g), need_w=False)
    rx, ry, _ = oracle.tp_backward(q, d["x"][rows], d["y"][rows], d["w"], g[rows])
    assert rel_err(h(gx[ridx]), rx) <= 1e-5
    assert rel_err(h(gy[ridx]), ry) <= 1e-5
    sub = 512
    _, _, gw = e3b.tp_backward(p, x[:sub], y[:sub], w, t(g[:sub]), need_x=False, need_y=False)
    _, _, rw = oracle.tp_backward(q, d["x"][:sub], d["y"][:sub], d["w"], g[:sub])
    assert rel_err(h(gw), rw) <= 1e-5


def test_uvw_unsupported(e3b):
    with pytest.raises(e3b.E3Error, match="UNSUPPORTED"):
        e3b.Plan("32x0e+32x1o", "1x0e+1x1o", "32x0e+32x1o", mode="uvw")  # per-sample weights
    with pytest.raises(e3b.E3Error, match="UNSUPPORTED"):
        e3b.Plan("16x0e+16x1o", "1x0e+1x1o", "32x0e+32x1o", mode="uvw", shared_weights=True)
    with pytest.raises(e3b.E3Error, match="UNSUPPORTED"):
        e3b.Plan("32x0e+32x1o", "1x0e+1x1o", "32x0e+32x1o", mode="uvw", shared_weights=True, dtype=torch.float64)
    p = e3b.Plan("32x0e+32x1o", "1x0e+1x1o", "32x0e+32x1o", mode="uvw", shared_weights=True)
    with pytest.raises(e3b.E3Error, match="UNSUPPORTED"):
        e3b.conv_workspace(p, 10, 20, DEV)


def test_uvw_explicit_instructions_and_path_weight(e3b):
    """An explicit instruction list (a subset of the fully connected one, out of loop order, one
    path weight given) goes through the library's explicit path: same plan as the oracle's."""
    ir1, ir2, irout = "32x0e+32x1o+32x2e", "1x0e+1x1o+1x2e", "64x1o+64x0e+64x2e"
    ins = [(2, 1, 0), (0, 0, 1), (1, 1, 1, 0.7), (1, 0, 0), (2, 2, 2), (0, 2, 2)]
    p = e3b.Plan(ir1, ir2, irout, instructions=ins, mode="uvw", shared_weights=True)
    q = oracle.make_plan(ir1, ir2, irout, instructions=[oracle.Instruction(*i[:3], True, i[3] if len(i) > 3 else -1.0)
                                                         for i in ins], mode="uvw", shared_weights=True)
    assert p.n_paths == q.n_paths == len(ins) and p.weight_numel == q.weight_numel
    np.testing.assert_allclose(p.alphas, q.alphas, rtol=1e-15)
    x, y, w = inputs(p, 77, seed=4)
    assert rel_err(h(e3b.tp_forward(p, t(x), t(y), t(w))), oracle.tp_forward(q, x, y, w)) <= 1e-5
    g = np.random.default_rng(5).standard_normal((77, p.dim_out)).astype(np.float32)
    for got, want in zip(e3b.tp_backward(p, t(x), t(y), t(w), t(g)), oracle.tp_backward(q, x, y, w, g)):
        assert rel_err(h(got), want) <= 1e-5


def test_uvw_as_a_per_irrep_linear(e3b):
    """The channel-mixing linear of a layer (per irrep, out_l = x_l W_l / sqrt(C)) is the fully
    connected product with y = 1x0e of ones: checked against plain float64 matrix products, at the
    shapes of the large graph's node features (128 -> 128 channels, degrees 0..3)."""
    ir = W.irreps_str(128, 3)
    p = e3b.Plan(ir, "1x0e", ir, mode="uvw", shared_weights=True)
    assert p.n_paths == 4
    rng = np.random.default_rng(15)
    B = 3000
    x = rng.standard_normal((B, p.dim_in1)).astype(np.float32)
    Wl = [rng.standard_normal((128, 128)).astype(np.float32) for _ in range(4)]
    w = np.concatenate([m.ravel() for m in Wl])
    out = h(e3b.tp_forward(p, t(x), t(np.ones((B, 1), np.float32)), t(w)))
    want, o = [], 0
    for l in range(4):
        d = 2 * l + 1
        xl = x[:, o:o + 128 * d].reshape(B, 128, d).astype(np.float64)
        want.append((np.einsum("uw,bum->bwm", Wl[l].astype(np.float64), xl) / np.sqrt(128.0)).reshape(B, -1))
        o += 128 * d
    assert rel_err(out, np.concatenate(want, axis=1)) <= 1e-5
