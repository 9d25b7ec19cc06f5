"""Parity of the CUDA path (through the C ABI) with the float64 oracle on the same seeded
inputs.  fp32 results must match to an infinity-norm relative error <= 1e-5, fp64 results to
<= 1e-12; CSR index arrays must match bit for bit."""

import math

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


def oplan(mul, lx, ly, lo):
    return oracle.make_plan(W.irreps_str(mul, lx), W.sh_irreps(ly), lmax_out=lo)


def gplan(e3b, mul, lx, ly, lo, dtype):
    return e3b.Plan(W.irreps_str(mul, lx), W.sh_irreps(ly), lmax_out=lo, dtype=dtype)


def t(a, dtype=None):
    x = torch.as_tensor(np.ascontiguousarray(a))
    if dtype is not None:
        x = x.to(dtype)
    return x.to(DEV)


def h(x):
    return x.detach().cpu().numpy().astype(np.float64)


# ------------------------------------------------------------------------- plans ---
def test_plan_matches_oracle_enumeration(e3b):
    for mul, lx, ly, lo in [(8, 1, 2, 2), (64, 2, 3, 2), (128, 3, 3, 3), (4, 1, 1, 2)]:
        p, q = gplan(e3b, mul, lx, ly, lo, torch.float32), oplan(mul, lx, ly, lo)
        assert p.irreps_out.replace(" ", "") == str(q.irreps_out).replace(" ", "")
        assert p.weight_numel == q.weight_numel and p.dim_out == q.irreps_out.dim
        np.testing.assert_allclose(p.alphas, q.alphas, rtol=1e-15)


# --------------------------------------------------------------------- harmonics ---
@pytest.mark.parametrize("dtype", [torch.float32, torch.float64])
@pytest.mark.parametrize("norm", ["component", "integral", "norm"])
def test_spherical_harmonics(e3b, dtype, norm):
    rng = np.random.default_rng(0)
    v = rng.standard_normal((5000, 3)).astype(NP[dtype])
    v[7] = 0.0
    got = h(e3b.spherical_harmonics(3, t(v), sh_norm=norm))
    ref = oracle.real_sh_all(3, v.astype(np.float64))
    if norm == "integral":
        ref = ref / math.sqrt(4 * math.pi)
    elif norm == "norm":
        ref = ref / np.sqrt(np.concatenate([[2 * l + 1] * (2 * l + 1) for l in range(4)]))
    assert rel_err(got, ref) < (2e-6 if dtype == torch.float32 else 1e-14)


@pytest.mark.parametrize("dtype", [torch.float32, torch.float64])
@pytest.mark.parametrize("norm", ["component", "integral", "norm"])
@pytest.mark.parametrize("lmax", [0, 1, 2, 3])
def test_spherical_harmonics_backward(e3b, dtype, norm, lmax):
    """grad_vec = sum_m grad_y[m] dY_m/dvec against the oracle's analytic Jacobian."""
    rng = np.random.default_rng(6 + lmax)
    n, ny = 3000, (lmax + 1) ** 2
    v = (rng.standard_normal((n, 3)) * rng.uniform(0.3, 4.0, (n, 1))).astype(NP[dtype])
    v[5] = 0.0
    gy = rng.standard_normal((n, ny)).astype(NP[dtype])
    got = h(e3b.spherical_harmonics_backward(lmax, t(v), t(gy), sh_norm=norm))
    deg = np.concatenate([[l] * (2 * l + 1) for l in range(lmax + 1)])
    if norm == "integral":
        scale = np.full(ny, 1 / math.sqrt(4 * math.pi))
    elif norm == "norm":
        scale = 1 / np.sqrt(2 * deg + 1)
    else:
        scale = np.ones(ny)
    ref = oracle.sh_backward(lmax, v.astype(np.float64), gy.astype(np.float64) * scale)
    assert np.all(got[5] == 0)
    if lmax == 0:
        assert np.all(got == 0)
    else:
        assert rel_err(got, ref) <= TOL[dtype]
        # the gradient is orthogonal to the vector (harmonics depend on the direction only)
        assert np.max(np.abs(np.sum(got * v, axis=1))) <= (1e-4 if dtype == torch.float32 else 1e-11)


# ------------------------------------------------------------- tensor product ---
@pytest.mark.parametrize("dtype", [torch.float32, torch.float64])
def test_tp_small_forward_backward(e3b, dtype):
    cfg = W.CONFIGS["tp_small"]
    mul, lx, ly, lo = cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"]
    d = W.tp_inputs(cfg["B"], mul, lx, ly, lo, cfg["seed"], cfg["vectors"], dtype=NP[dtype])
    y = oracle.real_sh_all(ly, d["vec"]).astype(NP[dtype])
    p, q = gplan(e3b, mul, lx, ly, lo, dtype), oplan(mul, lx, ly, lo)
    out = e3b.tp_forward(p, t(d["x"]), t(y), t(d["w"]))
    ref = oracle.tp_forward(q, d["x"], y, d["w"])
    assert rel_err(h(out), ref) <= TOL[dtype]
    g = np.random.default_rng(9).standard_normal(ref.shape).astype(NP[dtype])
    gx, gy, gw = e3b.tp_backward(p, t(d["x"]), t(y), t(d["w"]), t(g))
    rx, ry, rw = oracle.tp_backward(q, d["x"], y, d["w"], g)
    assert rel_err(h(gx), rx) <= TOL[dtype]
    assert rel_err(h(gy), ry) <= TOL[dtype]
    assert rel_err(h(gw), rw) <= TOL[dtype]


@pytest.mark.parametrize("B", [1, 2, 17, 33])
def test_tp_ragged_batches(e3b, B):
    # batches that leave part of a warp's sample slices idle
    d = W.tp_inputs(B, 8, 1, 2, 2, 3, dtype=np.float32)
    y = oracle.real_sh_all(2, d["vec"]).astype(np.float32)
    p, q = gplan(e3b, 8, 1, 2, 2, torch.float32), oplan(8, 1, 2, 2)
    assert rel_err(h(e3b.tp_forward(p, t(d["x"]), t(y), t(d["w"]))), oracle.tp_forward(q, d["x"], y, d["w"])) <= 1e-5
    g = np.random.default_rng(B).standard_normal((B, q.irreps_out.dim)).astype(np.float32)
    res = e3b.tp_backward(p, t(d["x"]), t(y), t(d["w"]), t(g))
    for a, b in zip(res, oracle.tp_backward(q, d["x"], y, d["w"], g)):
        assert rel_err(h(a), b) <= 1e-5


def test_tp_shared_weights(e3b):
    d = W.tp_inputs(300, 8, 1, 2, 2, 4, dtype=np.float32)
    y = oracle.real_sh_all(2, d["vec"]).astype(np.float32)
    p = e3b.Plan(W.irreps_str(8, 1), W.sh_irreps(2), lmax_out=2, shared_weights=True)
    q = oracle.make_plan(W.irreps_str(8, 1), W.sh_irreps(2), lmax_out=2, shared_weights=True)
    w = d["w"][0]
    assert rel_err(h(e3b.tp_forward(p, t(d["x"]), t(y), t(w))), oracle.tp_forward(q, d["x"], y, w)) <= 1e-5


def test_tp_batched_full_size_sampled(e3b):
    cfg = W.CONFIGS["tp_batched"]
    mul, lx, ly, lo = cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"]
    d = W.tp_inputs(cfg["B"], mul, lx, ly, lo, cfg["seed"], cfg["vectors"])
    vec = t(d["vec"], torch.float32)
    p, q = gplan(e3b, mul, lx, ly, lo, torch.float32), oplan(mul, lx, ly, lo)
    y = e3b.spherical_harmonics(ly, vec)  # the library's own harmonics feed the product
    x, w = t(d["x"]), t(d["w"])
    out = e3b.tp_forward(p, x, y, w)
    rows = np.unique(np.concatenate([[0, cfg["B"] - 1], np.random.default_rng(0).integers(0, cfg["B"], 1500)]))
    yh = h(y)[rows]
    ref = oracle.tp_forward(q, d["x"][rows], yh, d["w"][rows])
    assert rel_err(h(out[torch.as_tensor(rows, device=DEV)]), ref) <= 1e-5
    g = torch.randn_like(out)
    gx, gy, gw = e3b.tp_backward(p, x, y, w, g)
    ri = torch.as_tensor(rows, device=DEV)
    rx, ry, rw = oracle.tp_backward(q, d["x"][rows], yh, d["w"][rows], h(g[ri]))
    assert rel_err(h(gx[ri]), rx) <= 1e-5
    assert rel_err(h(gy[ri]), ry) <= 1e-5
    assert rel_err(h(gw[ri]), rw) <= 1e-5


# --------------------------------------------------------------------------- CSR ---
def _csr_case(e3b, n, src, dst):
    ref = oracle.csr_build(n, src, dst)
    got = e3b.csr_build(n, t(src), t(dst))
    for a, b in zip(got, ref):
        assert a.dtype == torch.int32
        assert np.array_equal(a.cpu().numpy(), b)


def test_csr_bit_exact(e3b):
    g = W.graph_inputs(3000, 4, 0, 0, 0, seed=2)
    _csr_case(e3b, 3000, g["src"], g["dst"])
    rng = np.random.default_rng(1)
    for n, e in [(1, 0), (1, 5), (7, 1), (300, 5000), (70000, 9000), (5, 4099)]:
        src = rng.integers(0, n, e).astype(np.int32)
        dst = rng.integers(0, n, e).astype(np.int32)
        _csr_case(e3b, n, src, dst)
    # a hub receiver with many duplicates (ties must keep input order)
    dst = np.zeros(20000, dtype=np.int32)
    dst[::3] = 5
    src = rng.integers(0, 9, 20000).astype(np.int32)
    _csr_case(e3b, 9, src, dst)


def test_csr_out_of_range_is_reported(e3b):
    src = np.array([0, 1, 2, 7], dtype=np.int32)
    dst = np.array([1, 2, 0, 1], dtype=np.int32)
    e3b.csr_build(3, t(src), t(dst))
    with pytest.raises(e3b.E3Error) as ei:
        e3b.device_status()
    assert ei.value.status == e3b.E3_ERR_INDEX
    e3b.device_status()  # cleared


# ------------------------------------------------------------------- convolution ---
def conv_setup(e3b, n_nodes, mul, lx, ly, lo, seed, dtype, weights="host"):
    g = W.graph_inputs(n_nodes, mul, lx, ly, lo, seed, dtype=NP[dtype], weights=weights, device=DEV)
    graph = e3b.Graph(n_nodes, t(g["src"]), t(g["dst"]))
    w_dev = g["w"] if weights == "torch" else t(g["w"])
    return g, graph, w_dev


@pytest.mark.parametrize("dtype", [torch.float32, torch.float64])
@pytest.mark.parametrize("mode", ["y", "vec"])
def test_conv_forward_backward_full(e3b, dtype, mode):
    # a small water box: several CTAs per SM, ragged degrees (about 52 +- 7)
    n, mul, lx, ly, lo = 400, 64, 2, 3, 2
    g, graph, w = conv_setup(e3b, n, mul, lx, ly, lo, 21, dtype)
    p, q = gplan(e3b, mul, lx, ly, lo, dtype), oplan(mul, lx, ly, lo)
    Y = oracle.real_sh_all(ly, g["vec"].astype(np.float64)).astype(NP[dtype])
    s = 1 / math.sqrt(52)
    wr = graph.to_receiver_order(w)
    kw = dict(y=graph.to_receiver_order(t(Y))) if mode == "y" else dict(edge_vec=graph.to_receiver_order(t(g["vec"])))
    out = e3b.conv_forward(p, graph, t(g["x"]), wr, out_scale=s, **kw)
    ref = oracle.conv_forward(q, n, g["src"], g["dst"], g["x"], Y, g["w"], s)
    assert rel_err(h(out), ref) <= TOL[dtype]
    go = W.grad_out(n, q.irreps_out.dim, 5, dtype=NP[dtype])
    gx, gy, gw = e3b.conv_backward(p, graph, t(g["x"]), wr, t(go), out_scale=s, **kw)
    rx, ry, rw = oracle.conv_backward(q, n, g["src"], g["dst"], g["x"], Y, g["w"], go, s)
    perm = graph.perm_dst.cpu().numpy()
    assert rel_err(h(gx), rx) <= TOL[dtype]
    assert rel_err(h(gy), ry[perm]) <= TOL[dtype]
    assert rel_err(h(gw), rw[perm]) <= TOL[dtype]


@pytest.mark.parametrize("mul", [64, 128])
def test_conv_backward_gradient_subsets(e3b, mul):
    """Multiplicities 64 and 128 run a separately compiled backward when grad_w and grad_y are
    both requested; every other subset runs the general one.  Each subset against the oracle."""
    n, lx, ly, lo = 400, 2, 3, 2
    g, graph, w = conv_setup(e3b, n, mul, lx, ly, lo, 23, torch.float32)
    p, q = gplan(e3b, mul, lx, ly, lo, torch.float32), oplan(mul, lx, ly, lo)
    Y = oracle.real_sh_all(ly, g["vec"].astype(np.float64))
    vec = graph.to_receiver_order(t(g["vec"]))
    wr = graph.to_receiver_order(w)
    go = W.grad_out(n, q.irreps_out.dim, 9)
    s = 1 / math.sqrt(52)
    rx, ry, rw = oracle.conv_backward(q, n, g["src"], g["dst"], g["x"], Y, g["w"], go, s)
    perm = graph.perm_dst.cpu().numpy()
    ref = (rx, ry[perm], rw[perm])
    for need in [(1, 1, 1), (1, 0, 0), (0, 1, 0), (0, 0, 1), (1, 0, 1), (1, 1, 0), (0, 1, 1)]:
        res = e3b.conv_backward(p, graph, t(g["x"]), wr, t(go), edge_vec=vec, out_scale=s,
                                need_x=bool(need[0]), need_y=bool(need[1]), need_w=bool(need[2]))
        for i in range(3):
            if need[i]:
                assert rel_err(h(res[i]), ref[i]) <= 1e-5, (need, i)
            else:
                assert res[i] is None, (need, i)


def test_conv_small_multiplicity_and_degrees(e3b):
    # C = 8 (16 edge slices per warp) on the (1, 2, 2) path set and C = 4 on (1, 1, 2)
    for mul, lx, ly, lo in [(8, 1, 2, 2), (4, 1, 1, 2), (32, 2, 3, 2)]:
        n = 400
        g = W.graph_inputs(n, mul, lx, ly, lo, 8, dtype=np.float32)
        graph = e3b.Graph(n, t(g["src"]), t(g["dst"]))
        p, q = gplan(e3b, mul, lx, ly, lo, torch.float32), oplan(mul, lx, ly, lo)
        vec = graph.to_receiver_order(t(g["vec"]))
        wr = graph.to_receiver_order(t(g["w"]))
        Y = oracle.real_sh_all(ly, g["vec"].astype(np.float64))
        out = e3b.conv_forward(p, graph, t(g["x"]), wr, edge_vec=vec, out_scale=0.2)
        assert rel_err(h(out), oracle.conv_forward(q, n, g["src"], g["dst"], g["x"], Y, g["w"], 0.2)) <= 1e-5
        go = W.grad_out(n, q.irreps_out.dim, 6)
        res = e3b.conv_backward(p, graph, t(g["x"]), wr, t(go), edge_vec=vec, out_scale=0.2)
        ref = oracle.conv_backward(q, n, g["src"], g["dst"], g["x"], Y, g["w"], go, 0.2)
        perm = graph.perm_dst.cpu().numpy()
        assert rel_err(h(res[0]), ref[0]) <= 1e-5
        assert rel_err(h(res[1]), ref[1][perm]) <= 1e-5
        assert rel_err(h(res[2]), ref[2][perm]) <= 1e-5


@pytest.mark.parametrize("dtype", [torch.float32, torch.float64])
def test_conv_l3_mul128_sampled(e3b, dtype):
    """The l <= 3 path set (34 paths) at multiplicity 128 -- the large-convolution kernels -- on a
    400-node box: forward on 40 sampled receivers (all their in-edges), backward on 40 sampled
    senders (all their out-edges: their grad_x and those edges' grad_y, grad_w are exact)."""
    n, mul, lx, ly, lo = 400, 128, 3, 3, 3
    g, graph, w = conv_setup(e3b, n, mul, lx, ly, lo, 31, dtype)
    p, q = gplan(e3b, mul, lx, ly, lo, dtype), oplan(mul, lx, ly, lo)
    s = 1 / math.sqrt(52)
    vec, wr = graph.to_receiver_order(t(g["vec"])), graph.to_receiver_order(w)
    out = e3b.conv_forward(p, graph, t(g["x"]), wr, edge_vec=vec, out_scale=s)
    go = W.grad_out(n, q.irreps_out.dim, 7, dtype=NP[dtype])
    gx, gy, gw = e3b.conv_backward(p, graph, t(g["x"]), wr, t(go), edge_vec=vec, out_scale=s)
    rng = np.random.default_rng(12)
    recv = np.sort(rng.choice(n, 40, replace=False))
    sel = np.flatnonzero(np.isin(g["dst"], recv))
    Y = oracle.real_sh_all(ly, g["vec"][sel].astype(np.float64))
    ref = oracle.conv_forward(q, n, g["src"][sel], g["dst"][sel], g["x"], Y, g["w"][sel], s)
    assert rel_err(h(out)[recv], ref[recv]) <= TOL[dtype]
    send = np.sort(rng.choice(n, 40, replace=False))
    sel = np.flatnonzero(np.isin(g["src"], send))
    Y = oracle.real_sh_all(ly, g["vec"][sel].astype(np.float64))
    rx, ry, rw = oracle.conv_backward(q, n, g["src"][sel], g["dst"][sel], g["x"], Y, g["w"][sel], go, s)
    pos = np.argsort(graph.perm_dst.cpu().numpy())  # original edge id -> receiver-order position
    assert rel_err(h(gx)[send], rx[send]) <= TOL[dtype]
    assert rel_err(h(gy)[pos[sel]], ry) <= TOL[dtype]
    assert rel_err(h(gw)[pos[sel]], rw) <= TOL[dtype]


@pytest.mark.parametrize("dtype", [torch.float32, torch.float64])
def test_morton_order_bit_exact(e3b, dtype):
    """Morton order of positions against the oracle, bit for bit: several sort tiles and a ragged
    tail, points outside the box (clamped), duplicated positions (ties keep ascending ids)."""
    rng = np.random.default_rng(70)
    pos = rng.uniform(-1.0, 11.0, (5003, 3)).astype(NP[dtype])
    pos[100:140] = pos[7]
    lo, ext = (0.0, 0.5, -0.25), (10.0, 9.0, 10.5)
    perm = e3b.morton_order(t(pos), lo, ext)
    ref = oracle.morton_order(pos.astype(np.float64), lo, ext)
    assert np.array_equal(perm.cpu().numpy(), ref)
    inv = e3b.invert_permutation(perm)
    assert np.array_equal(inv.cpu().numpy(), oracle.invert_permutation(ref))
    ids = t(rng.integers(0, 5003, 777).astype(np.int32))
    assert np.array_equal(e3b.remap_ids(ids, inv).cpu().numpy(), oracle.invert_permutation(ref)[ids.cpu().numpy()])
    e3b.device_status()
    ids[5] = 5003  # out of range: reported, not dereferenced
    e3b.remap_ids(ids, inv)
    with pytest.raises(e3b.E3Error):
        e3b.device_status()


def test_conv_on_morton_renumbered_graph(e3b):
    """Renumbering nodes along the Morton curve changes no result: the forward is bitwise the
    permuted original (each receiver keeps its in-edge order); the backward agrees to rounding."""
    n, mul, lx, ly, lo = 400, 64, 2, 3, 2
    g, graph, w = conv_setup(e3b, n, mul, lx, ly, lo, 21, torch.float32)
    p = gplan(e3b, mul, lx, ly, lo, torch.float32)
    x, vec_e, src, dst = t(g["x"]), t(g["vec"]), t(g["src"]), t(g["dst"])
    go = t(W.grad_out(n, p.dim_out, 5))
    out0 = e3b.conv_forward(p, graph, x, graph.to_receiver_order(w), edge_vec=graph.to_receiver_order(vec_e),
                            out_scale=0.2)
    b0 = e3b.conv_backward(p, graph, x, graph.to_receiver_order(w), go, edge_vec=graph.to_receiver_order(vec_e),
                           out_scale=0.2)
    perm, inv, src2, dst2 = e3b.reorder_graph(t(g["pos"]), (0, 0, 0), (g["side"],) * 3, src, dst)
    g2 = e3b.Graph(n, src2, dst2)
    x2, go2 = e3b.gather_rows(perm, x), e3b.gather_rows(perm, go)
    out2 = e3b.conv_forward(p, g2, x2, g2.to_receiver_order(w), edge_vec=g2.to_receiver_order(vec_e), out_scale=0.2)
    assert torch.equal(e3b.gather_rows(inv, out2), out0)
    gx2, gy2, gw2 = e3b.conv_backward(p, g2, x2, g2.to_receiver_order(w), go2, edge_vec=g2.to_receiver_order(vec_e),
                                      out_scale=0.2)
    assert rel_err(h(e3b.gather_rows(inv, gx2)), h(b0[0])) <= 1e-5
    # per-edge gradients: map both back to the original edge order
    o0, o2 = np.argsort(graph.perm_dst.cpu().numpy()), np.argsort(g2.perm_dst.cpu().numpy())
    assert rel_err(h(gy2)[o2], h(b0[1])[o0]) <= 1e-5
    assert rel_err(h(gw2)[o2], h(b0[2])[o0]) <= 1e-5


def test_csr_with_padding_bit_exact(e3b):
    """Padding edges (-1 as sender, receiver or both) after the valid ones in both orders."""
    rng = np.random.default_rng(80)
    n, E = 500, 20000
    src = rng.integers(0, n, E).astype(np.int32)
    dst = rng.integers(0, n, E).astype(np.int32)
    pad = rng.choice(E, 4000, replace=False)
    src[pad[:1500]] = -1
    dst[pad[1500:3000]] = -1
    src[pad[3000:]] = -1
    dst[pad[3000:]] = -1
    got = [a.cpu().numpy() for a in e3b.csr_build(n, t(src), t(dst))]
    e3b.device_status()  # padding is not an error
    for a, b in zip(got, oracle.csr_build(n, src, dst)):
        assert np.array_equal(a, b)


def test_conv_with_padding_edges(e3b):
    """A padded water box gives the unpadded results bit for bit; padding edges get zero
    gradients and no kernel walks them."""
    n, mul, lx, ly, lo = 400, 64, 2, 3, 2
    g, graph, w = conv_setup(e3b, n, mul, lx, ly, lo, 21, torch.float32)
    p = gplan(e3b, mul, lx, ly, lo, torch.float32)
    rng = np.random.default_rng(81)
    E = len(g["src"])
    k = E // 4
    src_p = np.concatenate([g["src"], rng.integers(-1, n, k).astype(np.int32)])
    dst_p = np.concatenate([g["dst"], np.full(k, -1, np.int32)])
    vec_p = np.concatenate([g["vec"], rng.standard_normal((k, 3)).astype(np.float32)])
    w_p = torch.cat([w, torch.randn(k, p.weight_numel, device=DEV)])
    gp = e3b.Graph(n, t(src_p), t(dst_p))
    x, go = t(g["x"]), t(W.grad_out(n, p.dim_out, 5))
    args = dict(out_scale=0.2)
    out0 = e3b.conv_forward(p, graph, x, graph.to_receiver_order(w), edge_vec=graph.to_receiver_order(t(g["vec"])),
                            **args)
    out1 = e3b.conv_forward(p, gp, x, gp.to_receiver_order(w_p), edge_vec=gp.to_receiver_order(t(vec_p)), **args)
    assert torch.equal(out0, out1)
    b0 = e3b.conv_backward(p, graph, x, graph.to_receiver_order(w), go, edge_vec=graph.to_receiver_order(t(g["vec"])),
                           **args)
    b1 = e3b.conv_backward(p, gp, x, gp.to_receiver_order(w_p), go, edge_vec=gp.to_receiver_order(t(vec_p)), **args)
    assert torch.equal(b0[0], b1[0])
    assert torch.equal(b0[1], b1[1][:E]) and torch.equal(b0[2], b1[2][:E])
    assert torch.all(b1[1][E:] == 0) and torch.all(b1[2][E:] == 0)
    e3b.device_status()


@pytest.mark.parametrize("dtype", [torch.float32, torch.float64])
def test_conv_hubs_split_into_segments(e3b, dtype):
    """A receiver with 5000 in-edges and a sender with 5000 out-edges (20 row segments each, added
    in order by separate CTAs) beside ordinary nodes: forward and backward against the oracle,
    bitwise equal on a second run."""
    rng = np.random.default_rng(90)
    n, mul, lx, ly, lo = 300, 32, 2, 3, 2
    src = np.concatenate([rng.integers(0, n, 6000), rng.integers(0, n, 5000), np.full(5000, 11)]).astype(np.int32)
    dst = np.concatenate([rng.integers(0, n, 6000), np.full(5000, 7), rng.integers(0, n, 5000)]).astype(np.int32)
    E = len(src)
    p, q = gplan(e3b, mul, lx, ly, lo, dtype), oplan(mul, lx, ly, lo)
    vec = rng.standard_normal((E, 3))
    x = rng.standard_normal((n, p.dim_in1))
    w = rng.standard_normal((E, p.weight_numel)) / 8
    go = rng.standard_normal((n, p.dim_out))
    graph = e3b.Graph(n, t(src), t(dst))
    args = (t(x, dtype), graph.to_receiver_order(t(w, dtype)))
    kw = dict(edge_vec=graph.to_receiver_order(t(vec, dtype)), out_scale=0.3)
    out = e3b.conv_forward(p, graph, *args, **kw)
    gx, gy, gw = e3b.conv_backward(p, graph, *args, t(go, dtype), **kw)
    Y = oracle.real_sh_all(ly, vec)
    ref = oracle.conv_forward(q, n, src, dst, x, Y, w, 0.3)
    rx, ry, rw = oracle.conv_backward(q, n, src, dst, x, Y, w, go, 0.3)
    perm = graph.perm_dst.cpu().numpy()
    assert rel_err(h(out), ref) <= TOL[dtype]
    assert rel_err(h(gx), rx) <= TOL[dtype]
    assert rel_err(h(gy), ry[perm]) <= TOL[dtype]
    assert rel_err(h(gw), rw[perm]) <= TOL[dtype]
    out2 = e3b.conv_forward(p, graph, *args, **kw)
    gx2, gy2, gw2 = e3b.conv_backward(p, graph, *args, t(go, dtype), **kw)
    assert torch.equal(out, out2) and torch.equal(gx, gx2) and torch.equal(gy, gy2) and torch.equal(gw, gw2)
    e3b.device_status()


def test_conv_forward_multiplicity_256(e3b):
    """C = 256: two warps per forward CTA (64 lanes of 4 channels) on a small box; the backward
    reports the multiplicity as unsupported."""
    n, mul, lx, ly, lo = 400, 256, 1, 2, 2
    g = W.graph_inputs(n, mul, lx, ly, lo, 14, dtype=np.float32)
    graph = e3b.Graph(n, t(g["src"]), t(g["dst"]))
    p, q = gplan(e3b, mul, lx, ly, lo, torch.float32), oplan(mul, lx, ly, lo)
    vec, wr = graph.to_receiver_order(t(g["vec"])), graph.to_receiver_order(t(g["w"]))
    out = e3b.conv_forward(p, graph, t(g["x"]), wr, edge_vec=vec, out_scale=0.2)
    Y = oracle.real_sh_all(ly, g["vec"].astype(np.float64))
    assert rel_err(h(out), oracle.conv_forward(q, n, g["src"], g["dst"], g["x"], Y, g["w"], 0.2)) <= 1e-5
    with pytest.raises(e3b.E3Error) as ei:
        e3b.conv_backward(p, graph, t(g["x"]), wr, torch.zeros_like(out), edge_vec=vec, out_scale=0.2)
    assert ei.value.status == e3b.E3_ERR_UNSUPPORTED


def test_conv_edge_cases(e3b):
    p = gplan(e3b, 8, 1, 2, 2, torch.float32)
    q = oplan(8, 1, 2, 2)
    rng = np.random.default_rng(3)
    # no edges at all: zero rows, no kernel reads of edge arrays
    n = 5
    graph = e3b.Graph(n, t(np.zeros(0, np.int32)), t(np.zeros(0, np.int32)))
    x = t(rng.standard_normal((n, p.dim_in1)).astype(np.float32))
    out = e3b.conv_forward(p, graph, x, torch.zeros((0, p.weight_numel), device=DEV),
                           edge_vec=torch.zeros((0, 3), device=DEV))
    assert out.shape == (n, p.dim_out) and torch.all(out == 0)
    gx, gy, gw = e3b.conv_backward(p, graph, x, torch.zeros((0, p.weight_numel), device=DEV),
                                   torch.ones((n, p.dim_out), device=DEV), edge_vec=torch.zeros((0, 3), device=DEV))
    assert torch.all(gx == 0) and gy.shape[0] == 0 and gw.shape[0] == 0
    # isolated receivers and senders, a single edge, a hub receiver with 300 in-edges
    src = np.array([0, 2, 2, 3] + [1] * 300, dtype=np.int32)
    dst = np.array([1, 1, 3, 0] + [4] * 300, dtype=np.int32)
    n = 6  # node 5 is isolated
    vec = rng.standard_normal((len(src), 3)).astype(np.float32)
    w = rng.standard_normal((len(src), p.weight_numel)).astype(np.float32)
    x = rng.standard_normal((n, p.dim_in1)).astype(np.float32)
    graph = e3b.Graph(n, t(src), t(dst))
    out = e3b.conv_forward(p, graph, t(x), graph.to_receiver_order(t(w)), edge_vec=graph.to_receiver_order(t(vec)))
    Y = oracle.real_sh_all(2, vec.astype(np.float64))
    ref = oracle.conv_forward(q, n, src, dst, x, Y, w, 1.0)
    assert rel_err(h(out), ref) <= 1e-5 and torch.all(out[5] == 0) and torch.all(out[2] == 0)


def test_backward_workspace_is_checked(e3b):
    """The backward refuses a missing, misaligned or short workspace before any launch."""
    p = gplan(e3b, 8, 1, 2, 2, torch.float32)
    n = 4
    graph = e3b.Graph(n, t(np.array([0, 1, 2, 3], np.int32)), t(np.array([1, 2, 3, 0], np.int32)))
    x = torch.randn(n, p.dim_in1, device=DEV)
    w = torch.randn(4, p.weight_numel, device=DEV)
    go = torch.randn(n, p.dim_out, device=DEV)
    vec = torch.randn(4, 3, device=DEV)
    gx = torch.empty_like(x)
    ws = e3b.conv_workspace(p, n, 4, DEV)
    P = e3b._ptr

    def call(wsp, nbytes):
        return e3b.lib.e3_conv_backward(p.handle, n, 4, P(graph.row_ptr_dst), P(graph.src), P(graph.dst),
                                        P(graph.row_ptr_src), P(graph.perm_src), P(x), None, P(vec), 0, P(w),
                                        P(go), 1.0, P(gx), None, None, P(graph.topo), wsp, nbytes, e3b._stream())

    assert call(None, ws.numel()) == e3b.E3_ERR_INVALID_ARG
    assert call(P(ws[8:]), ws.numel() - 8) == e3b.E3_ERR_INVALID_ARG
    assert call(P(ws), 16) == e3b.E3_ERR_INVALID_ARG
    assert call(P(ws), ws.numel()) == e3b.E3_OK
    torch.cuda.synchronize()
    ref, _, _ = e3b.conv_backward(p, graph, x, w, go, edge_vec=vec, need_y=False, need_w=False)
    assert torch.equal(gx, ref)


def test_conv_bad_index_is_reported_not_dereferenced(e3b):
    p = gplan(e3b, 8, 1, 2, 2, torch.float32)
    n = 4
    src = np.array([0, 1, 2, 3], dtype=np.int32)
    dst = np.array([1, 2, 3, 0], dtype=np.int32)
    graph = e3b.Graph(n, t(src), t(dst))
    graph.src[2] = 1000  # corrupt one sender id after the CSR was built
    x = torch.randn(n, p.dim_in1, device=DEV)
    w = torch.randn(4, p.weight_numel, device=DEV)
    out = e3b.conv_forward(p, graph, x, w, edge_vec=torch.randn(4, 3, device=DEV))
    with pytest.raises(e3b.E3Error) as ei:
        e3b.device_status()
    assert ei.value.status == e3b.E3_ERR_INDEX
    assert torch.isfinite(out).all()
    e3b.device_status()


def test_errors_are_attributed_to_the_plan(e3b):
    """Two plans used one after the other on one stream: the index error raised by a call on the
    first plan is reported by that plan's status only; the second plan's status stays clean, and the
    device-wide status is clean once the plan's word has been read."""
    pa = gplan(e3b, 8, 1, 2, 2, torch.float32)
    pb = gplan(e3b, 8, 1, 2, 2, torch.float32)
    n = 4
    src = np.array([0, 1, 2, 3], dtype=np.int32)
    dst = np.array([1, 2, 3, 0], dtype=np.int32)
    bad = e3b.Graph(n, t(src), t(dst))
    bad.src[2] = 1000  # a sender id out of range, after the CSR was built
    good = e3b.Graph(n, t(src), t(dst))
    x = torch.randn(n, pa.dim_in1, device=DEV)
    w = torch.randn(4, pa.weight_numel, device=DEV)
    vec = torch.randn(4, 3, device=DEV)
    e3b.conv_forward(pa, bad, x, w, edge_vec=vec)
    e3b.conv_forward(pb, good, x, w, edge_vec=vec)
    pb.status()  # clean
    with pytest.raises(e3b.E3Error) as ei:
        pa.status()
    assert ei.value.status == e3b.E3_ERR_INDEX
    pa.status()  # read and cleared
    e3b.device_status()
    # the device-wide read also drains a plan's word
    e3b.conv_forward(pa, bad, x, w, edge_vec=vec)
    with pytest.raises(e3b.E3Error) as ei:
        e3b.device_status()
    assert ei.value.status == e3b.E3_ERR_INDEX
    pa.status()


def test_conv_deterministic(e3b):
    g, graph, w = conv_setup(e3b, 400, 64, 2, 3, 2, 22, torch.float32)
    p = gplan(e3b, 64, 2, 3, 2, torch.float32)
    vec, wr, x = graph.to_receiver_order(t(g["vec"])), graph.to_receiver_order(w), t(g["x"])
    a = e3b.conv_forward(p, graph, x, wr, edge_vec=vec, out_scale=0.1)
    b = e3b.conv_forward(p, graph, x, wr, edge_vec=vec, out_scale=0.1)
    assert torch.equal(a, b)
    go = torch.randn_like(a)
    r1 = e3b.conv_backward(p, graph, x, wr, go, edge_vec=vec, out_scale=0.1)
    r2 = e3b.conv_backward(p, graph, x, wr, go, edge_vec=vec, out_scale=0.1)
    for u, v in zip(r1, r2):
        assert torch.equal(u, v)


def test_conv_waterbox_full_size_sampled(e3b):
    """The benchmark's workload and launch configuration (3000 nodes, ~156k edges, 64 channels,
    harmonics from edge vectors), checked on sampled receivers, senders and edges."""
    cfg = W.CONFIGS["conv_waterbox"]
    n, mul, lx, ly, lo = cfg["N"], cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"]
    g, graph, w = conv_setup(e3b, n, mul, lx, ly, lo, cfg["seed"], torch.float32)
    p, q = gplan(e3b, mul, lx, ly, lo, torch.float32), oplan(mul, lx, ly, lo)
    s = 1 / math.sqrt(52)
    vec, wr, x = graph.to_receiver_order(t(g["vec"])), graph.to_receiver_order(w), t(g["x"])
    out = e3b.conv_forward(p, graph, x, wr, edge_vec=vec, out_scale=s)
    rng = np.random.default_rng(0)
    nodes = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, 150)]))
    sel = np.flatnonzero(np.isin(g["dst"], nodes))
    Y = oracle.real_sh_all(ly, g["vec"][sel].astype(np.float64))
    full = oracle.conv_forward(q, n, g["src"][sel], g["dst"][sel], g["x"], Y, g["w"][sel], s)
    assert rel_err(h(out)[nodes], full[nodes]) <= 1e-5
    # backward: grad_x of sampled senders (all their out-edges), grad_y / grad_w of sampled edges
    go = W.grad_out(n, q.irreps_out.dim, W.CONFIGS["conv_waterbox_bwd"]["grad_seed"])
    gx, gy, gw = e3b.conv_backward(p, graph, x, wr, t(go), edge_vec=vec, out_scale=s)
    senders = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, 80)]))
    sel = np.flatnonzero(np.isin(g["src"], senders))
    Y = oracle.real_sh_all(ly, g["vec"][sel].astype(np.float64))
    rx, ry, rw = oracle.conv_backward(q, n, g["src"][sel], g["dst"][sel], g["x"], Y, g["w"][sel], go, s)
    assert rel_err(h(gx)[senders], rx[senders]) <= 1e-5
    inv = np.empty_like(graph.perm_dst.cpu().numpy())
    inv[graph.perm_dst.cpu().numpy()] = np.arange(len(inv))
    pos = torch.as_tensor(inv[sel], device=DEV)
    assert rel_err(h(gy[pos]), ry) <= 1e-5
    assert rel_err(h(gw[pos]), rw) <= 1e-5


@pytest.mark.parametrize("dtype", [torch.float32, torch.float64])
def test_conv_large_sampled(e3b, dtype):
    """24000 nodes, ~1.26M edges, 128 channels, l <= 3, at full size in the benchmark's launch
    configuration: the forward on 256 sampled receivers (all their in-edges), the backward's grad_x
    on 40 sampled senders (all their out-edges) and grad_y / grad_w on those out-edges."""
    cfg = W.CONFIGS["conv_large"]
    n, mul, lx, ly, lo = cfg["N"], cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"]
    torch.cuda.empty_cache()
    g, graph, w = conv_setup(e3b, n, mul, lx, ly, lo, cfg["seed"], dtype, weights="torch")
    p, q = gplan(e3b, mul, lx, ly, lo, dtype), oplan(mul, lx, ly, lo)
    s = 1 / math.sqrt(52)
    vec, x = graph.to_receiver_order(t(g["vec"])), t(g["x"])
    wr = graph.to_receiver_order(w)
    del w  # rows the oracle needs are read from the receiver-ordered copy
    torch.cuda.empty_cache()
    perm = graph.perm_dst.cpu().numpy()
    inv = np.empty_like(perm)
    inv[perm] = np.arange(len(perm))

    def w_rows(sel):
        return h(wr[torch.as_tensor(inv[sel], device=DEV)])

    out = e3b.conv_forward(p, graph, x, wr, edge_vec=vec, out_scale=s)
    nodes = np.sort(np.random.default_rng(1).choice(n, 256, replace=False))
    sel = np.flatnonzero(np.isin(g["dst"], nodes))
    Y = oracle.real_sh_all(ly, g["vec"][sel].astype(np.float64))
    ref = oracle.conv_forward(q, n, g["src"][sel], g["dst"][sel], g["x"], Y, w_rows(sel), s)
    assert rel_err(h(out[torch.as_tensor(nodes, device=DEV)]), ref[nodes]) <= TOL[dtype]
    del out
    torch.cuda.empty_cache()
    go = W.grad_out(n, q.irreps_out.dim, 5, dtype=NP[dtype])
    gx, gy, gw = e3b.conv_backward(p, graph, x, wr, t(go), edge_vec=vec, out_scale=s)
    senders = np.sort(np.random.default_rng(2).choice(n, 40, replace=False))
    sel = np.flatnonzero(np.isin(g["src"], senders))
    Y = oracle.real_sh_all(ly, g["vec"][sel].astype(np.float64))
    rx, ry, rw = oracle.conv_backward(q, n, g["src"][sel], g["dst"][sel], g["x"], Y, w_rows(sel), go, s)
    assert rel_err(h(gx[torch.as_tensor(senders, device=DEV)]), rx[senders]) <= TOL[dtype]
    pos = torch.as_tensor(inv[sel], device=DEV)
    assert rel_err(h(gy[pos]), ry) <= TOL[dtype]
    assert rel_err(h(gw[pos]), rw) <= TOL[dtype]
    del wr, gx, gy, gw
    torch.cuda.empty_cache()


def test_conv_backward_finite_differences_subgraph(e3b):
    """fp64 on the 50 nodes nearest to node 0 of the water box (every edge among them):
    the kernel gradients equal central differences of the kernel forward and the oracle."""
    cfg = W.CONFIGS["conv_waterbox"]
    g = W.graph_inputs(cfg["N"], cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"], cfg["seed"], dtype=np.float64)
    nodes, eids, s_src, s_dst = W.subgraph_nearest(g["pos"], g["side"], g["src"], g["dst"], 0, 50)
    n = len(nodes)
    x = g["x"][nodes]
    w = g["w"][eids]
    vec = g["vec"][eids]
    p = gplan(e3b, 64, 2, 3, 2, torch.float64)
    q = oplan(64, 2, 3, 2)
    graph = e3b.Graph(n, t(s_src), t(s_dst))
    Y = oracle.real_sh_all(3, vec)
    Yr, wr = graph.to_receiver_order(t(Y)), graph.to_receiver_order(t(w))
    go = np.random.default_rng(4).standard_normal((n, p.dim_out))
    s = 1 / math.sqrt(52)
    gx, gy, gw = e3b.conv_backward(p, graph, t(x), wr, t(go), y=Yr, out_scale=s)
    rng = np.random.default_rng(5)
    hstep = 1e-4

    def L(xx, yy, ww):
        return float((t(go) * e3b.conv_forward(p, graph, xx, ww, y=yy, out_scale=s)).sum())

    for which, grad in ((0, gx), (1, gy), (2, gw)):
        base = [t(x), Yr, wr]
        d = torch.as_tensor(rng.standard_normal(tuple(base[which].shape)), device=DEV)
        plus, minus = list(base), list(base)
        plus[which] = base[which] + hstep * d
        minus[which] = base[which] - hstep * d
        fd = (L(*plus) - L(*minus)) / (2 * hstep)
        an = float((grad * d).sum())
        assert abs(fd - an) <= 1e-8 * max(1.0, abs(an))
    rx, ry, rw = oracle.conv_backward(q, n, s_src, s_dst, x, Y, w, go, s)
    perm = graph.perm_dst.cpu().numpy()
    assert rel_err(h(gx), rx) <= 1e-12
    assert rel_err(h(gy), ry[perm]) <= 1e-12
    assert rel_err(h(gw), rw[perm]) <= 1e-12


@pytest.mark.parametrize("dtype", [torch.float32, torch.float64])
def test_conv_vec_gradients(e3b, dtype):
    """Autograd of the convolution with in-kernel harmonics: gradients with respect to x, the
    edge vectors (through the harmonics: forces) and w against the oracle, and the edge-vector
    gradient against central differences of the kernel forward (float64)."""
    n, mul, lx, ly, lo = 400, 64, 2, 3, 2
    g, graph, w = conv_setup(e3b, n, mul, lx, ly, lo, 23, dtype)
    p, q = gplan(e3b, mul, lx, ly, lo, dtype), oplan(mul, lx, ly, lo)
    s = 1 / math.sqrt(52)
    vec = graph.to_receiver_order(t(g["vec"])).requires_grad_()
    x = t(g["x"]).requires_grad_()
    wr = graph.to_receiver_order(w).requires_grad_()
    out = e3b.conv_vec(p, graph, x, vec, wr, s)
    go = np.random.default_rng(8).standard_normal((n, p.dim_out)).astype(NP[dtype])
    out.backward(t(go))
    Y = oracle.real_sh_all(ly, g["vec"].astype(np.float64))
    rx, ry, rw = oracle.conv_backward(q, n, g["src"], g["dst"], g["x"], Y, g["w"], go, s)
    rvec = oracle.sh_backward(ly, g["vec"].astype(np.float64), ry)
    perm = graph.perm_dst.cpu().numpy()
    assert rel_err(h(x.grad), rx) <= TOL[dtype]
    assert rel_err(h(wr.grad), rw[perm]) <= TOL[dtype]
    assert rel_err(h(vec.grad), rvec[perm]) <= TOL[dtype]
    if dtype == torch.float64:
        d = torch.as_tensor(np.random.default_rng(9).standard_normal(tuple(vec.shape)), device=DEV)
        hs = 1e-6
        xd, wd, gt = x.detach(), wr.detach(), t(go)

        def L(vv):
            return float((gt * e3b.conv_forward(p, graph, xd, wd, edge_vec=vv, out_scale=s)).sum())

        fd = (L(vec.detach() + hs * d) - L(vec.detach() - hs * d)) / (2 * hs)
        an = float((vec.grad * d).sum())
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an))


def test_autograd_wrapper(e3b):
    g, graph, w = conv_setup(e3b, 400, 32, 2, 3, 2, 9, torch.float32)
    p = gplan(e3b, 32, 2, 3, 2, torch.float32)
    Y = graph.to_receiver_order(e3b.spherical_harmonics(3, t(g["vec"])))
    x = t(g["x"]).requires_grad_()
    y = Y.clone().requires_grad_()
    wr = graph.to_receiver_order(w).requires_grad_()
    out = e3b.conv(p, graph, x, y, wr, 0.3)
    go = torch.randn_like(out)
    out.backward(go)
    gx, gy, gw = e3b.conv_backward(p, graph, x.detach(), wr.detach(), go, y=Y, out_scale=0.3)
    assert torch.equal(x.grad, gx) and torch.equal(y.grad, gy) and torch.equal(wr.grad, gw)


@pytest.mark.parametrize("dtype", [torch.float32, torch.float64])
def test_processing_order_changes_nothing(e3b, dtype):
    """Rows processed in another order (a random permutation, and the Morton order of the
    positions) give bitwise the results of node-id order, also for hub rows cut into segments;
    an order entry out of range is reported, not dereferenced."""
    n, mul, lx, ly, lo = 400, 32, 2, 3, 2
    g = W.graph_inputs(n, mul, lx, ly, lo, 21, dtype=NP[dtype])
    rng = np.random.default_rng(22)
    hub = 600  # node 7 receives and sends 600 extra edges: three segments each way
    src = np.concatenate([g["src"], rng.integers(0, n, hub), np.full(hub, 7)]).astype(np.int32)
    dst = np.concatenate([g["dst"], np.full(hub, 7), rng.integers(0, n, hub)]).astype(np.int32)
    keep = src != dst
    src, dst = src[keep], dst[keep]
    vec = rng.standard_normal((src.shape[0], 3)).astype(NP[dtype])
    p = gplan(e3b, mul, lx, ly, lo, dtype)
    w = rng.standard_normal((src.shape[0], p.weight_numel)).astype(NP[dtype])
    go = t(rng.standard_normal((n, p.dim_out)).astype(NP[dtype]))
    x = t(g["x"])

    def run(order):
        graph = e3b.Graph(n, t(src), t(dst), order=order)
        v, wr = graph.to_receiver_order(t(vec)), graph.to_receiver_order(t(w))
        out = e3b.conv_forward(p, graph, x, wr, edge_vec=v, out_scale=0.3)
        grads = e3b.conv_backward(p, graph, x, wr, go, edge_vec=v, out_scale=0.3)
        e3b.device_status()
        return [out, *grads]

    base = run(None)
    perm = torch.as_tensor(rng.permutation(n).astype(np.int32), device=DEV)
    morton = e3b.morton_order(t(g["pos"]), (0.0, 0.0, 0.0), (g["side"],) * 3)
    for order in (perm, morton):
        for a, b in zip(run(order), base):
            assert torch.equal(a, b)
    bad = perm.clone()
    bad[3] = n + 5
    graph = e3b.Graph(n, t(src), t(dst), order=bad)
    with pytest.raises(e3b.E3Error) as err:
        e3b.device_status()
    assert err.value.status == e3b.E3_ERR_INDEX
