"""Pins of the float64 oracle to facts that do not come from the oracle itself: closed forms
and textbook values, a library routine (sympy's Clebsch-Gordan), symmetry (rotations and
reflections), orthogonality, multilinearity, finite differences and brute force."""

import itertools
import math
import os

import numpy as np
import pytest

import oracle
from oracle.cg import complex_cg, real_basis_change, real_cg
from oracle.sh import real_sh, real_sh_all
from tests.conftest import rel_err

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_rot(rng):
    q, r = np.linalg.qr(rng.standard_normal((3, 3)))
    q = q * np.sign(np.diag(r))
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q


def wigner_real(l, R, rng):
    """D^l(R) in the real-harmonic basis, fitted from Y(R r) = D Y(r) on random points
    (exact up to rounding: the harmonics of one degree span a (2l+1)-dim space)."""
    r = rng.standard_normal((4 * (2 * l + 1) + 8, 3))
    A = real_sh(l, r)
    B = real_sh(l, r @ R.T)
    D, *_ = np.linalg.lstsq(A, B, rcond=None)
    return D.T


# ------------------------------------------------------------------------ harmonics ---
def test_sh_closed_forms_low_degree():
    rng = np.random.default_rng(0)
    v = rng.standard_normal((50, 3))
    u = v / np.linalg.norm(v, axis=1, keepdims=True)
    x, y, z = u.T
    np.testing.assert_allclose(real_sh(0, v)[:, 0], 1.0, atol=1e-15)
    np.testing.assert_allclose(real_sh(1, v), math.sqrt(3) * np.stack([y, z, x], 1), atol=1e-14)
    s15, s5 = math.sqrt(15), math.sqrt(5)
    y2 = np.stack([s15 * x * y, s15 * y * z, s5 / 2 * (3 * z * z - 1), s15 * x * z, s15 / 2 * (x * x - y * y)], 1)
    np.testing.assert_allclose(real_sh(2, v), y2, atol=1e-13)
    # textbook real harmonics of degree 3 (orthonormal table times sqrt(4 pi))
    y3 = np.stack([
        math.sqrt(70) / 4 * y * (3 * x * x - y * y),
        math.sqrt(105) * x * y * z,
        math.sqrt(42) / 4 * y * (5 * z * z - 1),
        math.sqrt(7) / 2 * z * (5 * z * z - 3),
        math.sqrt(42) / 4 * x * (5 * z * z - 1),
        math.sqrt(105) / 2 * z * (x * x - y * y),
        math.sqrt(70) / 4 * x * (x * x - 3 * y * y),
    ], 1)
    np.testing.assert_allclose(real_sh(3, v), y3, atol=1e-13)


@pytest.mark.parametrize("l", range(5))
def test_sh_norm_parity_and_scale_invariance(l):
    rng = np.random.default_rng(l)
    v = rng.standard_normal((40, 3))
    Y = real_sh(l, v)
    np.testing.assert_allclose((Y * Y).sum(1), 2 * l + 1, rtol=1e-13)
    np.testing.assert_allclose(real_sh(l, -v), (-1) ** l * Y, atol=1e-13)
    np.testing.assert_allclose(real_sh(l, 3.7 * v), Y, atol=1e-13)


@pytest.mark.parametrize("l", range(1, 5))
def test_sh_harmonic(l):
    # r^l Y_lm(r) is a harmonic polynomial: its Laplacian vanishes (central differences)
    rng = np.random.default_rng(10 + l)
    p = rng.standard_normal((10, 3))
    h = 1e-3
    f = lambda q: np.linalg.norm(q, axis=1, keepdims=True) ** l * real_sh(l, q)
    lap = sum(f(p + h * e) + f(p - h * e) - 2 * f(p) for e in np.eye(3)) / h ** 2
    assert np.abs(lap).max() < 1e-5 * max(1.0, np.abs(f(p)).max())


def test_sh_zero_vector():
    Y = real_sh_all(3, np.zeros((2, 3)))
    assert Y[0, 0] == 1.0 and np.all(Y[:, 1:] == 0.0)


@pytest.mark.parametrize("l", range(4))
def test_sh_equivariance_and_wigner_homomorphism(l):
    rng = np.random.default_rng(20 + l)
    R1, R2 = rand_rot(rng), rand_rot(rng)
    D1, D2, D12 = wigner_real(l, R1, rng), wigner_real(l, R2, rng), wigner_real(l, R1 @ R2, rng)
    v = rng.standard_normal((30, 3))
    np.testing.assert_allclose(real_sh(l, v @ R1.T), real_sh(l, v) @ D1.T, atol=1e-12)
    np.testing.assert_allclose(D1 @ D1.T, np.eye(2 * l + 1), atol=1e-12)
    np.testing.assert_allclose(D12, D1 @ D2, atol=1e-12)
    if l == 1:
        P = np.array([[0, 1, 0], [0, 0, 1], [1, 0, 0]], dtype=float)  # (x,y,z) -> (y,z,x)
        np.testing.assert_allclose(D1, P @ R1 @ P.T, atol=1e-12)


@pytest.mark.parametrize("l", [0, 1, 2, 3])
def test_sh_grad_matches_central_differences(l):
    """The analytic Jacobian against central differences of real_sh (an independent
    computation; h = 1e-6: truncation below 1e-9 down to |v| = 0.2, rounding ~1e-10)."""
    rng = np.random.default_rng(40 + l)
    v = rng.standard_normal((40, 3)) * rng.uniform(0.5, 3.0, (40, 1))
    J = oracle.real_sh_grad(l, v)
    h = 1e-6
    fd = np.zeros_like(J)
    for k in range(3):
        e = np.zeros(3)
        e[k] = h
        fd[:, :, k] = (real_sh(l, v + e) - real_sh(l, v - e)) / (2 * h)
    assert np.max(np.abs(J - fd)) <= 1e-8


def test_sh_grad_closed_form_l1():
    """Y^1 = sqrt(3) (y, z, x) / r, so dY_(i)/dv = sqrt(3) (e_i / r - v_i v / r^3)."""
    rng = np.random.default_rng(44)
    v = rng.standard_normal((20, 3))
    r = np.linalg.norm(v, axis=1)
    J = oracle.real_sh_grad(1, v)
    for comp, axis in enumerate((1, 2, 0)):
        ref = -v[:, axis, None] * v / r[:, None] ** 3
        ref[:, axis] += 1 / r
        np.testing.assert_allclose(J[:, comp, :], math.sqrt(3) * ref, atol=1e-13)


@pytest.mark.parametrize("l", [1, 2, 3])
def test_sh_grad_radial_scaling_and_rotation(l):
    """Y(c v) = Y(v): the Jacobian is orthogonal to v and scales as 1/c; Y(R v) = D Y(v):
    J(R v) R = D J(v)."""
    rng = np.random.default_rng(50 + l)
    v = rng.standard_normal((25, 3))
    J = oracle.real_sh_grad(l, v)
    assert np.max(np.abs(np.einsum("nmk,nk->nm", J, v))) <= 1e-12
    np.testing.assert_allclose(oracle.real_sh_grad(l, 2.5 * v), J / 2.5, atol=1e-13)
    R = rand_rot(rng)
    D = wigner_real(l, R, rng)
    lhs = np.einsum("nmk,kj->nmj", oracle.real_sh_grad(l, v @ R.T), R)
    rhs = np.einsum("ab,nbk->nak", D, J)
    np.testing.assert_allclose(lhs, rhs, atol=1e-11)


def test_sh_grad_zero_vector_and_backward_contraction():
    v = np.array([[0.0, 0.0, 0.0], [0.3, -1.2, 0.7]])
    J = oracle.real_sh_all_grad(3, v)
    assert J.shape == (2, 16, 3) and np.all(J[0] == 0) and np.all(J[1, 0] == 0)
    g = np.random.default_rng(45).standard_normal((2, 16))
    np.testing.assert_allclose(oracle.sh_backward(3, v, g), np.einsum("nm,nmk->nk", g, J), atol=1e-15)


# ------------------------------------------------------------------ Clebsch-Gordan ---
def test_complex_cg_matches_sympy():
    from sympy.physics.quantum.cg import CG
    for l1, l2 in itertools.product(range(4), range(4)):
        for l3 in range(abs(l1 - l2), l1 + l2 + 1):
            for m1 in range(-l1, l1 + 1):
                for m2 in range(-l2, l2 + 1):
                    m3 = m1 + m2
                    if abs(m3) > l3:
                        continue
                    ref = float(CG(l1, m1, l2, m2, l3, m3).doit())
                    assert abs(complex_cg(l1, m1, l2, m2, l3, m3) - ref) < 1e-14


def test_complex_cg_textbook_values():
    assert abs(complex_cg(1, 1, 1, -1, 0, 0) - 1 / math.sqrt(3)) < 1e-15
    assert abs(complex_cg(1, 0, 1, 0, 0, 0) + 1 / math.sqrt(3)) < 1e-15
    assert abs(complex_cg(1, 1, 1, 0, 2, 1) - 1 / math.sqrt(2)) < 1e-15
    assert abs(complex_cg(1, 0, 1, 0, 2, 0) - math.sqrt(2 / 3)) < 1e-15
    assert abs(complex_cg(1, 0, 1, 0, 1, 0)) < 1e-15


def test_real_basis_change_is_unitary_and_real_sh_follows():
    for l in range(5):
        U = real_basis_change(l)
        np.testing.assert_allclose(U @ U.conj().T, np.eye(2 * l + 1), atol=1e-15)


def _golden_1x1():
    vals = {0: np.zeros((3, 3, 1)), 1: np.zeros((3, 3, 3)), 2: np.zeros((3, 3, 5))}
    with open(os.path.join(GOLDEN, "one_times_one.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            l3, m1, m2, m3, a, b = (int(t) for t in line.split())
            vals[l3][m1 + 1, m2 + 1, m3 + l3] = math.copysign(math.sqrt(abs(a) / b), a)
    return vals


def test_real_cg_1x1_is_dot_cross_symtraceless():
    gold = _golden_1x1()
    for l3 in range(3):
        np.testing.assert_allclose(real_cg(1, 1, l3), gold[l3], atol=1e-15)
    rng = np.random.default_rng(3)
    a, b = rng.standard_normal(3), rng.standard_normal(3)
    P = [1, 2, 0]  # (y, z, x) order of the real basis
    ar, br = a[P], b[P]
    np.testing.assert_allclose(np.einsum("i,j,ijk->k", ar, br, real_cg(1, 1, 0)), [a @ b / math.sqrt(3)], atol=1e-14)
    np.testing.assert_allclose(np.einsum("i,j,ijk->k", ar, br, real_cg(1, 1, 1)), np.cross(a, b)[P] / math.sqrt(6),
                               atol=1e-14)


@pytest.mark.parametrize("l1,l2", list(itertools.product(range(4), range(4))))
def test_real_cg_orthogonality(l1, l2):
    for l3 in range(abs(l1 - l2), l1 + l2 + 1):
        for l3b in range(abs(l1 - l2), l1 + l2 + 1):
            g = np.einsum("ijk,ijl->kl", real_cg(l1, l2, l3), real_cg(l1, l2, l3b))
            ref = np.eye(2 * l3 + 1) / (2 * l3 + 1) if l3 == l3b else np.zeros((2 * l3 + 1, 2 * l3b + 1))
            np.testing.assert_allclose(g, ref, atol=1e-14)


@pytest.mark.parametrize("l1,l2", list(itertools.product(range(4), range(4))))
def test_real_cg_equivariance(l1, l2):
    rng = np.random.default_rng(100 + 4 * l1 + l2)
    R = rand_rot(rng)
    D1, D2 = wigner_real(l1, R, rng), wigner_real(l2, R, rng)
    for l3 in range(abs(l1 - l2), l1 + l2 + 1):
        D3 = wigner_real(l3, R, rng)
        C = real_cg(l1, l2, l3)
        # f(D1 a, D2 b) = D3 f(a, b) with f(a, b)_k = sum_ij C[i, j, k] a_i b_j
        lhs = np.einsum("ia,jb,ijk->abk", D1, D2, C)
        rhs = np.einsum("kc,abc->abk", D3, C)
        np.testing.assert_allclose(lhs, rhs, atol=1e-12)


@pytest.mark.parametrize("l1,l2", [(1, 1), (1, 2), (2, 2), (2, 3), (3, 3)])
def test_real_cg_gaunt_property(l1, l2):
    # for even l1+l2+l3, contracting C with Y^l1(r) Y^l2(r) gives a multiple of Y^l3(r)
    rng = np.random.default_rng(7)
    v = rng.standard_normal((25, 3))
    for l3 in range(abs(l1 - l2), l1 + l2 + 1, 2):
        f = np.einsum("ni,nj,ijk->nk", real_sh(l1, v), real_sh(l2, v), real_cg(l1, l2, l3))
        Y3 = real_sh(l3, v)
        c = (f * Y3).sum() / (Y3 * Y3).sum()
        assert abs(c) > 1e-3
        np.testing.assert_allclose(f, c * Y3, atol=1e-12)


# --------------------------------------------------------------- tensor product ---
def _channel_triples(mode, a, bb, c):
    """(u, v, w_out, weight index within the path) of every channel coupling of one instruction:
    uvu ties w_out = u and sums v; uuu ties all three; uvw couples every (u, v) with every w_out
    (e3nn course, lesson 03b: the connection mode of an instruction)."""
    if mode == "uvu":
        return [(u, v, u, u * bb.mul + v) for u in range(a.mul) for v in range(bb.mul)]
    if mode == "uuu":
        return [(u, u, u, u) for u in range(a.mul)]
    return [(u, v, k, (u * bb.mul + v) * c.mul + k)
            for u in range(a.mul) for v in range(bb.mul) for k in range(c.mul)]


def brute_tp(plan, x, y, w):
    """Pure-Python loops over every index of the definition (tiny inputs only)."""
    out = np.zeros((x.shape[0], plan.irreps_out.dim))
    o1s, o2s, o3s = plan.irreps_in1.offsets(), plan.irreps_in2.offsets(), plan.irreps_out.offsets()
    for b in range(x.shape[0]):
        for p, ins in enumerate(plan.instructions):
            a, c = plan.irreps_in1[ins.i_in1], plan.irreps_out[ins.i_out]
            bb = plan.irreps_in2[ins.i_in2]
            C = real_cg(a.l, bb.l, c.l)
            for u, v, wo, q in _channel_triples(plan.mode, a, bb, c):
                wt = w[b, plan.weight_offsets[p] + q]
                for i in range(2 * a.l + 1):
                    for j in range(2 * bb.l + 1):
                        for k in range(2 * c.l + 1):
                            out[b, o3s[ins.i_out] + wo * (2 * c.l + 1) + k] += (
                                plan.alphas[p] * wt * C[i, j, k]
                                * x[b, o1s[ins.i_in1] + u * (2 * a.l + 1) + i]
                                * y[b, o2s[ins.i_in2] + v * (2 * bb.l + 1) + j])
    return out


def mode_plan(mode):
    """A small plan of each connection mode: several channels, a collapsed output (two paths into
    one block), and for uvw output multiplicities that differ from the inputs'."""
    if mode == "uuu":
        return oracle.make_plan("2x0e+2x1o+2x2e", "2x0e+2x1o+2x2e", lmax_out=2, mode="uuu")
    if mode == "uvw":
        return oracle.make_plan("2x0e+2x1o", "2x1o+2x0e", "1x1o+3x0e+2x1e",
                                instructions=[(0, 0, 0), (1, 1, 0), (1, 0, 1), (1, 0, 2)], mode="uvw")
    if mode == "uvw_fans":  # two paths into one block with channel fans 2 x 3 and 1 x 2
        return oracle.make_plan("2x0e+1x1o", "3x1o+2x0e", "1x1o+3x0e+2x1e",
                                instructions=[(0, 0, 0), (1, 1, 0), (1, 0, 1), (1, 0, 2)], mode="uvw")
    return oracle.make_plan("2x0e+2x1o", "3x1o", "2x1o+2x0e+2x1e",
                            instructions=[(0, 0, 0), (1, 0, 1), (1, 0, 2)], mode="uvu")


def test_tp_matches_brute_force_loops():
    rng = np.random.default_rng(5)
    plan = oracle.make_plan("2x0e+2x1o+2x2e", "1x0e+1x1o+1x2e", lmax_out=2)
    x = rng.standard_normal((3, plan.irreps_in1.dim))
    y = rng.standard_normal((3, plan.irreps_in2.dim))
    w = rng.standard_normal((3, plan.weight_numel))
    np.testing.assert_allclose(oracle.tp_forward(plan, x, y, w), brute_tp(plan, x, y, w), atol=1e-13)


def test_tp_multiplicity_two_inputs_brute_force():
    # uvu with mul_y = 2 (sum over v with one weight per (u, v)) and a collapsed output
    rng = np.random.default_rng(6)
    plan = oracle.make_plan("2x1o", "2x1o", "2x0e+2x1e", instructions=[(0, 0, 0), (0, 0, 1)])
    x = rng.standard_normal((2, plan.irreps_in1.dim))
    y = rng.standard_normal((2, plan.irreps_in2.dim))
    w = rng.standard_normal((2, plan.weight_numel))
    np.testing.assert_allclose(oracle.tp_forward(plan, x, y, w), brute_tp(plan, x, y, w), atol=1e-13)


@pytest.mark.parametrize("mode", ["uvu", "uuu", "uvw", "uvw_fans"])
def test_tp_modes_brute_force(mode):
    rng = np.random.default_rng(7)
    plan = mode_plan(mode)
    x = rng.standard_normal((2, plan.irreps_in1.dim))
    y = rng.standard_normal((2, plan.irreps_in2.dim))
    w = rng.standard_normal((2, plan.weight_numel))
    assert plan.weight_numel == sum(len(_channel_triples(plan.mode, plan.irreps_in1[i.i_in1], plan.irreps_in2[i.i_in2],
                                                         plan.irreps_out[i.i_out])) for i in plan.instructions)
    np.testing.assert_allclose(oracle.tp_forward(plan, x, y, w), brute_tp(plan, x, y, w), atol=1e-13)


def test_modes_coincide_at_multiplicity_one():
    """With one channel everywhere the three connection modes are the same map, default path
    weights included (each output element then sums exactly one channel product)."""
    rng = np.random.default_rng(8)
    plans = [oracle.make_plan("1x0e+1x1o+1x2e", "1x0e+1x1o+1x2e", lmax_out=2, mode=m) for m in ("uvu", "uuu", "uvw")]
    x = rng.standard_normal((3, plans[0].irreps_in1.dim))
    y = rng.standard_normal((3, plans[0].irreps_in2.dim))
    w = rng.standard_normal((3, plans[0].weight_numel))
    outs = [oracle.tp_forward(p, x, y, w) for p in plans]
    assert plans[0].alphas == plans[1].alphas == plans[2].alphas
    np.testing.assert_allclose(outs[1], outs[0], atol=1e-14)
    np.testing.assert_allclose(outs[2], outs[0], atol=1e-14)


def test_uuu_is_uvu_on_the_diagonal():
    """uuu equals uvu whose weight matrix per path is diagonal in (u, v), up to the default path
    weight: uvu normalises by the channel count of y, uuu by one channel."""
    rng = np.random.default_rng(9)
    pu = oracle.make_plan("3x0e+3x1o", "3x0e+3x1o", lmax_out=1, mode="uuu")
    pv = oracle.make_plan("3x0e+3x1o", "3x0e+3x1o", lmax_out=1, mode="uvu")
    x = rng.standard_normal((2, pu.irreps_in1.dim))
    y = rng.standard_normal((2, pu.irreps_in2.dim))
    wu = rng.standard_normal((2, pu.weight_numel))
    wv = np.zeros((2, pv.weight_numel))
    for p in range(pu.n_paths):
        for u in range(3):
            wv[:, pv.weight_offsets[p] + u * 3 + u] = wu[:, pu.weight_offsets[p] + u] * pu.alphas[p] / pv.alphas[p]
    np.testing.assert_allclose(oracle.tp_forward(pu, x, y, wu), oracle.tp_forward(pv, x, y, wv), atol=1e-13)
    assert all(abs(a / b - math.sqrt(3)) < 1e-14 for a, b in zip(pu.alphas, pv.alphas))


def test_scalar_path_modes_closed_forms():
    """0e x 0e -> 0e with C = 1: uuu is the channelwise product w_u x_u y_u (alpha 1); uvw is the
    bilinear form sum_uv W_uvw x_u y_v / sqrt(mul_x mul_y)."""
    rng = np.random.default_rng(10)
    x, y = rng.standard_normal((4, 3)), rng.standard_normal((4, 3))
    pu = oracle.make_plan("3x0e", "3x0e", lmax_out=0, mode="uuu")
    w = rng.standard_normal((4, 3))
    np.testing.assert_allclose(oracle.tp_forward(pu, x, y, w), w * x * y, atol=1e-15)
    pw = oracle.make_plan("3x0e", "3x0e", "2x0e", instructions=[(0, 0, 0)], mode="uvw")
    W = rng.standard_normal((4, 3, 3, 2))
    want = np.einsum("buvw,bu,bv->bw", W, x, y) / 3.0
    np.testing.assert_allclose(oracle.tp_forward(pw, x, y, W.reshape(4, -1)), want, atol=1e-14)


def test_uvw_with_scalar_y_is_a_per_irrep_linear():
    """With y = 1x0e the only paths are l x 0 -> l, whose coefficients are delta(m1, m3)/sqrt(2l+1)
    (course 03a: coupling with a scalar), and the fan of an output element is mul_x: the fully
    connected product is then the per-irrep channel mixing out_l[w, m] = sum_u W_l[u, w] x_l[u, m] y /
    sqrt(mul_x), written here with plain matrix products."""
    rng = np.random.default_rng(14)
    ir1, irout = "4x0e+4x1o+4x2e", "3x0e+3x1o+3x2e"
    plan = oracle.make_plan(ir1, "1x0e", irout, instructions=[(0, 0, 0), (1, 0, 1), (2, 0, 2)], mode="uvw")
    B = 5
    x = rng.standard_normal((B, plan.irreps_in1.dim))
    y = rng.standard_normal((B, 1))
    W = [rng.standard_normal((4, 3)) for _ in range(3)]
    w = np.concatenate([m.ravel() for m in W])[None].repeat(B, axis=0)
    got = oracle.tp_forward(plan, x, y, w)
    want, o1 = [], 0
    for l in range(3):
        d = 2 * l + 1
        xl = x[:, o1:o1 + 4 * d].reshape(B, 4, d)
        want.append((np.einsum("uw,bum->bwm", W[l], xl) * y[:, :, None] / 2.0).reshape(B, -1))
        o1 += 4 * d
    np.testing.assert_allclose(got, np.concatenate(want, axis=1), atol=1e-13)


def test_mode_validation():
    with pytest.raises(ValueError):
        oracle.make_plan("2x1o", "3x1o", lmax_out=2, mode="uuu")  # uuu ties x and y channels
    with pytest.raises(ValueError):
        oracle.make_plan("2x1o", "1x1o", "3x0e", instructions=[(0, 0, 0)], mode="uvu")  # uvu ties x and out
    with pytest.raises(ValueError):
        oracle.make_plan("1x1o", "1x1o", lmax_out=2, mode="uvv")


def test_tp_scalar_path():
    plan = oracle.make_plan("3x0e", "1x0e", lmax_out=0)
    rng = np.random.default_rng(1)
    x, y, w = rng.standard_normal((4, 3)), rng.standard_normal((4, 1)), rng.standard_normal((4, 3))
    np.testing.assert_allclose(oracle.tp_forward(plan, x, y, w), x * y * w, atol=1e-15)


def _trilinear_coefficients(plan):
    """T[k, i, j, q] = out_k for x = e_i, y = e_j, w = e_q (the oracle as a black box).  The
    tensor product is linear in each input, so these basis evaluations fix it completely."""
    d1, d2, nw, do = plan.irreps_in1.dim, plan.irreps_in2.dim, plan.weight_numel, plan.irreps_out.dim
    T = np.zeros((do, d1, d2, nw))
    eye1, eye2 = np.eye(d1), np.eye(d2)
    for q in range(nw):
        wq = np.zeros((d1 * d2, nw))
        wq[:, q] = 1.0
        xs = np.repeat(eye1, d2, axis=0)
        ys = np.tile(eye2, (d1, 1))
        T[:, :, :, q] = oracle.tp_forward(plan, xs, ys, wq).reshape(d1, d2, do).transpose(2, 0, 1)
    return T


@pytest.mark.parametrize("case", ["uncollapsed", "collapsed", "mul_y2", "uuu", "uvw", "uvw_fans"])
def test_default_path_weight_gives_unit_second_moment(case):
    """The default path weight alpha_p is fixed by one property (e3nn course, lesson 03b: paths
    are normalised so that the output keeps the scale of the inputs): when every component of x,
    y and w is an independent zero-mean unit-variance variable, every output component has second
    moment 1.  For a trilinear map out_k = sum T[k,i,j,q] x_i y_j w_q that moment is exactly
    sum_{ijq} T[k,i,j,q]^2, so the check is exact, with T read off the oracle by basis inputs."""
    if case == "uncollapsed":
        plan = oracle.make_plan("1x0e+1x1o+1x2e", "1x0e+1x1o+1x2e+1x3o", lmax_out=3)
    elif case == "collapsed":  # two paths share each output block: n_out = 2
        plan = oracle.make_plan("1x1o+1x2o", "1x1o", "1x1e+1x2e",
                                instructions=[(0, 0, 0), (1, 0, 0), (1, 0, 1)])
    elif case == "mul_y2":  # uvu with two channels of y: sum over v with a weight per (u, v)
        plan = oracle.make_plan("2x1o", "2x1o+2x2e", "2x0e+2x1e+2x2o+2x3o",
                                instructions=[(0, 0, 0), (0, 0, 1), (0, 1, 2), (0, 1, 3)])
    else:  # the other connection modes (uuu: one channel per output; uvw: mul_x * mul_y)
        plan = mode_plan(case)
    T = _trilinear_coefficients(plan)
    moment = (T * T).sum(axis=(1, 2, 3))
    np.testing.assert_allclose(moment, 1.0, rtol=1e-12)


def test_default_path_weight_unit_moment_over_the_sphere():
    """The same property with y the component-normalised harmonics of a direction uniform on the
    sphere (the convolution's input), averaged exactly by a product quadrature (Gauss-Legendre in
    cos(theta) times equally spaced phi; exact for the degree-6 polynomials Y_m Y_m' with l <= 3),
    and x, w independent N(0, 1), whose average is again the sum of squares of the coefficients."""
    plan = oracle.make_plan("1x0e+1x1o+1x2e+1x3o", "1x0e+1x1o+1x2e+1x3o", lmax_out=3)
    t, tw = np.polynomial.legendre.leggauss(6)
    phi = np.arange(12) * (2 * np.pi / 12)
    st = np.sqrt(1 - t * t)
    dirs = np.stack([np.outer(st, np.cos(phi)).ravel(), np.outer(st, np.sin(phi)).ravel(),
                     np.repeat(t, phi.size)], 1)
    qw = np.repeat(tw, phi.size) / (2 * phi.size)  # weights sum to 1: the average over the sphere
    Y = real_sh_all(3, dirs)
    T = _trilinear_coefficients(plan)  # [k, i, j, q]
    # out_k(x, w | y) = sum_{i,q} (sum_j T[k,i,j,q] y_j) x_i w_q
    Ty = np.einsum("kijq,nj->nkiq", T, Y)
    moment = np.einsum("n,nkiq->k", qw, Ty * Ty)
    np.testing.assert_allclose(moment, 1.0, rtol=1e-12)


def test_default_path_weight_closed_forms_1x1():
    """1o x 1o with unit weights.  The outer product a b^T splits into its trace part, its
    antisymmetric part and its symmetric traceless part (e3nn course, lesson 03a: the dot, cross
    and symmetric traceless products); with the default path weights (1, sqrt(3), sqrt(5)) each
    output block is an isometric image of one part, so its norm equals that part's Frobenius
    norm, the three squared norms add up to |a|^2 |b|^2, and the scalar block is a.b/sqrt(3)."""
    plan = oracle.make_plan("1x1o", "1x1o", lmax_out=2)
    rng = np.random.default_rng(21)
    for _ in range(5):
        a, b = rng.standard_normal(3), rng.standard_normal(3)
        out = oracle.tp_forward(plan, a[None], b[None], np.ones((1, 3)))[0]
        M = np.outer(a, b)
        tr = np.trace(M) / 3 * np.eye(3)
        anti = 0.5 * (M - M.T)
        sym = 0.5 * (M + M.T) - tr
        assert abs(out[0] - a @ b / math.sqrt(3)) < 1e-14
        assert abs(np.linalg.norm(out[1:4]) - np.linalg.norm(anti)) < 1e-14
        assert abs(np.linalg.norm(out[4:9]) - np.linalg.norm(sym)) < 1e-14
        assert abs(out @ out - (a @ a) * (b @ b)) < 1e-12


def test_default_path_enumeration_counts():
    p0 = oracle.make_plan("8x0e+8x1o", "1x0e+1x1o+1x2e", lmax_out=2)
    assert [(plan_l(p0, i)) for i in range(p0.n_paths)] == [
        (0, 0, 0), (0, 1, 1), (0, 2, 2), (1, 0, 1), (1, 1, 0), (1, 1, 1), (1, 1, 2), (1, 2, 1), (1, 2, 2)]
    assert p0.irreps_out.dim == 29 * 8
    p2 = oracle.make_plan("64x0e+64x1o+64x2e", "1x0e+1x1o+1x2e+1x3o", lmax_out=2)
    assert p2.n_paths == 18 and p2.irreps_out.dim == 64 * 64
    p3 = oracle.make_plan("128x0e+128x1o+128x2e+128x3o", "1x0e+1x1o+1x2e+1x3o", lmax_out=3)
    assert p3.n_paths == 34 and p3.irreps_out.dim == 156 * 128
    # parity rule: 1o x 1o -> 1e (pseudovector)
    assert str(p0.irreps_out).split(" + ")[5] == "8x1e"


def plan_l(plan, p):
    ins = plan.instructions[p]
    return plan.irreps_in1[ins.i_in1].l, plan.irreps_in2[ins.i_in2].l, plan.irreps_out[ins.i_out].l


def test_instruction_validation():
    with pytest.raises(ValueError):
        oracle.make_plan("1x1o", "1x1o", "1x0o", instructions=[(0, 0, 0)])  # parity
    with pytest.raises(ValueError):
        oracle.make_plan("1x1o", "1x1o", "1x3e", instructions=[(0, 0, 0)])  # triangle
    with pytest.raises(ValueError):
        oracle.parse_irreps("3x1q")


def _rep(plan_irreps, Ds, parity_flip, x):
    """Apply the O(3) element (R, or -R when parity_flip) to features in mul_ir layout."""
    out = np.empty_like(x)
    for ir, off in zip(plan_irreps, plan_irreps.offsets()):
        d = 2 * ir.l + 1
        blk = x[:, off:off + ir.dim].reshape(x.shape[0], ir.mul, d)
        s = ir.p if parity_flip else 1
        out[:, off:off + ir.dim] = (s * blk @ Ds[ir.l].T).reshape(x.shape[0], -1)
    return out


@pytest.mark.parametrize("flip", [False, True])
def test_tp_equivariance_o3(flip):
    rng = np.random.default_rng(11 + flip)
    plan = oracle.make_plan("3x0e+3x1o+3x2e+3x3o", "1x0e+1x1o+1x2e+1x3o", lmax_out=3)
    R = rand_rot(rng)
    Ds = {l: wigner_real(l, R, rng) for l in range(4)}
    v = rng.standard_normal((5, 3))
    x = rng.standard_normal((5, plan.irreps_in1.dim))
    w = rng.standard_normal((5, plan.weight_numel))
    g = -R if flip else R
    y, y_rot = real_sh_all(3, v), real_sh_all(3, v @ g.T)
    out = oracle.tp_forward(plan, x, y, w)
    out_rot = oracle.tp_forward(plan, _rep(plan.irreps_in1, Ds, flip, x), y_rot, w)
    np.testing.assert_allclose(out_rot, _rep(plan.irreps_out, Ds, flip, out), atol=1e-12)


@pytest.mark.parametrize("mode", ["uuu", "uvw"])
def test_tp_modes_equivariance_o3(mode):
    """Rotating (and reflecting) both inputs of a uuu or uvw product rotates its output; y here is
    a general feature (several channels), not only harmonics."""
    rng = np.random.default_rng(13)
    plan = (oracle.make_plan("2x0e+2x1o+2x2e+2x3o", "2x0e+2x1o+2x2e+2x3o", lmax_out=3, mode="uuu") if mode == "uuu"
            else oracle.make_plan("2x0e+2x1o+1x2e", "2x1o+1x2o", lmax_out=3, mode="uvw"))
    R = rand_rot(rng)
    Ds = {l: wigner_real(l, R, rng) for l in range(4)}
    x = rng.standard_normal((3, plan.irreps_in1.dim))
    y = rng.standard_normal((3, plan.irreps_in2.dim))
    w = rng.standard_normal((3, plan.weight_numel))
    out = oracle.tp_forward(plan, x, y, w)
    for flip in (False, True):
        out_rot = oracle.tp_forward(plan, _rep(plan.irreps_in1, Ds, flip, x), _rep(plan.irreps_in2, Ds, flip, y), w)
        np.testing.assert_allclose(out_rot, _rep(plan.irreps_out, Ds, flip, out), atol=1e-12)


@pytest.mark.parametrize("mode", ["uvu", "uuu", "uvw"])
def test_tp_backward_euler_identities_and_fd(mode):
    rng = np.random.default_rng(12)
    plan = {"uvu": lambda: oracle.make_plan("2x0e+2x1o+2x2e", "1x0e+1x1o+1x2e+1x3o", lmax_out=2),
            "uuu": lambda: mode_plan("uuu"), "uvw": lambda: mode_plan("uvw")}[mode]()
    B = 4
    x = rng.standard_normal((B, plan.irreps_in1.dim))
    y = rng.standard_normal((B, plan.irreps_in2.dim))
    w = rng.standard_normal((B, plan.weight_numel))
    g = rng.standard_normal((B, plan.irreps_out.dim))
    dx, dy, dw = oracle.tp_backward(plan, x, y, w, g)
    L = float((g * oracle.tp_forward(plan, x, y, w)).sum())
    # the map is linear in each input separately: <grad, input> = L (Euler)
    for d, t in ((dx, x), (dy, y), (dw, w)):
        assert abs(float((d * t).sum()) - L) < 1e-11 * max(1.0, abs(L))
    # central differences along random directions (exact for a linear function up to rounding)
    h = 1e-3
    for which, d in ((0, dx), (1, dy), (2, dw)):
        args = [x, y, w]
        dirn = rng.standard_normal(args[which].shape)
        plus = list(args)
        minus = list(args)
        plus[which] = args[which] + h * dirn
        minus[which] = args[which] - h * dirn
        fd = ((g * oracle.tp_forward(plan, *plus)).sum() - (g * oracle.tp_forward(plan, *minus)).sum()) / (2 * h)
        assert abs(fd - (d * dirn).sum()) < 1e-9 * max(1.0, abs(fd))


# ------------------------------------------------------------------- convolution ---
def small_graph(seed, n=40, e=300):
    rng = np.random.default_rng(seed)
    src = rng.integers(0, n, e).astype(np.int32)
    dst = rng.integers(0, n, e).astype(np.int32)
    return rng, src, dst


def test_csr_bit_exact_against_loops():
    rng, src, dst = small_graph(1)
    n = 40
    perm_dst, rp_dst, perm_src, rp_src = oracle.csr_build(n, src, dst)
    # brute force: receivers ascending, ties in input order
    ref = [e for v in range(n) for e in range(len(dst)) if dst[e] == v]
    assert perm_dst.tolist() == ref
    srt = src[perm_dst]
    ref_s = [i for v in range(n) for i in range(len(srt)) if srt[i] == v]
    assert perm_src.tolist() == ref_s
    assert rp_dst[0] == 0 and rp_dst[-1] == len(dst) and np.all(np.diff(rp_dst) >= 0)
    assert rp_dst.tolist() == [sum(1 for d in dst if d < v) for v in range(n + 1)]
    assert rp_src.tolist() == [sum(1 for s in src if s < v) for v in range(n + 1)]


def test_csr_with_padding_against_loops():
    """Edges with sender or receiver -1 are padding: outside every row, after the valid edges."""
    rng, src, dst = small_graph(3)
    n = 40
    src, dst = src.copy(), dst.copy()
    pad = rng.choice(len(src), 25, replace=False)
    src[pad[:10]] = -1
    dst[pad[10:20]] = -1
    src[pad[20:]] = -1
    dst[pad[20:]] = -1
    perm_dst, rp_dst, perm_src, rp_src = oracle.csr_build(n, src, dst)
    valid = [e for e in range(len(src)) if src[e] != -1 and dst[e] != -1]
    ref = [e for v in range(n) for e in valid if dst[e] == v] + [e for e in range(len(src)) if e not in valid]
    assert perm_dst.tolist() == ref
    nv = len(valid)
    srt = src[perm_dst[:nv]]
    assert perm_src.tolist() == [i for v in range(n) for i in range(nv) if srt[i] == v] + list(range(nv, len(src)))
    assert rp_dst.tolist() == [sum(1 for e in valid if dst[e] < v) for v in range(n + 1)]
    assert rp_src.tolist() == [sum(1 for e in valid if src[e] < v) for v in range(n + 1)]


def test_conv_padding_edges_change_nothing():
    rng, src, dst = small_graph(4)
    n = 40
    plan = oracle.make_plan("2x0e+2x1o", "1x0e+1x1o+1x2e", lmax_out=2)
    x = rng.standard_normal((n, plan.irreps_in1.dim))
    k = len(src)
    y = real_sh_all(2, rng.standard_normal((k + 12, 3)))
    w = rng.standard_normal((k + 12, plan.weight_numel))
    ps = np.concatenate([src, rng.integers(-1, n, 12)])
    pd = np.concatenate([dst, np.full(12, -1)])
    ps[k::3] = -1
    g = rng.standard_normal((n, plan.irreps_out.dim))
    np.testing.assert_allclose(oracle.conv_forward(plan, n, ps, pd, x, y, w, 0.5),
                               oracle.conv_forward(plan, n, src, dst, x, y[:k], w[:k], 0.5), atol=1e-13)
    dx, dy, dw = oracle.conv_backward(plan, n, ps, pd, x, y, w, g, 0.5)
    rx, ry, rw = oracle.conv_backward(plan, n, src, dst, x, y[:k], w[:k], g, 0.5)
    np.testing.assert_allclose(dx, rx, atol=1e-13)
    np.testing.assert_allclose(dy[:k], ry, atol=1e-13)
    np.testing.assert_allclose(dw[:k], rw, atol=1e-13)
    assert np.all(dy[k:] == 0) and np.all(dw[k:] == 0)


def test_conv_edge_order_invariance_isolated_and_empty():
    rng, src, dst = small_graph(2)
    n = 40
    dst[dst == 7] = 8  # node 7 has no in-edges
    plan = oracle.make_plan("2x0e+2x1o", "1x0e+1x1o+1x2e", lmax_out=2)
    x = rng.standard_normal((n, plan.irreps_in1.dim))
    v = rng.standard_normal((len(src), 3))
    y = real_sh_all(2, v)
    w = rng.standard_normal((len(src), plan.weight_numel))
    out = oracle.conv_forward(plan, n, src, dst, x, y, w, 0.5)
    p = rng.permutation(len(src))
    out2 = oracle.conv_forward(plan, n, src[p], dst[p], x, y[p], w[p], 0.5)
    np.testing.assert_allclose(out2, out, atol=1e-13)
    assert np.all(out[7] == 0.0)
    e0 = np.zeros(0, dtype=np.int32)
    z = oracle.conv_forward(plan, n, e0, e0, x, y[:0], w[:0], 0.5)
    assert z.shape == out.shape and np.all(z == 0.0)
    # sum over edges: equals the per-edge products accumulated by receiver with loops
    ref = np.zeros_like(out)
    msg = oracle.tp_forward(plan, x[src], y, w)
    for e in range(len(src)):
        ref[dst[e]] += 0.5 * msg[e]
    np.testing.assert_allclose(out, ref, atol=1e-13)


def test_conv_equivariance_rotated_positions():
    rng = np.random.default_rng(13)
    n = 12
    pos = rng.uniform(0, 3, (n, 3))
    src, dst = np.nonzero(np.ones((n, n)) - np.eye(n))
    src, dst = src.astype(np.int32), dst.astype(np.int32)
    plan = oracle.make_plan("2x0e+2x1o+2x2e", "1x0e+1x1o+1x2e+1x3o", lmax_out=2)
    x = rng.standard_normal((n, plan.irreps_in1.dim))
    w = rng.standard_normal((len(src), plan.weight_numel))
    R = rand_rot(rng)
    Ds = {l: wigner_real(l, R, rng) for l in range(4)}
    vec = pos[dst] - pos[src]
    out = oracle.conv_forward(plan, n, src, dst, x, real_sh_all(3, vec), w, 1.0)
    out_r = oracle.conv_forward(plan, n, src, dst, _rep(plan.irreps_in1, Ds, False, x),
                                real_sh_all(3, (pos @ R.T)[dst] - (pos @ R.T)[src]), w, 1.0)
    np.testing.assert_allclose(out_r, _rep(plan.irreps_out, Ds, False, out), atol=1e-12)


def test_conv_backward_euler_and_fd():
    rng, src, dst = small_graph(3, n=15, e=80)
    n = 15
    plan = oracle.make_plan("2x0e+2x1o+2x2e", "1x0e+1x1o+1x2e+1x3o", lmax_out=2)
    x = rng.standard_normal((n, plan.irreps_in1.dim))
    y = real_sh_all(3, rng.standard_normal((len(src), 3)))
    w = rng.standard_normal((len(src), plan.weight_numel))
    g = rng.standard_normal((n, plan.irreps_out.dim))
    s = 0.3
    dx, dy, dw = oracle.conv_backward(plan, n, src, dst, x, y, w, g, s)
    L = float((g * oracle.conv_forward(plan, n, src, dst, x, y, w, s)).sum())
    for d, t in ((dx, x), (dy, y), (dw, w)):
        assert abs(float((d * t).sum()) - L) < 1e-11 * max(1.0, abs(L))
    h = 1e-3
    for which, d in ((0, dx), (1, dy), (2, dw)):
        args = [x, y, w]
        dirn = rng.standard_normal(args[which].shape)
        pl, mi = list(args), list(args)
        pl[which] = args[which] + h * dirn
        mi[which] = args[which] - h * dirn
        f = lambda a: float((g * oracle.conv_forward(plan, n, src, dst, a[0], a[1], a[2], s)).sum())
        fd = (f(pl) - f(mi)) / (2 * h)
        assert abs(fd - float((d * dirn).sum())) < 1e-9 * max(1.0, abs(fd))


# ------------------------------------------------------------------- reordering ---
def _octree_less(qa, qb):
    """Z-order by recursive octant subdivision: at the coarsest level where the cells differ,
    the octant index x + 2 y + 4 z decides (an independent formulation of the curve)."""
    for b in range(oracle.reorder.BITS - 1, -1, -1):
        oa = sum(((int(qa[k]) >> b) & 1) << k for k in range(3))
        ob = sum(((int(qb[k]) >> b) & 1) << k for k in range(3))
        if oa != ob:
            return -1 if oa < ob else 1
    return 0


def test_morton_order_equals_octree_order():
    import functools
    import oracle.reorder  # noqa: F401
    rng = np.random.default_rng(60)
    pos = rng.uniform(-2.0, 5.0, (300, 3))
    lo, ext = (-2.0, -2.0, -2.0), (7.0, 7.0, 7.0)
    q = oracle.reorder.quantise(pos, lo, ext)
    ref = sorted(range(len(pos)), key=functools.cmp_to_key(lambda a, b: _octree_less(q[a], q[b]) or (a > b) - (a < b)))
    assert np.array_equal(oracle.morton_order(pos, lo, ext), np.array(ref, dtype=np.int32))


def test_morton_codes_known_cells_and_clamping():
    import oracle.reorder  # noqa: F401
    lo, ext = (0.0, 0.0, 0.0), (1024.0, 1024.0, 1024.0)  # one unit per cell
    pts = np.array([[0.5, 0.5, 0.5], [1.5, 0.5, 0.5], [0.5, 1.5, 0.5], [0.5, 0.5, 1.5], [2.5, 0.5, 0.5],
                    [1023.9, 1023.9, 1023.9], [-5.0, 2000.0, 0.0]])
    codes = oracle.morton_codes(pts, lo, ext)
    # x -> bit 0, y -> bit 1, z -> bit 2, x = 2 -> bit 3; the last cell has all 30 bits set;
    # out-of-box coordinates clamp to the first / last cell
    assert list(codes[:5]) == [0, 1, 2, 4, 8]
    assert codes[5] == (1 << 30) - 1
    assert codes[6] == oracle.morton_codes(np.array([[0.0, 1023.5, 0.0]]), lo, ext)[0]


def test_invert_permutation():
    perm = np.random.default_rng(61).permutation(50).astype(np.int32)
    inv = oracle.invert_permutation(perm)
    assert np.array_equal(perm[inv], np.arange(50)) and np.array_equal(inv[perm], np.arange(50))


# ----------------------------------------------------------------- radial network ---
def test_bessel_basis_orthonormal_and_limits():
    """sqrt(2/c) sin(n pi r / c) / r are orthonormal on [0, c] with weight r^2 (Gauss-Legendre,
    exact for the trigonometric products to rounding at this order), vanish at r = c and tend to
    sqrt(2/c) n pi / c at r = 0."""
    c, nb = 5.0, 8
    t, wq = np.polynomial.legendre.leggauss(200)
    r = 0.5 * c * (t + 1.0)
    b = oracle.bessel_basis(r, c, nb)
    gram = (b * (r * r * 0.5 * c * wq)[:, None]).T @ b
    np.testing.assert_allclose(gram, np.eye(nb), atol=1e-12)
    np.testing.assert_allclose(oracle.bessel_basis(np.array([c]), c, nb), 0.0, atol=1e-14)
    lim = np.sqrt(2 / c) * np.arange(1, nb + 1) * np.pi / c
    np.testing.assert_allclose(oracle.bessel_basis(np.array([0.0]), c, nb)[0], lim, rtol=1e-15)
    np.testing.assert_allclose(oracle.bessel_basis(np.array([1e-7]), c, nb)[0], lim, rtol=1e-10)


@pytest.mark.parametrize("p", [3, 5, 6, 8])
def test_polynomial_envelope_smooth_at_cutoff(p):
    """The envelope itself (no formula retyped): u(0) = 1; near the cutoff u(1 - e) shrinks like
    e^3, i.e. u, u' and u'' all vanish at d = 1 (C^2, more than the C^1 the forces need); zero
    from the cutoff on; decreasing on [0, 1)."""
    u = lambda d: oracle.polynomial_envelope(np.asarray(d, dtype=np.float64), p)
    assert u([0.0])[0] == 1.0
    e = np.array([2e-3, 1e-3, 5e-4])
    ratio = u(1.0 - e) / e ** 3
    np.testing.assert_allclose(ratio[1:], ratio[:-1], rtol=0.02)  # cubic order
    # near d = 0 the envelope leaves 1 at order p (the order the reading fixes)
    d0 = np.array([0.02, 0.01])
    slope = np.log((1 - u(d0[0:1])[0]) / (1 - u(d0[1:2])[0])) / np.log(2.0)
    assert abs(slope - p) < 0.1
    assert np.all(u([1.0, 1.5, 7.0]) == 0.0)
    d = np.linspace(0, 0.999, 200)
    assert np.all(np.diff(u(d)) <= 0) and np.all(np.diff(u(np.linspace(0.2, 0.999, 100))) < 0)


def test_silu_closed_forms():
    x = np.array([-30.0, -1.0, 0.0, 1.0, 30.0])
    np.testing.assert_allclose(oracle.silu(x), x / (1 + np.exp(-x)), rtol=1e-15)
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(oracle.silu(np.array([40.0])), 40.0, rtol=1e-15)
    h = 1e-6  # SiLU'(0) = 1/2
    assert abs((oracle.silu(np.array([h]))[0] - oracle.silu(np.array([-h]))[0]) / (2 * h) - 0.5) < 1e-9


def test_radial_weights_brute_force_and_cutoff():
    rng = np.random.default_rng(31)
    vec = rng.standard_normal((7, 3)) * 2.0
    vec[0] = [5.5, 0.0, 0.0]  # beyond the cutoff: envelope 0, SiLU(0) = 0, so w = 0
    w1 = rng.standard_normal((8, 6))
    w2 = rng.standard_normal((6, 5))
    got = oracle.radial_weights(vec, 5.0, 8, 6, w1, w2)
    for e in range(vec.shape[0]):
        r = math.sqrt(sum(v * v for v in vec[e]))
        d = r / 5.0
        u = 1 - 28 * d ** 6 + 48 * d ** 7 - 21 * d ** 8 if d < 1 else 0.0
        f = [math.sqrt(2 / 5.0) * math.sin(n * math.pi * r / 5.0) / r * u for n in range(1, 9)]
        h = []
        for j in range(6):
            a = sum(f[n] * w1[n, j] for n in range(8))
            h.append(a / (1 + math.exp(-a)))
        for k in range(5):
            assert abs(got[e, k] - sum(h[j] * w2[j, k] for j in range(6))) < 1e-13
    assert np.all(got[0] == 0.0)
