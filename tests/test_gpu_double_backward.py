"""Second derivatives through the library (float64): the convolution's backward and the harmonics'
backward are themselves differentiated (force training runs through them), and every second
derivative is checked against central differences of the float64 oracle's FIRST derivatives along
random directions (the oracle's backward, not the library's)."""

import math

import numpy as np
import pytest
import torch

import oracle
from mlip_message_passing_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def e3b():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from mlip_message_passing_b200 import e3b
    return e3b


def _close(a, b, tol):
    assert abs(a - b) <= tol * max(1.0, abs(b)), (a, b)


def test_conv_double_backward_against_oracle_first_derivatives(e3b):
    n, mul, lx, ly, lo = 120, 8, 2, 3, 2
    rng = np.random.default_rng(61)
    src = rng.integers(0, n, 1500).astype(np.int32)
    dst = rng.integers(0, n, 1500).astype(np.int32)
    keep = src != dst
    src, dst = src[keep], dst[keep]
    E = src.shape[0]
    q = oracle.make_plan(W.irreps_str(mul, lx), W.sh_irreps(ly), lmax_out=lo)
    p = e3b.Plan(W.irreps_str(mul, lx), W.sh_irreps(ly), lmax_out=lo, dtype=torch.float64)
    x = rng.standard_normal((n, p.dim_in1))
    y = rng.standard_normal((E, p.dim_in2))
    w = rng.standard_normal((E, p.weight_numel))
    g = rng.standard_normal((n, p.dim_out))
    ux, uy, uw = (rng.standard_normal(a.shape) for a in (x, y, w))
    s = 0.37
    graph = e3b.Graph(n, torch.as_tensor(src, device=DEV), torch.as_tensor(dst, device=DEV))
    perm = graph.perm_dst.cpu().numpy()  # library edge arrays are in receiver order

    def dev(a, edge=False):
        return torch.as_tensor(a[perm] if edge else a, device=DEV).requires_grad_()

    xt, yt, wt, gt = dev(x), dev(y, True), dev(w, True), dev(g)
    out = e3b.conv(p, graph, xt, yt, wt, s)
    gx, gy, gw = torch.autograd.grad(out, (xt, yt, wt), gt, create_graph=True)
    L2 = (gx * dev(ux)).sum() + (gy * dev(uy, True)).sum() + (gw * dev(uw, True)).sum()
    dx, dy, dw, dg = torch.autograd.grad(L2, (xt, yt, wt, gt))
    e3b.device_status()

    def L2_oracle(xx, yy, ww, gg):
        rx, ry, rw = oracle.conv_backward(q, n, src, dst, xx, yy, ww, gg, s)
        return float((rx * ux).sum() + (ry * uy).sum() + (rw * uw).sum())

    h = 1e-3  # L2 is linear in each argument: central differences are exact up to rounding
    base = [x, y, w, g]
    for k, (name, grad, edge) in enumerate((("x", dx, False), ("y", dy, True), ("w", dw, True), ("g", dg, False))):
        d = rng.standard_normal(base[k].shape)
        plus, minus = list(base), list(base)
        plus[k], minus[k] = base[k] + h * d, base[k] - h * d
        fd = (L2_oracle(*plus) - L2_oracle(*minus)) / (2 * h)
        an = float((grad.detach().cpu().numpy() * (d[perm] if edge else d)).sum())
        _close(an, fd, 1e-10)


@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_sh_double_backward_against_oracle_first_derivative(e3b, lmax):
    rng = np.random.default_rng(70 + lmax)
    nv = 64
    vec = rng.standard_normal((nv, 3)) * rng.uniform(0.5, 3.0, (nv, 1))
    gy = rng.standard_normal((nv, (lmax + 1) ** 2))
    u = rng.standard_normal((nv, 3))
    vt = torch.as_tensor(vec, device=DEV).requires_grad_()
    gyt = torch.as_tensor(gy, device=DEV).requires_grad_()
    Y = e3b.sh(lmax, vt)
    (gv,) = torch.autograd.grad(Y, vt, gyt, create_graph=True)
    phi = (gv * torch.as_tensor(u, device=DEV)).sum()
    d_vec, d_gy = torch.autograd.grad(phi, (vt, gyt))
    e3b.device_status()

    def phi_oracle(vv, gg):
        return float((oracle.sh_backward(lmax, vv, gg) * u).sum())

    for which, grad, h, tol in ((0, d_vec, 1e-6, 1e-7), (1, d_gy, 1e-3, 1e-11)):
        d = rng.standard_normal(vec.shape if which == 0 else gy.shape)
        args_p, args_m = [vec, gy], [vec, gy]
        args_p[which] = args_p[which] + h * d
        args_m[which] = args_m[which] - h * d
        fd = (phi_oracle(*args_p) - phi_oracle(*args_m)) / (2 * h)
        _close(float((grad.cpu().numpy() * d).sum()), fd, tol)


def test_conv_with_harmonics_from_vectors_twice_differentiable(e3b):
    """conv(x, sh(vec), w): second derivative with respect to the edge vectors (the force-training
    term) against central differences of the oracle's first derivative (conv backward, then the
    harmonics' chain rule), float64."""
    n, mul, lx, ly, lo = 100, 4, 2, 3, 2
    rng = np.random.default_rng(81)
    src = rng.integers(0, n, 900).astype(np.int32)
    dst = rng.integers(0, n, 900).astype(np.int32)
    keep = src != dst
    src, dst = src[keep], dst[keep]
    E = src.shape[0]
    q = oracle.make_plan(W.irreps_str(mul, lx), W.sh_irreps(ly), lmax_out=lo)
    p = e3b.Plan(W.irreps_str(mul, lx), W.sh_irreps(ly), lmax_out=lo, dtype=torch.float64)
    x = rng.standard_normal((n, p.dim_in1))
    vec = rng.standard_normal((E, 3)) * 1.5
    w = rng.standard_normal((E, p.weight_numel))
    g = rng.standard_normal((n, p.dim_out))
    uv = rng.standard_normal((E, 3))
    s = 0.5
    graph = e3b.Graph(n, torch.as_tensor(src, device=DEV), torch.as_tensor(dst, device=DEV))
    perm = graph.perm_dst.cpu().numpy()
    vt = torch.as_tensor(vec[perm], device=DEV).requires_grad_()
    out = e3b.conv(p, graph, torch.as_tensor(x, device=DEV), e3b.sh(ly, vt), torch.as_tensor(w[perm], device=DEV), s)
    (gvec,) = torch.autograd.grad(out, vt, torch.as_tensor(g, device=DEV), create_graph=True)
    (hv,) = torch.autograd.grad((gvec * torch.as_tensor(uv[perm], device=DEV)).sum(), vt)
    e3b.device_status()

    def first(vv):
        Y = oracle.real_sh_all(ly, vv)
        _, ry, _ = oracle.conv_backward(q, n, src, dst, x, Y, w, g, s)
        return float((oracle.sh_backward(ly, vv, ry) * uv).sum())

    d = rng.standard_normal(vec.shape)
    h = 1e-6
    fd = (first(vec + h * d) - first(vec - h * d)) / (2 * h)
    _close(float((hv.cpu().numpy() * d[perm]).sum()), fd, 1e-7)
