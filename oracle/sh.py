"""Real spherical harmonics in float64 (oracle side; test infrastructure only).

e3nn course, "Curriculum at a glance", lesson 02b: Y^l(R r) = D^l(R) Y^l(r), parity (-1)^l, and
three normalisations; the convolution uses "component" normalisation ("Modular v2106 point
models", Scope), i.e. sum_m Y_lm(r)^2 = 2l+1 for a unit vector.

Definition used here (the textbook real harmonics with the z axis as the pole, no
Condon-Shortley phase, m = -l..l):

    Y_lm(r) = N_lm * d^{|m|}P_l/dt^{|m|}(z) * { Re (x + i y)^m      m > 0
                                              { 1                   m = 0
                                              { Im (x + i y)^{|m|}  m < 0
    N_lm    = sqrt((2l+1) (l-|m|)! / (l+|m|)!) * (sqrt(2) if m != 0 else 1)

for the unit vector (x, y, z) = r/|r|; (1-z^2)^{|m|/2} cos(|m| phi) = Re (x+iy)^{|m|} turns the
associated Legendre form into a polynomial.  P_l is the Legendre polynomial from its explicit sum.
With this choice Y^1 = sqrt(3) (y, z, x).  For r = 0 the oracle returns Y^0 = 1 and Y^{l>0} = 0
(the sources are silent; loop-free radius graphs never produce r = 0).
"""

from math import comb, factorial, sqrt

import numpy as np


def _legendre_coeffs(l):
    """Power-series coefficients (ascending) of the Legendre polynomial P_l."""
    c = np.zeros(l + 1)
    for k in range(l // 2 + 1):
        c[l - 2 * k] += (-1) ** k * comb(l, k) * comb(2 * l - 2 * k, l) / 2.0 ** l
    return c


def real_sh(l, vec):
    """Component-normalised real SH of degree l for vectors ``vec`` [n, 3] -> [n, 2l+1]."""
    vec = np.asarray(vec, dtype=np.float64)
    n = vec.shape[0]
    r = np.sqrt(np.sum(vec * vec, axis=1))
    out = np.zeros((n, 2 * l + 1))
    nz = r > 0
    if l == 0:
        out[:, 0] = 1.0
        return out
    u = np.zeros_like(vec)
    u[nz] = vec[nz] / r[nz, None]
    x, y, z = u[:, 0], u[:, 1], u[:, 2]
    pl = np.polynomial.polynomial.Polynomial(_legendre_coeffs(l))
    xy = x + 1j * y
    for m in range(-l, l + 1):
        am = abs(m)
        dp = pl.deriv(am) if am > 0 else pl
        norm = sqrt((2 * l + 1) * factorial(l - am) / factorial(l + am))
        if m != 0:
            norm *= sqrt(2.0)
        trig = xy ** am
        if m > 0:
            ang = trig.real
        elif m < 0:
            ang = trig.imag
        else:
            ang = np.ones(n)
        out[:, m + l] = norm * dp(z) * ang
    out[~nz] = 0.0
    return out


def real_sh_all(lmax, vec):
    """Concatenated [Y^0 | Y^1 | ... | Y^lmax] -> [n, (lmax+1)^2] (irreps 1x0e+1x1o+...)."""
    return np.concatenate([real_sh(l, vec) for l in range(lmax + 1)], axis=1)


def real_sh_grad(l, vec):
    """Jacobian d Y^l / d vec of the component-normalised harmonics -> [n, 2l+1, 3].

    Y depends on vec only through u = vec/|vec|, so dY/dvec = (1/r) (I - u u^T) grad_u F(u) for
    any smooth F that equals Y on the unit sphere.  F is the formula of ``real_sh`` read as a
    function of independent (x, y, z):
        F_lm = N_lm * P_l^{(|m|)}(z) * A_m(x, y),   A_m = Re / Im (x + i y)^{|m|}, A_0 = 1,
        dF/dx = N P^{(|m|)}(z) * Re / Im (|m| (x + i y)^{|m|-1}),
        dF/dy = N P^{(|m|)}(z) * Re / Im (i |m| (x + i y)^{|m|-1}),
        dF/dz = N P^{(|m|+1)}(z) * A_m.
    At vec = 0 (where Y is set to Y^0 = 1, Y^{l>0} = 0) the gradient is defined as 0.
    """
    vec = np.asarray(vec, dtype=np.float64)
    n = vec.shape[0]
    out = np.zeros((n, 2 * l + 1, 3))
    if l == 0:
        return out
    r = np.sqrt(np.sum(vec * vec, axis=1))
    nz = r > 0
    u = np.zeros_like(vec)
    u[nz] = vec[nz] / r[nz, None]
    x, y, z = u[:, 0], u[:, 1], u[:, 2]
    pl = np.polynomial.polynomial.Polynomial(_legendre_coeffs(l))
    xy = x + 1j * y
    gu = np.zeros((n, 2 * l + 1, 3))
    for m in range(-l, l + 1):
        am = abs(m)
        dp = pl.deriv(am) if am > 0 else pl
        dp1 = pl.deriv(am + 1)
        norm = sqrt((2 * l + 1) * factorial(l - am) / factorial(l + am))
        if m != 0:
            norm *= sqrt(2.0)
        if m == 0:
            ang, dax, day = np.ones(n), np.zeros(n), np.zeros(n)
        else:
            trig = xy ** am
            dtrig = am * xy ** (am - 1)
            pick = (lambda c: c.real) if m > 0 else (lambda c: c.imag)
            ang, dax, day = pick(trig), pick(dtrig), pick(1j * dtrig)
        gu[:, m + l, 0] = norm * dp(z) * dax
        gu[:, m + l, 1] = norm * dp(z) * day
        gu[:, m + l, 2] = norm * dp1(z) * ang
    # project out the radial part and scale by 1/r
    radial = np.einsum("nmk,nk->nm", gu, u)
    out[nz] = (gu[nz] - radial[nz][:, :, None] * u[nz][:, None, :]) / r[nz, None, None]
    return out


def real_sh_all_grad(lmax, vec):
    """Jacobian of ``real_sh_all`` -> [n, (lmax+1)^2, 3]."""
    return np.concatenate([real_sh_grad(l, vec) for l in range(lmax + 1)], axis=1)


def sh_backward(lmax, vec, grad_y):
    """grad_vec[i] = sum_m grad_y[i, m] dY_m(vec_i)/dvec_i for the concatenated harmonics."""
    return np.einsum("nm,nmk->nk", np.asarray(grad_y, dtype=np.float64), real_sh_all_grad(lmax, vec))
