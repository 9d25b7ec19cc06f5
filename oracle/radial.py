"""Radial network of the point convolution in float64 (oracle side; test infrastructure only).

e3nn course, "Curriculum at a glance": lesson 06a writes the convolution message as
m_ij = (R(|r_ij|) Y(r_ij)) (x)_w h_j, with the path weights produced per edge by a radial function
R of the distance; lesson 05b feeds R a Bessel basis (the DimeNet one) instead of the raw distance
and multiplies it by a polynomial envelope so that the energy stays smooth at the cutoff.  The
pages name the parts, not their formulas; the readings taken (the published DimeNet forms):

* Bessel basis, n = 1 .. n_basis:  b_n(r) = sqrt(2 / c) sin(n pi r / c) / r  (its r -> 0 limit
  sqrt(2 / c) n pi / c at r = 0); orthonormal on [0, c] with weight r^2;
* polynomial envelope of order p, d = r / c:
  u(d) = 1 - (p + 1)(p + 2)/2 d^p + p (p + 2) d^(p+1) - p (p + 1)/2 d^(p+2) for d < 1, else 0,
  so u(0) = 1 and u, u', u'' vanish at d = 1;
* network: f = b(r) u(r / c) (n_basis features), h = SiLU(f W1) with SiLU(x) = x / (1 + e^-x),
  w = h W2 (no biases), W1 [n_basis, hidden], W2 [hidden, n_out].
"""

import numpy as np


def bessel_basis(r, cutoff, n_basis):
    """[n, n_basis] Bessel features of distances r [n]."""
    r = np.asarray(r, dtype=np.float64)
    n = np.arange(1, n_basis + 1, dtype=np.float64)
    out = np.empty((r.shape[0], n_basis))
    small = r < 1e-12
    rr = np.where(small, 1.0, r)
    out[:] = np.sqrt(2.0 / cutoff) * np.sin(np.outer(rr, n) * np.pi / cutoff) / rr[:, None]
    out[small] = np.sqrt(2.0 / cutoff) * n * np.pi / cutoff
    return out


def polynomial_envelope(d, p):
    """u(d) for scaled distances d = r / c (zero from d = 1 on)."""
    d = np.asarray(d, dtype=np.float64)
    u = 1.0 - (p + 1) * (p + 2) / 2.0 * d ** p + p * (p + 2) * d ** (p + 1) - p * (p + 1) / 2.0 * d ** (p + 2)
    return np.where(d < 1.0, u, 0.0)


def silu(x):
    return x / (1.0 + np.exp(-x))


def radial_weights(vec, cutoff, n_basis, p, w1, w2):
    """[E, n_out] per-edge path weights from edge vectors [E, 3]."""
    vec = np.asarray(vec, dtype=np.float64)
    r = np.sqrt(np.sum(vec * vec, axis=1))
    f = bessel_basis(r, cutoff, n_basis) * polynomial_envelope(r / cutoff, p)[:, None]
    h = silu(f @ np.asarray(w1, dtype=np.float64))
    return h @ np.asarray(w2, dtype=np.float64)
