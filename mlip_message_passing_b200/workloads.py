"""Seeded synthetic inputs for the tensor product and the convolution.

This module generates inputs only; it holds none of the method's arithmetic (no harmonics, no
Clebsch-Gordan coefficients, no tensor product).  It is shared by the tests, the benchmark and
the smoke check so that the CUDA path and the float64 oracle see the same bytes.

Recipes (numpy PCG64, ``default_rng(seed)``; draws in the order listed):

* channelwise (uuu) product: x, y, w ~ N(0, 1) in that order;
* fully connected (uvw) product, shared weights: x, y, w ~ N(0, 1) in that order;
* batched product: edge-like vectors ~ N(0, 1) (or uniform on the sphere), then x ~ N(0, 1)
  [B, dim_x], then w ~ N(0, 1) [B, weight_numel];
* water-box-like graph: N positions uniform in a periodic cube of side (N / 0.1)^(1/3) Angstrom
  (density 0.1 atoms / A^3), directed loop-free radius graph at 5 A with the minimum-image
  convention (e3nn course, lesson 05a: r_ij = r_j - r_i for sender i, receiver j), edges sorted by
  (sender, receiver); then x ~ N(0, 1) [N, dim_x]; then the radial MLP weights;
* per-edge weights: a radial MLP on 8 Bessel functions sqrt(2/rc) sin(n pi r / rc) / r times the
  polynomial envelope of order p = 6, u(d) = 1 - (p+1)(p+2)/2 d^p + p(p+2) d^(p+1) - p(p+1)/2 d^(p+2),
  d = r / rc (lesson 05b names Bessel bases and polynomial envelopes): h = SiLU(f W1),
  w = h W2 with W1 [8, 64], W2 [64, weight_numel] ~ N(0, 1) / sqrt(fan_in), no biases;
* upstream gradient of the convolution ~ N(0, 1) [N, dim_out], its own seed.
"""

import math

import numpy as np

DENSITY = 0.1
CUTOFF = 5.0
N_BASIS = 8
HIDDEN = 64
ENVELOPE_P = 6


def box_side(n_nodes, density=DENSITY):
    return (n_nodes / density) ** (1.0 / 3.0)


def radius_graph_pbc(pos, side, cutoff):
    """Directed, loop-free radius graph in a periodic cube (minimum image).

    Returns (src, dst, vec) with vec = pos[dst] - pos[src] wrapped to the nearest image, edges
    sorted by (src, dst).  Needs side >= 3 * cutoff so that each pair has one image within the
    cutoff and the 27 neighbouring cells are distinct.
    """
    pos = np.asarray(pos, dtype=np.float64)
    n = pos.shape[0]
    ncell = int(math.floor(side / cutoff))
    if ncell < 3:
        raise ValueError("box too small for the cell list")
    csize = side / ncell
    cidx = np.floor(pos / csize).astype(np.int64) % ncell
    flat = (cidx[:, 0] * ncell + cidx[:, 1]) * ncell + cidx[:, 2]
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=ncell ** 3)
    maxocc = int(counts.max())
    starts = np.concatenate([[0], np.cumsum(counts)[:-1]])
    members = -np.ones((ncell ** 3, maxocc), dtype=np.int64)
    rank = np.arange(n) - starts[flat[order]]
    members[flat[order], rank] = order
    cells = np.arange(ncell ** 3)
    cx, cy, cz = cells // (ncell * ncell), (cells // ncell) % ncell, cells % ncell
    src_l, dst_l = [], []
    for dx in (-1, 0, 1):
        for dy in (-1, 0, 1):
            for dz in (-1, 0, 1):
                nb = (((cx + dx) % ncell) * ncell + (cy + dy) % ncell) * ncell + (cz + dz) % ncell
                a = members[:, :, None]          # senders in cell c
                b = members[nb][:, None, :]      # receivers in the neighbour cell
                valid = (a >= 0) & (b >= 0) & (a != b)
                ai = np.broadcast_to(a, valid.shape)[valid]
                bi = np.broadcast_to(b, valid.shape)[valid]
                d = pos[bi] - pos[ai]
                d -= side * np.round(d / side)
                keep = np.einsum("ij,ij->i", d, d) < cutoff * cutoff
                src_l.append(ai[keep])
                dst_l.append(bi[keep])
    src = np.concatenate(src_l)
    dst = np.concatenate(dst_l)
    key = src * n + dst
    key, first = np.unique(key, return_index=True)  # sorted by (src, dst); pairs are unique
    src, dst = key // n, key % n
    vec = pos[dst] - pos[src]
    vec -= side * np.round(vec / side)
    return src.astype(np.int32), dst.astype(np.int32), vec


def bessel_envelope(r, cutoff=CUTOFF, n_basis=N_BASIS, p=ENVELOPE_P):
    """[E, n_basis] radial features: Bessel functions times the polynomial envelope."""
    r = np.asarray(r, dtype=np.float64)[:, None]
    n = np.arange(1, n_basis + 1, dtype=np.float64)[None, :]
    b = math.sqrt(2.0 / cutoff) * np.sin(n * math.pi * r / cutoff) / r
    d = r / cutoff
    u = 1.0 - (p + 1) * (p + 2) / 2.0 * d ** p + p * (p + 2) * d ** (p + 1) - p * (p + 1) / 2.0 * d ** (p + 2)
    return b * np.where(d < 1.0, u, 0.0)


def mlp_params(rng, n_out, n_basis=N_BASIS, hidden=HIDDEN):
    w1 = rng.standard_normal((n_basis, hidden)) / math.sqrt(n_basis)
    w2 = rng.standard_normal((hidden, n_out)) / math.sqrt(hidden)
    return w1, w2


def mlp_apply(feat, w1, w2, dtype=np.float32):
    h = feat @ w1
    h = h / (1.0 + np.exp(-h))  # SiLU
    return (h @ w2).astype(dtype)


def mlp_apply_torch(feat, w1, w2, dtype, device, chunk=1 << 16):
    """Same MLP evaluated with torch on `device` (large edge counts); returns [E, n_out]."""
    import torch
    f = torch.as_tensor(feat, dtype=torch.float64, device=device)
    a = torch.as_tensor(w1, dtype=torch.float64, device=device)
    b = torch.as_tensor(w2, dtype=torch.float64, device=device)
    out = torch.empty((f.shape[0], b.shape[1]), dtype=dtype, device=device)
    for s in range(0, f.shape[0], chunk):
        h = torch.nn.functional.silu(f[s:s + chunk] @ a)
        out[s:s + chunk] = (h @ b).to(dtype)
    return out


def irreps_str(mul, lmax, natural_parity=True):
    return "+".join(f"{mul}x{l}{'e' if (l % 2 == 0 or not natural_parity) else 'o'}" for l in range(lmax + 1))


def sh_irreps(lmax):
    return "+".join(f"1x{l}{'e' if l % 2 == 0 else 'o'}" for l in range(lmax + 1))


# --------------------------------------------------------------------- named workloads ---
# Each entry: the degrees, multiplicity and sizes of one configuration.
CONFIGS = {
    "tp_small": dict(kind="tp", B=1024, mul=8, lx=1, ly=2, lo=2, seed=0, vectors="normal"),
    "tp_batched": dict(kind="tp", B=200_000, mul=128, lx=2, ly=3, lo=2, seed=1, vectors="sphere"),
    "conv_waterbox": dict(kind="conv", N=3000, mul=64, lx=2, ly=3, lo=2, seed=2),
    "conv_large": dict(kind="conv", N=24_000, mul=128, lx=3, ly=3, lo=3, seed=3),
    "conv_waterbox_bwd": dict(kind="conv", N=3000, mul=64, lx=2, ly=3, lo=2, seed=2, grad_seed=4),
    # channelwise (uuu) product of two node-feature sets of 128 channels, degrees 0..3
    "tp_uuu": dict(kind="tp_uuu", B=32_768, mul=128, lx=3, ly=3, lo=3, seed=5),
    # fully connected (uvw) product, shared weights: 128 channels of degrees 0..3 with one
    # harmonic-like channel of degrees 0..3 into 128 channels of every (l3 <= 3, parity) block
    "tp_uvw": dict(kind="tp_uvw", B=65_536, mul=128, lx=3, ly=3, seed=6,
                   irreps_out="128x0e+128x1o+128x1e+128x2e+128x2o+128x3o+128x3e"),
}


def n_paths(lx, ly, lo):
    return sum(1 for l1 in range(lx + 1) for l2 in range(ly + 1)
               for l3 in range(abs(l1 - l2), min(l1 + l2, lo) + 1))


def out_dim(mul, lx, ly, lo):
    return mul * sum(2 * l3 + 1 for l1 in range(lx + 1) for l2 in range(ly + 1)
                     for l3 in range(abs(l1 - l2), min(l1 + l2, lo) + 1))


def tp_inputs(B, mul, lx, ly, lo, seed, vectors="normal", dtype=np.float32):
    """vectors [B, 3] (float64), x [B, dim_x], w [B, P*mul] in `dtype`."""
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((B, 3))
    if vectors == "sphere":
        v /= np.linalg.norm(v, axis=1, keepdims=True)
    x = rng.standard_normal((B, mul * (lx + 1) ** 2)).astype(dtype)
    w = rng.standard_normal((B, n_paths(lx, ly, lo) * mul)).astype(dtype)
    return dict(vec=v, x=x, w=w)


def channel_inputs(B, mul, lx, ly, lo, seed, dtype=np.float32):
    """Inputs of a channelwise (uuu) product: x [B, mul (lx+1)^2], y [B, mul (ly+1)^2] and
    w [B, P mul], all N(0, 1), drawn in that order."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, mul * (lx + 1) ** 2)).astype(dtype)
    y = rng.standard_normal((B, mul * (ly + 1) ** 2)).astype(dtype)
    w = rng.standard_normal((B, n_paths(lx, ly, lo) * mul)).astype(dtype)
    return dict(x=x, y=y, w=w)


def uvw_inputs(B, dim_x, dim_y, weight_numel, seed, dtype=np.float32):
    """Inputs of a fully connected product with shared weights: x [B, dim_x], y [B, dim_y] and
    w [weight_numel], all N(0, 1), drawn in that order."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, dim_x)).astype(dtype)
    y = rng.standard_normal((B, dim_y)).astype(dtype)
    w = rng.standard_normal(weight_numel).astype(dtype)
    return dict(x=x, y=y, w=w)


def graph_inputs(N, mul, lx, ly, lo, seed, dtype=np.float32, weights="host", device=None):
    """Water-box-like graph: src, dst (int32, sorted by (src, dst)), vec [E, 3] (dtype), x, w.

    weights="host" evaluates the radial MLP with numpy; "torch" evaluates it on `device` and
    returns a torch tensor (for edge counts whose weights do not fit comfortably on the host);
    "none" skips it (w is None; mlp_apply on the returned parameters gives any subset of rows).
    """
    rng = np.random.default_rng(seed)
    side = box_side(N)
    pos = rng.uniform(0.0, side, size=(N, 3))
    src, dst, vec = radius_graph_pbc(pos, side, CUTOFF)
    x = rng.standard_normal((N, mul * (lx + 1) ** 2)).astype(dtype)
    w1, w2 = mlp_params(rng, n_paths(lx, ly, lo) * mul)
    feat = bessel_envelope(np.linalg.norm(vec, axis=1))
    if weights == "host":
        w = mlp_apply(feat, w1, w2, dtype)
    elif weights == "none":
        w = None
    else:
        import torch
        w = mlp_apply_torch(feat, w1, w2, torch.float32 if dtype == np.float32 else torch.float64, device)
    return dict(pos=pos, side=side, src=src, dst=dst, vec=vec.astype(dtype), x=x, w=w, mlp=(w1, w2))


def grad_out(N, dim_out, seed, dtype=np.float32):
    return np.random.default_rng(seed).standard_normal((N, dim_out)).astype(dtype)


def subgraph_nearest(pos, side, src, dst, center=0, k=50):
    """The k nodes nearest to `center` (minimum image, center included), every edge among them,
    nodes relabelled by ascending original id.  Returns (nodes, edge_ids, new_src, new_dst)."""
    d = pos - pos[center]
    d -= side * np.round(d / side)
    nodes = np.sort(np.argsort(np.einsum("ij,ij->i", d, d), kind="stable")[:k])
    remap = -np.ones(pos.shape[0], dtype=np.int64)
    remap[nodes] = np.arange(len(nodes))
    keep = np.flatnonzero((remap[src] >= 0) & (remap[dst] >= 0))
    return nodes, keep, remap[src[keep]].astype(np.int32), remap[dst[keep]].astype(np.int32)
