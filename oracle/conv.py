"""Message-passing convolution and its CSR segmentation in float64 (oracle side; test
infrastructure only).

e3nn course, "Curriculum at a glance", lesson 06a: the point convolution forms, for each edge,
the tensor product of the edge's spherical harmonics (scaled by radial weights) with the
sender's features, and sums the messages over each receiver's neighbours.  "Modular v2106
point models" (Scope) divides by sqrt(num_neighbors); the E3J summary, section E.2.2, names the
receiver-ordered CSR aggregation that the GPU path uses.  Here the sum is the literal
definition: messages are accumulated with ``np.add.at`` in the input edge order.

Edge i -> j has sender ``src = i`` and receiver ``dst = j`` (lesson 05a: r_ij = r_j - r_i).

Padding edges: batches of fixed shape pad the edge list (the E3J summary, sections 3.1.2 and 3.2,
measures the cost of padding edges that point to a shared padding node).  Here an edge whose sender or
receiver is -1 is padding: it belongs to no node, contributes nothing and gets zero gradients.
"""

import numpy as np

from .tp import tp_backward, tp_forward


def csr_build(n_nodes, src, dst):
    """Receiver (dst) CSR and sender (src) CSR of an edge list.

    perm_dst: stable argsort of dst (original edge ids in dst-sorted order).
    row_ptr_dst[n]..row_ptr_dst[n+1]: positions of node n's in-edges in that order.
    perm_src: stable argsort by src of the dst-sorted list (positions in dst-sorted order).
    row_ptr_src: the same offsets per sender.
    Ties keep input order (stable), which makes every array unique.
    """
    src = np.asarray(src, dtype=np.int64)
    dst = np.asarray(dst, dtype=np.int64)
    valid = (src != -1) & (dst != -1)
    ids = np.flatnonzero(valid)
    pad = np.flatnonzero(~valid)
    # valid edges stably by receiver, then the padding edges in input order (outside every row)
    perm_dst = np.concatenate([ids[np.argsort(dst[ids], kind="stable")], pad])
    row_ptr_dst = np.concatenate([[0], np.cumsum(np.bincount(dst[ids], minlength=n_nodes))])
    nv = len(ids)
    perm_src = np.concatenate([np.argsort(src[perm_dst[:nv]], kind="stable"), np.arange(nv, len(src))])
    row_ptr_src = np.concatenate([[0], np.cumsum(np.bincount(src[ids], minlength=n_nodes))])
    return (perm_dst.astype(np.int32), row_ptr_dst.astype(np.int32),
            perm_src.astype(np.int32), row_ptr_src.astype(np.int32))


def conv_forward(plan, n_nodes, src, dst, x, y, w, scale, chunk=4096):
    """out[n] = scale * sum_{e: dst_e = n} TP(x[src_e], y_e, w_e)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros((n_nodes, plan.irreps_out.dim))
    n_edges = len(src)
    src, dst = np.asarray(src), np.asarray(dst)
    for s in range(0, n_edges, chunk):
        e = np.arange(s, min(s + chunk, n_edges))
        e = e[(src[e] != -1) & (dst[e] != -1)]  # padding edges contribute nothing
        msg = tp_forward(plan, x[src[e]], y[e], w[e])
        np.add.at(out, dst[e], msg)
    return scale * out


def conv_backward(plan, n_nodes, src, dst, x, y, w, grad_out, scale, chunk=4096):
    """(dx [N, dim1], dy [E, dim2], dw [E, weight_numel]) for conv_forward."""
    x = np.asarray(x, dtype=np.float64)
    g = np.asarray(grad_out, dtype=np.float64)
    n_edges = len(src)
    dx = np.zeros_like(x)
    dy = np.zeros((n_edges, plan.irreps_in2.dim))
    dw = np.zeros((n_edges, plan.weight_numel))
    src, dst = np.asarray(src), np.asarray(dst)
    for s in range(0, n_edges, chunk):
        e = np.arange(s, min(s + chunk, n_edges))
        e = e[(src[e] != -1) & (dst[e] != -1)]  # padding edges: zero gradients
        ddx, ddy, ddw = tp_backward(plan, x[src[e]], y[e], w[e], g[dst[e]])
        np.add.at(dx, src[e], scale * ddx)
        dy[e] = scale * ddy
        dw[e] = scale * ddw
    return dx, dy, dw
