"""Node reordering along a Morton (Z-order) curve, float64/integer oracle (test infrastructure).

Sparse, irregular gathers bound message-passing layers (Sobek: Streaming Equivariant Tensor
Product Convolutions, abstract); numbering nodes along a space-filling curve puts the senders of
neighbouring receivers close together in memory, so gathered rows are reused from L2.

Definition used here (the pages name the goal, not a curve; the plainest choice is the Z-order
curve): each coordinate is quantised to B = 10 bits inside the box [lo, lo + extent),
q_k = clamp(floor((p_k - lo_k) * (2^B / extent_k)), 0, 2^B - 1), the scale 2^B / extent_k taken in
float64 first; the code interleaves the bits, bit b of axis k going to bit 3 b + k.  The order is
the stable sort of the codes (equal codes keep ascending node ids).
"""

import numpy as np

BITS = 10


def quantise(pos, lo, extent):
    """Integer cell coordinates [n, 3] in [0, 2^BITS)."""
    pos = np.asarray(pos, dtype=np.float64)
    scale = np.array([float(1 << BITS) / float(e) for e in extent])
    q = np.floor((pos - np.asarray(lo, dtype=np.float64)) * scale)
    return np.clip(q, 0, (1 << BITS) - 1).astype(np.int64)


def morton_codes(pos, lo, extent):
    """30-bit Morton codes: bit b of axis k -> bit 3 b + k."""
    q = quantise(pos, lo, extent)
    code = np.zeros(q.shape[0], dtype=np.int64)
    for b in range(BITS):
        for k in range(3):
            code |= ((q[:, k] >> b) & 1) << (3 * b + k)
    return code


def morton_order(pos, lo, extent):
    """perm[i] = id of the node with the i-th smallest code (stable)."""
    return np.argsort(morton_codes(pos, lo, extent), kind="stable").astype(np.int32)


def invert_permutation(perm):
    inv = np.empty_like(perm)
    inv[perm] = np.arange(len(perm), dtype=perm.dtype)
    return inv
