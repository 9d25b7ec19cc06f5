"""Weighted tensor product in float64 (oracle side; test infrastructure only).

e3nn course, "Curriculum at a glance", lesson 03b: a learnable tensor product x (x)_w y is a list
of instructions (i1, i2, i_out); each instruction couples irrep i1 of x with irrep i2 of y into
irrep i_out through the Clebsch-Gordan tensor, scaled by a weight; the connection mode says how
channels are tied.  In "uvu" mode output channel u takes input channel u of x and sums over the
channels v of y with one weight per (u, v):

    out[b, i_out, u, m3] += alpha_p * sum_v w[b, p, u, v]
                            * sum_{m1, m2} C_p[m1, m2, m3] x[b, i1, u, m1] y[b, i2, v, m2]

"uuu" ties all three channels (both inputs and the output have the same multiplicity), one weight
per (p, u):

    out[b, i_out, u, m3] += alpha_p * w[b, p, u] * sum_{m1, m2} C_p[m1, m2, m3] x[b, i1, u, m1] y[b, i2, u, m2]

"uvw" (fully connected) mixes every pair of input channels into every output channel, one weight
per (p, u, v, w):

    out[b, i_out, w, m3] += alpha_p * sum_{u, v} W[b, p, u, v, w]
                            * sum_{m1, m2} C_p[m1, m2, m3] x[b, i1, u, m1] y[b, i2, v, m2]

Lesson 03a fixes the parity rule p3 = p1 p2 and the triangle rule |l1-l2| <= l3 <= l1+l2.
The sum over (m1, m2, m3) is written densely (no use of sparsity).  Readings taken where the
sources are silent:

* instructions, when none are given: for i1 over x irreps, for i2 over y irreps, for l3 from
  |l1-l2| to min(l1+l2, lmax_out): one instruction with its own output block ("uncollapsed"
  output, irrep (mul_x, l3, p1 p2)); E3J summary, section B.3, treats collapsed (shared) output
  blocks as a special case, which explicit instruction lists may request by sharing i_out;
* weights flattened path-major, then the mode's channel indices in the order written above
  (uvu: u, v; uuu: u; uvw: u, v, w);
* alpha_p = sqrt((2 l3 + 1) / (fan_in * n_out)), n_out = number of instructions writing i_out and
  fan_in the channel sum of one output element (uvu: mul_y; uuu: 1; uvw: mul_x * mul_y), so that
  unit-variance inputs give unit-variance outputs; an instruction may override it.
"""

from dataclasses import dataclass, field

import numpy as np

from .cg import real_cg
from .irreps import Irrep, Irreps, parse_irreps


@dataclass(frozen=True)
class Instruction:
    i_in1: int
    i_in2: int
    i_out: int
    has_weight: bool = True
    path_weight: float = -1.0  # < 0: default alpha


@dataclass
class TPPlan:
    irreps_in1: Irreps
    irreps_in2: Irreps
    irreps_out: Irreps
    instructions: list
    alphas: list = field(default_factory=list)
    weight_offsets: list = field(default_factory=list)
    weight_numel: int = 0
    shared_weights: bool = False
    mode: str = "uvu"

    @property
    def n_paths(self):
        return len(self.instructions)


def _enumerate(ir1, ir2, lmax_out):
    out, ins = [], []
    for i1, a in enumerate(ir1):
        for i2, b in enumerate(ir2):
            for l3 in range(abs(a.l - b.l), min(a.l + b.l, lmax_out) + 1):
                ins.append(Instruction(i1, i2, len(out)))
                out.append(Irrep(a.mul, l3, a.p * b.p))
    return Irreps(out), ins


def make_plan(irreps_in1, irreps_in2, irreps_out=None, instructions=None, lmax_out=None,
              shared_weights=False, mode="uvu"):
    """Build the oracle's plan.  ``irreps_out``/``instructions`` None -> default enumeration."""
    if mode not in ("uvu", "uuu", "uvw"):
        raise ValueError(f"unknown connection mode {mode!r}")
    ir1 = parse_irreps(irreps_in1) if isinstance(irreps_in1, str) else irreps_in1
    ir2 = parse_irreps(irreps_in2) if isinstance(irreps_in2, str) else irreps_in2
    if instructions is None:
        if lmax_out is None:
            lmax_out = max(a.l for a in ir1) + max(b.l for b in ir2)
        irout, ins = _enumerate(ir1, ir2, lmax_out)
    else:
        irout = parse_irreps(irreps_out) if isinstance(irreps_out, str) else irreps_out
        ins = [i if isinstance(i, Instruction) else Instruction(*i) for i in instructions]
    for ins_ in ins:
        a, b, c = ir1[ins_.i_in1], ir2[ins_.i_in2], irout[ins_.i_out]
        if not (abs(a.l - b.l) <= c.l <= a.l + b.l):
            raise ValueError(f"instruction {ins_} breaks the triangle rule")
        if c.p != a.p * b.p:
            raise ValueError(f"instruction {ins_} breaks the parity rule p3 = p1 p2")
        if mode in ("uvu", "uuu") and c.mul != a.mul:
            raise ValueError(f"{mode} instruction {ins_} needs mul_out == mul_in1")
        if mode == "uuu" and b.mul != a.mul:
            raise ValueError(f"uuu instruction {ins_} needs mul_in2 == mul_in1")
    n_out = {}
    for ins_ in ins:
        n_out[ins_.i_out] = n_out.get(ins_.i_out, 0) + 1
    alphas, woffs, wn = [], [], 0
    for ins_ in ins:
        a, b, c = ir1[ins_.i_in1], ir2[ins_.i_in2], irout[ins_.i_out]
        fan_in = {"uvu": b.mul, "uuu": 1, "uvw": a.mul * b.mul}[mode]
        if ins_.path_weight >= 0:
            alphas.append(float(ins_.path_weight))
        else:
            alphas.append(float(np.sqrt((2 * c.l + 1) / (fan_in * n_out[ins_.i_out]))))
        woffs.append(wn)
        if ins_.has_weight:
            wn += {"uvu": a.mul * b.mul, "uuu": a.mul, "uvw": a.mul * b.mul * c.mul}[mode]
    return TPPlan(ir1, ir2, irout, ins, alphas, woffs, wn, shared_weights, mode)


def _blocks(plan, p):
    ins = plan.instructions[p]
    a, b, c = plan.irreps_in1[ins.i_in1], plan.irreps_in2[ins.i_in2], plan.irreps_out[ins.i_out]
    o1 = plan.irreps_in1.offsets()[ins.i_in1]
    o2 = plan.irreps_in2.offsets()[ins.i_in2]
    o3 = plan.irreps_out.offsets()[ins.i_out]
    return ins, a, b, c, o1, o2, o3


def _weights(plan, w, p, bsz):
    """The path's weights as [B, u, v] (uvu), [B, u] (uuu) or [B, u, v, w] (uvw)."""
    ins = plan.instructions[p]
    a, b, c = plan.irreps_in1[ins.i_in1], plan.irreps_in2[ins.i_in2], plan.irreps_out[ins.i_out]
    shape = {"uvu": (a.mul, b.mul), "uuu": (a.mul,), "uvw": (a.mul, b.mul, c.mul)}[plan.mode]
    size = int(np.prod(shape))
    if not ins.has_weight:
        return np.ones((bsz,) + shape)
    off = plan.weight_offsets[p]
    if plan.shared_weights:
        return np.broadcast_to(w[off:off + size].reshape((1,) + shape), (bsz,) + shape)
    return w[:, off:off + size].reshape((bsz,) + shape)


# einsum of each mode: x "bui", y "bvj", C "ijk", weights, output "b?k"
_FWD = {"uvu": "bui,bvj,ijk,buv->buk", "uuu": "bui,buj,ijk,bu->buk", "uvw": "bui,bvj,ijk,buvw->bwk"}
_DX = {"uvu": "bvj,ijk,buv,buk->bui", "uuu": "buj,ijk,bu,buk->bui", "uvw": "bvj,ijk,buvw,bwk->bui"}
_DY = {"uvu": "bui,ijk,buv,buk->bvj", "uuu": "bui,ijk,bu,buk->buj", "uvw": "bui,ijk,buvw,bwk->bvj"}
_DW = {"uvu": "bui,bvj,ijk,buk->buv", "uuu": "bui,buj,ijk,buk->bu", "uvw": "bui,bvj,ijk,bwk->buvw"}


def tp_forward(plan, x, y, w):
    """out [B, dim_out] from x [B, dim1], y [B, dim2], w [B, weight_numel] (or [weight_numel])."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    bsz = x.shape[0]
    out = np.zeros((bsz, plan.irreps_out.dim))
    for p in range(plan.n_paths):
        ins, a, b, c, o1, o2, o3 = _blocks(plan, p)
        C = real_cg(a.l, b.l, c.l)
        xs = x[:, o1:o1 + a.dim].reshape(bsz, a.mul, 2 * a.l + 1)
        ys = y[:, o2:o2 + b.dim].reshape(bsz, b.mul, 2 * b.l + 1)
        ws = _weights(plan, w, p, bsz)
        blk = plan.alphas[p] * np.einsum(_FWD[plan.mode], xs, ys, C, ws, optimize=True)
        out[:, o3:o3 + c.dim] += blk.reshape(bsz, -1)
    return out


def tp_backward(plan, x, y, w, grad_out):
    """(dx, dy, dw) of <grad_out, tp_forward(x, y, w)>: the transposes of the trilinear map
    (E3J summary, section E.1: reverse mode by transposing the linearised operation)."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    g = np.asarray(grad_out, dtype=np.float64)
    bsz = x.shape[0]
    dx, dy = np.zeros_like(x), np.zeros_like(y)
    dw = np.zeros((plan.weight_numel,)) if plan.shared_weights else np.zeros((bsz, plan.weight_numel))
    for p in range(plan.n_paths):
        ins, a, b, c, o1, o2, o3 = _blocks(plan, p)
        C = real_cg(a.l, b.l, c.l)
        al = plan.alphas[p]
        xs = x[:, o1:o1 + a.dim].reshape(bsz, a.mul, 2 * a.l + 1)
        ys = y[:, o2:o2 + b.dim].reshape(bsz, b.mul, 2 * b.l + 1)
        gs = g[:, o3:o3 + c.dim].reshape(bsz, c.mul, 2 * c.l + 1)
        ws = _weights(plan, w, p, bsz)
        dx[:, o1:o1 + a.dim] += al * np.einsum(_DX[plan.mode], ys, C, ws, gs, optimize=True).reshape(bsz, -1)
        dy[:, o2:o2 + b.dim] += al * np.einsum(_DY[plan.mode], xs, C, ws, gs, optimize=True).reshape(bsz, -1)
        if ins.has_weight:
            off = plan.weight_offsets[p]
            dwp = al * np.einsum(_DW[plan.mode], xs, ys, C, gs, optimize=True).reshape(bsz, -1)
            if plan.shared_weights:
                dw[off:off + dwp.shape[1]] += dwp.sum(axis=0)
            else:
                dw[:, off:off + dwp.shape[1]] += dwp
    return dx, dy, dw
