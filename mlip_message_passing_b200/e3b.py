"""Thin PyTorch binding of the C ABI in ``include/e3b.h`` (``libe3b.so``).

Every function here only checks and marshals arguments (device, dtype, shape, contiguity),
then calls the library on the current CUDA stream; all arithmetic runs in the library's CUDA
kernels.  If the shared library is missing this module fails to import: there is no CPU path.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libe3b.so")

E3_OK, E3_ERR_INVALID_ARG, E3_ERR_IRREPS_PARSE, E3_ERR_INSTRUCTION, E3_ERR_UNSUPPORTED, \
    E3_ERR_SHAPE, E3_ERR_INDEX, E3_ERR_CUDA, E3_ERR_TIMEOUT = range(9)
STATUS_NAMES = ["OK", "INVALID_ARG", "IRREPS_PARSE", "INSTRUCTION", "UNSUPPORTED", "SHAPE", "INDEX",
                "CUDA", "TIMEOUT"]
_DTYPES = {torch.float32: 0, torch.float64: 1}
_SH_NORMS = {"component": 0, "integral": 1, "norm": 2}

# every symbol include/e3b.h declares
SYMBOLS = [
    "e3_plan_create", "e3_plan_destroy", "e3_plan_info", "e3_plan_irreps_out", "e3_plan_paths",
    "e3_device_status", "e3_cg_dense", "e3_supported", "e3_tp_forward", "e3_tp_backward",
    "e3_spherical_harmonics", "e3_csr_workspace_size", "e3_csr_build", "e3_gather_rows",
    "e3_conv_forward", "e3_conv_backward", "e3_last_error", "e3_csr_build_static",
    "e3_backward_workspace_size", "e3_spherical_harmonics_backward", "e3_morton_workspace_size",
    "e3_morton_order", "e3_invert_permutation", "e3_remap_ids", "e3_conv_workspace_size",
    "e3_conv_topology_size", "e3_conv_topology_build", "e3_set_test_knobs", "e3_add_rows",
    "e3_conv_topology_build_ordered", "e3_radial_prep_size", "e3_radial_prepare", "e3_radial_weights",
    "e3_spherical_harmonics_double_backward", "e3_plan_status",
]


class E3Error(RuntimeError):
    def __init__(self, status, message):
        self.status = status
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        super().__init__(f"e3b {name}: {message}")


class Instruction(ctypes.Structure):
    _fields_ = [("i_in1", ctypes.c_int32), ("i_in2", ctypes.c_int32), ("i_out", ctypes.c_int32),
                ("has_weight", ctypes.c_int32), ("path_weight", ctypes.c_double)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m mlip_message_passing_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, D, VP = ctypes.c_char_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    sig = {
        "e3_plan_create": [P, P, P, ctypes.POINTER(Instruction), I32, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                           ctypes.POINTER(VP)],
        "e3_plan_destroy": [VP],
        "e3_plan_info": [VP, ctypes.POINTER(I64), ctypes.POINTER(I64), ctypes.POINTER(I64), ctypes.POINTER(I64),
                         ctypes.POINTER(I32)],
        "e3_plan_irreps_out": [VP, ctypes.c_char_p, ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t)],
        "e3_plan_paths": [VP, ctypes.POINTER(I32), ctypes.POINTER(D)],
        "e3_device_status": [VP],
        "e3_plan_status": [VP, VP],
        "e3_cg_dense": [I32, I32, I32, ctypes.POINTER(D)],
        "e3_supported": [],
        "e3_tp_forward": [VP, I64, VP, VP, VP, VP, VP],
        "e3_tp_backward": [VP, I64, VP, VP, VP, VP, VP, VP, VP, VP, ctypes.c_size_t, VP],
        "e3_backward_workspace_size": [I64, ctypes.POINTER(ctypes.c_size_t)],
        "e3_spherical_harmonics": [I32, I64, VP, ctypes.c_int, ctypes.c_int, VP, VP],
        "e3_spherical_harmonics_backward": [I32, I64, VP, ctypes.c_int, VP, ctypes.c_int, VP, VP],
        "e3_spherical_harmonics_double_backward": [I32, I64, VP, ctypes.c_int, VP, VP, ctypes.c_int, VP, VP, VP],
        "e3_csr_workspace_size": [I64, I64, ctypes.POINTER(ctypes.c_size_t)],
        "e3_csr_build": [I64, I64, VP, VP, VP, VP, VP, VP, VP, ctypes.c_size_t, VP],
        "e3_csr_build_static": [I64, I64, VP, VP, VP, VP, VP, VP, VP],
        "e3_gather_rows": [I64, I64, I64, VP, VP, VP, VP],
        "e3_add_rows": [I64, I64, I64, ctypes.c_int, VP, VP, VP, VP],
        "e3_radial_prep_size": [I32, I32, ctypes.POINTER(ctypes.c_size_t)],
        "e3_radial_prepare": [I32, I32, VP, VP, ctypes.c_size_t, VP],
        "e3_radial_weights": [I64, VP, D, I32, I32, I32, VP, VP, I32, VP, VP],
        "e3_conv_forward": [VP, I64, I64, VP, VP, VP, VP, VP, ctypes.c_int, VP, D, VP, VP, VP, ctypes.c_size_t,
                            VP],
        "e3_conv_workspace_size": [VP, I64, I64, ctypes.POINTER(ctypes.c_size_t)],
        "e3_conv_topology_size": [I64, I64, ctypes.POINTER(ctypes.c_size_t)],
        "e3_conv_topology_build": [I64, I64, VP, VP, VP, ctypes.c_size_t, VP],
        "e3_conv_topology_build_ordered": [I64, I64, VP, VP, VP, VP, ctypes.c_size_t, VP],
        "e3_conv_backward": [VP, I64, I64, VP, VP, VP, VP, VP, VP, VP, VP, ctypes.c_int, VP, VP, D, VP, VP, VP,
                             VP, VP, ctypes.c_size_t, VP],
        "e3_morton_workspace_size": [I64, ctypes.POINTER(ctypes.c_size_t)],
        "e3_morton_order": [I64, VP, ctypes.c_int, ctypes.POINTER(D), ctypes.POINTER(D), VP, VP, ctypes.c_size_t,
                            VP],
        "e3_invert_permutation": [I64, VP, VP, VP],
        "e3_remap_ids": [I64, VP, I64, VP, VP, VP],
        "e3_set_test_knobs": [I64, I32],
        "e3_last_error": [],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name in ("e3_last_error", "e3_supported") else ctypes.c_int
    return lib


lib = _load()


def _check(status):
    if status != E3_OK:
        raise E3Error(status, lib.e3_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t, name, dtype, shape, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def supported():
    """Degree triples (Lx, Ly, Lo) with compiled kernels."""
    return [tuple(int(v) for v in s.split(",")) for s in lib.e3_supported().decode().split()]


def cg_dense(l1, l2, l3):
    """The library's real CG tensor (ladder construction) as a float64 CPU tensor."""
    out = (ctypes.c_double * ((2 * l1 + 1) * (2 * l2 + 1) * (2 * l3 + 1)))()
    _check(lib.e3_cg_dense(l1, l2, l3, out))
    return torch.tensor(list(out), dtype=torch.float64).reshape(2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1)


def device_status():
    """Synchronise the current stream; raise E3Error if a kernel recorded an error."""
    _check(lib.e3_device_status(_stream()))


class Plan:
    """A tensor-product plan (irreps, instructions, dtype) bound to the current CUDA device.

    ``irreps_out`` with ``instructions=None`` filters the enumerated output irreps; pass
    ``lmax_out`` instead to keep every output irrep of degree <= lmax_out.
    ``instructions``: list of (i_in1, i_in2, i_out[, path_weight]) tuples.
    """

    def __init__(self, irreps_in1, irreps_in2, irreps_out=None, instructions=None, lmax_out=None,
                 dtype=torch.float32, mode="uvu", shared_weights=False):
        if lmax_out is not None:
            if irreps_out is not None or instructions is not None:
                raise ValueError("give lmax_out or irreps_out/instructions, not both")
            irreps_out = "+".join(f"1x{l}{p}" for l in range(lmax_out + 1) for p in "eo")
        modes = {"uvu": 0, "uvw": 1, "uuu": 2, "uuw": 3}
        if mode not in modes:
            raise ValueError(f"unknown mode {mode!r}")
        if dtype not in _DTYPES:
            raise ValueError("dtype must be torch.float32 or torch.float64")
        n = 0
        arr = None
        if instructions is not None:
            n = len(instructions)
            arr = (Instruction * n)()
            for i, ins in enumerate(instructions):
                pw = float(ins[3]) if len(ins) > 3 else -1.0
                arr[i] = Instruction(int(ins[0]), int(ins[1]), int(ins[2]), 1, pw)
        handle = ctypes.c_void_p()
        self._handle = None
        _check(lib.e3_plan_create(irreps_in1.encode(), irreps_in2.encode(),
                                  None if irreps_out is None else irreps_out.encode(), arr, n, modes[mode],
                                  _DTYPES[dtype], 1 if shared_weights else 0, ctypes.byref(handle)))
        self._handle = handle
        self.dtype = dtype
        self.shared_weights = shared_weights
        self.device = torch.device("cuda", torch.cuda.current_device())
        d1, d2, do, wn = (ctypes.c_int64() for _ in range(4))
        npth = ctypes.c_int32()
        _check(lib.e3_plan_info(handle, ctypes.byref(d1), ctypes.byref(d2), ctypes.byref(do), ctypes.byref(wn),
                                ctypes.byref(npth)))
        self.dim_in1, self.dim_in2, self.dim_out = d1.value, d2.value, do.value
        self.weight_numel, self.n_paths = wn.value, npth.value
        need = ctypes.c_size_t()
        _check(lib.e3_plan_irreps_out(handle, None, 0, ctypes.byref(need)))
        buf = ctypes.create_string_buffer(need.value)
        _check(lib.e3_plan_irreps_out(handle, buf, need.value, None))
        self.irreps_out = buf.value.decode()
        lls = (ctypes.c_int32 * (3 * self.n_paths))()
        al = (ctypes.c_double * self.n_paths)()
        _check(lib.e3_plan_paths(handle, lls, al))
        self.paths = [tuple(lls[3 * p:3 * p + 3]) for p in range(self.n_paths)]
        self.alphas = list(al)
        self.irreps_in1, self.irreps_in2 = irreps_in1, irreps_in2

    def __del__(self):
        if getattr(self, "_handle", None) and lib is not None:
            try:
                lib.e3_plan_destroy(self._handle)
            except Exception:  # interpreter shutdown
                pass
            self._handle = None

    @property
    def handle(self):
        return self._handle

    def status(self):
        """Synchronise the current stream; raise E3Error if a kernel of a call made with this plan
        recorded an error since the last read (e3_plan_status)."""
        _check(lib.e3_plan_status(self._handle, _stream()))

    def _w_shape(self, rows):
        return (self.weight_numel,) if self.shared_weights else (rows, self.weight_numel)


def tp_forward(plan, x, y, w, out=None):
    """out[b] = TP(x[b], y[b], w[b]) (e3_tp_forward)."""
    B = x.shape[0]
    dev, dt = plan.device, plan.dtype
    _need(x, "x", dt, (B, plan.dim_in1), dev)
    _need(y, "y", dt, (B, plan.dim_in2), dev)
    _need(w, "w", dt, plan._w_shape(B), dev)
    if out is None:
        out = torch.empty((B, plan.dim_out), dtype=dt, device=dev)
    _need(out, "out", dt, (B, plan.dim_out), dev)
    _check(lib.e3_tp_forward(plan.handle, B, _ptr(x), _ptr(y), _ptr(w), _ptr(out), _stream()))
    return out


def tp_backward(plan, x, y, w, grad_out, need_x=True, need_y=True, need_w=True):
    """(grad_x, grad_y, grad_w) of <grad_out, TP(x, y, w)> (e3_tp_backward); skipped ones are None."""
    B = x.shape[0]
    dev, dt = plan.device, plan.dtype
    _need(x, "x", dt, (B, plan.dim_in1), dev)
    _need(y, "y", dt, (B, plan.dim_in2), dev)
    _need(w, "w", dt, plan._w_shape(B), dev)
    _need(grad_out, "grad_out", dt, (B, plan.dim_out), dev)
    gx = torch.empty_like(x) if need_x else None
    gy = torch.empty_like(y) if need_y else None
    gw = torch.empty_like(w) if need_w else None
    ws = backward_workspace(B, dev)
    _check(lib.e3_tp_backward(plan.handle, B, _ptr(x), _ptr(y), _ptr(w), _ptr(grad_out), _ptr(gx), _ptr(gy),
                              _ptr(gw), _ptr(ws), ws.numel(), _stream()))
    return gx, gy, gw


def conv_workspace(plan, n_nodes, n_edges, device):
    """Device workspace for e3_conv_forward / e3_conv_backward, from torch's allocator."""
    nbytes = ctypes.c_size_t()
    _check(lib.e3_conv_workspace_size(plan.handle, n_nodes, n_edges, ctypes.byref(nbytes)))
    return torch.empty(nbytes.value, dtype=torch.uint8, device=device)


def backward_workspace(n, device):
    """Device workspace for e3_tp_backward (n = B) / e3_conv_backward (n = N), from torch's allocator."""
    nbytes = ctypes.c_size_t()
    _check(lib.e3_backward_workspace_size(n, ctypes.byref(nbytes)))
    return torch.empty(nbytes.value, dtype=torch.uint8, device=device)


def spherical_harmonics(lmax, vec, sh_norm="component", out=None):
    """[n, (lmax+1)^2] real harmonics of vec [n, 3] (e3_spherical_harmonics)."""
    if vec.dtype not in _DTYPES:
        raise ValueError("vec must be float32 or float64")
    n = vec.shape[0]
    _need(vec, "vec", vec.dtype, (n, 3), vec.device)
    if out is None:
        out = torch.empty((n, (lmax + 1) ** 2), dtype=vec.dtype, device=vec.device)
    _need(out, "out", vec.dtype, (n, (lmax + 1) ** 2), vec.device)
    _check(lib.e3_spherical_harmonics(lmax, n, _ptr(vec), _SH_NORMS[sh_norm], _DTYPES[vec.dtype], _ptr(out),
                                      _stream()))
    return out


def spherical_harmonics_backward(lmax, vec, grad_y, sh_norm="component", out=None):
    """[n, 3] gradient of sum(grad_y * Y(vec)) with respect to vec (e3_spherical_harmonics_backward)."""
    if vec.dtype not in _DTYPES:
        raise ValueError("vec must be float32 or float64")
    n = vec.shape[0]
    _need(vec, "vec", vec.dtype, (n, 3), vec.device)
    _need(grad_y, "grad_y", vec.dtype, (n, (lmax + 1) ** 2), vec.device)
    if out is None:
        out = torch.empty((n, 3), dtype=vec.dtype, device=vec.device)
    _need(out, "out", vec.dtype, (n, 3), vec.device)
    _check(lib.e3_spherical_harmonics_backward(lmax, n, _ptr(vec), _SH_NORMS[sh_norm], _ptr(grad_y),
                                               _DTYPES[vec.dtype], _ptr(out), _stream()))
    return out


def spherical_harmonics_double_backward(lmax, vec, grad_y, u, sh_norm="component"):
    """(d_grad_y, d_vec): the backward of grad_vec = J(vec)^T grad_y for upstream u
    (e3_spherical_harmonics_double_backward)."""
    n = vec.shape[0]
    for t_, nm, sh_ in ((vec, "vec", (n, 3)), (grad_y, "grad_y", (n, (lmax + 1) ** 2)), (u, "u", (n, 3))):
        _need(t_, nm, vec.dtype, sh_, vec.device)
    d_gy = torch.empty((n, (lmax + 1) ** 2), dtype=vec.dtype, device=vec.device)
    d_vec = torch.empty((n, 3), dtype=vec.dtype, device=vec.device)
    _check(lib.e3_spherical_harmonics_double_backward(lmax, n, _ptr(vec), _SH_NORMS[sh_norm], _ptr(grad_y), _ptr(u),
                                                      _DTYPES[vec.dtype], _ptr(d_gy), _ptr(d_vec), _stream()))
    return d_gy, d_vec


class _ShFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, vec, lmax, sh_norm):
        ctx.lmax, ctx.sh_norm = lmax, sh_norm
        ctx.save_for_backward(vec)
        return spherical_harmonics(lmax, vec, sh_norm)

    @staticmethod
    def backward(ctx, g):
        (vec,) = ctx.saved_tensors
        return _ShBwdFn.apply(vec, g.contiguous(), ctx.lmax, ctx.sh_norm), None, None


class _ShBwdFn(torch.autograd.Function):
    """grad_vec = J(vec)^T grad_y as a differentiable function of (vec, grad_y)."""

    @staticmethod
    def forward(ctx, vec, gy, lmax, sh_norm):
        ctx.lmax, ctx.sh_norm = lmax, sh_norm
        ctx.save_for_backward(vec, gy)
        return spherical_harmonics_backward(lmax, vec, gy, sh_norm)

    @staticmethod
    def backward(ctx, u):
        vec, gy = ctx.saved_tensors
        d_gy, d_vec = spherical_harmonics_double_backward(ctx.lmax, vec, gy, u.contiguous(), ctx.sh_norm)
        return d_vec, d_gy, None, None


def sh(lmax, vec, sh_norm="component"):
    """Twice-differentiable real harmonics of vec [n, 3]."""
    return _ShFn.apply(vec, lmax, sh_norm)


def morton_order(pos, lo, extent):
    """int32 [N] node order along the Morton curve of pos [N, 3] inside the box [lo, lo + extent)
    (e3_morton_order): perm[i] is the id of the i-th node on the curve."""
    if pos.dtype not in _DTYPES:
        raise ValueError("pos must be float32 or float64")
    N = pos.shape[0]
    _need(pos, "pos", pos.dtype, (N, 3), pos.device)
    nbytes = ctypes.c_size_t()
    _check(lib.e3_morton_workspace_size(N, ctypes.byref(nbytes)))
    ws = torch.empty(nbytes.value, dtype=torch.uint8, device=pos.device)
    perm = torch.empty(N, dtype=torch.int32, device=pos.device)
    lo3, ext3 = (ctypes.c_double * 3)(*map(float, lo)), (ctypes.c_double * 3)(*map(float, extent))
    _check(lib.e3_morton_order(N, _ptr(pos), _DTYPES[pos.dtype], lo3, ext3, _ptr(perm), _ptr(ws), ws.numel(),
                               _stream()))
    return perm


def invert_permutation(perm):
    """inv with inv[perm[i]] = i (e3_invert_permutation)."""
    _need(perm, "perm", torch.int32, (perm.shape[0],), perm.device)
    inv = torch.empty_like(perm)
    _check(lib.e3_invert_permutation(perm.shape[0], _ptr(perm), _ptr(inv), _stream()))
    return inv


def remap_ids(ids, mapping):
    """mapping[ids] for int32 tensors (e3_remap_ids)."""
    _need(ids, "ids", torch.int32, (ids.shape[0],), ids.device)
    _need(mapping, "mapping", torch.int32, (mapping.shape[0],), ids.device)
    out = torch.empty_like(ids)
    _check(lib.e3_remap_ids(ids.shape[0], _ptr(ids), mapping.shape[0], _ptr(mapping), _ptr(out), _stream()))
    return out


def reorder_graph(pos, lo, extent, src, dst):
    """Morton renumbering of a graph: (perm, inv, src', dst') with src' = inv[src], dst' = inv[dst].
    Node rows of the new numbering are rows[perm] (gather_rows); results map back with rows[inv]."""
    perm = morton_order(pos, lo, extent)
    inv = invert_permutation(perm)
    return perm, inv, remap_ids(src, inv), remap_ids(dst, inv)


def csr_build(n_nodes, src, dst):
    """(perm_dst, row_ptr_dst, perm_src, row_ptr_src) of an int32 edge list (e3_csr_build)."""
    E = src.shape[0]
    dev = src.device
    _need(src, "src", torch.int32, (E,), dev)
    _need(dst, "dst", torch.int32, (E,), dev)
    nbytes = ctypes.c_size_t()
    _check(lib.e3_csr_workspace_size(n_nodes, E, ctypes.byref(nbytes)))
    ws = torch.empty((nbytes.value + 255) // 4 + 64, dtype=torch.int32, device=dev)
    off = (-ws.data_ptr()) % 256 // 4
    wsv = ws[off:]
    perm_dst = torch.empty(E, dtype=torch.int32, device=dev)
    perm_src = torch.empty(E, dtype=torch.int32, device=dev)
    rp_dst = torch.empty(n_nodes + 1, dtype=torch.int32, device=dev)
    rp_src = torch.empty(n_nodes + 1, dtype=torch.int32, device=dev)
    _check(lib.e3_csr_build(n_nodes, E, _ptr(src), _ptr(dst), _ptr(perm_dst), _ptr(rp_dst), _ptr(perm_src),
                            _ptr(rp_src), _ptr(wsv), nbytes.value, _stream()))
    return perm_dst, rp_dst, perm_src, rp_src


def gather_rows(perm, t, out=None):
    """out[i] = t[perm[i]] for a contiguous tensor t (e3_gather_rows)."""
    n = perm.shape[0]
    _need(perm, "perm", torch.int32, (n,), t.device)
    if not t.is_contiguous():
        raise ValueError("t must be contiguous")
    if out is None:
        out = torch.empty((n,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    row_bytes = t.element_size() * (t[0].numel() if t.dim() > 1 else 1)
    _check(lib.e3_gather_rows(n, t.shape[0], row_bytes, _ptr(perm), _ptr(t), _ptr(out), _stream()))
    return out


def add_rows_(out, idx, t):
    """out[idx[i]] += t[i] for distinct int32 indices (e3_add_rows); returns out."""
    n = idx.shape[0]
    _need(idx, "idx", torch.int32, (n,), out.device)
    if out.dtype not in _DTYPES:
        raise ValueError("out must be float32 or float64")
    _need(t, "t", out.dtype, (n,) + tuple(out.shape[1:]), out.device)
    if not out.is_contiguous():
        raise ValueError("out must be contiguous")
    row = out[0].numel() if out.dim() > 1 else 1
    _check(lib.e3_add_rows(n, out.shape[0], row, _DTYPES[out.dtype], _ptr(idx), _ptr(t), _ptr(out), _stream()))
    return out


class Radial:
    """The radial network w = SiLU(f(|v|) W1) W2 (Bessel basis x polynomial envelope) with W2 laid
    out once for the tensor cores (e3_radial_prepare); call ``weights(edge_vec)`` per step."""

    def __init__(self, w1, w2, cutoff, envelope_p=6):
        if w1.dtype != torch.float32 or w2.dtype != torch.float32:
            raise ValueError("the radial network runs in float32")
        if not (w1.is_contiguous() and w2.is_contiguous()) or w1.device != w2.device or w1.device.type != "cuda":
            raise ValueError("w1, w2 must be contiguous CUDA tensors on one device")
        self.n_basis, self.hidden = w1.shape
        if w2.shape[0] != self.hidden:
            raise ValueError("w2 must be [hidden, n_out]")
        self.n_out = w2.shape[1]
        self.cutoff, self.p, self.w1 = float(cutoff), int(envelope_p), w1
        nbytes = ctypes.c_size_t()
        _check(lib.e3_radial_prep_size(self.hidden, self.n_out, ctypes.byref(nbytes)))
        self.prep = torch.empty(nbytes.value, dtype=torch.uint8, device=w1.device)
        _check(lib.e3_radial_prepare(self.hidden, self.n_out, _ptr(w2), _ptr(self.prep), nbytes.value, _stream()))

    def weights(self, edge_vec, out=None):
        E = edge_vec.shape[0]
        _need(edge_vec, "edge_vec", torch.float32, (E, 3), self.w1.device)
        if out is None:
            out = torch.empty((E, self.n_out), dtype=torch.float32, device=self.w1.device)
        _need(out, "out", torch.float32, (E, self.n_out), self.w1.device)
        _check(lib.e3_radial_weights(E, _ptr(edge_vec), self.cutoff, self.n_basis, self.p, self.hidden, _ptr(self.w1),
                                     _ptr(self.prep), self.n_out, _ptr(out), _stream()))
        return out


class Graph:
    """A fixed topology in receiver order: CSR arrays plus src/dst permuted once (E3J,
    section E.2.2: CSR receiver aggregation).  ``perm_dst[i]`` is the original id of the
    i-th edge in receiver order; use ``to_receiver_order`` on per-edge arrays.  ``order``: an
    optional int32 permutation of the nodes in which the kernels process rows (for example the
    Morton order of the positions, ``morton_order``); results do not depend on it."""

    def __init__(self, n_nodes, src, dst, order=None):
        self.n_nodes = int(n_nodes)
        self.n_edges = int(src.shape[0])
        self.perm_dst, self.row_ptr_dst, self.perm_src, self.row_ptr_src = csr_build(self.n_nodes, src, dst)
        self.src = gather_rows(self.perm_dst, src)
        self.dst = gather_rows(self.perm_dst, dst)
        # the convolution's work units (rows cut into segments), built once for the topology
        nbytes = ctypes.c_size_t()
        _check(lib.e3_conv_topology_size(self.n_nodes, self.n_edges, ctypes.byref(nbytes)))
        self.topo = torch.empty(nbytes.value, dtype=torch.uint8, device=src.device)
        if order is not None:
            _need(order, "order", torch.int32, (self.n_nodes,), src.device)
        _check(lib.e3_conv_topology_build_ordered(self.n_nodes, self.n_edges, _ptr(self.row_ptr_dst),
                                                  _ptr(self.row_ptr_src), _ptr(order), _ptr(self.topo),
                                                  self.topo.numel(), _stream()))

    def to_receiver_order(self, t):
        return gather_rows(self.perm_dst, t.contiguous())


def conv_forward(plan, graph, x, w, y=None, edge_vec=None, sh_norm="component", out_scale=1.0, out=None):
    """out[n] = out_scale * sum_{e: dst_e = n} TP(x[src_e], Y_e, w_e) (e3_conv_forward).
    Edge arrays (w, y or edge_vec) are in the graph's receiver order."""
    N, E = graph.n_nodes, graph.n_edges
    dev, dt = plan.device, plan.dtype
    _need(x, "x", dt, (N, plan.dim_in1), dev)
    _need(w, "w", dt, plan._w_shape(E), dev)
    if (y is None) == (edge_vec is None):
        raise ValueError("give exactly one of y and edge_vec")
    if y is not None:
        _need(y, "y", dt, (E, plan.dim_in2), dev)
    else:
        _need(edge_vec, "edge_vec", dt, (E, 3), dev)
    if out is None:
        out = torch.empty((N, plan.dim_out), dtype=dt, device=dev)
    _need(out, "out", dt, (N, plan.dim_out), dev)
    ws = conv_workspace(plan, N, E, dev)
    _check(lib.e3_conv_forward(plan.handle, N, E, _ptr(graph.row_ptr_dst), _ptr(graph.src), _ptr(x), _ptr(y),
                               _ptr(edge_vec), _SH_NORMS[sh_norm], _ptr(w), float(out_scale), _ptr(out),
                               _ptr(graph.topo), _ptr(ws), ws.numel(), _stream()))
    return out


def conv_backward(plan, graph, x, w, grad_out, y=None, edge_vec=None, sh_norm="component", out_scale=1.0,
                  need_x=True, need_y=True, need_w=True):
    """(grad_x, grad_y, grad_w) of <grad_out, conv_forward(...)> (e3_conv_backward)."""
    N, E = graph.n_nodes, graph.n_edges
    dev, dt = plan.device, plan.dtype
    _need(x, "x", dt, (N, plan.dim_in1), dev)
    _need(w, "w", dt, (E, plan.weight_numel), dev)
    _need(grad_out, "grad_out", dt, (N, plan.dim_out), dev)
    if (y is None) == (edge_vec is None):
        raise ValueError("give exactly one of y and edge_vec")
    if y is not None:
        _need(y, "y", dt, (E, plan.dim_in2), dev)
    else:
        _need(edge_vec, "edge_vec", dt, (E, 3), dev)
    gx = torch.empty_like(x) if need_x else None
    gy = torch.empty((E, plan.dim_in2), dtype=dt, device=dev) if need_y else None
    gw = torch.empty_like(w) if need_w else None
    ws = conv_workspace(plan, N, E, dev)
    _check(lib.e3_conv_backward(plan.handle, N, E, _ptr(graph.row_ptr_dst), _ptr(graph.src), _ptr(graph.dst),
                                _ptr(graph.row_ptr_src), _ptr(graph.perm_src), _ptr(x), _ptr(y), _ptr(edge_vec),
                                _SH_NORMS[sh_norm], _ptr(w), _ptr(grad_out), float(out_scale), _ptr(gx),
                                _ptr(gy), _ptr(gw), _ptr(graph.topo), _ptr(ws), ws.numel(), _stream()))
    return gx, gy, gw


def _accumulate(acc, t):
    """acc + t for same-shape tensors through the library (e3_add_rows with the identity rows)."""
    if t is None:
        return acc
    if acc is None:
        return t.contiguous().clone()
    n = acc.shape[0]
    idx = torch.arange(n, dtype=torch.int32, device=acc.device)
    return add_rows_(acc.contiguous(), idx, t.contiguous())


class _ConvFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, y, w, plan, graph, out_scale):
        ctx.plan, ctx.graph, ctx.out_scale = plan, graph, out_scale
        ctx.save_for_backward(x, y, w)
        return conv_forward(plan, graph, x, w, y=y, out_scale=out_scale)

    @staticmethod
    def backward(ctx, g):
        x, y, w = ctx.saved_tensors
        gx, gy, gw = _ConvBwdFn.apply(x, y, w, g.contiguous(), ctx.plan, ctx.graph, ctx.out_scale,
                                      tuple(ctx.needs_input_grad[:3]))
        return gx, gy, gw, None, None, None


class _ConvBwdFn(torch.autograd.Function):
    """The convolution's backward as a differentiable function of (x, y, w, grad_out), so that the
    convolution is twice differentiable (xnn, "Run Models on Fused GPU Kernels", Training: force
    training runs through the fast path).  The convolution F(x, y, w) is linear in each argument,
    so with B_x, B_y, B_w its three gradients and upstream (u_x, u_y, u_w) for them,
        d/dg = F(u_x, y, w) + F(x, u_y, w) + F(x, y, u_w)
        d/dx = B_x(x, u_y, w, g) + B_x(x, y, u_w, g)
        d/dy = B_y(u_x, y, w, g) + B_y(x, y, u_w, g)
        d/dw = B_w(u_x, y, w, g) + B_w(x, u_y, w, g)
    (e.g. <u_y, B_y(x, w, g)> = <g, F(x, u_y, w)>, whose x-gradient is B_x with y -> u_y), each
    term one call of the library's forward or backward kernels, sums by e3_add_rows."""

    @staticmethod
    def forward(ctx, x, y, w, g, plan, graph, out_scale, needs):
        ctx.plan, ctx.graph, ctx.out_scale = plan, graph, out_scale
        ctx.save_for_backward(x, y, w, g)
        gx, gy, gw = conv_backward(plan, graph, x, w, g, y=y, out_scale=out_scale, need_x=needs[0], need_y=needs[1],
                                   need_w=needs[2])
        return gx, gy, gw

    @staticmethod
    def backward(ctx, ux, uy, uw):
        x, y, w, g = ctx.saved_tensors
        P, G, s = ctx.plan, ctx.graph, ctx.out_scale
        nx, ny, nw, ng = ctx.needs_input_grad[:4]
        ux = None if ux is None else ux.contiguous()
        uy = None if uy is None else uy.contiguous()
        uw = None if uw is None else uw.contiguous()
        dx = dy = dw = dg = None
        if ng:
            if ux is not None:
                dg = _accumulate(dg, conv_forward(P, G, ux, w, y=y, out_scale=s))
            if uy is not None:
                dg = _accumulate(dg, conv_forward(P, G, x, w, y=uy, out_scale=s))
            if uw is not None:
                dg = _accumulate(dg, conv_forward(P, G, x, uw, y=y, out_scale=s))
        if uy is not None and (nx or nw):  # y -> u_y: its x- and w-gradients
            bx, _, bw = conv_backward(P, G, x, w, g, y=uy, out_scale=s, need_x=nx, need_y=False, need_w=nw)
            dx, dw = _accumulate(dx, bx), _accumulate(dw, bw)
        if uw is not None and (nx or ny):  # w -> u_w: its x- and y-gradients
            bx, by, _ = conv_backward(P, G, x, uw, g, y=y, out_scale=s, need_x=nx, need_y=ny, need_w=False)
            dx, dy = _accumulate(dx, bx), _accumulate(dy, by)
        if ux is not None and (ny or nw):  # x -> u_x: its y- and w-gradients
            _, by, bw = conv_backward(P, G, ux, w, g, y=y, out_scale=s, need_x=False, need_y=ny, need_w=nw)
            dy, dw = _accumulate(dy, by), _accumulate(dw, bw)
        return dx, dy, dw, dg, None, None, None, None


def conv(plan, graph, x, y, w, out_scale=1.0):
    """Twice-differentiable convolution with respect to x, y (harmonics) and w."""
    return _ConvFn.apply(x, y, w, plan, graph, out_scale)


class _ConvVecFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, vec, w, plan, graph, out_scale, sh_norm):
        ctx.plan, ctx.graph, ctx.out_scale, ctx.sh_norm = plan, graph, out_scale, sh_norm
        ctx.save_for_backward(x, vec, w)
        return conv_forward(plan, graph, x, w, edge_vec=vec, sh_norm=sh_norm, out_scale=out_scale)

    @staticmethod
    def backward(ctx, g):
        x, vec, w = ctx.saved_tensors
        need_vec = ctx.needs_input_grad[1]
        gx, gy, gw = conv_backward(ctx.plan, ctx.graph, x, w, g.contiguous(), edge_vec=vec, sh_norm=ctx.sh_norm,
                                   out_scale=ctx.out_scale, need_x=ctx.needs_input_grad[0], need_y=need_vec,
                                   need_w=ctx.needs_input_grad[2])
        lmax = int(ctx.plan.dim_in2 ** 0.5 + 0.5) - 1  # harmonics irreps 1x0e+1x1o+... of dim (lmax+1)^2
        gvec = spherical_harmonics_backward(lmax, vec, gy, ctx.sh_norm) if need_vec else None
        return gx, gvec, gw, None, None, None, None


def conv_vec(plan, graph, x, edge_vec, w, out_scale=1.0, sh_norm="component"):
    """Differentiable convolution with harmonics computed in the kernels from edge vectors
    (receiver order): gradients with respect to x, edge_vec (through the harmonics) and w."""
    return _ConvVecFn.apply(x, edge_vec, w, plan, graph, out_scale, sh_norm)
