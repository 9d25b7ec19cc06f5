"""The radial network on the tensor cores (e3_radial_weights) against the float64 oracle: the
Bessel basis times the polynomial envelope, the SiLU hidden layer and the output layer, whose
contraction runs as three tf32 passes with float32 accumulation.  fp32 results must match to an
infinity-norm relative error <= 1e-5 (per output column block and overall)."""

import math

import numpy as np
import pytest
import torch

import oracle
from mlip_message_passing_b200 import workloads as W
from tests.conftest import rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def e3b():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from mlip_message_passing_b200 import e3b
    return e3b


def _case(e3b, E, n_basis, hidden, n_out, seed, cutoff=5.0, p=6):
    rng = np.random.default_rng(seed)
    vec = rng.standard_normal((E, 3)) * 2.2
    vec[0] = 0.0                      # zero vector: the r -> 0 limit of the basis
    vec[1] = [cutoff * 1.01, 0, 0]    # beyond the cutoff: zero weights
    vec = vec.astype(np.float32)
    w1 = (rng.standard_normal((n_basis, hidden)) / math.sqrt(n_basis)).astype(np.float32)
    w2 = (rng.standard_normal((hidden, n_out)) / math.sqrt(hidden)).astype(np.float32)
    rad = e3b.Radial(torch.as_tensor(w1, device=DEV), torch.as_tensor(w2, device=DEV), cutoff, p)
    out = rad.weights(torch.as_tensor(vec, device=DEV))
    e3b.device_status()
    ref = oracle.radial_weights(vec.astype(np.float64), cutoff, n_basis, p, w1, w2)
    return out.cpu().numpy().astype(np.float64), ref


@pytest.mark.parametrize("E,n_basis,hidden,n_out", [
    (1000, 8, 64, 1152),   # water-box weights (18 paths x 64 channels); ragged last edge tile
    (777, 8, 64, 4352),    # large-convolution weights (34 paths x 128 channels)
    (300, 5, 32, 100),     # one partial column tile, K = 32
    (129, 16, 8, 4),       # the smallest shapes: K = 8, n_out = 4
])
def test_radial_weights_match_oracle(e3b, E, n_basis, hidden, n_out):
    got, ref = _case(e3b, E, n_basis, hidden, n_out, seed=E + n_out)
    assert rel_err(got, ref) <= 1e-5
    for c0 in range(0, n_out, 128):  # every output column tile on its own scale
        assert rel_err(got[:, c0:c0 + 128], ref[:, c0:c0 + 128]) <= 1e-5
    assert np.all(got[1] == 0.0)      # beyond the cutoff


def test_radial_weights_full_size_sampled(e3b):
    """All 1.26 M edges of the large convolution's graph, 4352 weights each (21.9 GB), in one
    launch; 3000 sampled edges against the oracle."""
    cfg = W.CONFIGS["conv_large"]
    g = W.graph_inputs(cfg["N"], cfg["mul"], cfg["lx"], cfg["ly"], cfg["lo"], cfg["seed"], weights="none")
    w1, w2 = (m.astype(np.float32) for m in g["mlp"])
    rad = e3b.Radial(torch.as_tensor(w1, device=DEV), torch.as_tensor(w2, device=DEV), W.CUTOFF, W.ENVELOPE_P)
    vec = torch.as_tensor(g["vec"].astype(np.float32), device=DEV)
    out = rad.weights(vec)
    e3b.device_status()
    idx = np.sort(np.random.default_rng(3).choice(vec.shape[0], 3000, replace=False))
    got = out[torch.as_tensor(idx, device=DEV)].cpu().numpy().astype(np.float64)
    ref = oracle.radial_weights(g["vec"][idx].astype(np.float32).astype(np.float64), W.CUTOFF, W.N_BASIS,
                                W.ENVELOPE_P, w1, w2)
    assert rel_err(got, ref) <= 1e-5
    del out
    torch.cuda.empty_cache()


def test_radial_rejects_unsupported_shapes(e3b):
    import ctypes
    nb = ctypes.c_size_t()
    assert e3b.lib.e3_radial_prep_size(12, 64, ctypes.byref(nb)) == e3b.E3_ERR_UNSUPPORTED
    assert e3b.lib.e3_radial_prep_size(72, 64, ctypes.byref(nb)) == e3b.E3_ERR_UNSUPPORTED
    assert e3b.lib.e3_radial_prep_size(64, 6, ctypes.byref(nb)) == e3b.E3_ERR_SHAPE
    assert e3b.lib.e3_radial_prep_size(64, 1152, ctypes.byref(nb)) == e3b.E3_OK
    assert nb.value == 9 * 2 * 128 * 64 * 4
