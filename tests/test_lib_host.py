"""Host-side checks of the C-ABI library that need no GPU: every declared symbol is exported,
argument validation returns the documented status before any launch, and the library's CG
table (ladder construction) equals the oracle's (Racah formula) -- two independent generators."""

import ctypes
import itertools
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "e3b.h")


@pytest.fixture(scope="module")
def e3b():
    from mlip_message_passing_b200 import e3b
    return e3b


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^E3_API\s+[\w\s\*]+?\b(e3_\w+)\s*\(", txt, flags=re.M)))


def test_library_exports_every_declared_symbol(e3b):
    decl = declared_symbols()
    assert len(decl) >= 15
    raw = ctypes.CDLL(e3b.LIB_PATH)
    for name in decl:
        assert hasattr(raw, name), name
    assert sorted(e3b.SYMBOLS) == decl


def test_ladder_cg_equals_racah_cg(e3b):
    import oracle
    for l1, l2 in itertools.product(range(4), range(4)):
        for l3 in range(abs(l1 - l2), min(l1 + l2, 3) + 1):
            lib = e3b.cg_dense(l1, l2, l3).numpy()
            np.testing.assert_allclose(lib, oracle.real_cg(l1, l2, l3), atol=1e-14, rtol=0)


def test_cg_dense_errors(e3b):
    out = (ctypes.c_double * 64)()
    assert e3b.lib.e3_cg_dense(1, 1, 3, out) == e3b.E3_ERR_INSTRUCTION
    assert e3b.lib.e3_cg_dense(4, 0, 4, out) == e3b.E3_ERR_UNSUPPORTED
    assert e3b.lib.e3_cg_dense(1, 1, 1, None) == e3b.E3_ERR_INVALID_ARG


def _create(e3b, a, b, c=None, instr=None, mode=0, dtype=0, wmode=0):
    h = ctypes.c_void_p()
    arr, n = None, 0
    if instr is not None:
        n = len(instr)
        arr = (e3b.Instruction * n)(*[e3b.Instruction(i, j, k, 1, -1.0) for i, j, k in instr])
    st = e3b.lib.e3_plan_create(a.encode(), b.encode(), None if c is None else c.encode(), arr, n, mode, dtype,
                                wmode, ctypes.byref(h))
    return st, e3b.lib.e3_last_error().decode()


@pytest.mark.parametrize("a,b,code", [
    ("8x0e+8x1q", "1x0e", "IRREPS_PARSE"),
    ("8x0e+", "1x0e", "IRREPS_PARSE"),
    ("", "1x0e", "IRREPS_PARSE"),
    ("8x0e", "x1o", "IRREPS_PARSE"),
])
def test_plan_parse_errors(e3b, a, b, code):
    st, msg = _create(e3b, a, b)
    assert e3b.STATUS_NAMES[st] == code and msg


def test_plan_instruction_errors(e3b):
    st, msg = _create(e3b, "8x1o", "1x1o", "8x0o", instr=[(0, 0, 0)])
    assert st == e3b.E3_ERR_INSTRUCTION and "parity" in msg
    st, msg = _create(e3b, "8x1o", "1x1o", "8x3e", instr=[(0, 0, 0)])
    assert st == e3b.E3_ERR_INSTRUCTION and "triangle" in msg
    st, msg = _create(e3b, "8x1o", "1x1o", "8x0e", instr=[(0, 1, 0)])
    assert st == e3b.E3_ERR_INSTRUCTION and "range" in msg
    st, msg = _create(e3b, "8x1o", "1x1o", "4x0e", instr=[(0, 0, 0)])
    assert st == e3b.E3_ERR_INSTRUCTION


def test_plan_unsupported(e3b):
    # unsupported layouts, degrees without compiled kernels
    assert _create(e3b, "8x0e+4x1o", "1x0e+1x1o+1x2e")[0] == e3b.E3_ERR_UNSUPPORTED
    assert _create(e3b, "8x1o+8x0e", "1x0e+1x1o+1x2e")[0] == e3b.E3_ERR_UNSUPPORTED
    assert _create(e3b, "6x0e+6x1o", "1x0e+1x1o+1x2e")[0] == e3b.E3_ERR_UNSUPPORTED
    assert _create(e3b, "8x0e+8x1o+8x2e+8x3o+8x4e", "1x0e+1x1o")[0] == e3b.E3_ERR_UNSUPPORTED
    # an output filter that drops a path of the enumeration
    st, msg = _create(e3b, "8x0e+8x1o", "1x0e+1x1o+1x2e", "1x0e+1x1o+1x2e")
    assert st == e3b.E3_ERR_UNSUPPORTED and "every path" in msg
    assert _create(e3b, "8x0e+8x1o", "1x0e+1x1o+1x2e", dtype=7)[0] == e3b.E3_ERR_INVALID_ARG
    assert _create(e3b, "8x0e+8x1o", "1x0e+1x1o+1x2e", mode=3)[0] == e3b.E3_ERR_UNSUPPORTED
    assert _create(e3b, "8x0e+8x1o", "1x0e+1x1o+1x2e", mode=9)[0] == e3b.E3_ERR_INVALID_ARG


def test_plan_uvw_validation(e3b):
    # the fully connected mode needs output blocks, shared float32 weights and multiplicities in {32..128}
    st, msg = _create(e3b, "32x0e+32x1o", "1x0e+1x1o", mode=1)
    assert st == e3b.E3_ERR_INSTRUCTION and "irreps_out" in msg
    st, msg = _create(e3b, "32x0e+32x1o", "1x0e+1x1o", "32x0e+32x1o", mode=1)
    assert st == e3b.E3_ERR_UNSUPPORTED and "shared" in msg
    st, msg = _create(e3b, "32x0e+32x1o", "1x0e+1x1o", "32x0e+32x1o", mode=1, wmode=1, dtype=1)
    assert st == e3b.E3_ERR_UNSUPPORTED and "float32" in msg
    st, msg = _create(e3b, "16x0e+16x1o", "1x0e+1x1o", "32x0e+32x1o", mode=1, wmode=1)
    assert st == e3b.E3_ERR_UNSUPPORTED and "multiplicities" in msg
    st, msg = _create(e3b, "32x0e+32x1o", "1x0e+1x1o", "32x0e+64x1o", mode=1, wmode=1)
    assert st == e3b.E3_ERR_UNSUPPORTED and "common multiplicity" in msg
    st, msg = _create(e3b, "32x0e", "1x0e", "32x1o", mode=1, wmode=1)
    assert st == e3b.E3_ERR_INSTRUCTION and "no allowed path" in msg
    st, msg = _create(e3b, "32x1o", "1x1o", "32x0o", instr=[(0, 0, 0)], mode=1, wmode=1)
    assert st == e3b.E3_ERR_INSTRUCTION and "parity" in msg


def test_plan_uuu_validation(e3b):
    # uuu ties the channels of both inputs: y needs the multiplicity of x
    st, msg = _create(e3b, "8x0e+8x1o", "1x0e+1x1o", mode=2)
    assert st == e3b.E3_ERR_UNSUPPORTED and "uuu" in msg
    st, msg = _create(e3b, "8x1o", "4x1o", "8x0e", instr=[(0, 0, 0)], mode=2)
    assert st == e3b.E3_ERR_INSTRUCTION and "mul_in2" in msg
    st, msg = _create(e3b, "8x1o", "8x1o", "4x0e", instr=[(0, 0, 0)], mode=2)
    assert st == e3b.E3_ERR_INSTRUCTION and "mul_out" in msg


def test_supported_list(e3b):
    s = e3b.supported()
    assert (1, 2, 2) in s and (2, 3, 2) in s and (3, 3, 3) in s


def test_csr_workspace_and_argument_errors(e3b):
    n = ctypes.c_size_t()
    assert e3b.lib.e3_csr_workspace_size(3000, 156278, ctypes.byref(n)) == e3b.E3_OK and n.value > 4 * 156278 * 4
    assert e3b.lib.e3_csr_workspace_size(-1, 5, ctypes.byref(n)) == e3b.E3_ERR_SHAPE
    assert e3b.lib.e3_gather_rows(4, 4, 6, None, None, None, None) == e3b.E3_ERR_SHAPE
    assert e3b.lib.e3_spherical_harmonics(4, 10, None, 0, 0, None, None) == e3b.E3_ERR_UNSUPPORTED
    assert e3b.lib.e3_tp_forward(None, 1, None, None, None, None, None) == e3b.E3_ERR_INVALID_ARG


def test_backward_workspace_size(e3b):
    n = ctypes.c_size_t()
    for units in (0, 1, 3000, 1 << 20):
        assert e3b.lib.e3_backward_workspace_size(units, ctypes.byref(n)) == e3b.E3_OK
        assert n.value >= 16 + 4 * units and n.value % 256 == 0
    assert e3b.lib.e3_backward_workspace_size(-1, ctypes.byref(n)) == e3b.E3_ERR_SHAPE
    assert e3b.lib.e3_backward_workspace_size(1 << 31, ctypes.byref(n)) == e3b.E3_ERR_SHAPE
    assert e3b.lib.e3_backward_workspace_size(5, None) == e3b.E3_ERR_INVALID_ARG


def test_conv_topology_and_workspace_sizes(e3b):
    n = ctypes.c_size_t()
    assert e3b.lib.e3_conv_topology_size(3000, 156278, ctypes.byref(n)) == e3b.E3_OK
    # two directions, each: units (N + E/256 + 1) x (16 + 4 bytes) + row offsets (N + 1) x 4 bytes
    units = 3000 + 156278 // 256 + 1
    assert n.value >= 2 * (20 * units + 4 * 3001) and n.value % 256 == 0
    assert e3b.lib.e3_conv_topology_size(-1, 5, ctypes.byref(n)) == e3b.E3_ERR_SHAPE
    assert e3b.lib.e3_conv_topology_size(5, 5, None) == e3b.E3_ERR_INVALID_ARG
    assert e3b.lib.e3_conv_topology_build(4, 4, None, None, None, 0, None) == e3b.E3_ERR_INVALID_ARG
    assert e3b.lib.e3_conv_workspace_size(None, 5, 5, ctypes.byref(n)) == e3b.E3_ERR_INVALID_ARG


def test_c_abi_from_plain_c(e3b, tmp_path):
    """The header compiles as C (gcc, -std=c11), the library links, host-only calls answer."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    exe = tmp_path / "abi_host"
    src = os.path.join(ROOT, "tests", "c", "abi_host.c")
    lib_dir = os.path.dirname(e3b.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src, "-o", str(exe),
                        "-L", lib_dir, "-l:libe3b.so", "-Wl,-rpath," + lib_dir, "-lm"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FAIL" not in r.stdout


def test_test_knobs_validate_and_reset(e3b):
    # host-only: negative values are refused before anything changes; (0, 0) restores the defaults
    assert e3b.lib.e3_set_test_knobs(-1, 0) == e3b.E3_ERR_INVALID_ARG
    assert e3b.lib.e3_set_test_knobs(0, -3) == e3b.E3_ERR_INVALID_ARG
    assert e3b.lib.e3_set_test_knobs(5_000_000, 1) == e3b.E3_OK
    assert e3b.lib.e3_set_test_knobs(0, 0) == e3b.E3_OK
