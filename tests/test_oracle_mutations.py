"""Planted mistakes in the oracle must be caught by its pins.

Each case patches one oracle routine with a plausible bug (a flipped sign, transposed operands, a
dropped factor or term, a wrong index) and runs the pins that should see it; the case passes only
if at least one of them fails.  Everything runs on the CPU."""

import numpy as np
import pytest

import oracle
import oracle.cg as ocg
import oracle.conv as oconv
import oracle.sh as osh
import oracle.tp as otp
from tests import test_oracle_pins as pins


def _caught(checks):
    """True when one check fails an assertion.  A check that raises ValueError (a mutation that
    breaks the shapes of that check's inputs) does not count as catching it."""
    for fn in checks:
        try:
            fn()
        except AssertionError:
            return True
        except ValueError:
            continue
    return False


def _patch_cg(monkeypatch, fn):
    orig = ocg.real_cg

    def bad(l1, l2, l3):
        return fn(l1, l2, l3, np.array(orig(l1, l2, l3)))

    monkeypatch.setattr(ocg, "real_cg", bad)
    monkeypatch.setattr(otp, "real_cg", bad)
    monkeypatch.setattr(pins, "real_cg", bad)


CG_PINS = [pins.test_real_cg_1x1_is_dot_cross_symtraceless,
           lambda: pins.test_real_cg_orthogonality(1, 2),
           lambda: pins.test_real_cg_equivariance(1, 2),
           lambda: pins.test_real_cg_equivariance(2, 2),
           lambda: pins.test_tp_equivariance_o3(False)]


def test_flipped_cg_entry(monkeypatch):
    def f(l1, l2, l3, t):
        if (l1, l2, l3) == (1, 2, 2):
            idx = tuple(np.argwhere(np.abs(t) > 1e-9)[0])
            t[idx] = -t[idx]
        return t
    _patch_cg(monkeypatch, f)
    assert _caught(CG_PINS)


def test_transposed_cg_operands(monkeypatch):
    _patch_cg(monkeypatch, lambda l1, l2, l3, t: t.transpose(1, 0, 2) if l1 == l2 else t)
    assert _caught([pins.test_real_cg_1x1_is_dot_cross_symtraceless])


def test_cg_wrong_sign_convention(monkeypatch):
    _patch_cg(monkeypatch, lambda l1, l2, l3, t: -t if (l1 + l2 + l3) % 2 else t)
    assert _caught([pins.test_real_cg_1x1_is_dot_cross_symtraceless])


def test_sh_wrong_sin_sign(monkeypatch):
    orig = osh.real_sh

    def bad(l, vec):
        y = orig(l, vec)
        if l >= 1:
            y[:, :l] = -y[:, :l]
        return y

    monkeypatch.setattr(osh, "real_sh", bad)
    monkeypatch.setattr(pins, "real_sh", bad)
    assert _caught([pins.test_sh_closed_forms_low_degree])


def test_sh_dropped_sqrt2(monkeypatch):
    orig = osh.real_sh

    def bad(l, vec):
        y = orig(l, vec)
        if l >= 1:
            y[:, l + 1:] /= np.sqrt(2.0)
        return y

    monkeypatch.setattr(pins, "real_sh", bad)
    assert _caught([lambda: pins.test_sh_norm_parity_and_scale_invariance(2)])


def test_tp_dropped_path_weight(monkeypatch):
    orig = otp.tp_forward

    def bad(plan, x, y, w):
        saved = list(plan.alphas)
        plan.alphas = [1.0] * len(saved)
        try:
            return orig(plan, x, y, w)
        finally:
            plan.alphas = saved

    monkeypatch.setattr(oracle, "tp_forward", bad)
    assert _caught([pins.test_tp_matches_brute_force_loops])


def test_tp_transposed_uv_weights(monkeypatch):
    orig = otp._weights

    def bad2(plan, w, p, bsz):
        ws = orig(plan, w, p, bsz)
        a, b = ws.shape[1], ws.shape[2]
        return ws.reshape(bsz, -1)[:, ::-1].reshape(bsz, a, b)

    monkeypatch.setattr(otp, "_weights", bad2)
    assert _caught([pins.test_tp_multiplicity_two_inputs_brute_force])


def test_backward_dropped_alpha_in_dy(monkeypatch):
    orig = otp.tp_backward

    def bad(plan, x, y, w, g):
        dx, dy, dw = orig(plan, x, y, w, g)
        return dx, dy * 0.5, dw

    monkeypatch.setattr(oracle, "tp_backward", bad)
    assert _caught([lambda: pins.test_tp_backward_euler_identities_and_fd("uvu")])


def test_conv_double_scale(monkeypatch):
    orig = oconv.conv_forward

    def bad(plan, n, src, dst, x, y, w, scale, chunk=4096):
        return orig(plan, n, src, dst, x, y, w, scale * scale, chunk)

    monkeypatch.setattr(oracle, "conv_forward", bad)
    assert _caught([pins.test_conv_edge_order_invariance_isolated_and_empty])


def test_csr_unstable_sort(monkeypatch):
    def bad(n, src, dst):
        src = np.asarray(src)
        dst = np.asarray(dst)
        perm_dst = np.lexsort((-np.arange(len(dst)), dst))  # ties in reverse input order
        rp = np.concatenate([[0], np.cumsum(np.bincount(dst, minlength=n))])
        perm_src = np.argsort(src[perm_dst], kind="stable")
        rps = np.concatenate([[0], np.cumsum(np.bincount(src, minlength=n))])
        return perm_dst.astype(np.int32), rp.astype(np.int32), perm_src.astype(np.int32), rps.astype(np.int32)

    monkeypatch.setattr(oracle, "csr_build", bad)
    assert _caught([pins.test_csr_bit_exact_against_loops])


SH_GRAD_PINS = [lambda: pins.test_sh_grad_matches_central_differences(2),
                lambda: pins.test_sh_grad_matches_central_differences(3),
                pins.test_sh_grad_closed_form_l1,
                lambda: pins.test_sh_grad_radial_scaling_and_rotation(2)]


def _patch_sh_grad(monkeypatch, src_old, src_new):
    """Recompile real_sh_grad with one line changed."""
    import inspect
    import textwrap
    src = textwrap.dedent(inspect.getsource(osh.real_sh_grad))
    assert src_old in src
    ns = dict(vars(osh))
    exec(compile(src.replace(src_old, src_new), "mutant", "exec"), ns)
    monkeypatch.setattr(osh, "real_sh_grad", ns["real_sh_grad"])
    monkeypatch.setattr(oracle, "real_sh_grad", ns["real_sh_grad"])


def test_sh_grad_without_radial_projection(monkeypatch):
    _patch_sh_grad(monkeypatch, "(gu[nz] - radial[nz][:, :, None] * u[nz][:, None, :])", "gu[nz]")
    assert _caught(SH_GRAD_PINS)


def test_sh_grad_y_derivative_missing_i(monkeypatch):
    _patch_sh_grad(monkeypatch, "pick(1j * dtrig)", "pick(dtrig)")
    assert _caught(SH_GRAD_PINS)


def test_sh_grad_wrong_legendre_derivative(monkeypatch):
    _patch_sh_grad(monkeypatch, "dp1 = pl.deriv(am + 1)", "dp1 = pl.deriv(am)")
    assert _caught(SH_GRAD_PINS)


def test_morton_axes_swapped(monkeypatch):
    import inspect
    import textwrap
    import oracle.reorder as ore
    src = textwrap.dedent(inspect.getsource(ore.morton_codes))
    ns = dict(vars(ore))
    exec(compile(src.replace("<< (3 * b + k)", "<< (3 * b + 2 - k)"), "mutant", "exec"), ns)
    monkeypatch.setattr(ore, "morton_codes", ns["morton_codes"])
    monkeypatch.setattr(oracle, "morton_codes", ns["morton_codes"])
    bad_order = lambda pos, lo, ext: np.argsort(ns["morton_codes"](pos, lo, ext), kind="stable").astype(np.int32)
    monkeypatch.setattr(ore, "morton_order", bad_order)
    monkeypatch.setattr(oracle, "morton_order", bad_order)
    assert _caught([pins.test_morton_order_equals_octree_order, pins.test_morton_codes_known_cells_and_clamping])


ALPHA_PINS = [lambda: pins.test_default_path_weight_gives_unit_second_moment("uncollapsed"),
              lambda: pins.test_default_path_weight_gives_unit_second_moment("collapsed"),
              lambda: pins.test_default_path_weight_gives_unit_second_moment("mul_y2"),
              pins.test_default_path_weight_unit_moment_over_the_sphere,
              pins.test_default_path_weight_closed_forms_1x1]


def _patch_alpha(monkeypatch, formula):
    """Recompute every default path weight of the plans make_plan builds with another formula
    of (l3, mul_y, n_out)."""
    orig = otp.make_plan

    def bad(*args, **kwargs):
        plan = orig(*args, **kwargs)
        n_out = {}
        for ins in plan.instructions:
            n_out[ins.i_out] = n_out.get(ins.i_out, 0) + 1
        plan.alphas = [formula(plan.irreps_out[ins.i_out].l, plan.irreps_in2[ins.i_in2].mul, n_out[ins.i_out])
                       if ins.path_weight < 0 else a for ins, a in zip(plan.instructions, plan.alphas)]
        return plan

    monkeypatch.setattr(otp, "make_plan", bad)
    monkeypatch.setattr(oracle, "make_plan", bad)


@pytest.mark.parametrize("name,formula", [
    ("inverted", lambda l3, mv, no: np.sqrt(1.0 / ((2 * l3 + 1) * mv * no))),
    ("no_n_out", lambda l3, mv, no: np.sqrt((2 * l3 + 1) / mv)),
    ("no_mul_y", lambda l3, mv, no: np.sqrt((2 * l3 + 1) / no)),
    ("dimension_not_sqrt", lambda l3, mv, no: (2 * l3 + 1) / (mv * no)),
    ("l3_plus_one", lambda l3, mv, no: np.sqrt((l3 + 1) / (mv * no))),
])
def test_wrong_default_path_weight(monkeypatch, name, formula):
    _patch_alpha(monkeypatch, formula)
    assert _caught(ALPHA_PINS)


def test_right_default_path_weight_passes(monkeypatch):
    # the harness itself: the stated formula re-applied leaves every pin green
    _patch_alpha(monkeypatch, lambda l3, mv, no: np.sqrt((2 * l3 + 1) / (mv * no)))
    assert not _caught(ALPHA_PINS)


MODE_PINS = [lambda: pins.test_tp_modes_brute_force("uuu"), lambda: pins.test_tp_modes_brute_force("uvw"),
             lambda: pins.test_tp_modes_brute_force("uvw_fans"),
             lambda: pins.test_default_path_weight_gives_unit_second_moment("uvw_fans"),
             pins.test_modes_coincide_at_multiplicity_one, pins.test_uuu_is_uvu_on_the_diagonal,
             pins.test_scalar_path_modes_closed_forms,
             lambda: pins.test_default_path_weight_gives_unit_second_moment("uuu"),
             lambda: pins.test_default_path_weight_gives_unit_second_moment("uvw"),
             lambda: pins.test_tp_modes_equivariance_o3("uuu"), lambda: pins.test_tp_modes_equivariance_o3("uvw"),
             lambda: pins.test_tp_backward_euler_identities_and_fd("uuu"),
             lambda: pins.test_tp_backward_euler_identities_and_fd("uvw")]


@pytest.mark.parametrize("mode,eq", [
    ("uuu", "bui,bvj,ijk,bu->buk"),      # y summed over all channels instead of tied
    ("uvw", "bui,bvj,ijk,bvuw->bwk"),    # u and v of the weights transposed
])
def test_mode_forward_wrong_contraction(monkeypatch, mode, eq):
    monkeypatch.setitem(otp._FWD, mode, eq)
    assert _caught(MODE_PINS)


@pytest.mark.parametrize("mode", ["uuu", "uvw"])
def test_mode_weights_reversed(monkeypatch, mode):
    orig = otp._weights

    def bad(plan, w, p, bsz):
        ws = orig(plan, w, p, bsz)
        if plan.mode != mode:
            return ws
        return np.ascontiguousarray(ws.reshape(bsz, -1)[:, ::-1]).reshape(ws.shape)

    monkeypatch.setattr(otp, "_weights", bad)
    assert _caught(MODE_PINS)


@pytest.mark.parametrize("mode,table,eq", [
    ("uuu", "_DX", "bvj,ijk,bu,buk->bui"),      # y summed over channels
    ("uuu", "_DW", "bui,bvj,ijk,buk->bu"),      # y summed over channels
    ("uvw", "_DY", "bui,ijk,bvuw,bwk->bvj"),    # weights' u and v transposed (square paths)
    ("uvw", "_DW", "bui,bvj,ijk,bwk->bvuw"),    # weights' u and v transposed (square paths)
])
def test_mode_backward_wrong_contraction(monkeypatch, mode, table, eq):
    monkeypatch.setitem(getattr(otp, table), mode, eq)
    assert _caught(MODE_PINS)


@pytest.mark.parametrize("mode,fan_in,wrong", [
    ("uuu", lambda a, b: b, True), ("uvw", lambda a, b: b, True), ("uvw", lambda a, b: a, True),
    ("uuu", lambda a, b: 1, False), ("uvw", lambda a, b: a * b, False),   # the harness: the stated fans pass
])
def test_mode_wrong_default_path_weight(monkeypatch, mode, fan_in, wrong):
    orig = otp.make_plan

    def bad(*args, **kwargs):
        plan = orig(*args, **kwargs)
        if plan.mode == mode:
            n_out = {}
            for ins in plan.instructions:
                n_out[ins.i_out] = n_out.get(ins.i_out, 0) + 1
            plan.alphas = [np.sqrt((2 * plan.irreps_out[i.i_out].l + 1)
                                   / (fan_in(plan.irreps_in1[i.i_in1].mul, plan.irreps_in2[i.i_in2].mul) * n_out[i.i_out]))
                           for i in plan.instructions]
        return plan

    monkeypatch.setattr(otp, "make_plan", bad)
    monkeypatch.setattr(oracle, "make_plan", bad)
    assert _caught(MODE_PINS) == wrong


def _patch_radial(monkeypatch, name, fn):
    import oracle.radial as orad
    monkeypatch.setattr(orad, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def test_bessel_without_normalisation(monkeypatch):
    import oracle.radial as orad
    orig = orad.bessel_basis
    _patch_radial(monkeypatch, "bessel_basis", lambda r, c, n: orig(r, c, n) / np.sqrt(2.0 / c))
    assert _caught([pins.test_bessel_basis_orthonormal_and_limits])


def test_bessel_wrong_frequency(monkeypatch):
    import oracle.radial as orad
    orig = orad.bessel_basis
    _patch_radial(monkeypatch, "bessel_basis", lambda r, c, n: orig(r, 2 * c, n))
    assert _caught([pins.test_bessel_basis_orthonormal_and_limits])


@pytest.mark.parametrize("which", ["sign", "order"])
def test_envelope_wrong_polynomial(monkeypatch, which):
    import oracle.radial as orad
    orig = orad.polynomial_envelope
    if which == "sign":
        bad = lambda d, p: np.where(np.asarray(d) < 1, 1.0 - (orig(d, p) - 1.0) * 0.9 - 0.1 * np.asarray(d) ** p, 0.0)
    else:
        bad = lambda d, p: orig(d, p - 1) if p > 3 else 1 - np.asarray(d)
    _patch_radial(monkeypatch, "polynomial_envelope", bad)
    assert _caught([lambda: pins.test_polynomial_envelope_smooth_at_cutoff(6)])
