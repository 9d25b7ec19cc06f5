"""Float64 CPU oracle for the channelwise ("uvu") Clebsch-Gordan tensor product and the
message-passing convolution built on it.

This package is TEST INFRASTRUCTURE.  It is a plain, slow, obviously-correct restatement of
what the method computes, written from the mathematics the sources state and nothing else:

* irreps strings and the mul_ir layout (e3nn course, "Curriculum at a glance", lesson 02a);
* real spherical harmonics, component normalisation (lesson 02b; "Modular v2106 point
  models", Scope);
* Clebsch-Gordan coefficients from the Racah closed form, moved to the real basis (lesson 03a;
  the E3J summary, section G.2, builds the same objects a different way);
* the weighted tensor product with instructions and the "uvu" connection mode (lesson 03b);
* the point convolution with receiver aggregation (lesson 06a; E3J summary, section E.2.2);
* reverse mode by transposition of the multilinear map (E3J summary, section E.1);
* the radial network (Bessel basis, polynomial envelope, SiLU MLP) that gives the per-edge path
  weights (lessons 05b and 06a).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  It shares no code with the CUDA library and must never
sit on the product path.
"""

from .irreps import Irreps, parse_irreps
from .sh import real_sh, real_sh_all, real_sh_grad, real_sh_all_grad, sh_backward
from .cg import complex_cg, real_cg, real_basis_change
from .tp import Instruction, TPPlan, make_plan, tp_forward, tp_backward
from .conv import csr_build, conv_forward, conv_backward
from .reorder import morton_codes, morton_order, invert_permutation
from .radial import bessel_basis, polynomial_envelope, silu, radial_weights

__all__ = [
    "Irreps", "parse_irreps", "real_sh", "real_sh_all", "real_sh_grad", "real_sh_all_grad", "sh_backward",
    "complex_cg", "real_cg",
    "real_basis_change", "Instruction", "TPPlan", "make_plan", "tp_forward", "tp_backward",
    "csr_build", "conv_forward", "conv_backward", "morton_codes", "morton_order", "invert_permutation",
    "bessel_basis", "polynomial_envelope", "silu", "radial_weights",
]
