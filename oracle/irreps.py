"""Irreps strings such as ``"16x0e + 8x1o"`` (oracle side; test infrastructure only).

e3nn course, "Curriculum at a glance", lesson 02a: an irreps string lists terms
``<mul>x<l><p>``; ``mul`` is a multiplicity, ``l`` the degree (dimension 2l+1) and ``p`` the
parity, ``e`` (+1) or ``o`` (-1).  A bare ``<l><p>`` means multiplicity 1 (the "1e" edge
attribute in "Modular v2106 point models", NetworkForAGraphWithAttributes).  Features are laid
out ``mul_ir``: irrep blocks in order, inside a block ``[u][m]`` with ``m = -l..l`` fastest
(lesson 12a names this layout and warns that a mismatch silently gives wrong numbers).
"""

import re
from dataclasses import dataclass

_TERM = re.compile(r"^\s*(?:(\d+)\s*x\s*)?(\d+)\s*([eo])\s*$")


@dataclass(frozen=True)
class Irrep:
    mul: int
    l: int
    p: int  # +1 even, -1 odd

    @property
    def dim(self):
        return self.mul * (2 * self.l + 1)


class Irreps(tuple):
    @property
    def dim(self):
        return sum(ir.dim for ir in self)

    def offsets(self):
        offs, o = [], 0
        for ir in self:
            offs.append(o)
            o += ir.dim
        return offs

    def __str__(self):
        return " + ".join(f"{ir.mul}x{ir.l}{'e' if ir.p == 1 else 'o'}" for ir in self)


def parse_irreps(text):
    """Parse an irreps string; raises ValueError on any malformed term."""
    if not isinstance(text, str) or not text.strip():
        raise ValueError("empty irreps string")
    out = []
    for term in text.split("+"):
        m = _TERM.match(term)
        if m is None:
            raise ValueError(f"bad irreps term {term!r}")
        mul = int(m.group(1)) if m.group(1) is not None else 1
        if mul <= 0:
            raise ValueError(f"multiplicity must be positive in {term!r}")
        out.append(Irrep(mul, int(m.group(2)), 1 if m.group(3) == "e" else -1))
    return Irreps(out)
