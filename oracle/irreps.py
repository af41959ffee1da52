"""Irreps strings and path validation for the oracle (test infrastructure only).

An irreps string such as "32x0e+32x1o+32x2e" lists blocks (mul, l, parity).  A feature
row stores the blocks in string order; inside a block the layout is [u][m] with m the
fastest index, m = -l..l.  Parity rule for a path (in a, SH b -> out o): the triangle
rule |l_a - l_b| <= l_o <= l_a + l_b and p_o = p_a * p_b (E(3) equivariance, as in "The
Price of Freedom", abstract: tensor products that interact two geometric features in an
equivariant manner).  "uvu" paths need mul_in == mul_out; "uvw" paths take a shared
[mul_in, mul_out] matrix.
"""
from __future__ import annotations

import re
from typing import List, Sequence, Tuple

_TERM = re.compile(r"^(\d+)x(\d+)([eo])$")


class Irreps:
    def __init__(self, s: str):
        self.blocks: List[Tuple[int, int, int]] = []
        s = s.replace(" ", "")
        if not s:
            raise ValueError("empty irreps string")
        for term in s.split("+"):
            m = _TERM.match(term)
            if not m:
                raise ValueError(f"bad irreps term {term!r}")
            mul, l, p = int(m.group(1)), int(m.group(2)), 1 if m.group(3) == "e" else -1
            if mul <= 0:
                raise ValueError("multiplicity must be positive")
            self.blocks.append((mul, l, p))
        self.offsets = []
        off = 0
        for mul, l, _ in self.blocks:
            self.offsets.append(off)
            off += mul * (2 * l + 1)
        self.dim = off

    def __len__(self):
        return len(self.blocks)


class OraclePlan:
    """Parsed + validated convolution description (oracle's own, independent of the C ABI)."""

    def __init__(self, irreps_in: str, irreps_sh: str, irreps_out: str,
                 paths: Sequence[Sequence[int]], mode: str = "uvu", path_coeff=None):
        self.irr_in, self.irr_sh, self.irr_out = Irreps(irreps_in), Irreps(irreps_sh), Irreps(irreps_out)
        if mode not in ("uvu", "uvw"):
            raise ValueError("mode must be uvu or uvw")
        self.mode = mode
        for mul, l, p in self.irr_sh.blocks:
            if mul != 1 or p != (-1) ** l:
                raise ValueError("spherical-harmonic irreps must be 1x(l)(parity (-1)^l)")
        self.paths = [tuple(int(v) for v in p) for p in paths]
        if not self.paths:
            raise ValueError("no paths")
        self.triples = []
        self.w_off = []
        nw = 0
        for a, b, o in self.paths:
            if not (0 <= a < len(self.irr_in) and 0 <= b < len(self.irr_sh) and 0 <= o < len(self.irr_out)):
                raise ValueError("path index out of range")
            ma, la, pa = self.irr_in.blocks[a]
            _, lb, pb = self.irr_sh.blocks[b]
            mo, lo, po = self.irr_out.blocks[o]
            if not (abs(la - lb) <= lo <= la + lb):
                raise ValueError(f"path {(a, b, o)} violates the triangle rule")
            if po != pa * pb:
                raise ValueError(f"path {(a, b, o)} violates parity")
            if mode == "uvu" and ma != mo:
                raise ValueError("uvu path needs equal input and output multiplicity")
            self.triples.append((la, lb, lo))
            self.w_off.append(nw)
            nw += ma if mode == "uvu" else 1
        self.n_weights = nw
        if mode == "uvw":
            shapes = {(self.irr_in.blocks[a][0], self.irr_out.blocks[o][0]) for a, _, o in self.paths}
            if len(shapes) != 1:
                raise ValueError("oracle uvw supports one common [mul_in, mul_out] shape")
            self.W_shape = (len(self.paths),) + shapes.pop()
        self.coeff = [1.0] * len(self.paths) if path_coeff is None else [float(c) for c in path_coeff]
        self.lmax_sh = max(l for _, l, _ in self.irr_sh.blocks)
