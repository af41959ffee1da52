"""Generator for the compile-time tables and unrolled per-path bodies of the CUDA kernels.

Product code (build step).  It computes, on its own route:
  * complex Clebsch-Gordan coefficients by the Racah closed form (exact rationals under
    one square root), turned into the real basis of the spherical harmonics below, then
    normalised (||C||_F^2 = 2 l3 + 1 by construction) and signed so that the first
    non-zero entry in row-major (m1, m2, m3) order is positive;
  * real spherical harmonics as Cartesian polynomials P_lm(r_hat) for l <= 3 (component
    normalisation, no Condon-Shortley phase, m = -l..l), with exact gradients and
    Hessians taken symbolically, for the backward and double-backward passes.

These are the ingredients named by "The GPU Workload That Rewrites Molecular Physics"
(section "Equivariant feature transforms": spherical harmonics and Clebsch-Gordan tensor
products) and "FlashTP" (abstract: sparse computation -- only non-zero CG entries are
emitted).  For every supported path list ("spec") the generator writes one header with
straight-line device functions: loads and stores of a channel's slice of a feature row,
the SH evaluation, and the contraction bodies of forward, backward, double backward and
the uvw edge pass, each a chain of FFMAs over the non-zero CG entries only.

Usage: python codegen.py OUTDIR
"""
from __future__ import annotations

import math
import os
import sys
from fractions import Fraction
from itertools import product
from typing import Dict, List, Tuple

# ---------------------------------------------------------------------------
# Clebsch-Gordan by the Racah formula
# ---------------------------------------------------------------------------


def _f(n: int) -> int:
    return math.factorial(n)


def cg_complex(j1: int, m1: int, j2: int, m2: int, J: int, M: int) -> float:
    """<j1 m1 j2 m2 | J M> (Condon-Shortley convention), Racah's closed form."""
    if m1 + m2 != M or not (abs(j1 - j2) <= J <= j1 + j2):
        return 0.0
    if abs(m1) > j1 or abs(m2) > j2 or abs(M) > J:
        return 0.0
    pre = Fraction((2 * J + 1) * _f(J + j1 - j2) * _f(J - j1 + j2) * _f(j1 + j2 - J), _f(j1 + j2 + J + 1))
    pre *= _f(J + M) * _f(J - M) * _f(j1 - m1) * _f(j1 + m1) * _f(j2 - m2) * _f(j2 + m2)
    s = Fraction(0)
    for k in range(0, j1 + j2 + J + 1):
        args = [k, j1 + j2 - J - k, j1 - m1 - k, j2 + m2 - k, J - j2 + m1 + k, J - j1 - m2 + k]
        if min(args) < 0:
            continue
        den = 1
        for a in args:
            den *= _f(a)
        s += Fraction((-1) ** k, den)
    return float(s) * math.sqrt(float(pre))


def _real_basis(l: int):
    """Rows: real index m; columns: complex index mu.  Real SH (no Condon-Shortley phase)
    in terms of complex SH (with it): m>0 -> ((-1)^m Y^m + Y^-m)/sqrt2,
    m<0 (k=|m|) -> ((-1)^k Y^k - Y^-k)/(i sqrt2), m=0 -> Y^0."""
    d = 2 * l + 1
    U = [[0j] * d for _ in range(d)]
    r2 = math.sqrt(2.0)
    for m in range(-l, l + 1):
        if m > 0:
            U[m + l][m + l] = (-1) ** m / r2
            U[m + l][-m + l] = 1 / r2
        elif m < 0:
            k = -m
            U[m + l][k + l] = (-1) ** k / (1j * r2)
            U[m + l][-k + l] = -1 / (1j * r2)
        else:
            U[l][l] = 1.0
    return U


_CG_CACHE: Dict[Tuple[int, int, int], List[List[List[float]]]] = {}


def cg_real(l1: int, l2: int, l3: int):
    """Real CG tensor as nested lists [m1][m2][m3] (indices 0..2l)."""
    key = (l1, l2, l3)
    if key in _CG_CACHE:
        return _CG_CACHE[key]
    d1, d2, d3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
    U1, U2, U3 = _real_basis(l1), _real_basis(l2), _real_basis(l3)
    Cc = {}
    for a in range(d1):
        for b in range(d2):
            c = (a - l1) + (b - l2) + l3
            if 0 <= c < d3:
                v = cg_complex(l1, a - l1, l2, b - l2, l3, c - l3)
                if v != 0.0:
                    Cc[(a, b, c)] = v
    R = [[[0j] * d3 for _ in range(d2)] for _ in range(d1)]
    for i in range(d1):
        for j in range(d2):
            for k in range(d3):
                acc = 0j
                for (a, b, c), v in Cc.items():
                    acc += U3[k][c] * v * U1[i][a].conjugate() * U2[j][b].conjugate()
                R[i][j][k] = acc
    mre = max(abs(R[i][j][k].real) for i in range(d1) for j in range(d2) for k in range(d3))
    mim = max(abs(R[i][j][k].imag) for i in range(d1) for j in range(d2) for k in range(d3))
    take_im = mim > mre
    out = [[[0.0] * d3 for _ in range(d2)] for _ in range(d1)]
    for i in range(d1):
        for j in range(d2):
            for k in range(d3):
                z = R[i][j][k]
                main, other = (z.imag, z.real) if take_im else (z.real, z.imag)
                if abs(other) > 1e-12:
                    raise ArithmeticError("real change of basis left a mixed phase")
                out[i][j][k] = main if abs(main) > 1e-12 else 0.0
    first = next(v for i in range(d1) for j in range(d2) for k in range(d3)
                 for v in [out[i][j][k]] if v != 0.0)
    if first < 0:
        out = [[[-v + 0.0 for v in row] for row in pl] for pl in out]
    _CG_CACHE[key] = out
    return out


def cg_nonzeros(l1, l2, l3):
    C = cg_real(l1, l2, l3)
    return [(i, j, k, C[i][j][k]) for i in range(2 * l1 + 1) for j in range(2 * l2 + 1)
            for k in range(2 * l3 + 1) if C[i][j][k] != 0.0]


# ---------------------------------------------------------------------------
# Spherical-harmonic polynomials with symbolic derivatives
# ---------------------------------------------------------------------------

Poly = Dict[Tuple[int, int, int], float]      # monomial (i,j,k) of (x,y,z) -> coefficient


def _p(*terms) -> Poly:
    out: Poly = {}
    for c, mono in terms:
        out[mono] = out.get(mono, 0.0) + c
    return out


def sh_polys() -> Dict[int, List[Poly]]:
    s = math.sqrt
    X, Y, Z = (1, 0, 0), (0, 1, 0), (0, 0, 1)
    return {
        0: [_p((1.0, (0, 0, 0)))],
        1: [_p((s(3), Y)), _p((s(3), Z)), _p((s(3), X))],
        2: [_p((s(15), (1, 1, 0))), _p((s(15), (0, 1, 1))),
            _p((s(5), (0, 0, 2)), (-s(5) / 2, (2, 0, 0)), (-s(5) / 2, (0, 2, 0))),
            _p((s(15), (1, 0, 1))), _p((s(15) / 2, (2, 0, 0)), (-s(15) / 2, (0, 2, 0)))],
        3: [_p((3 * s(70) / 4, (2, 1, 0)), (-s(70) / 4, (0, 3, 0))),
            _p((s(105), (1, 1, 1))),
            _p((s(42), (0, 1, 2)), (-s(42) / 4, (2, 1, 0)), (-s(42) / 4, (0, 3, 0))),
            _p((s(7), (0, 0, 3)), (-3 * s(7) / 2, (2, 0, 1)), (-3 * s(7) / 2, (0, 2, 1))),
            _p((s(42), (1, 0, 2)), (-s(42) / 4, (3, 0, 0)), (-s(42) / 4, (1, 2, 0))),
            _p((s(105) / 2, (2, 0, 1)), (-s(105) / 2, (0, 2, 1))),
            _p((s(70) / 4, (3, 0, 0)), (-3 * s(70) / 4, (1, 2, 0)))],
    }


def dpoly(p: Poly, axis: int) -> Poly:
    out: Poly = {}
    for mono, c in p.items():
        if mono[axis] == 0:
            continue
        m = list(mono)
        k = m[axis]
        m[axis] -= 1
        out[tuple(m)] = out.get(tuple(m), 0.0) + c * k
    return {k: v for k, v in out.items() if v != 0.0}


def _flt(v: float) -> str:
    if v == 0.0:
        return "0.0f"
    return f"{v:.9e}f"


MONO_NAMES = {(0, 0, 0): "1.0f"}


def _mono_expr(mono) -> str:
    i, j, k = mono
    if mono == (0, 0, 0):
        return "1.0f"
    return "m_" + "x" * i + "y" * j + "z" * k


def _poly_expr(p: Poly) -> str:
    terms = [(c, mono) for mono, c in sorted(p.items()) if c != 0.0]
    if not terms:
        return "0.0f"
    out = ""
    for c, mono in terms:
        me = _mono_expr(mono)
        term = _flt(c) if me == "1.0f" else f"{_flt(c)} * {me}"
        out = term if not out else f"{out} + {term}"
    return out


def _monomials_code(maxdeg: int, indent="    ") -> List[str]:
    """Declares every monomial of (x,y,z) up to maxdeg as m_xxy... from rx, ry, rz."""
    lines = []
    names = {}
    for deg in range(1, maxdeg + 1):
        for i in range(deg + 1):
            for j in range(deg + 1 - i):
                k = deg - i - j
                mono = (i, j, k)
                name = _mono_expr(mono)
                if deg == 1:
                    src = {(1, 0, 0): "rx", (0, 1, 0): "ry", (0, 0, 1): "rz"}[mono]
                else:
                    # build from a lower monomial times one variable
                    if i > 0:
                        lower, var = (i - 1, j, k), "rx"
                    elif j > 0:
                        lower, var = (i, j - 1, k), "ry"
                    else:
                        lower, var = (i, j, k - 1), "rz"
                    src = f"{_mono_expr(lower)} * {var}"
                lines.append(f"{indent}const float {name} = {src};")
                names[mono] = name
    return lines


# ---------------------------------------------------------------------------
# Specs
# ---------------------------------------------------------------------------


class Spec:
    def __init__(self, name, in_ls, sh_ls, out_ls, paths, fast_muls=()):
        self.name = name
        self.fast_muls = list(fast_muls) + [0] * (2 - len(fast_muls))
        self.in_ls, self.sh_ls, self.out_ls = list(in_ls), list(sh_ls), list(out_ls)
        self.paths = [tuple(p) for p in paths]
        self.in_d = [2 * l + 1 for l in self.in_ls]
        self.sh_d = [2 * l + 1 for l in self.sh_ls]
        self.out_d = [2 * l + 1 for l in self.out_ls]
        self.in_cum = [sum(self.in_d[:i]) for i in range(len(self.in_d))]
        self.sh_cum = [sum(self.sh_d[:i]) for i in range(len(self.sh_d))]
        self.out_cum = [sum(self.out_d[:i]) for i in range(len(self.out_d))]
        self.IN_PC, self.NSH, self.OUT_PC = sum(self.in_d), sum(self.sh_d), sum(self.out_d)
        self.P = len(self.paths)
        self.triples = [(self.in_ls[a], self.sh_ls[b], self.out_ls[o]) for a, b, o in self.paths]
        for (a, b, o), (l1, l2, l3) in zip(self.paths, self.triples):
            if not abs(l1 - l2) <= l3 <= l1 + l2:
                raise ValueError(f"{name}: path {(a, b, o)} breaks the triangle rule")
        # uvw: per-path accumulator blocks (d3 per path)
        self.a_d = [2 * t[2] + 1 for t in self.triples]
        self.a_cum = [sum(self.a_d[:p]) for p in range(self.P)]
        self.A_PC = sum(self.a_d)
        self.LMAX_SH = max(self.sh_ls)

    def nnz_total(self):
        return sum(len(cg_nonzeros(*t)) for t in self.triples)


def _lines_load(name, n_blocks, d, cum, arr, const=True, shared=False):
    """Straight-line load of one channel's slice of a [u][m] row (read-only global path, or
    plain loads for a row staged in shared memory)."""
    out = [f"  __device__ __forceinline__ static void {name}(const float* __restrict__ row, int mul, int c, float (&{arr})[{sum(d)}]) {{"]
    for a in range(n_blocks):
        out.append(f"    {{ const float* p = row + mul * {cum[a]} + c * {d[a]};")
        for m in range(d[a]):
            out.append(f"      {arr}[{cum[a] + m}] = p[{m}];" if shared else f"      {arr}[{cum[a] + m}] = __ldg(p + {m});")
        out.append("    }")
    out.append("  }")
    return out


def _lines_store(name, n_blocks, d, cum, arr):
    out = [f"  __device__ __forceinline__ static void {name}(float* __restrict__ row, int mul, int c, const float (&{arr})[{sum(d)}]) {{"]
    for a in range(n_blocks):
        out.append(f"    {{ float* p = row + mul * {cum[a]} + c * {d[a]};")
        for m in range(d[a]):
            out.append(f"      p[{m}] = {arr}[{cum[a] + m}];")
        out.append("    }")
    out.append("  }")
    return out


def _gen_sh(spec: Spec) -> List[str]:
    polys = sh_polys()
    L = []
    maxdeg = spec.LMAX_SH
    # Y
    L.append(f"  __device__ __forceinline__ static void sh(float rx, float ry, float rz, float (&Y)[{spec.NSH}]) {{")
    L += _monomials_code(maxdeg)
    for b, l in enumerate(spec.sh_ls):
        for m in range(2 * l + 1):
            L.append(f"    Y[{spec.sh_cum[b] + m}] = {_poly_expr(polys[l][m])};")
    L.append("  }")
    # gradient of P at r_hat: G[k][3]
    L.append(f"  __device__ __forceinline__ static void sh_grad(float rx, float ry, float rz, float (&G)[{spec.NSH}][3]) {{")
    L += _monomials_code(max(maxdeg - 1, 1))
    for b, l in enumerate(spec.sh_ls):
        for m in range(2 * l + 1):
            for ax in range(3):
                L.append(f"    G[{spec.sh_cum[b] + m}][{ax}] = {_poly_expr(dpoly(polys[l][m], ax))};")
    L.append("  }")
    # Hessian of P at r_hat times d: HD[k][3]
    L.append(f"  __device__ __forceinline__ static void sh_hess_dot(float rx, float ry, float rz, float dx, float dy, float dz, float (&HD)[{spec.NSH}][3]) {{")
    L += _monomials_code(max(maxdeg - 2, 1))
    L.append("    (void)rx; (void)ry; (void)rz;")
    dn = ["dx", "dy", "dz"]
    for b, l in enumerate(spec.sh_ls):
        for m in range(2 * l + 1):
            for ax in range(3):
                terms = []
                g = dpoly(polys[l][m], ax)
                for ax2 in range(3):
                    h = dpoly(g, ax2)
                    if h:
                        terms.append(f"({_poly_expr(h)}) * {dn[ax2]}")
                expr = " + ".join(terms) if terms else "0.0f"
                L.append(f"    HD[{spec.sh_cum[b] + m}][{ax}] = {expr};")
    L.append("  }")
    # degree of each SH component (for the homogeneous derivative formulas)
    degs = []
    for l in spec.sh_ls:
        degs += [l] * (2 * l + 1)
    L.append(f"  __device__ __forceinline__ static float sh_degree(int k) {{ constexpr float d[{spec.NSH}] = {{{', '.join(f'{v}.0f' for v in degs)}}}; return d[k]; }}")
    return L


def _group(spec: Spec, key):
    groups: Dict[Tuple[int, int], List[int]] = {}
    for p, path in enumerate(spec.paths):
        groups.setdefault(key(path), []).append(p)
    return groups


def _chain(terms, tgt, decl=True):
    """Emit tgt = sum_i c_i * q_i as an FMUL followed by FFMAs."""
    out = []
    first = True
    for c, q in terms:
        if first:
            out.append(f"      {'float ' if decl else ''}{tgt} = {_flt(c)} * {q};")
            first = False
        else:
            out.append(f"      {tgt} = fmaf({_flt(c)}, {q}, {tgt});")
    if first:
        out.append(f"      {'float ' if decl else ''}{tgt} = 0.0f;")
    return out


def _gen_fwd(spec: Spec, name="fwd", weighted_out="acc", per_path_out=False) -> List[str]:
    """acc[out(p), m3] += w[p] * sum C x[in(p), m1] Y[sh(p), m2]  (per_path_out: A blocks)."""
    OUT = spec.A_PC if per_path_out else spec.OUT_PC
    L = [f"  __device__ __forceinline__ static void {name}(const float (&x)[{spec.IN_PC}], const float (&Y)[{spec.NSH}], const float (&w)[{spec.P}], float (&{weighted_out})[{OUT}]) {{"]
    groups = _group(spec, lambda p: (p[0], p[1]))
    for (a, b), plist in groups.items():
        la, lb = spec.in_ls[a], spec.sh_ls[b]
        L.append(f"    {{ // in block {a} (l={la}) x SH block {b} (l={lb})")
        used = set()
        for p in plist:
            for (i, j, k, c) in cg_nonzeros(*spec.triples[p]):
                used.add((i, j))
        for (i, j) in sorted(used):
            xs, ys = f"x[{spec.in_cum[a] + i}]", f"Y[{spec.sh_cum[b] + j}]"
            if lb == 0:
                L.append(f"      const float q{i}_{j} = {xs};")
            else:
                L.append(f"      const float q{i}_{j} = {xs} * {ys};")
        for p in plist:
            o = spec.paths[p][2]
            nz = cg_nonzeros(*spec.triples[p])
            d3 = 2 * spec.triples[p][2] + 1
            base = spec.a_cum[p] if per_path_out else spec.out_cum[o]
            for k in range(d3):
                terms = [(c, f"q{i}_{j}") for (i, j, kk, c) in nz if kk == k]
                if not terms:
                    continue
                L += _chain(terms, f"t{p}_{k}")
                L.append(f"      {weighted_out}[{base + k}] = fmaf(w[{p}], t{p}_{k}, {weighted_out}[{base + k}]);")
        L.append("    }")
    L.append("  }")
    return L


def _gen_bwd(spec: Spec) -> List[str]:
    """Sender-side backward for one edge and one channel:
       gw[p]        = sum C x[m1] Y[m2] gy[m3]
       gx[in(p)]   += w[p] * sum_{m2,m3} C Y[m2] gy[m3]
       gY[sh(p)]   += w[p] * sum_{m1,m3} C x[m1] gy[m3]      (WITH_GY)"""
    L = ["  template <bool WITH_GY>",
         f"  __device__ __forceinline__ static void bwd(const float (&x)[{spec.IN_PC}], const float (&Y)[{spec.NSH}], const float (&w)[{spec.P}], const float (&gy)[{spec.OUT_PC}], float (&gx)[{spec.IN_PC}], float (&gw)[{spec.P}], float (&gY)[{spec.NSH}]) {{"]
    # Z_p[m1] = sum C Y[m2] gy[m3]  with products r = Y[m2] gy[m3] grouped by (b, o)
    groups = _group(spec, lambda p: (p[1], p[2]))
    for (b, o), plist in groups.items():
        lb = spec.sh_ls[b]
        L.append(f"    {{ // SH block {b} x out block {o}")
        used = set()
        for p in plist:
            for (i, j, k, c) in cg_nonzeros(*spec.triples[p]):
                used.add((j, k))
        for (j, k) in sorted(used):
            gs, ys = f"gy[{spec.out_cum[o] + k}]", f"Y[{spec.sh_cum[b] + j}]"
            L.append(f"      const float r{j}_{k} = {gs};" if lb == 0 else f"      const float r{j}_{k} = {ys} * {gs};")
        for p in plist:
            a = spec.paths[p][0]
            nz = cg_nonzeros(*spec.triples[p])
            d1 = 2 * spec.triples[p][0] + 1
            gwterms = []
            for i in range(d1):
                terms = [(c, f"r{j}_{k}") for (ii, j, k, c) in nz if ii == i]
                if not terms:
                    continue
                L += _chain(terms, f"z{p}_{i}")
                L.append(f"      gx[{spec.in_cum[a] + i}] = fmaf(w[{p}], z{p}_{i}, gx[{spec.in_cum[a] + i}]);")
                gwterms.append(i)
            if gwterms:
                i0 = gwterms[0]
                L.append(f"      float gwp{p} = x[{spec.in_cum[a] + i0}] * z{p}_{i0};")
                for i in gwterms[1:]:
                    L.append(f"      gwp{p} = fmaf(x[{spec.in_cum[a] + i}], z{p}_{i}, gwp{p});")
                L.append(f"      gw[{p}] = gwp{p};")
            else:
                L.append(f"      gw[{p}] = 0.0f;")
        L.append("    }")
    # gY: products s = x[m1] gy[m3] grouped by (a, o)
    L.append("    if constexpr (WITH_GY) {")
    groups = _group(spec, lambda p: (p[0], p[2]))
    for (a, o), plist in groups.items():
        L.append(f"    {{ // in block {a} x out block {o}")
        used = set()
        for p in plist:
            if spec.sh_ls[spec.paths[p][1]] == 0:
                continue            # Y_0 is constant: no contribution to the direction gradient
            for (i, j, k, c) in cg_nonzeros(*spec.triples[p]):
                used.add((i, k))
        for (i, k) in sorted(used):
            L.append(f"      const float s{i}_{k} = x[{spec.in_cum[a] + i}] * gy[{spec.out_cum[o] + k}];")
        for p in plist:
            b = spec.paths[p][1]
            if spec.sh_ls[b] == 0:
                continue
            nz = cg_nonzeros(*spec.triples[p])
            d2 = 2 * spec.triples[p][1] + 1
            for j in range(d2):
                terms = [(c, f"s{i}_{k}") for (i, jj, k, c) in nz if jj == j]
                if not terms:
                    continue
                L += _chain(terms, f"qq{p}_{j}")
                L.append(f"      gY[{spec.sh_cum[b] + j}] = fmaf(w[{p}], qq{p}_{j}, gY[{spec.sh_cum[b] + j}]);")
        L.append("    }")
    L.append("    }")
    L.append("  }")
    return L


def _gen_dbwd_recv(spec: Spec) -> List[str]:
    """Receiver-side double backward for one edge and one channel:
       acc[out(p)] += ggw[p] * C(x, Y) + w[p] * (C(ggx, Y) + C(x, Yp))"""
    L = [f"  __device__ __forceinline__ static void dbwd_recv(const float (&x)[{spec.IN_PC}], const float (&ggx)[{spec.IN_PC}], const float (&Y)[{spec.NSH}], const float (&Yp)[{spec.NSH}], const float (&w)[{spec.P}], const float (&ggw)[{spec.P}], float (&acc)[{spec.OUT_PC}]) {{"]
    groups = _group(spec, lambda p: (p[0], p[1]))
    for (a, b), plist in groups.items():
        lb = spec.sh_ls[b]
        L.append(f"    {{ // in block {a} x SH block {b}")
        used = set()
        for p in plist:
            for (i, j, k, c) in cg_nonzeros(*spec.triples[p]):
                used.add((i, j))
        for (i, j) in sorted(used):
            xs, gs = f"x[{spec.in_cum[a] + i}]", f"ggx[{spec.in_cum[a] + i}]"
            ys, yps = f"Y[{spec.sh_cum[b] + j}]", f"Yp[{spec.sh_cum[b] + j}]"
            if lb == 0:
                L.append(f"      const float q{i}_{j} = {xs};")
                L.append(f"      const float h{i}_{j} = {gs};")
            else:
                L.append(f"      const float q{i}_{j} = {xs} * {ys};")
                L.append(f"      const float h{i}_{j} = fmaf({gs}, {ys}, {xs} * {yps});")
        for p in plist:
            o = spec.paths[p][2]
            nz = cg_nonzeros(*spec.triples[p])
            d3 = 2 * spec.triples[p][2] + 1
            for k in range(d3):
                t1 = [(c, f"q{i}_{j}") for (i, j, kk, c) in nz if kk == k]
                t2 = [(c, f"h{i}_{j}") for (i, j, kk, c) in nz if kk == k]
                if not t1:
                    continue
                L += _chain(t1, f"t{p}_{k}")
                L += _chain(t2, f"u{p}_{k}")
                L.append(f"      acc[{spec.out_cum[o] + k}] = fmaf(ggw[{p}], t{p}_{k}, fmaf(w[{p}], u{p}_{k}, acc[{spec.out_cum[o] + k}]));")
        L.append("    }")
    L.append("  }")
    return L


def _gen_dbwd_send(spec: Spec) -> List[str]:
    """Sender-side double backward for one edge and one channel:
       gx[in(p)]  += sum_{m2,m3} C (ggw[p] Y[m2] + w[p] Yp[m2]) gy[m3]
       gw[p]       = sum C (ggx[m1] Y[m2] + x[m1] Yp[m2]) gy[m3]
       G1[sh(p)]  += ggw[p] Q(x, gy) + w[p] Q(ggx, gy);  G2[sh(p)] += w[p] Q(x, gy)
       with Q(a, g)[m2] = sum_{m1,m3} C a[m1] g[m3].
    Emitted three ways: dbwd_send (all of it), dbwd_send_gx (gx and gw only) and
    dbwd_send_gv (G1 and G2 only), so that a large spec can run the two halves as two
    kernels with half the straight-line code each."""
    sig = "(const float (&x)[{i}], const float (&ggx)[{i}], const float (&Y)[{n}], const float (&Yp)[{n}], const float (&w)[{p}], const float (&ggw)[{p}], const float (&gy)[{o}], float (&gx)[{i}], float (&gw)[{p}], float (&G1)[{n}], float (&G2)[{n}])".format(
        i=spec.IN_PC, n=spec.NSH, p=spec.P, o=spec.OUT_PC)
    s1 = _dbwd_send_gx_lines(spec)
    s2 = _dbwd_send_gv_lines(spec)
    L = []
    for name, parts in (("dbwd_send", s1 + s2), ("dbwd_send_gx", s1), ("dbwd_send_gv", s2)):
        L.append(f"  __device__ __forceinline__ static void {name}{sig} {{")
        L += parts
        L.append("  }")
    return L


def _dbwd_send_gx_lines(spec: Spec) -> List[str]:
    L = []
    groups = _group(spec, lambda p: (p[1], p[2]))
    for (b, o), plist in groups.items():
        lb = spec.sh_ls[b]
        L.append(f"    {{ // SH block {b} x out block {o}")
        used = set()
        for p in plist:
            for (i, j, k, c) in cg_nonzeros(*spec.triples[p]):
                used.add((j, k))
        for (j, k) in sorted(used):
            gs = f"gy[{spec.out_cum[o] + k}]"
            ys, yps = f"Y[{spec.sh_cum[b] + j}]", f"Yp[{spec.sh_cum[b] + j}]"
            if lb == 0:
                L.append(f"      const float r{j}_{k} = {gs};")
            else:
                L.append(f"      const float r{j}_{k} = {ys} * {gs};")
                L.append(f"      const float rp{j}_{k} = {yps} * {gs};")
        for p in plist:
            a = spec.paths[p][0]
            nz = cg_nonzeros(*spec.triples[p])
            d1 = 2 * spec.triples[p][0] + 1
            gw_terms = []
            for i in range(d1):
                t1 = [(c, f"r{j}_{k}") for (ii, j, k, c) in nz if ii == i]
                if not t1:
                    continue
                L += _chain(t1, f"z{p}_{i}")
                if lb == 0:
                    L.append(f"      const float zp{p}_{i} = 0.0f;")
                else:
                    L += _chain([(c, f"rp{j}_{k}") for (ii, j, k, c) in nz if ii == i], f"zp{p}_{i}")
                ia = spec.in_cum[a] + i
                L.append(f"      gx[{ia}] = fmaf(ggw[{p}], z{p}_{i}, fmaf(w[{p}], zp{p}_{i}, gx[{ia}]));")
                gw_terms.append(i)
            if gw_terms:
                L.append(f"      float gwp{p} = 0.0f;")
                for i in gw_terms:
                    ia = spec.in_cum[a] + i
                    L.append(f"      gwp{p} = fmaf(ggx[{ia}], z{p}_{i}, fmaf(x[{ia}], zp{p}_{i}, gwp{p}));")
                L.append(f"      gw[{p}] = gwp{p};")
            else:
                L.append(f"      gw[{p}] = 0.0f;")
        L.append("    }")
    return L


def _dbwd_send_gv_lines(spec: Spec) -> List[str]:
    L = []
    groups = _group(spec, lambda p: (p[0], p[2]))
    for (a, o), plist in groups.items():
        plist = [p for p in plist if spec.sh_ls[spec.paths[p][1]] != 0]
        if not plist:
            continue
        L.append(f"    {{ // in block {a} x out block {o}")
        used = set()
        for p in plist:
            for (i, j, k, c) in cg_nonzeros(*spec.triples[p]):
                used.add((i, k))
        for (i, k) in sorted(used):
            L.append(f"      const float s{i}_{k} = x[{spec.in_cum[a] + i}] * gy[{spec.out_cum[o] + k}];")
            L.append(f"      const float sg{i}_{k} = ggx[{spec.in_cum[a] + i}] * gy[{spec.out_cum[o] + k}];")
        for p in plist:
            b = spec.paths[p][1]
            nz = cg_nonzeros(*spec.triples[p])
            d2 = 2 * spec.triples[p][1] + 1
            for j in range(d2):
                t1 = [(c, f"s{i}_{k}") for (i, jj, k, c) in nz if jj == j]
                if not t1:
                    continue
                L += _chain(t1, f"qa{p}_{j}")
                L += _chain([(c, f"sg{i}_{k}") for (i, jj, k, c) in nz if jj == j], f"qb{p}_{j}")
                kb = spec.sh_cum[b] + j
                L.append(f"      G1[{kb}] = fmaf(ggw[{p}], qa{p}_{j}, fmaf(w[{p}], qb{p}_{j}, G1[{kb}]));")
                L.append(f"      G2[{kb}] = fmaf(w[{p}], qa{p}_{j}, G2[{kb}]);")
        L.append("    }")
    return L


def _uvw_tables(spec: Spec):
    """Per output irrep o: paths into o (in path order), d3, count, and the per-(node, channel)
    offset of its region in the uvw node state A (regions in output order)."""
    outs = []
    cum = 0
    for o, l3 in enumerate(spec.out_ls):
        plist = [p for p, path in enumerate(spec.paths) if path[2] == o]
        d3 = 2 * l3 + 1
        outs.append(dict(o=o, d3=d3, paths=plist, cnt=len(plist), cumA=cum))
        cum += d3 * len(plist)
    assert cum == spec.A_PC
    return outs


def _gen_uvw_layout(spec: Spec) -> List[str]:
    outs = _uvw_tables(spec)
    n = len(outs)
    maxc = max(1, max(t["cnt"] for t in outs))
    L = [f"  static constexpr int N_OUT = {n};",
         f"  static constexpr int MAX_CNT = {maxc};"]
    for name, vals in (("out_d3_at", [t["d3"] for t in outs]), ("out_cnt_at", [t["cnt"] for t in outs]),
                       ("out_cumA_at", [t["cumA"] for t in outs]), ("out_cumY_at", list(spec.out_cum))):
        L.append(f"  __host__ __device__ static int {name}(int o) {{ constexpr int v[{n}] = "
                 f"{{{', '.join(map(str, vals))}}}; return v[o]; }}")
    flat = []
    for t in outs:
        flat += t["paths"] + [-1] * (maxc - t["cnt"])
    L.append(f"  __host__ __device__ static int path_of_at(int o, int pl) {{ constexpr int v[{n * maxc}] = "
             f"{{{', '.join(map(str, flat))}}}; return v[o * {maxc} + pl]; }}")
    # store / load of one channel's per-path state, [N*mul*cumA_o] + ((i*d3+m3)*cnt + pl)*mul + c
    for name, const, arr in (("store_uvw", False, "a"), ("load_uvw", True, "a")):
        sig = (f"  __device__ __forceinline__ static void {name}({'const ' if const else ''}float* __restrict__ base, "
               f"int64_t N, int mul, int64_t i, int c, {'float' if const else 'const float'} (&{arr})[{spec.A_PC}]) {{")
        L.append(sig)
        for t in outs:
            for pl, p in enumerate(t["paths"]):
                for m3 in range(t["d3"]):
                    idx = (f"N * mul * {t['cumA']} + ((i * {t['d3']} + {m3}) * {t['cnt']} + {pl}) * (int64_t)mul + c")
                    k = spec.a_cum[p] + m3
                    if const:
                        L.append(f"    {arr}[{k}] = __ldg(base + {idx});")
                    else:
                        L.append(f"    base[{idx}] = {arr}[{k}];")
        L.append("  }")
    return L


def _uvw_in_tables(spec: Spec):
    """Per input irrep a: paths reading a (in path order), d1, count, and the per-(node, channel)
    offset of its region in the sender-side state (x W and its gradient partner B)."""
    ins = []
    cum = 0
    for a, l1 in enumerate(spec.in_ls):
        plist = [p for p, path in enumerate(spec.paths) if path[0] == a]
        d1 = 2 * l1 + 1
        ins.append(dict(a=a, d1=d1, paths=plist, cnt=len(plist), cumX=cum))
        cum += d1 * len(plist)
    return ins, cum


def _gen_uvw_send_layout(spec: Spec) -> List[str]:
    ins, xt_pc = _uvw_in_tables(spec)
    n = len(ins)
    maxc = max(1, max(t["cnt"] for t in ins))
    # per path: block offset inside one channel's xt row (path order)
    xt_cum = [0] * spec.P
    c = 0
    for p in range(spec.P):
        xt_cum[p] = c
        c += 2 * spec.triples[p][0] + 1
    L = [f"  static constexpr int XT_PC = {xt_pc};",
         f"  static constexpr int N_IN = {n};",
         f"  static constexpr int MAX_CNT_IN = {maxc};"]
    for name, vals in (("in_d1_at", [t["d1"] for t in ins]), ("in_cnt_at", [t["cnt"] for t in ins]),
                       ("in_cumX_at", [t["cumX"] for t in ins]), ("in_cum_at", list(spec.in_cum))):
        L.append(f"  __host__ __device__ static int {name}(int a) {{ constexpr int v[{n}] = "
                 f"{{{', '.join(map(str, vals))}}}; return v[a]; }}")
    flat = []
    for t in ins:
        flat += t["paths"] + [-1] * (maxc - t["cnt"])
    L.append(f"  __host__ __device__ static int path_in_at(int a, int pl) {{ constexpr int v[{n * maxc}] = "
             f"{{{', '.join(map(str, flat))}}}; return v[a * {maxc} + pl]; }}")
    # region a of the sender state: N*mul*cumX_a + ((j*d1 + m1)*cnt_a + pl)*mul + c ; register xt[xt_cum[p] + m1]
    for name, const in (("load_xt", True), ("store_xt", False)):
        L.append(f"  __device__ __forceinline__ static void {name}({'const ' if const else ''}float* __restrict__ base, "
                 f"int64_t N, int mul, int64_t j, int c, {'float' if const else 'const float'} (&v)[{xt_pc}]) {{")
        for t in ins:
            for pl, p in enumerate(t["paths"]):
                for m1 in range(t["d1"]):
                    idx = f"N * mul * {t['cumX']} + ((j * {t['d1']} + {m1}) * {t['cnt']} + {pl}) * (int64_t)mul + c"
                    k = xt_cum[p] + m1
                    L.append(f"    v[{k}] = __ldg(base + {idx});" if const else f"    base[{idx}] = v[{k}];")
        L.append("  }")
    return L, xt_cum, xt_pc


def _gen_uvw_send(spec: Spec, xt_cum, xt_pc) -> List[str]:
    """uvw sender pass for one edge and one output channel w, with xt = (x W)[sender] per path:
       Z_p[m1]  = sum_{m2,m3} C Y[m2] gy[out(p), m3]
       bt[p]   += s[p] Z_p            (sender state; gx = bt W^T, gW = x^T bt)
       gs[p]   += sum_m1 xt_p[m1] Z_p[m1]      (partial over this channel)
       gY[sh(p)] += s[p] sum_{m1,m3} C xt_p[m1] gy[m3]   (WITH_GY)"""
    L = ["  template <bool WITH_GY>",
         f"  __device__ __forceinline__ static void uvw_send(const float (&xt)[{xt_pc}], const float (&Y)[{spec.NSH}], const float (&s)[{spec.P}], const float (&gy)[{spec.OUT_PC}], float (&bt)[{xt_pc}], float (&gs)[{spec.P}], float (&gY)[{spec.NSH}]) {{"]
    groups = _group(spec, lambda p: (p[1], p[2]))
    for (b, o), plist in groups.items():
        lb = spec.sh_ls[b]
        L.append(f"    {{ // SH block {b} x out block {o}")
        used = set()
        for p in plist:
            for (i, j, k, c) in cg_nonzeros(*spec.triples[p]):
                used.add((j, k))
        for (j, k) in sorted(used):
            gs_ = f"gy[{spec.out_cum[o] + k}]"
            L.append(f"      const float r{j}_{k} = {gs_};" if lb == 0 else f"      const float r{j}_{k} = Y[{spec.sh_cum[b] + j}] * {gs_};")
        for p in plist:
            nz = cg_nonzeros(*spec.triples[p])
            d1 = 2 * spec.triples[p][0] + 1
            zs = []
            for i in range(d1):
                terms = [(c, f"r{j}_{k}") for (ii, j, k, c) in nz if ii == i]
                if not terms:
                    continue
                L += _chain(terms, f"z{p}_{i}")
                L.append(f"      bt[{xt_cum[p] + i}] = fmaf(s[{p}], z{p}_{i}, bt[{xt_cum[p] + i}]);")
                zs.append(i)
            for i in zs:
                L.append(f"      gs[{p}] = fmaf(xt[{xt_cum[p] + i}], z{p}_{i}, gs[{p}]);")
        L.append("    }")
    L.append("    if constexpr (WITH_GY) {")
    for p, (a, b, o) in enumerate(spec.paths):
        if spec.sh_ls[b] == 0:
            continue
        nz = cg_nonzeros(*spec.triples[p])
        d2 = 2 * spec.triples[p][1] + 1
        L.append(f"    {{ // path {p}")
        for (i, k) in sorted({(i, k) for (i, j, k, c) in nz}):
            L.append(f"      const float t{i}_{k} = xt[{xt_cum[p] + i}] * gy[{spec.out_cum[o] + k}];")
        for j in range(d2):
            terms = [(c, f"t{i}_{k}") for (i, jj, k, c) in nz if jj == j]
            if not terms:
                continue
            L += _chain(terms, f"q{j}")
            L.append(f"      gY[{spec.sh_cum[b] + j}] = fmaf(s[{p}], q{j}, gY[{spec.sh_cum[b] + j}]);")
        L.append("    }")
    L.append("    }")
    L.append("  }")
    return L


# ---------------------------------------------------------------------------
# Edge-pair variants: every value is a float2 holding the same quantity for two edges of
# one row, so each CG FMA is one packed __ffma2_rn (two FMAs per lane and instruction).
# ---------------------------------------------------------------------------

def _c2(c):
    return f"make_float2({_flt(c)}, {_flt(c)})"


def _chain2(terms, tgt):
    out = []
    first = True
    for c, q in terms:
        if first:
            out.append(f"      float2 {tgt} = {q};" if c == 1.0 else f"      float2 {tgt} = __fmul2_rn({_c2(c)}, {q});")
            first = False
        else:
            out.append(f"      {tgt} = __fadd2_rn({q}, {tgt});" if c == 1.0 else f"      {tgt} = __ffma2_rn({_c2(c)}, {q}, {tgt});")
    if first:
        out.append(f"      float2 {tgt} = make_float2(0.0f, 0.0f);")
    return out


def _gen_fwd2(spec: Spec) -> List[str]:
    """Edge-pair forward: acc[out(p), m3] += w[p] * sum C x[in(p), m1] Y[sh(p), m2] (float2)."""
    L = [f"  __device__ __forceinline__ static void fwd2(const float2 (&x)[{spec.IN_PC}], const float2 (&Y)[{spec.NSH}], const float2 (&w)[{spec.P}], float2 (&acc)[{spec.OUT_PC}]) {{"]
    groups = _group(spec, lambda p: (p[0], p[1]))
    for (a, b), plist in groups.items():
        lb = spec.sh_ls[b]
        L.append(f"    {{ // in block {a} x SH block {b}")
        used = set()
        for p in plist:
            for (i, j, k, c) in cg_nonzeros(*spec.triples[p]):
                used.add((i, j))
        for (i, j) in sorted(used):
            xs, ys = f"x[{spec.in_cum[a] + i}]", f"Y[{spec.sh_cum[b] + j}]"
            L.append(f"      const float2 q{i}_{j} = {xs};" if lb == 0 else f"      const float2 q{i}_{j} = __fmul2_rn({xs}, {ys});")
        for p in plist:
            o = spec.paths[p][2]
            nz = cg_nonzeros(*spec.triples[p])
            d3 = 2 * spec.triples[p][2] + 1
            for k in range(d3):
                terms = [(c, f"q{i}_{j}") for (i, j, kk, c) in nz if kk == k]
                if not terms:
                    continue
                L += _chain2(terms, f"t{p}_{k}")
                idx = spec.out_cum[o] + k
                L.append(f"      acc[{idx}] = __ffma2_rn(w[{p}], t{p}_{k}, acc[{idx}]);")
        L.append("    }")
    L.append("  }")
    return L


def _km_blocks(spec: Spec):
    """Per input block a of the uvw receiver pass: the rows r = (p, m3) of the paths reading a
    (path order), their count n, the padded width W (a multiple of 4), the offset of the block's
    d1 x W matrix in an edge's K row and the index of its first accumulator pair."""
    blocks, off, pb = [], 0, 0
    for a, l1 in enumerate(spec.in_ls):
        rows = [(p, m3) for p in range(spec.P) if spec.paths[p][0] == a for m3 in range(spec.a_d[p])]
        if not rows:
            continue
        n, d1 = len(rows), 2 * l1 + 1
        W = (n + 3) // 4 * 4
        blocks.append(dict(a=a, d1=d1, rows=rows, n=n, W=W, off=off, pb=pb))
        off += d1 * W
        pb += (n + 1) // 2
    return blocks, off, pb


def _gen_km(spec: Spec) -> List[str]:
    """uvw receiver pass with the per-edge coupling matrix
         K_e[(a, m1), (p, m3)] = c_p s[e, p] sum_m2 C_p[m1, m2, m3] Y(v_e)[m2]      (in(p) = a)
       so that, per channel, A[(p, m3)] += sum_m1 x[a, m1] K_e[(a, m1), (p, m3)]: the edge's
       harmonics, path scalars and CG entries are folded once per edge (shared by all channels)
       and the per-channel work is a dense d1 x n product per input block, evaluated two
       accumulator rows at a time (FFMA2).  K rows: [block][m1][W] floats, zero padded."""
    blocks, krow, pairs = _km_blocks(spec)
    L = [f"  static constexpr int KM_ROW = {krow};",
         f"  static constexpr int KM_PAIRS = {pairs};"]
    # entries of the K row, in order, as (cost, expression); pads are 0
    entries = []
    for B in blocks:
        for m1 in range(B["d1"]):
            for r in range(B["W"]):
                if r >= B["n"]:
                    entries.append((0, "0.0f"))
                    continue
                p, m3 = B["rows"][r]
                b = spec.paths[p][1]
                lb = spec.sh_ls[b]
                nz = [(j, c) for (i, j, k, c) in cg_nonzeros(*spec.triples[p]) if i == m1 and k == m3]
                if not nz:
                    entries.append((0, "0.0f"))
                    continue
                if lb == 0:
                    expr = f"{_flt(nz[0][1])} * cs[{p}]"
                else:
                    t = " + ".join(f"{_flt(c)} * Y[{spec.sh_cum[b] + j}]" for j, c in nz)
                    expr = f"cs[{p}] * ({t})"
                entries.append((len(nz) + 1, expr))
    groups = [entries[4 * g:4 * g + 4] for g in range(krow // 4)]
    gcost = [1 + sum(c for c, _ in grp) for grp in groups]
    # K row of one edge, built by H threads: thread h writes a contiguous run of float4 groups
    L.append("  template <int H>")
    L.append(f"  __device__ __forceinline__ static void km_build(int h, const float (&Y)[{spec.NSH}], "
             f"const float (&cs)[{spec.P}], float4* __restrict__ k) {{")
    L.append("    (void)Y;")
    for H in (1, 2, 4, 8):
        total = sum(gcost)
        cuts, acc, part = [0], 0, 1
        for g, c in enumerate(gcost):
            acc += c
            if part < H and acc >= total * part / H:
                cuts.append(g + 1)
                part += 1
        while len(cuts) < H:
            cuts.append(len(groups))
        cuts.append(len(groups))
        L.append(f"    if constexpr (H == {H}) {{")
        for h in range(H):
            L.append(f"      if (h == {h}) {{")
            for g in range(cuts[h], cuts[h + 1]):
                ex = [e for _, e in groups[g]]
                L.append(f"        k[{g}] = make_float4({ex[0]}, {ex[1]}, {ex[2]}, {ex[3]});")
            L.append("      }")
        L.append("    }")
    L.append("  }")
    # per-channel products, one and two channels sharing the K loads
    for nch in (1, 2):
        if nch == 1:
            L.append(f"  __device__ __forceinline__ static void km_apply1(const float (&x0)[{spec.IN_PC}], "
                     f"const float4* __restrict__ k, float2 (&a0)[{pairs}]) {{")
        else:
            L.append(f"  __device__ __forceinline__ static void km_apply2(const float (&x0)[{spec.IN_PC}], "
                     f"const float (&x1)[{spec.IN_PC}], const float4* __restrict__ k, float2 (&a0)[{pairs}], "
                     f"float2 (&a1)[{pairs}]) {{")
        for B in blocks:
            npair = (B["n"] + 1) // 2
            for m1 in range(B["d1"]):
                xi = spec.in_cum[B["a"]] + m1
                L.append("    {")
                for ch in range(nch):
                    L.append(f"      const float2 u{ch} = make_float2(x{ch}[{xi}], x{ch}[{xi}]);")
                for q in range(B["W"] // 4):
                    g = (B["off"] + m1 * B["W"]) // 4 + q
                    L.append(f"      {{ const float4 v = k[{g}];")
                    for half, (lo, hi) in enumerate((("x", "y"), ("z", "w"))):
                        pi = 2 * q + half
                        if pi >= npair:
                            continue
                        for ch in range(nch):
                            L.append(f"        a{ch}[{B['pb'] + pi}] = __ffma2_rn(u{ch}, make_float2(v.{lo}, v.{hi}), a{ch}[{B['pb'] + pi}]);")
                    L.append("      }")
                L.append("    }")
        L.append("  }")
    # store into the node state A (the store_uvw layout)
    outs = _uvw_tables(spec)
    L.append(f"  __device__ __forceinline__ static void km_store(float* __restrict__ base, int64_t N, int mul, "
             f"int64_t i, int c, const float2 (&acc)[{pairs}]) {{")
    for B in blocks:
        for r, (p, m3) in enumerate(B["rows"]):
            o = spec.paths[p][2]
            t = outs[o]
            pl = t["paths"].index(p)
            idx = f"N * mul * {t['cumA']} + ((i * {t['d3']} + {m3}) * {t['cnt']} + {pl}) * (int64_t)mul + c"
            L.append(f"    base[{idx}] = acc[{B['pb'] + r // 2}].{'x' if r % 2 == 0 else 'y'};")
    L.append("  }")
    return L


def _kmt_blocks(spec: Spec):
    """Per output block o of the uvw sender pass: the rows r = (p, m1) of the paths into o (path
    order), their count n, padded width W, the offset of the block's d3 x W matrix in an edge's
    K row and the index of its first row pair."""
    blocks, off, pb = [], 0, 0
    for o, l3 in enumerate(spec.out_ls):
        rows = [(p, m1) for p in range(spec.P) if spec.paths[p][2] == o
                for m1 in range(2 * spec.triples[p][0] + 1)]
        if not rows:
            continue
        n, d3 = len(rows), 2 * l3 + 1
        W = (n + 3) // 4 * 4
        blocks.append(dict(o=o, d3=d3, rows=rows, n=n, W=W, off=off, pb=pb))
        off += d3 * W
        pb += (n + 1) // 2
    return blocks, off, pb


def _gen_kmt(spec: Spec) -> List[str]:
    """uvw sender pass with the transposed per-edge coupling matrix
         K_e[(o, m3), (p, m1)] = c_p sum_m2 C_p[m1, m2, m3] Y(v_e)[m2]      (out(p) = o)
       per channel w:  z[(p, m1)] = sum_m3 K_e[(o, m3), (p, m1)] gy[o, m3]   (two rows per FFMA2)
                       bt[(p, m1)] += s[e, p] z[(p, m1)],   gs[p] += sum_m1 xt[(p, m1)] z[(p, m1)].
       The sender state xt / bt is held in the same row-pair order.  An edge's row in shared
       memory: the K entries ([block][m3][W], zero padded), then s[e, p] per row pair."""
    blocks, krow, pairs = _kmt_blocks(spec)
    srow = (2 * pairs + 3) // 4 * 4
    L = [f"  static constexpr int KMT_ROW = {krow + srow};",
         f"  static constexpr int KMT_PAIRS = {pairs};"]
    rows_flat = []                       # (pair index, half) -> (p, m1) or None
    for B in blocks:
        for q in range((B["n"] + 1) // 2):
            for h in range(2):
                r = 2 * q + h
                rows_flat.append(B["rows"][r] if r < B["n"] else None)
    entries = []
    for B in blocks:
        for m3 in range(B["d3"]):
            for r in range(B["W"]):
                if r >= B["n"]:
                    entries.append((0, "0.0f"))
                    continue
                p, m1 = B["rows"][r]
                b = spec.paths[p][1]
                lb = spec.sh_ls[b]
                nz = [(j, c) for (i, j, k, c) in cg_nonzeros(*spec.triples[p]) if i == m1 and k == m3]
                if not nz:
                    entries.append((0, "0.0f"))
                elif lb == 0:
                    entries.append((2, f"{_flt(nz[0][1])} * cf[{p}]"))
                else:
                    t = " + ".join(f"{_flt(c)} * Y[{spec.sh_cum[b] + j}]" for j, c in nz)
                    entries.append((len(nz) + 1, f"cf[{p}] * ({t})"))
    for rf in rows_flat:
        entries.append((1, "0.0f" if rf is None else f"s[{rf[0]}]"))
    while len(entries) % 4:
        entries.append((0, "0.0f"))
    assert len(entries) == krow + srow
    groups = [entries[4 * g:4 * g + 4] for g in range(len(entries) // 4)]
    gcost = [1 + sum(c for c, _ in grp) for grp in groups]
    L.append("  template <int H>")
    L.append(f"  __device__ __forceinline__ static void kmt_build(int h, const float (&Y)[{spec.NSH}], "
             f"const float (&cf)[{spec.P}], const float (&s)[{spec.P}], float4* __restrict__ k) {{")
    L.append("    (void)Y;")
    for H in (1, 2, 4):
        total = sum(gcost)
        cuts, acc, part = [0], 0, 1
        for g, c in enumerate(gcost):
            acc += c
            if part < H and acc >= total * part / H:
                cuts.append(g + 1)
                part += 1
        while len(cuts) < H:
            cuts.append(len(groups))
        cuts.append(len(groups))
        L.append(f"    if constexpr (H == {H}) {{")
        for h in range(H):
            L.append(f"      if (h == {h}) {{")
            for g in range(cuts[h], cuts[h + 1]):
                ex = [e for _, e in groups[g]]
                L.append(f"        k[{g}] = make_float4({ex[0]}, {ex[1]}, {ex[2]}, {ex[3]});")
            L.append("      }")
        L.append("    }")
    L.append("  }")
    # per channel: z, bt, gs
    L.append(f"  __device__ __forceinline__ static void kmt_apply(const float (&gy)[{spec.OUT_PC}], "
             f"const float4* __restrict__ k, const float2 (&xt)[{pairs}], float2 (&bt)[{pairs}], "
             f"float (&gs)[{spec.P}]) {{")
    L.append(f"    float2 z[{pairs}];")
    for B in blocks:
        npair = (B["n"] + 1) // 2
        for m3 in range(B["d3"]):
            gi = spec.out_cum[B["o"]] + m3
            L.append("    {")
            L.append(f"      const float2 g = make_float2(gy[{gi}], gy[{gi}]);")
            for q in range(B["W"] // 4):
                g = (B["off"] + m3 * B["W"]) // 4 + q
                L.append(f"      {{ const float4 v = k[{g}];")
                for half, (lo, hi) in enumerate((("x", "y"), ("z", "w"))):
                    pi = 2 * q + half
                    if pi >= npair:
                        continue
                    zi = B["pb"] + pi
                    if m3 == 0:
                        L.append(f"        z[{zi}] = __fmul2_rn(g, make_float2(v.{lo}, v.{hi}));")
                    else:
                        L.append(f"        z[{zi}] = __ffma2_rn(g, make_float2(v.{lo}, v.{hi}), z[{zi}]);")
                L.append("      }")
            L.append("    }")
    sg = krow // 4
    for q4 in range((pairs + 1) // 2):
        L.append(f"    {{ const float4 v = k[{sg + q4}];")
        for half, (lo, hi) in enumerate((("x", "y"), ("z", "w"))):
            q = 2 * q4 + half
            if q >= pairs:
                continue
            L.append(f"      bt[{q}] = __ffma2_rn(make_float2(v.{lo}, v.{hi}), z[{q}], bt[{q}]);")
        L.append("    }")
    # gs: products in pairs, then the halves summed per path
    terms = {p: [] for p in range(spec.P)}
    for q in range(pairs):
        L.append(f"    const float2 h{q} = __fmul2_rn(xt[{q}], z[{q}]);")
        for half in range(2):
            rf = rows_flat[2 * q + half]
            if rf is not None:
                terms[rf[0]].append(f"h{q}.{'x' if half == 0 else 'y'}")
    for p in range(spec.P):
        t = terms[p]
        L.append(f"    gs[{p}] = {' + '.join(t) if t else '0.0f'};")
    L.append("  }")
    # sender state in row-pair order (the load_xt / store_xt layout in memory)
    ins, _ = _uvw_in_tables(spec)
    for name, const in (("kmt_load_xt", True), ("kmt_store_bt", False)):
        L.append(f"  __device__ __forceinline__ static void {name}({'const ' if const else ''}float* __restrict__ base, "
                 f"int64_t N, int mul, int64_t j, int c, {'float2' if const else 'const float2'} (&v)[{pairs}]) {{")
        for q in range(pairs):
            for half in range(2):
                rf = rows_flat[2 * q + half]
                comp = f"v[{q}].{'x' if half == 0 else 'y'}"
                if rf is None:
                    if const:
                        L.append(f"    {comp} = 0.0f;")
                    continue
                p, m1 = rf
                t = ins[spec.paths[p][0]]
                pl = t["paths"].index(p)
                idx = f"N * mul * {t['cumX']} + ((j * {t['d1']} + {m1}) * {t['cnt']} + {pl}) * (int64_t)mul + c"
                L.append(f"    {comp} = __ldg(base + {idx});" if const else f"    base[{idx}] = {comp};")
        L.append("  }")
    return L


def gen_spec_header(spec: Spec) -> str:
    L = [f"// Generated by codegen.py for spec '{spec.name}'.  Do not edit.",
         f"// inputs l={spec.in_ls}  SH l={spec.sh_ls}  outputs l={spec.out_ls}",
         f"// paths (in, sh, out) = {spec.paths}",
         f"// non-zero CG entries: {spec.nnz_total()}",
         "#pragma once",
         f"struct Spec_{spec.name} {{",
         f"  static constexpr int IN_PC = {spec.IN_PC};",
         f"  static constexpr int OUT_PC = {spec.OUT_PC};",
         f"  static constexpr int NSH = {spec.NSH};",
         f"  static constexpr int P = {spec.P};",
         f"  static constexpr int A_PC = {spec.A_PC};",
         f"  static constexpr int LMAX_SH = {spec.LMAX_SH};",
         f"  static constexpr int NNZ = {spec.nnz_total()};",
         f"  static constexpr int FAST_MUL0 = {spec.fast_muls[0]};",
         f"  static constexpr int FAST_MUL1 = {spec.fast_muls[1]};"]
    L += _lines_load("load_in", len(spec.in_ls), spec.in_d, spec.in_cum, "x")
    L += _lines_load("load_in_shared", len(spec.in_ls), spec.in_d, spec.in_cum, "x", shared=True)
    L += _lines_store("store_in", len(spec.in_ls), spec.in_d, spec.in_cum, "x")
    L += _lines_load("load_out", len(spec.out_ls), spec.out_d, spec.out_cum, "y")
    L += _lines_load("load_out_shared", len(spec.out_ls), spec.out_d, spec.out_cum, "y", shared=True)
    L += _lines_store("store_out", len(spec.out_ls), spec.out_d, spec.out_cum, "y")
    # uvw per-path state rows [p][u][m3]
    L += _lines_load("load_a", spec.P, spec.a_d, spec.a_cum, "a")
    L += _lines_store("store_a", spec.P, spec.a_d, spec.a_cum, "a")
    L += _gen_sh(spec)
    L += _gen_fwd(spec)
    L += _gen_fwd(spec, name="uvw_edge", weighted_out="A", per_path_out=True)
    L += _gen_bwd(spec)
    L += _gen_fwd2(spec)
    L += _gen_dbwd_recv(spec)
    L += _gen_dbwd_send(spec)
    L += _gen_uvw_layout(spec)
    lay, xt_cum, xt_pc = _gen_uvw_send_layout(spec)
    L += lay
    L += _gen_uvw_send(spec, xt_cum, xt_pc)
    L += _gen_km(spec)
    L += _gen_kmt(spec)
    L.append("};")
    return "\n".join(L) + "\n"


# ---------------------------------------------------------------------------
# Runtime path table: one set of contractions per (l1, l2, l3) triple
# ---------------------------------------------------------------------------

def all_triples():
    """Every (l1, l2, l3) with l <= 3 that satisfies the triangle rule, lexicographic (34)."""
    return [(a, b, c) for a in range(4) for b in range(4) for c in range(4) if abs(a - b) <= c <= a + b]


def _gen_triple(l1, l2, l3) -> List[str]:
    """fwd: t[m3] = sum C x[m1] Y[m2];  tx: z[m1] = sum C Y[m2] g[m3];  ty: q[m2] = sum C x[m1] g[m3]."""
    nz = cg_nonzeros(l1, l2, l3)
    d1, d2, d3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
    L = [f"template <> struct Cg<{l1}, {l2}, {l3}> {{",
         f"  static constexpr int L1 = {l1}, L2 = {l2}, L3 = {l3}, D1 = {d1}, D2 = {d2}, D3 = {d3}, NNZ = {len(nz)};"]

    def body(name, a, an, b, bn, out, on, key_pair, key_out):
        L.append(f"  __device__ __forceinline__ static void {name}(const float (&{a})[{an}], const float (&{b})[{bn}], "
                 f"float (&{out})[{on}]) {{")
        used = sorted({key_pair(i, j, k) for i, j, k, c in nz})
        for (u, v) in used:
            # no shortcut for l2 = 0: the double backward passes dY (zero for l = 0) in place of Y
            L.append(f"    const float p{u}_{v} = {a}[{u}] * {b}[{v}];")
        for m in range(on):
            terms = [(c, "p%d_%d" % key_pair(i, j, k)) for (i, j, k, c) in nz if key_out(i, j, k) == m]
            L.extend(line.replace("      ", "    ", 1) for line in _chain(terms, f"{out}[{m}]", decl=False))
        L.append("  }")

    body("fwd", "x", d1, "Y", d2, "t", d3, lambda i, j, k: (i, j), lambda i, j, k: k)
    body("tx", "Y", d2, "g", d3, "z", d1, lambda i, j, k: (j, k), lambda i, j, k: i)
    body("ty", "x", d1, "g", d3, "q", d2, lambda i, j, k: (i, k), lambda i, j, k: j)
    L.append("};")
    return L


def _gen_sh_block(l) -> List[str]:
    """Real SH of one degree l as Cartesian polynomials of r_hat, their gradient and the Hessian
    applied to a direction d (for the double backward)."""
    polys = sh_polys()[l]
    d = 2 * l + 1
    L = [f"template <> struct ShBlock<{l}> {{", f"  static constexpr int L = {l}, D = {d};",
         f"  __device__ __forceinline__ static void sh(float rx, float ry, float rz, float (&Y)[{d}]) {{"]
    L += _monomials_code(max(l, 1))
    L.append("    (void)rx; (void)ry; (void)rz;")
    for m in range(d):
        L.append(f"    Y[{m}] = {_poly_expr(polys[m])};")
    L.append("  }")
    L.append(f"  __device__ __forceinline__ static void grad(float rx, float ry, float rz, float (&G)[{d}][3]) {{")
    L += _monomials_code(max(l - 1, 1))
    L.append("    (void)rx; (void)ry; (void)rz;")
    for m in range(d):
        for ax in range(3):
            L.append(f"    G[{m}][{ax}] = {_poly_expr(dpoly(polys[m], ax))};")
    L.append("  }")
    L.append("};")
    return L


def gen_generic_header() -> str:
    tr = all_triples()
    L = ["// Generated by codegen.py.  Do not edit.",
         "// Contractions of the real Clebsch-Gordan tensor of every (l1, l2, l3) triple with l <= 3 (non-zero",
         "// entries only, unrolled), for the runtime path table of plans without a compiled specialisation,",
         "// and the real spherical harmonics of each degree, all degrees at once (ShAll) with gradients and",
         "// Hessian-direction products.",
         "#pragma once",
         "namespace tp {",
         "namespace gen {",
         f"constexpr int kNumTriples = {len(tr)};",
         "template <int L1, int L2, int L3> struct Cg;"]
    for t in tr:
        L += _gen_triple(*t)
    ids = [-1] * 64
    for k, (a, b, c) in enumerate(tr):
        ids[a * 16 + b * 4 + c] = k
    L.append("__host__ __device__ inline int triple_id(int l1, int l2, int l3) {")
    L.append(f"  constexpr int v[64] = {{{', '.join(map(str, ids))}}};")
    L.append("  return (l1 | l2 | l3) >= 0 && l1 < 4 && l2 < 4 && l3 < 4 ? v[l1 * 16 + l2 * 4 + l3] : -1;")
    L.append("}")
    L.append("// Calls f(Cg<l1, l2, l3>{}) for the triple with id `id` (warp-uniform in every caller).")
    L.append("template <class F>")
    L.append("__device__ __forceinline__ void with_triple(int id, F&& f) {")
    L.append("  switch (id) {")
    for k, (a, b, c) in enumerate(tr):
        L.append(f"    case {k}: f(Cg<{a}, {b}, {c}>{{}}); break;")
    L.append("    default: break;")
    L.append("  }")
    L.append("}")
    L.append("template <int L> struct ShBlock;")
    for l in range(4):
        L += _gen_sh_block(l)
    allsh = Spec("all", [0], [0, 1, 2, 3], [0], [(0, 0, 0)])
    L.append("struct ShAll {")
    L.append("  static constexpr int NSH = 16;")
    L += _gen_sh(allsh)
    L.append("};")
    L.append("}  // namespace gen")
    L.append("}  // namespace tp")
    return "\n".join(L) + "\n"


# ---------------------------------------------------------------------------
# Spherical grid of the Gaunt (grid) convolution
# ---------------------------------------------------------------------------

def _gauss_legendre(n: int):
    """Nodes and weights of n-point Gauss-Legendre on [-1, 1], by Newton's iteration on P_n
    from the Chebyshev guesses (the textbook recurrence; float64)."""
    nodes, weights = [], []
    for k in range(n):
        t = math.cos(math.pi * (k + 0.75) / (n + 0.5))
        for _ in range(100):
            p0, p1 = 1.0, t
            for j in range(2, n + 1):
                p0, p1 = p1, ((2 * j - 1) * t * p1 - (j - 1) * p0) / j
            dp = n * (t * p1 - p0) / (t * t - 1.0) if n > 1 else 1.0
            step = p1 / dp
            t -= step
            if abs(step) < 1e-16:
                break
        p0, p1 = 1.0, t
        for j in range(2, n + 1):
            p0, p1 = p1, ((2 * j - 1) * t * p1 - (j - 1) * p0) / j
        dp = n * (t * p1 - p0) / (t * t - 1.0) if n > 1 else 1.0
        nodes.append(t)
        weights.append(2.0 / ((1.0 - t * t) * dp * dp))
    return nodes, weights


def _poly_value(p: Poly, x: float, y: float, z: float) -> float:
    return sum(c * x ** i * y ** j * z ** k for (i, j, k), c in p.items())


def gaunt_grid(L: int):
    """Points (x, y, z), weights summing to 1 and the harmonics of degrees 0..L at every point,
    for a grid that integrates polynomials of degree <= 3 L exactly on the sphere (products
    of three degree-L functions): ceil((3L+1)/2) Gauss-Legendre nodes in cos(theta) times
    3L+1 equispaced azimuths."""
    D = 3 * L
    n_t, n_p = D // 2 + 1, D + 1
    nodes, wts = _gauss_legendre(n_t)
    polys = sh_polys()
    pts, q, Y = [], [], []
    for t, a in zip(nodes, wts):
        st = math.sqrt(max(0.0, 1.0 - t * t))
        for j in range(n_p):
            ph = 2.0 * math.pi * j / n_p
            x, y, z = st * math.cos(ph), st * math.sin(ph), t
            pts.append((x, y, z))
            q.append(a / (2.0 * n_p))
            Y.append([_poly_value(polys[l][m], x, y, z) for l in range(L + 1) for m in range(2 * l + 1)])
    return pts, q, Y


def gen_gaunt_header() -> str:
    L_ = ["// Generated by codegen.py.  Do not edit.",
          "// Spherical grids of the Gaunt (grid) convolution: for L = 1, 2, 3 the points, quadrature weights",
          "// (summing to 1) and the real spherical harmonics of degrees 0..L at the points, exact for",
          "// polynomials of degree 3L on the sphere.",
          "#pragma once",
          "namespace tp {",
          "namespace gaunt {",
          "template <int L> struct Grid;"]
    for Lg in (1, 2, 3):
        pts, q, Y = gaunt_grid(Lg)
        ng, nsh = len(pts), (Lg + 1) ** 2
        L_.append(f"template <> struct Grid<{Lg}> {{")
        L_.append(f"  static constexpr int NG = {ng}, NSH = {nsh};")
        for name, vals in (("px", [p[0] for p in pts]), ("py", [p[1] for p in pts]), ("pz", [p[2] for p in pts]), ("q", q)):
            L_.append(f"  __device__ __forceinline__ static float {name}(int g) {{ constexpr float v[{ng}] = {{"
                      + ", ".join(_flt(v) for v in vals) + "}; return v[g]; }")
        # the grid is a product: point g = k * NP + j has cos(theta) = ct(k), azimuth phi_j
        D = 3 * Lg
        n_t, n_p = D // 2 + 1, D + 1
        nodes, _ = _gauss_legendre(n_t)
        L_.append(f"  static constexpr int NT = {n_t}, NP = {n_p};")
        for name, vals in (("ct", nodes), ("st", [math.sqrt(max(0.0, 1.0 - t * t)) for t in nodes]),
                           ("cp", [math.cos(2.0 * math.pi * j / n_p) for j in range(n_p)]),
                           ("sp", [math.sin(2.0 * math.pi * j / n_p) for j in range(n_p)])):
            L_.append(f"  __device__ __forceinline__ static float {name}(int i) {{ constexpr float v[{len(vals)}] = {{"
                      + ", ".join(_flt(v) for v in vals) + "}; return v[i]; }")
        flat = [Y[g][k] for g in range(ng) for k in range(nsh)]
        L_.append(f"  __device__ __forceinline__ static float Y(int g, int k) {{ constexpr float v[{ng * nsh}] = {{"
                  + ", ".join(_flt(v) for v in flat) + f"}}; return v[g * {nsh} + k]; }}")
        L_.append("};")
    L_ += ["}  // namespace gaunt", "}  // namespace tp"]
    return "\n".join(L_) + "\n"


# ---------------------------------------------------------------------------
# The compiled specialisations
# ---------------------------------------------------------------------------

def _all_paths(in_ls, in_par, sh_ls, out_irreps):
    """(in, sh, out) index triples in (l1, l2, l3) lexicographic order over the given irreps."""
    out = []
    for a, (l1, p1) in enumerate(zip(in_ls, in_par)):
        for b, l2 in enumerate(sh_ls):
            for o, (l3, p3) in enumerate(out_irreps):
                if abs(l1 - l2) <= l3 <= l1 + l2 and p3 == p1 * (-1) ** l2:
                    out.append((a, b, o))
    return out


def builtin_specs() -> List[Spec]:
    specs = []
    # lmax 1: c1-style (4 paths into 0e + 1o)
    specs.append(Spec("l1_c1", [0, 1], [0, 1], [0, 1], [(0, 0, 0), (0, 1, 1), (1, 0, 1), (1, 1, 0)]))
    for L in (1, 2, 3):
        ins = list(range(L + 1))
        par = [(-1) ** l for l in ins]
        outs = []
        for l in range(L + 1):
            for p in (1, -1):
                if l == 0 and p == -1:
                    continue
                outs.append((l, p))
        paths = _all_paths(ins, par, ins, outs)
        # keep only reachable outputs
        reach = sorted({o for _, _, o in paths})
        remap = {o: k for k, o in enumerate(reach)}
        paths = [(a, b, remap[o]) for a, b, o in paths]
        # channel counts compiled as constants: 32 and 128 for lmax 2, 32 and 64 for lmax 3
        fast = {1: (), 2: (32, 128), 3: (32, 64)}[L]
        specs.append(Spec(f"full_l{L}", ins, ins, [outs[o][0] for o in reach], paths, fast))
    return specs


def _ops_initializer(s: Spec, fns) -> str:
    def arr(v, n):
        v = list(v) + [0] * (n - len(v))
        return "{" + ", ".join(map(str, v)) + "}"
    paths = "{" + ", ".join("{%d, %d, %d}" % p for p in s.paths) + "}"
    xt_pc = _uvw_in_tables(s)[1]
    return (f"  \"{s.name}\", {len(s.in_ls)}, {arr(s.in_ls, 16)}, {len(s.sh_ls)}, {arr(s.sh_ls, 16)}, "
            f"{len(s.out_ls)}, {arr(s.out_ls, 16)}, {s.P}, {paths},\n"
            f"  {s.IN_PC}, {s.OUT_PC}, {s.NSH}, {s.P}, {s.A_PC}, {xt_pc},\n  " + ", ".join(fns))


# kernels of each spec, split into translation units that compile in parallel
PARTS = {
    "fwd": [("fwd_uvu", "launch_fwd_uvu")],
    "bwd": [("bwd_uvu", "launch_bwd_uvu")],
    "dbwd": [("dbwd_recv", "launch_dbwd_recv"), ("dbwd_send", "launch_dbwd_send")],
    "uvw": [("uvw_fwd", "launch_uvw_fwd"), ("uvw_bwd", "launch_uvw_bwd")],
}
SLOTS = ["fwd_uvu", "bwd_uvu", "dbwd_recv", "dbwd_send", "uvw_fwd", "uvw_bwd"]


def main(outdir: str):
    os.makedirs(outdir, exist_ok=True)
    specs = builtin_specs()
    written = []

    def write(name, text):
        path = os.path.join(outdir, name)
        old = open(path).read() if os.path.exists(path) else None
        if old != text:                      # keep mtimes stable for incremental builds
            with open(path, "w") as f:
                f.write(text)
        written.append(name)

    for s in specs:
        write(f"spec_{s.name}.h", gen_spec_header(s))
        for part, fns in PARTS.items():
            inc = "tp_uvw.cuh" if part == "uvw" else "tp_kernels.cuh"
            body = [f"// Generated by codegen.py: {part} kernels of spec '{s.name}'.",
                    f'#include "{inc}"', f'#include "spec_{s.name}.h"', "namespace tp {"]
            for slot, tmpl in fns:
                body.append(f"cudaError_t {s.name}_{slot}(const LaunchArgs& a, cudaStream_t st) "
                            f"{{ return {tmpl}<Spec_{s.name}>(a, st); }}")
            body.append("}  // namespace tp")
            write(f"k_{s.name}_{part}.cu", "\n".join(body) + "\n")
    reg = ["// Generated by codegen.py: registry of compiled specialisations.",
           '#include "tp_common.h"', "namespace tp {"]
    have = {slot for fns in PARTS.values() for slot, _ in fns}
    for s in specs:
        for slot in SLOTS:
            if slot in have:
                reg.append(f"cudaError_t {s.name}_{slot}(const LaunchArgs&, cudaStream_t);")
    for s in specs:
        fns = [f"&{s.name}_{slot}" if slot in have else "nullptr" for slot in SLOTS]
        reg.append(f"static const SpecOps ops_{s.name} = {{\n{_ops_initializer(s, fns)}}};")
    reg.append("const SpecOps* const kRegistry[] = {" + ", ".join(f"&ops_{s.name}" for s in specs) + "};")
    reg.append(f"const int kRegistrySize = {len(specs)};")
    reg.append("}  // namespace tp")
    write("registry.cu", "\n".join(reg) + "\n")
    write("generic_cg.h", gen_generic_header())
    write("gaunt_grid.h", gen_gaunt_header())
    # CG table dump (text) for the host-side table tests
    lines = []
    for l1, l2, l3 in product(range(4), repeat=3):
        if abs(l1 - l2) <= l3 <= l1 + l2:
            for (i, j, k, c) in cg_nonzeros(l1, l2, l3):
                lines.append(f"{l1} {l2} {l3} {i} {j} {k} {c:.17e}")
    write("cg_tables.txt", "\n".join(lines) + "\n")
    return specs, written


if __name__ == "__main__":
    main(sys.argv[1] if len(sys.argv) > 1 else os.path.join(os.path.dirname(__file__), "gen"))
