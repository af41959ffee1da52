"""The CUDA path's compile-time tables (Racah-route CG, Cartesian SH polynomials and their
symbolic derivatives) against the oracle's independent routes (null-space CG, Legendre
SH, autograd derivatives)."""
import math
import os
import sys

import numpy as np
import pytest
import torch

from oracle.so3 import cg_real, real_sh

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.join(ROOT, "equivariant_tensor_product_b200", "csrc"))
import codegen  # noqa: E402

TRIPLES = [(a, b, c) for a in range(4) for b in range(4) for c in range(4) if abs(a - b) <= c <= a + b]


@pytest.mark.parametrize("t", TRIPLES)
def test_cg_tables_match_oracle(t):
    gen = np.array(codegen.cg_real(*t))
    ref = cg_real(*t)
    np.testing.assert_array_equal(gen != 0, ref != 0)
    np.testing.assert_allclose(gen, ref, atol=1e-12)


def test_cg_dump_file_matches(tmp_path):
    codegen.main(str(tmp_path))
    rows = [l.split() for l in open(tmp_path / "cg_tables.txt")]
    assert len(rows) == sum(int((cg_real(*t) != 0).sum()) for t in TRIPLES)
    for r in rows:
        l1, l2, l3, i, j, k = map(int, r[:6])
        assert abs(float(r[6]) - cg_real(l1, l2, l3)[i, j, k]) < 1e-12


def _eval(poly, r):
    out = np.zeros(len(r))
    for (i, j, k), c in poly.items():
        out += c * r[:, 0] ** i * r[:, 1] ** j * r[:, 2] ** k
    return out


def _dirs(n=32, seed=0):
    v = np.random.default_rng(seed).standard_normal((n, 3))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


@pytest.mark.parametrize("l", [0, 1, 2, 3])
def test_sh_polynomials_match_oracle(l):
    r = _dirs()
    polys = codegen.sh_polys()[l]
    gen = np.stack([_eval(p, r) for p in polys], 1)
    ref = real_sh(l, torch.as_tensor(r)).numpy()
    np.testing.assert_allclose(gen, ref, atol=1e-13)


@pytest.mark.parametrize("l", [1, 2, 3])
def test_sh_derivative_formulas_match_autograd(l):
    """dY/dv = (grad P - l Y r)/|v| and the Hessian-vector form used by the kernels, built from
    the generator's symbolic derivatives, against autograd of the oracle SH."""
    rng = np.random.default_rng(l)
    v = rng.standard_normal((8, 3)) * 2.0
    d = rng.standard_normal((8, 3))
    polys = codegen.sh_polys()[l]
    rr = np.linalg.norm(v, axis=1)
    r = v / rr[:, None]
    rd = (r * d).sum(1)
    vt = torch.as_tensor(v, dtype=torch.float64).requires_grad_(True)
    Y = real_sh(l, vt)
    for m, p in enumerate(polys):
        G = np.stack([_eval(codegen.dpoly(p, a), r) for a in range(3)], 1)
        H = np.zeros((len(r), 3, 3))
        for a in range(3):
            for b in range(3):
                H[:, a, b] = _eval(codegen.dpoly(codegen.dpoly(p, a), b), r)
        Ym = _eval(p, r)
        J = (G - l * Ym[:, None] * r) / rr[:, None]
        (gref,) = torch.autograd.grad(Y[:, m].sum(), vt, create_graph=True)
        np.testing.assert_allclose(J, gref.detach().numpy(), atol=1e-12)
        Hd = np.einsum("nab,nb->na", H, d)
        Gd = (G * d).sum(1)
        K = (Hd - l * (G * rd[:, None] + r * Gd[:, None] + Ym[:, None] * d)
             + l * (l + 2) * Ym[:, None] * r * rd[:, None]) / (rr ** 2)[:, None]
        (kref,) = torch.autograd.grad((gref * torch.as_tensor(d)).sum(), vt, retain_graph=True)
        np.testing.assert_allclose(K, kref.numpy(), atol=1e-11)


def test_builtin_specs_cover_the_workloads():
    import synth
    names = {s.name: s for s in codegen.builtin_specs()}
    assert [tuple(p) for p in names["full_l2"].paths] == [tuple(p) for p in synth.L2_PATHS]
    assert [tuple(p) for p in names["full_l3"].paths] == [tuple(p) for p in synth.L3_PATHS]
    assert [tuple(p) for p in names["l1_c1"].paths] == [tuple(p) for p in synth.C1_PATHS]
    assert names["full_l3"].nnz_total() == 611 and names["full_l2"].nnz_total() == 137
