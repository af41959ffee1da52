"""Pins for the float64 spherical-grid (Gaunt) convolution oracle (oracle/gaunt.py).

The Gaunt coefficients the oracle integrates on its grid are checked against sympy's
complex Gaunt coefficients (a closed form) taken into this package's real basis; the
operator against rotation equivariance, two closed-form special cases (a weighted SpMV and
a pure filter), and its backward against finite differences."""
import math

import numpy as np
import pytest
import scipy.sparse as sp
import torch

from oracle.gaunt import GauntPlan, gaunt_backward, gaunt_forward, gaunt_tensor, quadrature
from oracle.so3 import random_rotation, real_sh, wigner_D


def _U(l):
    """Real SH (component normalisation, no Condon-Shortley phase) = sqrt(4 pi) U . complex
    orthonormal SH with the Condon-Shortley phase."""
    d = 2 * l + 1
    M = np.zeros((d, d), dtype=complex)
    for m in range(-l, l + 1):
        if m > 0:
            M[m + l, m + l] = (-1) ** m / math.sqrt(2)
            M[m + l, -m + l] = 1 / math.sqrt(2)
        elif m < 0:
            k = -m
            M[m + l, k + l] = (-1) ** k / (1j * math.sqrt(2))
            M[m + l, -k + l] = -1 / (1j * math.sqrt(2))
        else:
            M[l, l] = 1
    return M


def _sympy_real_gaunt(l1, l2, l3):
    from sympy.physics.wigner import gaunt
    d1, d2, d3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
    Gc = np.zeros((d1, d2, d3))
    for a in range(d1):
        for b in range(d2):
            for c in range(d3):
                Gc[a, b, c] = float(gaunt(l1, l2, l3, a - l1, b - l2, c - l3))
    Gr = math.sqrt(4 * math.pi) * np.einsum("ia,jb,kc,abc->ijk", _U(l1), _U(l2), _U(l3), Gc)
    assert np.abs(Gr.imag).max() < 1e-12
    return Gr.real


TRIPLES = [(a, b, c) for a in range(4) for b in range(4) for c in range(4)]


@pytest.mark.parametrize("t", TRIPLES)
def test_gaunt_tensor_matches_sympy(t):
    G = gaunt_tensor(*t).numpy()
    np.testing.assert_allclose(G, _sympy_real_gaunt(*t), atol=1e-12)
    if sum(t) % 2 or not abs(t[0] - t[1]) <= t[2] <= t[0] + t[1]:
        assert np.abs(G).max() < 1e-12


def test_quadrature_is_exact_and_normalised():
    pts, w = quadrature(9)
    assert abs(w.sum() - 1.0) < 1e-14
    np.testing.assert_allclose(np.linalg.norm(pts, axis=1), 1.0, atol=1e-14)
    # orthonormality of the harmonics against dOmega / 4 pi up to l = 4 (products of degree 8)
    for l in range(5):
        Y = real_sh(l, torch.as_tensor(pts)).numpy()
        np.testing.assert_allclose(np.einsum("g,ga,gb->ab", w, Y, Y), np.eye(2 * l + 1), atol=1e-12)


def _graph(seed, N, deg):
    rng = np.random.default_rng(seed)
    d = rng.integers(0, deg + 1, N)
    rowptr = np.concatenate([[0], np.cumsum(d)])
    src = rng.integers(0, N, rowptr[-1])
    vec = rng.standard_normal((rowptr[-1], 3)) * rng.uniform(0.5, 3.0, (rowptr[-1], 1))
    return rowptr, src, vec, rng


def test_scalar_case_is_a_weighted_spmv():
    plan = GauntPlan("3x0e", 0, "3x0e")
    rowptr, src, vec, rng = _graph(0, 20, 6)
    x = rng.standard_normal((20, 3))
    w = rng.standard_normal((len(src), 3))
    y = gaunt_forward(plan, rowptr, src, x, vec, w).numpy()
    for u in range(3):
        A = sp.csr_matrix((w[:, u], src, rowptr), shape=(20, 20))
        np.testing.assert_allclose(y[:, u], A @ x[:, u], atol=1e-12)


@pytest.mark.parametrize("L", [1, 2, 3])
def test_pure_filter_case(L):
    """Scalar inputs into degree L: y[i, u, m] = sum_e x[src, u] w[e, L, u] Y_Lm(v_e)."""
    plan = GauntPlan("2x0e", L, f"2x{L}{'e' if L % 2 == 0 else 'o'}")
    rowptr, src, vec, rng = _graph(1, 15, 5)
    x = rng.standard_normal((15, 2))
    w = rng.standard_normal((len(src), (L + 1) * 2))
    y = gaunt_forward(plan, rowptr, src, x, vec, w).numpy().reshape(15, 2, 2 * L + 1)
    Y = real_sh(L, torch.as_tensor(vec)).numpy()
    ref = np.zeros_like(y)
    dst = np.repeat(np.arange(15), np.diff(rowptr))
    for e in range(len(src)):
        ref[dst[e]] += (x[src[e]] * w[e].reshape(L + 1, 2)[L])[:, None] * Y[e][None, :]
    np.testing.assert_allclose(y, ref, atol=1e-12)


@pytest.mark.parametrize("lin,L,lout", [("4x0e+4x1o+4x2e", 2, "4x0e+4x1o+4x2e"),
                                        ("3x1o+3x3o", 3, "3x0e+3x2e+3x3o")])
def test_equivariance(lin, L, lout):
    plan = GauntPlan(lin, L, lout)
    rowptr, src, vec, rng = _graph(2, 12, 5)
    x = rng.standard_normal((12, plan.in_dim))
    w = rng.standard_normal((len(src), plan.nw))
    R = random_rotation(rng)

    def rot(irreps, a):
        out, off = [], 0
        for term in irreps.split("+"):
            m, ir = term.split("x")
            l = int(ir[:-1])
            d = 2 * l + 1
            blk = a[:, off:off + int(m) * d].reshape(len(a), int(m), d)
            out.append(np.einsum("nud,ed->nue", blk, wigner_D(l, R)).reshape(len(a), -1))
            off += int(m) * d
        return np.concatenate(out, axis=1)

    y = gaunt_forward(plan, rowptr, src, x, vec, w).numpy()
    y_rot = gaunt_forward(plan, rowptr, src, rot(lin, x), vec @ R.T, w).numpy()
    np.testing.assert_allclose(y_rot, rot(lout, y), atol=1e-10)


def test_backward_matches_finite_differences():
    plan = GauntPlan("2x0e+2x1o+2x2e", 2, "2x0e+2x1o+2x2e")
    rowptr, src, vec, rng = _graph(3, 8, 4)
    x = rng.standard_normal((8, plan.in_dim))
    w = rng.standard_normal((len(src), plan.nw))
    gy = rng.standard_normal((8, plan.out_dim))
    g = gaunt_backward(plan, rowptr, src, x, vec, w, gy)
    f = lambda x_, v_, w_: float((gaunt_forward(plan, rowptr, src, x_, v_, w_) * torch.as_tensor(gy)).sum())
    h = 1e-6
    for name, arr in (("gx", x), ("gw", w), ("gvec", vec)):
        d = rng.standard_normal(arr.shape)
        args = lambda s: [x + s * d if name == "gx" else x, vec + s * d if name == "gvec" else vec,
                          w + s * d if name == "gw" else w]
        fd = (f(*args(h)) - f(*args(-h))) / (2 * h)
        an = float((g[name] * torch.as_tensor(d)).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_rejects_unnatural_parity():
    with pytest.raises(ValueError):
        GauntPlan("2x1e", 1, "2x0e")
