"""Pins for the oracle's spherical harmonics, Wigner-D and Clebsch-Gordan tables.

Each check compares the oracle with something other than itself: scipy's complex
spherical harmonics, textbook Cartesian closed forms, exact quadrature, sympy's
Clebsch-Gordan coefficients, group laws and hand-derived special cases.
"""
import math

import numpy as np
import pytest
import scipy.special as sps

from oracle.so3 import cg_real, random_rotation, real_sh_np, wigner_D

RNG = np.random.default_rng(0)


def _dirs(n=64, rng=RNG):
    v = rng.standard_normal((n, 3))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


def _real_from_scipy(l, r):
    """Real SH (component normalisation, no Condon-Shortley phase) from scipy's complex
    orthonormal SH, which carry the Condon-Shortley phase."""
    theta = np.arccos(np.clip(r[:, 2], -1, 1))
    phi = np.arctan2(r[:, 1], r[:, 0])
    out = np.zeros((len(r), 2 * l + 1))
    for m in range(-l, l + 1):
        k = abs(m)
        Yc = sps.sph_harm_y(l, k, theta, phi)
        if m > 0:
            val = math.sqrt(2) * (-1) ** k * Yc.real
        elif m < 0:
            val = math.sqrt(2) * (-1) ** k * Yc.imag
        else:
            val = Yc.real
        out[:, m + l] = math.sqrt(4 * math.pi) * val
    return out


@pytest.mark.parametrize("l", [0, 1, 2, 3, 4])
def test_sh_matches_scipy(l):
    r = _dirs()
    np.testing.assert_allclose(real_sh_np(l, r), _real_from_scipy(l, r), atol=1e-12)


@pytest.mark.parametrize("l", [0, 1, 2, 3, 4])
def test_sh_addition_theorem_and_scale_invariance(l):
    r = _dirs()
    Y = real_sh_np(l, r)
    np.testing.assert_allclose((Y ** 2).sum(1), 2 * l + 1, atol=1e-12)
    np.testing.assert_allclose(real_sh_np(l, 3.7 * r), Y, atol=1e-12)
    # addition theorem between two directions: sum_m Y(a) Y(b) = (2l+1) P_l(a.b)
    a, b = _dirs(8), _dirs(8)
    lhs = (real_sh_np(l, a) * real_sh_np(l, b)).sum(1)
    rhs = (2 * l + 1) * sps.eval_legendre(l, (a * b).sum(1))
    np.testing.assert_allclose(lhs, rhs, atol=1e-12)


def test_sh_quadrature_orthonormal():
    # Gauss-Legendre in cos(theta) x uniform phi is exact for these degrees
    xg, wg = np.polynomial.legendre.leggauss(12)
    nphi = 20
    phi = 2 * np.pi * np.arange(nphi) / nphi
    ct, ph = np.meshgrid(xg, phi, indexing="ij")
    st = np.sqrt(1 - ct ** 2)
    r = np.stack([st * np.cos(ph), st * np.sin(ph), ct], -1).reshape(-1, 3)
    wts = (np.repeat(wg, nphi) * (2 * np.pi / nphi)) / (4 * np.pi)
    Y = np.concatenate([real_sh_np(l, r) for l in range(5)], axis=1)
    G = (Y * wts[:, None]).T @ Y
    np.testing.assert_allclose(G, np.eye(G.shape[0]), atol=1e-12)


def test_sh_cartesian_closed_forms():
    """Textbook real solid harmonics on the unit sphere."""
    r = _dirs()
    x, y, z = r[:, 0], r[:, 1], r[:, 2]
    s3, s5, s15 = math.sqrt(3), math.sqrt(5), math.sqrt(15)
    Y1 = np.stack([s3 * y, s3 * z, s3 * x], 1)
    Y2 = np.stack([s15 * x * y, s15 * y * z, s5 / 2 * (2 * z * z - x * x - y * y), s15 * x * z,
                   s15 / 2 * (x * x - y * y)], 1)
    Y3 = np.stack([
        math.sqrt(70) / 4 * y * (3 * x * x - y * y), math.sqrt(105) * x * y * z,
        math.sqrt(42) / 4 * y * (4 * z * z - x * x - y * y),
        math.sqrt(7) / 2 * z * (2 * z * z - 3 * x * x - 3 * y * y),
        math.sqrt(42) / 4 * x * (4 * z * z - x * x - y * y), math.sqrt(105) / 2 * z * (x * x - y * y),
        math.sqrt(70) / 4 * x * (x * x - 3 * y * y)], 1)
    np.testing.assert_allclose(real_sh_np(0, r), np.ones((len(r), 1)), atol=1e-14)
    np.testing.assert_allclose(real_sh_np(1, r), Y1, atol=1e-13)
    np.testing.assert_allclose(real_sh_np(2, r), Y2, atol=1e-13)
    np.testing.assert_allclose(real_sh_np(3, r), Y3, atol=1e-13)


@pytest.mark.parametrize("l", [0, 1, 2, 3])
def test_sh_parity_and_zero_vector(l):
    r = _dirs()
    np.testing.assert_allclose(real_sh_np(l, -r), (-1) ** l * real_sh_np(l, r), atol=1e-13)
    z = real_sh_np(l, np.zeros((2, 3)))
    np.testing.assert_array_equal(z, np.ones((2, 1)) if l == 0 else np.zeros((2, 2 * l + 1)))


@pytest.mark.parametrize("l", [1, 2, 3])
def test_wigner_group_law(l):
    rng = np.random.default_rng(l)
    R1, R2 = random_rotation(rng), random_rotation(rng)
    D1, D2, D12 = wigner_D(l, R1), wigner_D(l, R2), wigner_D(l, R1 @ R2)
    np.testing.assert_allclose(D1 @ D1.T, np.eye(2 * l + 1), atol=1e-12)
    np.testing.assert_allclose(D12, D1 @ D2, atol=1e-12)
    np.testing.assert_allclose(abs(np.linalg.det(D1)), 1.0, atol=1e-12)


def test_wigner_l1_closed_form():
    rng = np.random.default_rng(3)
    R = random_rotation(rng)
    Pi = np.array([[0, 1, 0], [0, 0, 1], [1, 0, 0]], dtype=float)   # (x,y,z) -> (y,z,x)
    np.testing.assert_allclose(wigner_D(1, R), Pi @ R @ Pi.T, atol=1e-12)


TRIPLES = [(l1, l2, l3) for l1 in range(4) for l2 in range(4) for l3 in range(4)
           if abs(l1 - l2) <= l3 <= l1 + l2]


def test_cg_triple_count():
    assert len(TRIPLES) == 34


def _sympy_real_cg(l1, l2, l3):
    """Real CG from sympy's complex Clebsch-Gordan coefficients.

    Complex -> real change of basis for SH values without the Condon-Shortley phase:
    m>0: (( -1)^m Y^m + Y^-m)/sqrt2; m<0: ((-1)^k Y^k - Y^-k)/(i sqrt2), k=|m|; m=0: Y^0.
    C_r = sum U3[m3,mu3] CG[mu1,mu2,mu3] conj(U1[m1,mu1]) conj(U2[m2,mu2]).
    """
    from sympy.physics.wigner import clebsch_gordan

    def U(l):
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

    d1, d2, d3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
    CG = np.zeros((d1, d2, d3))
    for a in range(d1):
        for b in range(d2):
            c = (a - l1) + (b - l2) + l3
            if 0 <= c < d3:
                CG[a, b, c] = float(clebsch_gordan(l1, l2, l3, a - l1, b - l2, c - l3))
    Cr = np.einsum("kc,abc,ia,jb->ijk", U(l3), CG, U(l1).conj(), U(l2).conj())
    if np.abs(Cr.imag).max() > np.abs(Cr.real).max():
        Cr = Cr.imag + 0j
    assert np.abs(Cr.imag).max() < 1e-12
    C = Cr.real
    C[np.abs(C) < 1e-12] = 0
    first = C.reshape(-1)[np.nonzero(C.reshape(-1))[0][0]]
    return C * np.sign(first)


@pytest.mark.parametrize("t", TRIPLES)
def test_cg_matches_sympy(t):
    np.testing.assert_allclose(cg_real(*t), _sympy_real_cg(*t), atol=1e-12)


@pytest.mark.parametrize("l1,l2", [(a, b) for a in range(4) for b in range(4)])
def test_cg_orthogonal_change_of_basis(l1, l2):
    cols = [cg_real(l1, l2, l3).reshape((2 * l1 + 1) * (2 * l2 + 1), -1)
            for l3 in range(abs(l1 - l2), l1 + l2 + 1)]
    M = np.concatenate(cols, axis=1)
    assert M.shape[0] == M.shape[1]
    np.testing.assert_allclose(M.T @ M, np.eye(M.shape[1]), atol=1e-12)
    np.testing.assert_allclose(M @ M.T, np.eye(M.shape[0]), atol=1e-12)


@pytest.mark.parametrize("t", TRIPLES)
def test_cg_equivariant(t):
    l1, l2, l3 = t
    rng = np.random.default_rng(sum(t) + 11)
    C = cg_real(*t)
    for _ in range(2):
        R = random_rotation(rng)
        a, b = rng.standard_normal(2 * l1 + 1), rng.standard_normal(2 * l2 + 1)
        lhs = np.einsum("ijk,i,j->k", C, wigner_D(l1, R) @ a, wigner_D(l2, R) @ b)
        rhs = wigner_D(l3, R) @ np.einsum("ijk,i,j->k", C, a, b)
        np.testing.assert_allclose(lhs, rhs, atol=1e-12)


def test_cg_special_cases():
    for l in range(4):
        d = 2 * l + 1
        np.testing.assert_allclose(cg_real(0, l, l)[0], np.eye(d), atol=1e-14)
        np.testing.assert_allclose(cg_real(l, 0, l)[:, 0, :], np.eye(d), atol=1e-14)
        np.testing.assert_allclose(cg_real(l, l, 0)[:, :, 0], np.eye(d) / math.sqrt(d), atol=1e-14)
    eps = np.zeros((3, 3, 3))
    for i, j, k in [(0, 1, 2), (1, 2, 0), (2, 0, 1)]:
        eps[i, j, k], eps[j, i, k] = 1, -1
    np.testing.assert_allclose(cg_real(1, 1, 1), eps / math.sqrt(2), atol=1e-14)


@pytest.mark.parametrize("t", [t for t in TRIPLES if sum(t) % 2 == 0])
def test_cg_couples_harmonics_to_harmonics(t):
    """For even l1+l2+l3, coupling Y_l1(r) with Y_l2(r) gives a fixed multiple of Y_l3(r)."""
    l1, l2, l3 = t
    r = _dirs(16)
    f = np.einsum("ijk,ei,ej->ek", cg_real(*t), real_sh_np(l1, r), real_sh_np(l2, r))
    Y3 = real_sh_np(l3, r)
    ratio = (f * Y3).sum(1) / (2 * l3 + 1)
    assert np.ptp(ratio) < 1e-12
    np.testing.assert_allclose(f, ratio[:, None] * Y3, atol=1e-12)
    # |ratio| = sqrt((2l1+1)(2l2+1)/(2l3+1)) |<l1 0 l2 0 | l3 0>| (Gaunt)
    from sympy.physics.wigner import clebsch_gordan
    g = abs(float(clebsch_gordan(l1, l2, l3, 0, 0, 0)))
    expect = math.sqrt((2 * l1 + 1) * (2 * l2 + 1) / (2 * l3 + 1)) * g
    np.testing.assert_allclose(abs(ratio[0]), expect, atol=1e-12)
