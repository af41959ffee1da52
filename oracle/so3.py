"""Real spherical harmonics, Wigner-D matrices and real Clebsch-Gordan tensors (float64).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Conventions (the pages name spherical harmonics and Clebsch-Gordan coupling -- "The GPU
Workload That Rewrites Molecular Physics", section "Equivariant feature transforms" --
but fix no normalisation; the readings below are the plainest ones and are listed in the
design notes):
  * real SH, m = -l..l, z is the polar axis, no Condon-Shortley phase, "component"
    normalisation sum_m Y_lm(r)^2 = 2l+1 (so Y_0 = 1);
  * route: Y_lm = N_lm * (d^|m| P_l / dz^|m|)(z) * {Re, Im}((x + i y)^|m|) with
    N_lm = sqrt((2l+1) (l-|m|)!/(l+|m|)!) * (sqrt 2 if m != 0); Re for m >= 0, Im for m < 0;
  * a zero edge vector has r_hat := 0: Y_0 = 1 and Y_{l>0} = 0;
  * Wigner D^l(R) is defined by Y_l(R r) = D^l(R) Y_l(r) and fitted by least squares;
  * real CG C[m1,m2,m3] spans the one-dimensional space of tensors with
    C(D1 a, D2 b) = D3 C(a, b); normalised to ||C||_F^2 = 2 l3 + 1 (unitary coupling), and
    its first non-zero entry in row-major (m1, m2, m3) order is positive.
"""
from __future__ import annotations

import functools
import math

import numpy as np
import torch
from numpy.polynomial import legendre as npleg

__all__ = ["real_sh", "real_sh_np", "wigner_D", "cg_real", "random_rotation"]


@functools.lru_cache(maxsize=None)
def _legendre_deriv_power(l: int, m: int):
    """Power-series coefficients (in z) of d^m P_l / dz^m."""
    c = np.zeros(l + 1)
    c[l] = 1.0
    d = npleg.legder(c, m) if m > 0 else c
    return tuple(npleg.leg2poly(d).tolist())


def _norm(l: int, m: int) -> float:
    am = abs(m)
    n = math.sqrt((2 * l + 1) * math.factorial(l - am) / math.factorial(l + am))
    return n * (math.sqrt(2.0) if m != 0 else 1.0)


def real_sh(l: int, vec: torch.Tensor) -> torch.Tensor:
    """Y_l(vec/|vec|) as a [E, 2l+1] float64 tensor (differentiable in vec)."""
    vec = vec.to(torch.float64)
    r2 = (vec * vec).sum(-1, keepdim=True)
    nz = r2 > 0
    safe = torch.where(nz, r2, torch.ones_like(r2))
    rhat = torch.where(nz, vec / torch.sqrt(safe), torch.zeros_like(vec))
    x, y, z = rhat[..., 0], rhat[..., 1], rhat[..., 2]
    # (x + i y)^k for k = 0..l
    re = [torch.ones_like(x)]
    im = [torch.zeros_like(x)]
    for _ in range(l):
        re.append(re[-1] * x - im[-1] * y)
        im.append(re[-2] * y + im[-1] * x)
    cols = []
    for m in range(-l, l + 1):
        am = abs(m)
        coef = _legendre_deriv_power(l, am)
        q = torch.zeros_like(z)
        for k in range(len(coef) - 1, -1, -1):       # Horner in z
            q = q * z + coef[k]
        part = re[am] if m >= 0 else im[am]
        cols.append(_norm(l, m) * q * part)
    out = torch.stack(cols, dim=-1)
    if l > 0:
        out = out * nz.to(out.dtype)
    return out


def real_sh_np(l: int, vec) -> np.ndarray:
    with torch.no_grad():
        return real_sh(l, torch.as_tensor(np.asarray(vec, dtype=np.float64))).numpy()


def random_rotation(rng: np.random.Generator) -> np.ndarray:
    """Uniform random rotation matrix from a normalised Gaussian quaternion."""
    q = rng.standard_normal(4)
    q /= np.linalg.norm(q)
    a, b, c, d = q
    return np.array([
        [a * a + b * b - c * c - d * d, 2 * (b * c - a * d), 2 * (b * d + a * c)],
        [2 * (b * c + a * d), a * a - b * b + c * c - d * d, 2 * (c * d - a * b)],
        [2 * (b * d - a * c), 2 * (c * d + a * b), a * a - b * b - c * c + d * d],
    ])


_FIT_DIRS = None


def _fit_dirs() -> np.ndarray:
    global _FIT_DIRS
    if _FIT_DIRS is None:
        g = np.random.default_rng(12345).standard_normal((160, 3))
        _FIT_DIRS = g / np.linalg.norm(g, axis=1, keepdims=True)
    return _FIT_DIRS


def wigner_D(l: int, R: np.ndarray) -> np.ndarray:
    """D^l(R) with Y_l(R r) = D^l(R) Y_l(r), by least squares over 160 directions."""
    r = _fit_dirs()
    A = real_sh_np(l, r)                  # [K, d]
    B = real_sh_np(l, r @ np.asarray(R, dtype=np.float64).T)
    DT, *_ = np.linalg.lstsq(A, B, rcond=None)
    return DT.T


@functools.lru_cache(maxsize=None)
def _cg_cached(l1: int, l2: int, l3: int):
    d1, d2, d3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
    rng = np.random.default_rng(7 + 100 * l1 + 10 * l2 + l3)
    rows = []
    for _ in range(3):
        R = random_rotation(rng)
        K = np.kron(np.kron(wigner_D(l1, R), wigner_D(l2, R)), wigner_D(l3, R))
        rows.append(K.T - np.eye(d1 * d2 * d3))
    M = np.concatenate(rows, axis=0)
    _, sv, vt = np.linalg.svd(M)
    null = vt[-1]
    if sv[-1] > 1e-9 or (len(sv) > 1 and sv[-2] < 1e-6):
        raise ValueError(f"({l1},{l2},{l3}) has no unique coupling")
    C = null.reshape(d1, d2, d3)
    C *= math.sqrt(d3) / np.linalg.norm(C)
    C[np.abs(C) < 1e-12] = 0.0
    first = C.reshape(-1)[np.nonzero(C.reshape(-1))[0][0]]
    if first < 0:
        C = -C
    return C + 0.0          # no negative zeros


def cg_real(l1: int, l2: int, l3: int) -> np.ndarray:
    """Real Clebsch-Gordan tensor [2l1+1, 2l2+1, 2l3+1] (float64 copy)."""
    if not (abs(l1 - l2) <= l3 <= l1 + l2):
        raise ValueError("triangle rule violated")
    return _cg_cached(l1, l2, l3).copy()
