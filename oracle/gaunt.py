"""Plain float64 spherical-grid (Gaunt) tensor-product convolution.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

"The Price of Freedom: Exploring Expressivity and Runtime Tradeoffs in Equivariant Tensor
Products" (abstract) names the Gaunt tensor product: two equivariant features, read as
functions on the sphere, are multiplied pointwise and the product is expanded back into
spherical harmonics -- computed directly on a spherical grid.  The pages give no formula;
the plain reading used here, with the convolution's own ingredients:

  * a node feature with blocks of degrees l (natural parity (-1)^l, one multiplicity u for
    all blocks) is, per channel u, the function f_u(r) = sum_{l,m} x[u, l, m] Y_lm(r);
  * an edge e carries the filter g_{e,u}(r) = sum_{l2 <= L_sh} w[e, l2, u] sum_m2 Y_l2m2(v_e) Y_l2m2(r)
    (its spherical harmonics, scaled per degree and channel by the radial weights);
  * the message is the product projected onto the output degrees,
        t[e, u, l3, m3] = integral f_u(r) g_{e,u}(r) Y_l3m3(r) dOmega / (4 pi),
    and y[i] is the sum of the messages of the edges into i.

With the real Gaunt coefficients G(l1 m1, l2 m2, l3 m3) = integral Y_l1m1 Y_l2m2 Y_l3m3 dOmega/(4 pi)
this is
    y[i, u, l3, m3] = sum_e sum_{l1 m1 l2 m2} G(l1 m1, l2 m2, l3 m3) x[src_e, u, l1, m1] w[e, l2, u] Y_l2m2(v_e).

This module computes G by its integral (Gauss-Legendre in cos(theta) times an equispaced
azimuth grid, exact for these polynomial degrees, on this package's own spherical
harmonics) and the convolution by that sum, in float64, edges in receiver-aligned chunks;
the backward is torch autograd of it.
"""
from __future__ import annotations

import functools
from typing import Dict, List, Sequence, Tuple

import numpy as np
import torch

from .so3 import real_sh

__all__ = ["GauntPlan", "gaunt_tensor", "quadrature", "gaunt_forward", "gaunt_backward"]


def quadrature(degree: int) -> Tuple[np.ndarray, np.ndarray]:
    """Points [n, 3] and weights [n] (summing to 1) that integrate every polynomial of degree
    <= `degree` on the unit sphere exactly against dOmega / (4 pi)."""
    n_t = degree // 2 + 1
    n_p = degree + 1
    t, a = np.polynomial.legendre.leggauss(n_t)
    phi = 2.0 * np.pi * np.arange(n_p) / n_p
    st = np.sqrt(1.0 - t * t)
    pts = np.stack([np.outer(st, np.cos(phi)).ravel(), np.outer(st, np.sin(phi)).ravel(),
                    np.repeat(t, n_p)], axis=1)
    wts = np.repeat(a, n_p) / (2.0 * n_p)
    return pts, wts


@functools.lru_cache(maxsize=None)
def _gaunt_np(l1: int, l2: int, l3: int) -> np.ndarray:
    pts, wts = quadrature(l1 + l2 + l3 + 2)
    p = torch.as_tensor(pts)
    Y1, Y2, Y3 = (real_sh(l, p).numpy() for l in (l1, l2, l3))
    return np.einsum("g,ga,gb,gc->abc", wts, Y1, Y2, Y3)


def gaunt_tensor(l1: int, l2: int, l3: int) -> torch.Tensor:
    """G[m1, m2, m3] = integral Y_l1m1 Y_l2m2 Y_l3m3 dOmega / (4 pi) (float64)."""
    return torch.as_tensor(_gaunt_np(l1, l2, l3))


def _degrees(irreps: str) -> Tuple[int, List[int]]:
    mul, ls = None, []
    for term in irreps.replace(" ", "").split("+"):
        m, ir = term.split("x")
        l, par = int(ir[:-1]), ir[-1]
        if par != ("e" if l % 2 == 0 else "o"):
            raise ValueError(f"block {term}: the Gaunt product needs natural parity (-1)^l")
        if mul is not None and int(m) != mul:
            raise ValueError("one multiplicity for every block")
        mul = int(m)
        ls.append(l)
    return mul, ls


class GauntPlan:
    """Input degrees, filter degrees 0..lmax_sh, output degrees; one multiplicity."""

    def __init__(self, irreps_in: str, lmax_sh: int, irreps_out: str):
        self.mul, self.ls_in = _degrees(irreps_in)
        mo, self.ls_out = _degrees(irreps_out)
        if mo != self.mul:
            raise ValueError("input and output multiplicities differ")
        self.lmax_sh = lmax_sh
        self.in_off = np.concatenate([[0], np.cumsum([self.mul * (2 * l + 1) for l in self.ls_in])]).tolist()
        self.out_off = np.concatenate([[0], np.cumsum([self.mul * (2 * l + 1) for l in self.ls_out])]).tolist()
        self.in_dim, self.out_dim = self.in_off[-1], self.out_off[-1]
        self.nw = (lmax_sh + 1) * self.mul


def _t(a) -> torch.Tensor:
    """float64 tensor (a tensor keeps its autograd history)."""
    if isinstance(a, torch.Tensor):
        return a.to(torch.float64)
    return torch.as_tensor(np.asarray(a), dtype=torch.float64)


def _messages(plan: GauntPlan, xs: torch.Tensor, vec: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
    """Per-edge messages [Ec, out_dim]."""
    Ec, u = xs.shape[0], plan.mul
    w3 = w.reshape(Ec, plan.lmax_sh + 1, u)
    Ysh = [real_sh(l2, vec) for l2 in range(plan.lmax_sh + 1)]
    cols = []
    for l3 in plan.ls_out:
        acc = torch.zeros(Ec, u, 2 * l3 + 1, dtype=torch.float64)
        for k, l1 in enumerate(plan.ls_in):
            xa = xs[:, plan.in_off[k]:plan.in_off[k + 1]].reshape(Ec, u, 2 * l1 + 1)
            for l2 in range(plan.lmax_sh + 1):
                if (l1 + l2 + l3) % 2 or not abs(l1 - l2) <= l3 <= l1 + l2:
                    continue
                G = gaunt_tensor(l1, l2, l3)
                acc = acc + torch.einsum("eua,eb,abc->euc", xa, Ysh[l2], G) * w3[:, l2, :, None]
        cols.append(acc.reshape(Ec, u * (2 * l3 + 1)))
    return torch.cat(cols, dim=1)


def _dst(rowptr) -> torch.Tensor:
    rp = torch.as_tensor(np.asarray(rowptr, dtype=np.int64))
    return torch.repeat_interleave(torch.arange(len(rp) - 1), rp[1:] - rp[:-1])


def gaunt_forward(plan: GauntPlan, rowptr, src, x, vec, w, chunk: int = 1 << 13) -> torch.Tensor:
    """y[N, out_dim] in float64."""
    rowptr = np.asarray(rowptr, dtype=np.int64)
    N, E = len(rowptr) - 1, int(rowptr[-1])
    x, vec, w = _t(x), _t(vec), _t(w)
    src_t = torch.as_tensor(np.asarray(src, dtype=np.int64))
    dst = _dst(rowptr)
    y = torch.zeros(N, plan.out_dim, dtype=torch.float64)
    for e0 in range(0, E, chunk):
        e1 = min(E, e0 + chunk)
        y.index_add_(0, dst[e0:e1], _messages(plan, x[src_t[e0:e1]], vec[e0:e1], w[e0:e1]))
    return y


def gaunt_backward(plan: GauntPlan, rowptr, src, x, vec, w, gy) -> Dict[str, torch.Tensor]:
    """VJP of gaunt_forward against gy: gx, gw, gvec."""
    x, vec, w = (_t(a).detach().requires_grad_() for a in (x, vec, w))
    with torch.enable_grad():
        y = gaunt_forward(plan, rowptr, src, x, vec, w)
        gx, gw, gvec = torch.autograd.grad(y, (x, w, vec), _t(gy), allow_unused=True)
    z = lambda g, ref: torch.zeros_like(ref) if g is None else g.detach()
    return {"gx": z(gx, x), "gw": z(gw, w), "gvec": z(gvec, vec)}
