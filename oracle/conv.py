"""Plain float64 convolution: forward, backward (VJP) and double backward (VJP of the VJP).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Forward follows the definition written in oracle/__init__.py: per edge a dense einsum of
the gathered sender block, the edge's spherical harmonics and the CG tensor, scaled by
the radial weight, then ``index_add`` into the receiver ("Sobek", abstract: edge-local
products aggregated into receiver-side state; "FlashTP", abstract: the tensor-product
layer of equivariant interatomic potentials).  Edges are processed in receiver-aligned
chunks; every output is a sum of per-edge terms, so chunking is exact.

Backward = torch.autograd VJP with respect to (x, w, vec) -- or (x, s, W, vec) in uvw
mode.  Double backward = VJP of (x, vec, w[, W], gy) -> (gx, gw, gvec) against
(ggx, ggw, ggvec), by ``create_graph=True``.
"""
from __future__ import annotations

import os
from typing import Dict, Optional

import numpy as np
import torch

from .irreps import OraclePlan
from .so3 import cg_real, real_sh

__all__ = ["forward", "backward", "double_backward", "forward_uvw_reassociated", "set_threads"]


def set_threads(n: Optional[int] = None) -> int:
    n = n or len(os.sched_getaffinity(0))
    torch.set_num_threads(n)
    return n


def _t(a) -> torch.Tensor:
    if isinstance(a, torch.Tensor):
        return a.detach().to(torch.float64)
    return torch.as_tensor(np.asarray(a), dtype=torch.float64)


def _chunks(rowptr: np.ndarray, max_edges: int):
    """Receiver-aligned edge ranges [e0, e1) of at most ~max_edges edges (a single row may exceed)."""
    rowptr = np.asarray(rowptr, dtype=np.int64)
    n = len(rowptr) - 1
    E = int(rowptr[-1])
    out = []
    i = 0
    while i < n:
        e0 = int(rowptr[i])
        j = int(np.searchsorted(rowptr, e0 + max_edges, side="right")) - 1
        j = max(j, i + 1)
        j = min(j, n)
        out.append((i, j, e0, int(rowptr[j])))
        i = j
    if not out and E == 0:
        return []
    return out


def _edge_messages(plan: OraclePlan, xs, vec, wts, W) -> torch.Tensor:
    """Per-edge messages [Ec, out_dim] (plain form; the oracle may materialise them)."""
    Ec = xs.shape[0]
    Ysh = [real_sh(l, vec) for _, l, _ in plan.irr_sh.blocks]
    per_out = [None] * len(plan.irr_out)
    for p, (a, b, o) in enumerate(plan.paths):
        ma, la, _ = plan.irr_in.blocks[a]
        mo, lo, _ = plan.irr_out.blocks[o]
        d1, d3 = 2 * la + 1, 2 * lo + 1
        C = torch.as_tensor(cg_real(la, plan.triples[p][1], lo), dtype=torch.float64)
        xa = xs[:, plan.irr_in.offsets[a]: plan.irr_in.offsets[a] + ma * d1].reshape(Ec, ma, d1)
        if plan.mode == "uvu":
            T = torch.einsum("eum,en,mnk->euk", xa, Ysh[b], C)
            T = T * wts[:, plan.w_off[p]: plan.w_off[p] + ma, None]
        else:
            xm = torch.einsum("eum,uv->evm", xa, W[p])
            T = torch.einsum("evm,en,mnk->evk", xm, Ysh[b], C) * wts[:, p, None, None]
        T = plan.coeff[p] * T.reshape(Ec, mo * d3)
        per_out[o] = T if per_out[o] is None else per_out[o] + T
    cols = []
    for o, (mo, lo, _) in enumerate(plan.irr_out.blocks):
        cols.append(per_out[o] if per_out[o] is not None
                    else torch.zeros(Ec, mo * (2 * lo + 1), dtype=torch.float64))
    return torch.cat(cols, dim=1)


def _dst(rowptr: np.ndarray) -> torch.Tensor:
    rp = torch.as_tensor(np.asarray(rowptr, dtype=np.int64))
    return torch.repeat_interleave(torch.arange(len(rp) - 1), rp[1:] - rp[:-1])


def _weights(plan, w, s):
    return _t(w if plan.mode == "uvu" else s)


def forward(plan: OraclePlan, rowptr, src, x, vec, w=None, s=None, W=None,
            max_edges: int = 1 << 14) -> torch.Tensor:
    """y[N, out_dim] in float64."""
    rowptr = np.asarray(rowptr, dtype=np.int64)
    N = len(rowptr) - 1
    x, vec, wts = _t(x), _t(vec), _weights(plan, w, s)
    Wt = _t(W) if plan.mode == "uvw" else None
    src_t = torch.as_tensor(np.asarray(src, dtype=np.int64))
    dst = _dst(rowptr)
    y = torch.zeros(N, plan.irr_out.dim, dtype=torch.float64)
    with torch.no_grad():
        for _, _, e0, e1 in _chunks(rowptr, max_edges):
            if e1 == e0:
                continue
            m = _edge_messages(plan, x[src_t[e0:e1]], vec[e0:e1], wts[e0:e1], Wt)
            y.index_add_(0, dst[e0:e1], m)
    return y


def backward(plan: OraclePlan, rowptr, src, x, vec, gy, w=None, s=None, W=None,
             max_edges: int = 1 << 13) -> Dict[str, torch.Tensor]:
    """VJP of forward against gy: gx, gvec and gw (uvu) or gs, gW (uvw)."""
    rowptr = np.asarray(rowptr, dtype=np.int64)
    N = len(rowptr) - 1
    E = int(rowptr[-1])
    x0, vec0, wts0, gy = _t(x), _t(vec), _weights(plan, w, s), _t(gy)
    W0 = _t(W) if plan.mode == "uvw" else None
    src_t = torch.as_tensor(np.asarray(src, dtype=np.int64))
    dst = _dst(rowptr)
    gx = torch.zeros_like(x0)
    gwts = torch.zeros_like(wts0)
    gvec = torch.zeros(E, 3, dtype=torch.float64)
    gW = torch.zeros_like(W0) if W0 is not None else None
    for _, _, e0, e1 in _chunks(rowptr, max_edges):
        if e1 == e0:
            continue
        xl = x0.clone().requires_grad_(True)
        vl = vec0[e0:e1].clone().requires_grad_(True)
        wl = wts0[e0:e1].clone().requires_grad_(True)
        leaves = [xl, vl, wl]
        Wl = None
        if W0 is not None:
            Wl = W0.clone().requires_grad_(True)
            leaves.append(Wl)
        m = _edge_messages(plan, xl[src_t[e0:e1]], vl, wl, Wl)
        # <gy, y_chunk> = sum_e <gy[dst_e], m_e>
        L = (gy[dst[e0:e1]] * m).sum()
        g = torch.autograd.grad(L, leaves, allow_unused=True)
        gx += g[0]
        gvec[e0:e1] = g[1]
        gwts[e0:e1] = g[2]
        if W0 is not None:
            gW += g[3]
    out = {"gx": gx, "gvec": gvec}
    if plan.mode == "uvu":
        out["gw"] = gwts
    else:
        out["gs"] = gwts
        out["gW"] = gW
    return out


def double_backward(plan: OraclePlan, rowptr, src, x, vec, gy, ggx=None, ggw=None, ggvec=None,
                    w=None, max_edges: int = 1 << 12) -> Dict[str, torch.Tensor]:
    """uvu double backward: VJP of (x, vec, w, gy) -> (gx, gw, gvec) against (ggx, ggw, ggvec).

    Missing gg inputs are zero.  Returns g_gy, g_x, g_w, g_vec.
    """
    if plan.mode != "uvu":
        raise ValueError("oracle double backward is defined for uvu")
    rowptr = np.asarray(rowptr, dtype=np.int64)
    N = len(rowptr) - 1
    E = int(rowptr[-1])
    x0, vec0, w0, gy0 = _t(x), _t(vec), _t(w), _t(gy)
    ggx = torch.zeros_like(x0) if ggx is None else _t(ggx)
    ggw = torch.zeros_like(w0) if ggw is None else _t(ggw)
    ggvec = torch.zeros(E, 3, dtype=torch.float64) if ggvec is None else _t(ggvec)
    src_t = torch.as_tensor(np.asarray(src, dtype=np.int64))
    dst = _dst(rowptr)
    g_gy = torch.zeros_like(gy0)
    g_x = torch.zeros_like(x0)
    g_w = torch.zeros_like(w0)
    g_vec = torch.zeros(E, 3, dtype=torch.float64)
    for _, _, e0, e1 in _chunks(rowptr, max_edges):
        if e1 == e0:
            continue
        xl = x0.clone().requires_grad_(True)
        vl = vec0[e0:e1].clone().requires_grad_(True)
        wl = w0[e0:e1].clone().requires_grad_(True)
        gyl = gy0.clone().requires_grad_(True)
        m = _edge_messages(plan, xl[src_t[e0:e1]], vl, wl, None)
        L = (gyl[dst[e0:e1]] * m).sum()
        gx_c, gvec_c, gw_c = torch.autograd.grad(L, [xl, vl, wl], create_graph=True)
        L2 = (ggx * gx_c).sum() + (ggw[e0:e1] * gw_c).sum() + (ggvec[e0:e1] * gvec_c).sum()
        h = torch.autograd.grad(L2, [gyl, xl, wl, vl], allow_unused=True)
        zero = lambda t, ref: torch.zeros_like(ref) if t is None else t
        g_gy += zero(h[0], gyl)
        g_x += zero(h[1], xl)
        g_w[e0:e1] = zero(h[2], wl)
        g_vec[e0:e1] = zero(h[3], vl)
    return {"g_gy": g_gy, "g_x": g_x, "g_w": g_w, "g_vec": g_vec}


def forward_uvw_reassociated(plan: OraclePlan, rowptr, src, x, vec, s, W) -> torch.Tensor:
    """uvw forward in the node-side order: aggregate A[i,p,u,m3] over edges first, then mix
    with W_p per node ("Sobek", abstract: reassociating radial projection, SH coupling and
    aggregation).  Used only as a pin against the plain per-edge form."""
    if plan.mode != "uvw":
        raise ValueError("uvw only")
    rowptr = np.asarray(rowptr, dtype=np.int64)
    N = len(rowptr) - 1
    x, vec, s, W = _t(x), _t(vec), _t(s), _t(W)
    src_t = torch.as_tensor(np.asarray(src, dtype=np.int64))
    dst = _dst(rowptr)
    E = len(src_t)
    Ysh = [real_sh(l, vec) for _, l, _ in plan.irr_sh.blocks]
    y = torch.zeros(N, plan.irr_out.dim, dtype=torch.float64)
    with torch.no_grad():
        for p, (a, b, o) in enumerate(plan.paths):
            ma, la, _ = plan.irr_in.blocks[a]
            mo, lo, _ = plan.irr_out.blocks[o]
            d1, d3 = 2 * la + 1, 2 * lo + 1
            C = torch.as_tensor(cg_real(la, plan.triples[p][1], lo), dtype=torch.float64)
            xa = x[src_t, plan.irr_in.offsets[a]: plan.irr_in.offsets[a] + ma * d1].reshape(E, ma, d1)
            T = torch.einsum("eum,en,mnk->euk", xa, Ysh[b], C) * s[:, p, None, None]
            A = torch.zeros(N, ma, d3, dtype=torch.float64).index_add_(0, dst, T)
            Yo = plan.coeff[p] * torch.einsum("iuk,uv->ivk", A, W[p]).reshape(N, mo * d3)
            off = plan.irr_out.offsets[o]
            y[:, off: off + mo * d3] += Yo
    return y
