"""Float64 convolution with the radial projection fused in: the per-edge weights are formed from
the radial network's last hidden layer instead of being given.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

"Sobek: Streaming Equivariant Tensor Product Convolutions" (abstract) reorders the radial
projection so that edge-specific weights are never materialised.  The radial network ends in
a bias-free linear layer, so the uvu weights of edge e are

    w[e, p, u] = sum_k h[e, k] W_r[k, w_off(p) + u]

with h[E, H] the last hidden layer's activations and W_r[H, nw] that layer's matrix.  This
module composes that product (a float64 matmul) with the plain convolution of
``oracle.conv``; the backward is the torch autograd VJP with respect to (x, vec, h, W_r), the
same way ``oracle.conv.backward`` takes it.
"""
from __future__ import annotations

from typing import Dict

import numpy as np
import torch

from .conv import _chunks, _dst, _edge_messages, _t, forward
from .irreps import OraclePlan

__all__ = ["radial_weights", "forward_radial", "backward_radial"]


def radial_weights(h, Wr) -> torch.Tensor:
    """w[E, nw] = h[E, H] @ W_r[H, nw] in float64."""
    return _t(h) @ _t(Wr)


def forward_radial(plan: OraclePlan, rowptr, src, x, vec, h, Wr) -> torch.Tensor:
    """y[N, out_dim] of the uvu convolution whose weights are h @ W_r."""
    if plan.mode != "uvu":
        raise ValueError("the fused radial projection is defined for uvu plans")
    return forward(plan, rowptr, src, x, vec, w=radial_weights(h, Wr))


def backward_radial(plan: OraclePlan, rowptr, src, x, vec, h, Wr, gy,
                    max_edges: int = 1 << 13) -> Dict[str, torch.Tensor]:
    """VJP of forward_radial against gy: gx[N, in], gvec[E, 3], gh[E, H], gWr[H, nw]."""
    if plan.mode != "uvu":
        raise ValueError("the fused radial projection is defined for uvu plans")
    rowptr = np.asarray(rowptr, dtype=np.int64)
    E = int(rowptr[-1])
    x0, vec0, h0, Wr0, gy = _t(x), _t(vec), _t(h), _t(Wr), _t(gy)
    src_t = torch.as_tensor(np.asarray(src, dtype=np.int64))
    dst = _dst(rowptr)
    gx = torch.zeros_like(x0)
    gvec = torch.zeros(E, 3, dtype=torch.float64)
    gh = torch.zeros_like(h0)
    gWr = torch.zeros_like(Wr0)
    for _, _, e0, e1 in _chunks(rowptr, max_edges):
        if e1 == e0:
            continue
        xl = x0.clone().requires_grad_(True)
        vl = vec0[e0:e1].clone().requires_grad_(True)
        hl = h0[e0:e1].clone().requires_grad_(True)
        Wl = Wr0.clone().requires_grad_(True)
        m = _edge_messages(plan, xl[src_t[e0:e1]], vl, hl @ Wl, None)
        L = (gy[dst[e0:e1]] * m).sum()
        g = torch.autograd.grad(L, [xl, vl, hl, Wl], allow_unused=True)
        gx += g[0]
        gvec[e0:e1] = g[1]
        gh[e0:e1] = g[2]
        gWr += g[3]
    return {"gx": gx, "gvec": gvec, "gh": gh, "gWr": gWr}
