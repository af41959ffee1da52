"""Plain float64 node-side operators of an equivariant interaction layer: the irreps-wise
linear map (self-interaction, and the mixing of path-concatenated convolution outputs) and
the gate nonlinearity.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  Shares nothing with the CUDA library.

The pages place these around the convolution without defining them: "Accelerating Tensor
Products in E(3)-Equivariant Graph Neural Networks" (abstract) names NequIP's equivariant
interaction layers, of which the tensor-product convolution is the dominant part, and "The
GPU Workload That Rewrites Molecular Physics" (section "What Makes MLFF Workloads
Structurally Different") describes each atom aggregating its neighbours and transforming the
result through a neural network.  The forms below are the plainest
readings that keep E(3) equivariance:

Linear.  Instructions are all block pairs (i_in, i_out) with equal (l, parity), in
lexicographic (i_in, i_out) order; instruction k owns a weight matrix W_k[mul_in, mul_out]
(row-major, concatenated in instruction order) and an optional coefficient c_k (default 1):

    y[n, o, w, m] = sum_{k: out(k) = o} c_k sum_u W_k[u, w] x[n, in(k), u, m]

Output blocks that no instruction reaches are zero.  The same W_k acts on every m of the
block, which is what makes the map commute with rotations (Schur's lemma).

Gate.  The input row is [scalars | gates | gated]: scalar blocks (l = 0), gate blocks
(l = 0, even) whose total multiplicity equals that of the gated blocks, and gated blocks of
any l.  The output row is [act(scalars) | gated * sigmoid(gate)]: even scalars pass through
SiLU (x * sigmoid(x)), odd scalars through tanh (an odd function, so parity is kept), and
gated channel c (counting the channels of the gated blocks in order) is multiplied by
sigmoid of gate channel c.

Backward and double backward are torch autograd VJPs of these maps (``create_graph``).
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

from .irreps import Irreps

__all__ = ["linear_instructions", "linear_weight_count", "linear", "linear_backward", "linear_double_backward",
           "GateSpec", "gate", "gate_backward", "gate_double_backward"]


def _t(a) -> torch.Tensor:
    if isinstance(a, torch.Tensor):
        return a.detach().to(torch.float64)
    return torch.as_tensor(np.asarray(a), dtype=torch.float64)


def linear_instructions(irreps_in: str, irreps_out: str) -> List[Tuple[int, int]]:
    """All (i_in, i_out) with the same (l, parity), lexicographic."""
    a, b = Irreps(irreps_in), Irreps(irreps_out)
    return [(i, o) for i, (_, li, pi) in enumerate(a.blocks) for o, (_, lo, po) in enumerate(b.blocks)
            if li == lo and pi == po]


def linear_weight_count(irreps_in: str, irreps_out: str) -> int:
    a, b = Irreps(irreps_in), Irreps(irreps_out)
    return sum(a.blocks[i][0] * b.blocks[o][0] for i, o in linear_instructions(irreps_in, irreps_out))


def _linear_t(irreps_in: str, irreps_out: str, x: torch.Tensor, W: torch.Tensor,
              coeff: Optional[Sequence[float]]) -> torch.Tensor:
    a, b = Irreps(irreps_in), Irreps(irreps_out)
    ins = linear_instructions(irreps_in, irreps_out)
    N = x.shape[0]
    outs: List[Optional[torch.Tensor]] = [None] * len(b.blocks)
    off = 0
    for k, (i, o) in enumerate(ins):
        mi, l, _ = a.blocks[i]
        mo = b.blocks[o][0]
        d = 2 * l + 1
        Wk = W[off:off + mi * mo].reshape(mi, mo)
        off += mi * mo
        xb = x[:, a.offsets[i]:a.offsets[i] + mi * d].reshape(N, mi, d)
        c = 1.0 if coeff is None else float(coeff[k])
        term = c * torch.einsum("uw,num->nwm", Wk, xb)
        outs[o] = term if outs[o] is None else outs[o] + term
    cols = []
    for o, (mo, l, _) in enumerate(b.blocks):
        d = 2 * l + 1
        blk = outs[o] if outs[o] is not None else torch.zeros(N, mo, d, dtype=x.dtype)
        cols.append(blk.reshape(N, mo * d))
    return torch.cat(cols, dim=1)


def linear(irreps_in: str, irreps_out: str, x, W, coeff: Optional[Sequence[float]] = None) -> torch.Tensor:
    return _linear_t(irreps_in, irreps_out, _t(x), _t(W).reshape(-1), coeff)


def linear_backward(irreps_in: str, irreps_out: str, x, W, gy, coeff=None) -> Dict[str, torch.Tensor]:
    xt = _t(x).requires_grad_(True)
    Wt = _t(W).reshape(-1).requires_grad_(True)
    y = _linear_t(irreps_in, irreps_out, xt, Wt, coeff)
    gx, gW = torch.autograd.grad(y, (xt, Wt), _t(gy))
    return {"gx": gx, "gW": gW}


def linear_double_backward(irreps_in: str, irreps_out: str, x, W, gy, ggx=None, ggW=None,
                           coeff=None) -> Dict[str, torch.Tensor]:
    """VJP of (x, W, gy) -> (gx, gW) against (ggx, ggW)."""
    xt = _t(x).requires_grad_(True)
    Wt = _t(W).reshape(-1).requires_grad_(True)
    gyt = _t(gy).requires_grad_(True)
    y = _linear_t(irreps_in, irreps_out, xt, Wt, coeff)
    gx, gW = torch.autograd.grad(y, (xt, Wt), gyt, create_graph=True)
    s = torch.zeros((), dtype=torch.float64)
    if ggx is not None:
        s = s + (gx * _t(ggx)).sum()
    if ggW is not None:
        s = s + (gW * _t(ggW).reshape(-1)).sum()
    g = torch.autograd.grad(s, (gyt, xt, Wt), allow_unused=True)
    z = lambda t, ref: torch.zeros_like(ref) if t is None else t
    return {"g_gy": z(g[0], gyt), "g_x": z(g[1], xt), "g_W": z(g[2], Wt)}


class GateSpec:
    """Validated gate layout: input [scalars | gates | gated] -> output [act(scalars) | gated * sigmoid(gates)]."""

    def __init__(self, irreps_scalars: str, irreps_gates: str, irreps_gated: str):
        self.scalars = Irreps(irreps_scalars) if irreps_scalars else None
        self.gates = Irreps(irreps_gates) if irreps_gates else None
        self.gated = Irreps(irreps_gated) if irreps_gated else None
        sc = self.scalars.blocks if self.scalars else []
        gt = self.gates.blocks if self.gates else []
        gd = self.gated.blocks if self.gated else []
        if any(l != 0 for _, l, _ in sc):
            raise ValueError("scalar blocks must have l = 0")
        if any(l != 0 or p != 1 for _, l, p in gt):
            raise ValueError("gate blocks must be even scalars (0e)")
        if sum(m for m, _, _ in gt) != sum(m for m, _, _ in gd):
            raise ValueError("gate multiplicity must equal the gated multiplicity")
        self.n_scalar = sum(m for m, _, _ in sc)
        self.n_gate = sum(m for m, _, _ in gt)
        self.gated_dim = sum(m * (2 * l + 1) for m, l, _ in gd)
        self.in_dim = self.n_scalar + self.n_gate + self.gated_dim
        self.out_dim = self.n_scalar + self.gated_dim
        self.scalar_blocks = sc
        self.gated_blocks = gd


def _gate_t(spec: GateSpec, x: torch.Tensor) -> torch.Tensor:
    N = x.shape[0]
    cols = []
    off = 0
    for m, _, p in spec.scalar_blocks:
        s = x[:, off:off + m]
        cols.append(torch.nn.functional.silu(s) if p == 1 else torch.tanh(s))
        off += m
    gates = torch.sigmoid(x[:, off:off + spec.n_gate])
    off += spec.n_gate
    c = 0
    for m, l, _ in spec.gated_blocks:
        d = 2 * l + 1
        v = x[:, off:off + m * d].reshape(N, m, d)
        cols.append((v * gates[:, c:c + m, None]).reshape(N, m * d))
        off += m * d
        c += m
    if not cols:
        return torch.zeros(N, 0, dtype=x.dtype)
    return torch.cat(cols, dim=1)


def gate(spec: GateSpec, x) -> torch.Tensor:
    return _gate_t(spec, _t(x))


def gate_backward(spec: GateSpec, x, gy) -> torch.Tensor:
    xt = _t(x).requires_grad_(True)
    (gx,) = torch.autograd.grad(_gate_t(spec, xt), xt, _t(gy))
    return gx


def gate_double_backward(spec: GateSpec, x, gy, ggx) -> Dict[str, torch.Tensor]:
    """VJP of (x, gy) -> gx against ggx."""
    xt = _t(x).requires_grad_(True)
    gyt = _t(gy).requires_grad_(True)
    (gx,) = torch.autograd.grad(_gate_t(spec, xt), xt, gyt, create_graph=True)
    g_gy, g_x = torch.autograd.grad((gx * _t(ggx)).sum(), (gyt, xt), allow_unused=True)
    return {"g_gy": torch.zeros_like(gyt) if g_gy is None else g_gy,
            "g_x": torch.zeros_like(xt) if g_x is None else g_x}
