"""torch.autograd wrapper: forward -> tp_conv_fwd, backward -> tp_conv_bwd, and the backward's
own backward -> tp_conv_dbwd, so force training (a loss on d(energy)/d(positions)) can
differentiate twice through the convolution (uvu; uvw mode differentiates once, to x, the
edge vectors, the per-edge scalars and the shared mixing weights W; the radial-projection form
differentiates once, to x, the edge vectors, the hidden layer h and the output matrix W_r).
Marshalling only (see ops.py)."""
from __future__ import annotations

import torch

from ._lib import TP_MODE_UVW
from .ops import (Plan, tp_conv_bwd, tp_conv_bwd_radial, tp_conv_dbwd, tp_conv_fwd, tp_conv_fwd_radial,
                  tp_csr_transpose)


class Graph:
    """Receiver-sorted CSR plus a lazily built stable sender transpose (int32, on device)."""

    def __init__(self, rowptr: torch.Tensor, src: torch.Tensor):
        self.rowptr = rowptr.to(torch.int32).contiguous()
        self.src = src.to(torch.int32).contiguous()
        self.N = self.rowptr.numel() - 1
        self._colptr = None
        self._perm = None

    def transpose(self):
        if self._colptr is None:
            self._colptr, self._perm = tp_csr_transpose(self.rowptr, self.src, self.N)
        return self._colptr, self._perm


class _Bwd(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, vec, w, W, gy, plan, graph, needs):
        colptr, perm = graph.transpose()
        gx, gw, gvec, gW = tp_conv_bwd(plan, graph.rowptr, graph.src, x, vec, w, gy, W=W, colptr=colptr, perm=perm,
                                       need_gx=needs[0], need_gvec=needs[1], need_gw=needs[2],
                                       need_gW=W is not None and needs[3])
        ctx.save_for_backward(x, vec, w, gy)
        ctx.plan, ctx.graph = plan, graph
        return gx, gvec, gw, None if gW is None else gW.view(W.shape)

    @staticmethod
    def backward(ctx, ggx, ggvec, ggw, ggW):
        if ctx.plan.mode == TP_MODE_UVW:
            raise RuntimeError("second derivatives of the uvw convolution are not implemented (tp_conv_dbwd is uvu)")
        x, vec, w, gy = ctx.saved_tensors
        colptr, perm = ctx.graph.transpose()
        c = lambda t: None if t is None else t.contiguous()
        need = tuple(n for n, k in zip(("g_x", "g_vec", "g_w", "g_gy"), (0, 1, 2, 4)) if ctx.needs_input_grad[k])
        g_gy, g_x, g_w, g_vec = tp_conv_dbwd(ctx.plan, ctx.graph.rowptr, ctx.graph.src, x, vec, w, gy,
                                             ggx=c(ggx), ggw=c(ggw), ggvec=c(ggvec), colptr=colptr, perm=perm,
                                             need=need)
        return g_x, g_vec, g_w, None, g_gy, None, None, None


class TPConv(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, vec, w, W, plan, graph):
        W = None if W is None else W.contiguous()
        y = tp_conv_fwd(plan, graph.rowptr, graph.src, x.contiguous(), vec.contiguous(), w.contiguous(), W=W)
        ctx.save_for_backward(x, vec, w, W)
        ctx.plan, ctx.graph = plan, graph
        return y

    @staticmethod
    def backward(ctx, gy):
        x, vec, w, W = ctx.saved_tensors
        n = ctx.needs_input_grad
        gx, gvec, gw, gW = _Bwd.apply(x, vec, w, W, gy.contiguous(), ctx.plan, ctx.graph, (n[0], n[1], n[2], n[3]))
        return gx, gvec, gw, gW, None, None


def tp_conv(plan: Plan, graph: Graph, x, vec, w, W=None):
    """y = conv(x, vec, w) with derivatives through the CUDA kernels: first and second order in
    uvu mode (w = per-edge weights [E, n_edge_weights]); first order in uvw mode (w = per-edge
    path scalars s [E, P], W = shared mixing weights [P, mul_in, mul_out], gradients to both)."""
    if (plan.mode == TP_MODE_UVW) != (W is not None):
        raise ValueError("W is required in uvw mode and must be None in uvu mode")
    return TPConv.apply(x, vec, w, W, plan, graph)


# ---------------------------------------------------------------------------------------------
# Node-side operators (include/tp_block.h).  The linear map's second-order terms are again
# applications of the map and its adjoint: g_gy = fwd(ggx; W) + fwd(x; ggW),
# g_x = bwd(gy; ggW).gx, g_W = bwd(ggx, gy).gW -- the same two entry points with other
# arguments.  The gate's come from tp_gate_dbwd.
# ---------------------------------------------------------------------------------------------

from .block import Gate, Linear, tp_gate_bwd, tp_gate_dbwd, tp_gate_fwd, tp_linear_bwd, tp_linear_fwd  # noqa: E402


class _LinearBwd(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, W, gy, lin, needs):
        gx, gW = tp_linear_bwd(lin, x, W, gy, need_gx=needs[0], need_gW=needs[1])
        ctx.save_for_backward(x, W, gy)
        ctx.lin = lin
        return gx, gW

    @staticmethod
    def backward(ctx, ggx, ggW):
        x, W, gy = ctx.saved_tensors
        lin = ctx.lin
        c = lambda t: None if t is None else t.contiguous()
        ggx, ggW = c(ggx), c(ggW)
        g_x = g_W = g_gy = None
        if ctx.needs_input_grad[2]:
            if ggx is not None:
                g_gy = tp_linear_fwd(lin, ggx, W)
            if ggW is not None:
                g_gy = tp_linear_fwd(lin, x, ggW, y=g_gy, accumulate=g_gy is not None)
        if ctx.needs_input_grad[0] and ggW is not None:
            g_x, _ = tp_linear_bwd(lin, None, ggW, gy, need_gx=True, need_gW=False)
        if ctx.needs_input_grad[1] and ggx is not None:
            _, g_W = tp_linear_bwd(lin, ggx, None, gy, need_gx=False, need_gW=True)
        return g_x, g_W, g_gy, None, None


class LinearFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, W, lin):
        x, W = x.contiguous(), W.contiguous()
        y = tp_linear_fwd(lin, x, W)
        ctx.save_for_backward(x, W)
        ctx.lin = lin
        return y

    @staticmethod
    def backward(ctx, gy):
        x, W = ctx.saved_tensors
        needs = (ctx.needs_input_grad[0], ctx.needs_input_grad[1])
        gx, gW = _LinearBwd.apply(x, W, gy.contiguous(), ctx.lin, needs)
        return gx, gW, None


def tp_linear(lin: Linear, x, W):
    """y = linear(x; W) with first and second derivatives through the CUDA kernels."""
    return LinearFn.apply(x, W, lin)


class _GateBwd(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, gy, gate):
        gx = tp_gate_bwd(gate, x, gy)
        ctx.save_for_backward(x, gy)
        ctx.gate = gate
        return gx

    @staticmethod
    def backward(ctx, ggx):
        x, gy = ctx.saved_tensors
        g_gy, g_x = tp_gate_dbwd(ctx.gate, x, gy, ggx.contiguous(), need_g_gy=ctx.needs_input_grad[1],
                                 need_g_x=ctx.needs_input_grad[0])
        return g_x, g_gy, None


class GateFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, gate):
        x = x.contiguous()
        y = tp_gate_fwd(gate, x)
        ctx.save_for_backward(x)
        ctx.gate = gate
        return y

    @staticmethod
    def backward(ctx, gy):
        (x,) = ctx.saved_tensors
        return _GateBwd.apply(x, gy.contiguous(), ctx.gate), None


def tp_gate(gate: Gate, x):
    """y = gate(x) with first and second derivatives through the CUDA kernels."""
    return GateFn.apply(x, gate)


class TPConvRadial(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, vec, h, Wr, plan, graph):
        x, vec, h, Wr = x.contiguous(), vec.contiguous(), h.contiguous(), Wr.contiguous()
        y = tp_conv_fwd_radial(plan, graph.rowptr, graph.src, x, vec, h, Wr)
        ctx.save_for_backward(x, vec, h, Wr)
        ctx.plan, ctx.graph = plan, graph
        return y

    @staticmethod
    @torch.autograd.function.once_differentiable
    def backward(ctx, gy):
        x, vec, h, Wr = ctx.saved_tensors
        n = ctx.needs_input_grad
        colptr, perm = ctx.graph.transpose()
        gx, gh, gWr, gvec = tp_conv_bwd_radial(ctx.plan, ctx.graph.rowptr, ctx.graph.src, x, vec, h, Wr,
                                               gy.contiguous(), colptr=colptr, perm=perm, need_gx=n[0],
                                               need_gvec=n[1], need_gh=n[2], need_gWr=n[3])
        return gx, gvec, gh, gWr, None, None


def tp_conv_radial(plan: Plan, graph: Graph, x, vec, h, Wr):
    """y = conv(x, vec, w) with w = h @ Wr formed inside the kernels (uvu plans; h [E, H] the
    radial network's last hidden layer, Wr [H, n_edge_weights] its output layer); first-order
    derivatives to x, vec, h and Wr through the CUDA kernels."""
    if plan.mode == TP_MODE_UVW:
        raise ValueError("the fused radial projection is implemented for uvu plans")
    return TPConvRadial.apply(x, vec, h, Wr, plan, graph)
