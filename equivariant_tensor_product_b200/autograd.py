"""torch.autograd wrapper: forward -> tp_conv_fwd, backward -> tp_conv_bwd, and the backward's
own backward -> tp_conv_dbwd, so force training (a loss on d(energy)/d(positions)) can
differentiate twice through the convolution.  Marshalling only (see ops.py)."""
from __future__ import annotations

import torch

from .ops import Plan, tp_conv_bwd, tp_conv_dbwd, tp_conv_fwd, tp_csr_transpose


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
    def forward(ctx, x, vec, w, gy, plan, graph, needs):
        colptr, perm = graph.transpose()
        gx, gw, gvec, _ = tp_conv_bwd(plan, graph.rowptr, graph.src, x, vec, w, gy, colptr=colptr, perm=perm,
                                      need_gx=needs[0], need_gvec=needs[1], need_gw=needs[2])
        ctx.save_for_backward(x, vec, w, gy)
        ctx.plan, ctx.graph = plan, graph
        return gx, gvec, gw

    @staticmethod
    def backward(ctx, ggx, ggvec, ggw):
        x, vec, w, gy = ctx.saved_tensors
        colptr, perm = ctx.graph.transpose()
        c = lambda t: None if t is None else t.contiguous()
        need = tuple(n for n, k in zip(("g_x", "g_vec", "g_w", "g_gy"), range(4)) if ctx.needs_input_grad[k])
        g_gy, g_x, g_w, g_vec = tp_conv_dbwd(ctx.plan, ctx.graph.rowptr, ctx.graph.src, x, vec, w, gy,
                                             ggx=c(ggx), ggw=c(ggw), ggvec=c(ggvec), colptr=colptr, perm=perm,
                                             need=need)
        return g_x, g_vec, g_w, g_gy, None, None, None


class TPConv(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, vec, w, plan, graph):
        y = tp_conv_fwd(plan, graph.rowptr, graph.src, x.contiguous(), vec.contiguous(), w.contiguous())
        ctx.save_for_backward(x, vec, w)
        ctx.plan, ctx.graph = plan, graph
        return y

    @staticmethod
    def backward(ctx, gy):
        x, vec, w = ctx.saved_tensors
        needs = (ctx.needs_input_grad[0], ctx.needs_input_grad[1], ctx.needs_input_grad[2])
        gx, gvec, gw = _Bwd.apply(x, vec, w, gy.contiguous(), ctx.plan, ctx.graph, needs)
        return gx, gvec, gw, None, None


def tp_conv(plan: Plan, graph: Graph, x, vec, w):
    """y = conv(x, vec, w) with first and second derivatives through the CUDA kernels (uvu)."""
    return TPConv.apply(x, vec, w, plan, graph)
