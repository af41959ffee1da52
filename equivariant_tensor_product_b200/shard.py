"""Receiver-range sharding of the convolution over several GPUs, one process per GPU.

A graph too large for one device is split into contiguous ranges of receiver rows, balanced
by edges plus rows; every rank owns its rows, their incoming edges (the contiguous edge range
[e0, e1) of the receiver-sorted CSR, with their vec and w) and the feature rows of its nodes
("Sobek: Streaming Equivariant Tensor Product Convolutions", abstract: graphs far beyond what
fit before, with bounded state per device).  One step per rank:

  forward   the x rows of the senders it needs from other ranks (its halo) arrive by one
            all-to-all (each rank first gathers the rows its peers need, `tp_gather_rows`);
            the local graph -- owned rows, then the halo as rows without edges -- runs the
            unchanged single-GPU kernels;
  backward  the local backward leaves gradient partials on the halo rows; one all-to-all
            sends them back to their owners, who add them to their own rows peer by peer in
            rank order (`tp_add_rows`, distinct rows per call), so the sum is deterministic;
            gW (uvw) is summed over ranks by an all-reduce.

The exchanges are plain collectives of `torch.distributed` (NCCL over NVLink on GPUs, gloo on
the CPU in the tests); no remote memory is read by a kernel.  The row planning is host code
that every rank runs on the full CSR, once per graph.
"""
from __future__ import annotations

from typing import List, Optional

import numpy as np
import torch


def row_bounds(rowptr, world: int) -> np.ndarray:
    """world + 1 receiver-row boundaries: rank k owns rows [b[k], b[k+1]).  The cost of a row is
    1 + its degree, and every boundary is the first row whose cumulative cost reaches k / world
    of the total."""
    rowptr = np.asarray(rowptr, dtype=np.int64)
    N = len(rowptr) - 1
    cost = rowptr + np.arange(N + 1)                # cumulative cost before row i
    total = cost[-1]
    b = [0] + [int(np.searchsorted(cost, k * total / world, side="left")) for k in range(1, world)] + [N]
    return np.minimum(np.maximum.accumulate(np.asarray(b, dtype=np.int64)), N)


class ShardPlan:
    """Rows, edges, halo and exchange lists of one rank (host arrays).

    Local node numbering: the owned rows [r0, r1) first (as 0 .. n_own-1), then the halo
    senders in increasing global id.  recv_counts[q] / send_counts[q] are the rows this rank
    receives from / sends to rank q in the forward exchange (the backward runs it in reverse);
    send_idx lists, peer after peer, the owned local rows each peer needs."""

    def __init__(self, rowptr, src, world: int, rank: int):
        rowptr = np.asarray(rowptr, dtype=np.int64)
        src = np.asarray(src, dtype=np.int64)
        self.world, self.rank = world, rank
        self.N, self.E = len(rowptr) - 1, int(rowptr[-1])
        self.bounds = row_bounds(rowptr, world)
        b = self.bounds
        self.r0, self.r1 = int(b[rank]), int(b[rank + 1])
        self.e0, self.e1 = int(rowptr[self.r0]), int(rowptr[self.r1])
        self.n_own = self.r1 - self.r0
        owner = lambda ids: np.searchsorted(b, ids, side="right") - 1

        def halo_of(q):
            s = src[rowptr[b[q]]:rowptr[b[q + 1]]]
            return np.unique(s[owner(s) != q])

        loc = src[self.e0:self.e1]
        self.halo = halo_of(rank)
        self.n_halo = len(self.halo)
        self.n_ext = self.n_own + self.n_halo
        mine = owner(loc) == rank
        self.src_local = np.where(mine, loc - self.r0, self.n_own + np.searchsorted(self.halo, loc)).astype(np.int32)
        self.rowptr_local = np.concatenate([rowptr[self.r0:self.r1 + 1] - self.e0,
                                            np.full(self.n_halo, self.e1 - self.e0)]).astype(np.int32)
        self.recv_counts = np.bincount(owner(self.halo), minlength=world).astype(np.int64)
        send, counts = [], []
        for q in range(world):
            need = halo_of(q) if q != rank else np.zeros(0, np.int64)
            need = need[(need >= self.r0) & (need < self.r1)]
            send.append(need - self.r0)
            counts.append(len(need))
        self.send_idx = np.concatenate(send).astype(np.int32) if send else np.zeros(0, np.int32)
        self.send_counts = np.asarray(counts, dtype=np.int64)
        self.send_offsets = np.concatenate([[0], np.cumsum(self.send_counts)])


class TorchExchange:
    """The halo exchange through torch.distributed (NCCL on GPUs, gloo in the CPU tests)."""

    def all_to_all(self, out: torch.Tensor, inp: torch.Tensor, out_rows: List[int], in_rows: List[int]):
        import torch.distributed as dist
        dist.all_to_all_single(out, inp, out_rows, in_rows)

    def all_reduce(self, t: torch.Tensor):
        import torch.distributed as dist
        dist.all_reduce(t)


class CudaOps:
    """Row movement and the convolution through the library's C ABI (the default)."""

    def __init__(self):
        from . import ops
        from ._lib import check, load
        self.ops, self.lib, self.check = ops, load(), check

    def gather_rows(self, src: torch.Tensor, idx: torch.Tensor) -> torch.Tensor:
        out = torch.empty(idx.numel(), src.shape[1], dtype=src.dtype, device=src.device)
        if idx.numel():
            self.check(self.lib.tp_gather_rows(src.data_ptr(), src.shape[1], idx.data_ptr(), idx.numel(),
                                               out.data_ptr(), torch.cuda.current_stream().cuda_stream),
                       "tp_gather_rows")
        return out

    def add_rows(self, dst: torch.Tensor, idx: torch.Tensor, src: torch.Tensor):
        if idx.numel():
            self.check(self.lib.tp_add_rows(dst.data_ptr(), dst.shape[1], idx.data_ptr(), idx.numel(),
                                            src.data_ptr(), torch.cuda.current_stream().cuda_stream), "tp_add_rows")

    def fwd(self, plan, graph, x, vec, w, W):
        return self.ops.tp_conv_fwd(plan, graph.rowptr, graph.src, x, vec, w, W=W)

    def bwd(self, plan, graph, x, vec, w, W, gy, need_gvec, need_gW):
        colptr, perm = graph.transpose()
        return self.ops.tp_conv_bwd(plan, graph.rowptr, graph.src, x, vec, w, gy, W=W, colptr=colptr, perm=perm,
                                    need_gvec=need_gvec, need_gW=need_gW)


class ShardedConv:
    """The convolution of one rank's shard.  Inputs per call: x_own [n_own, in_dim] (the rows
    this rank owns), vec and w of its edges (rows e0..e1 of the global arrays), W (uvw), gy_own
    for the backward.  Outputs: y_own, gx_own, and gw / gvec of its edges."""

    def __init__(self, plan, rowptr, src, world: int, rank: int, device, exchange=None, ops=None):
        from .autograd import Graph
        self.plan = plan
        self.sp = ShardPlan(rowptr, src, world, rank)
        self.device = device
        self.exchange = exchange or TorchExchange()
        self.ops = ops or CudaOps()
        sp = self.sp
        self.graph = Graph(torch.as_tensor(sp.rowptr_local).to(device), torch.as_tensor(sp.src_local).to(device))
        self.send_idx = torch.as_tensor(sp.send_idx).to(device)
        self.seg = [(int(sp.send_offsets[q]), int(sp.send_offsets[q + 1])) for q in range(world)]

    def _extend(self, x_own: torch.Tensor) -> torch.Tensor:
        """[x_own; halo rows from the peers] (the forward exchange)."""
        sp = self.sp
        x_ext = torch.empty(sp.n_ext, x_own.shape[1], dtype=x_own.dtype, device=x_own.device)
        x_ext[:sp.n_own].copy_(x_own)
        send = self.ops.gather_rows(x_own, self.send_idx)
        self.exchange.all_to_all(x_ext[sp.n_own:], send, sp.recv_counts.tolist(), sp.send_counts.tolist())
        return x_ext

    def _return_halo(self, g_ext: torch.Tensor) -> torch.Tensor:
        """Owned rows of g_ext plus the halo partials the peers computed for them (the reverse
        exchange), added peer by peer in rank order."""
        sp = self.sp
        back = torch.empty(len(sp.send_idx), g_ext.shape[1], dtype=g_ext.dtype, device=g_ext.device)
        self.exchange.all_to_all(back, g_ext[sp.n_own:].contiguous(), sp.send_counts.tolist(),
                                 sp.recv_counts.tolist())
        g_own = g_ext[:sp.n_own]
        for a, b in self.seg:
            if b > a:
                self.ops.add_rows(g_own, self.send_idx[a:b], back[a:b])
        return g_own

    def forward(self, x_own, vec, w, W=None):
        y_ext = self.ops.fwd(self.plan, self.graph, self._extend(x_own), vec, w, W)
        return y_ext[:self.sp.n_own]

    def backward(self, x_own, vec, w, gy_own, W=None, need_gvec=False, need_gW=False):
        sp = self.sp
        x_ext = self._extend(x_own)
        gy_ext = torch.zeros(sp.n_ext, gy_own.shape[1], dtype=gy_own.dtype, device=gy_own.device)
        gy_ext[:sp.n_own].copy_(gy_own)           # halo rows have no edges: never read
        gx_ext, gw, gvec, gW = self.ops.bwd(self.plan, self.graph, x_ext, vec, w, W, gy_ext, need_gvec, need_gW)
        gx_own = self._return_halo(gx_ext)
        if gW is not None:
            self.exchange.all_reduce(gW)
        return gx_own, gw, gvec, gW

    def edge_range(self):
        return self.sp.e0, self.sp.e1

    def row_range(self):
        return self.sp.r0, self.sp.r1
