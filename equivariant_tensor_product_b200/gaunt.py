"""Python binding of the spherical-grid (Gaunt) convolution (include/tp_gaunt.h): argument
marshalling only; every step runs in libtp.so."""
from __future__ import annotations

import ctypes as C
from typing import Optional

import torch

from ._lib import TP_OP_BWD, TP_OP_FWD, check, load
from .ops import _ptr, _stream

__all__ = ["Gaunt", "tp_gaunt_fwd", "tp_gaunt_bwd", "tp_gaunt_workspace_size"]


class Gaunt:
    """Owns a tp_gaunt_t: natural-parity irreps with one multiplicity, filter degrees 0..lmax_sh."""

    def __init__(self, irreps_in: str, lmax_sh: int, irreps_out: str):
        lib = load()
        self._lib = lib
        self.handle = C.c_void_p()
        check(lib.tp_gaunt_create(C.byref(self.handle), irreps_in.encode(), int(lmax_sh), irreps_out.encode()),
              "tp_gaunt_create")
        v = [C.c_int64() for _ in range(3)]
        ng = C.c_int32()
        check(lib.tp_gaunt_query(self.handle, *[C.byref(t) for t in v], C.byref(ng)), "tp_gaunt_query")
        self.in_dim, self.out_dim, self.n_edge_weights = (t.value for t in v)
        self.grid_points = ng.value
        self.lmax_sh = int(lmax_sh)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            self._lib.tp_gaunt_destroy(h)
            self.handle = None


def tp_gaunt_workspace_size(g: Gaunt, N: int, E: int, op: int) -> int:
    out = C.c_size_t()
    check(load().tp_gaunt_workspace_size(g.handle, int(N), int(E), int(op), C.byref(out)), "tp_gaunt_workspace_size")
    return out.value


def _ws(g, N, E, op, ws, dev):
    need = tp_gaunt_workspace_size(g, N, E, op)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    elif ws.numel() < need:
        raise ValueError(f"workspace needs {need} bytes, got {ws.numel()}")
    return ws


def tp_gaunt_fwd(g: Gaunt, rowptr, src, x, vec, w, y=None, ws=None, stream=None):
    N, E = rowptr.numel() - 1, src.numel()
    y = torch.empty(N, g.out_dim, dtype=torch.float32, device=x.device) if y is None else y
    ws = _ws(g, N, E, TP_OP_FWD, ws, x.device)
    check(load().tp_gaunt_fwd(g.handle, N, E, _ptr(rowptr, torch.int32, "rowptr"), _ptr(src, torch.int32, "src"),
                              _ptr(x, torch.float32, "x"), _ptr(vec, torch.float32, "vec"),
                              _ptr(w, torch.float32, "w"), _ptr(y, torch.float32, "y"), _ptr(ws), ws.numel(),
                              _stream(stream)), "tp_gaunt_fwd")
    return y


def tp_gaunt_bwd(g: Gaunt, rowptr, src, x, vec, w, gy, colptr=None, perm=None, need_gx=True, need_gw=True,
                 need_gvec=False, gx: Optional[torch.Tensor] = None, gw=None, gvec=None, ws=None, stream=None):
    N, E = rowptr.numel() - 1, src.numel()
    dev = x.device
    if need_gx and gx is None:
        gx = torch.empty(N, g.in_dim, dtype=torch.float32, device=dev)
    if need_gw and gw is None:
        gw = torch.empty(E, g.n_edge_weights, dtype=torch.float32, device=dev)
    if need_gvec and gvec is None:
        gvec = torch.empty(E, 3, dtype=torch.float32, device=dev)
    ws = _ws(g, N, E, TP_OP_BWD, ws, dev)
    check(load().tp_gaunt_bwd(g.handle, N, E, _ptr(rowptr, torch.int32, "rowptr"), _ptr(src, torch.int32, "src"),
                              _ptr(colptr, torch.int32, "colptr"), _ptr(perm, torch.int32, "perm"),
                              _ptr(x, torch.float32, "x"), _ptr(vec, torch.float32, "vec"),
                              _ptr(w, torch.float32, "w"), _ptr(gy, torch.float32, "gy"),
                              _ptr(gx, torch.float32, "gx"), _ptr(gw, torch.float32, "gw"),
                              _ptr(gvec, torch.float32, "gvec"), _ptr(ws), ws.numel(), _stream(stream)),
          "tp_gaunt_bwd")
    return gx, gw, gvec
