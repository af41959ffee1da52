"""Python binding of the node-side operators (include/tp_block.h): the irreps-wise linear map
and the gate.  Same names as the C ABI, argument marshalling only: every step runs in
libtp.so, on the current torch stream."""
from __future__ import annotations

import ctypes as C
from typing import Optional, Sequence

import torch

from ._lib import TP_OP_BWD, TP_OP_FWD, check, load
from .ops import _ptr, _stream

__all__ = ["Linear", "Gate", "tp_linear_fwd", "tp_linear_bwd", "tp_linear_workspace_size", "tp_gate_fwd",
           "tp_gate_bwd", "tp_gate_dbwd"]


class Linear:
    """Owns a tp_linear_t: y[n, o, w, m] = sum_k c_k sum_u W_k[u, w] x[n, in(k), u, m] over all
    same-(l, parity) block pairs k = (i_in, i_out), lexicographic.  flags: 0 (form chosen per
    call by size), TP_LINEAR_TENSOR_CORES or TP_LINEAR_CUDA_CORES."""

    def __init__(self, irreps_in: str, irreps_out: str, coeff: Optional[Sequence[float]] = None, flags: int = 0):
        lib = load()
        self._lib = lib
        self.handle = C.c_void_p()
        self.irreps_in, self.irreps_out = irreps_in, irreps_out
        carr = (C.c_double * len(coeff))(*coeff) if coeff is not None else None
        check(lib.tp_linear_create(C.byref(self.handle), irreps_in.encode(), irreps_out.encode(),
                                   C.cast(carr, C.c_void_p) if carr is not None else None, int(flags)),
              "tp_linear_create")
        vals = [C.c_int64() for _ in range(3)]
        n_instr = C.c_int32()
        check(lib.tp_linear_query(self.handle, *[C.byref(v) for v in vals], C.byref(n_instr)), "tp_linear_query")
        self.in_dim, self.out_dim, self.n_weights = (v.value for v in vals)
        self.n_instructions = n_instr.value

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            self._lib.tp_linear_destroy(h)
            self.handle = None


def tp_linear_workspace_size(lin: Linear, N: int, op: int) -> int:
    out = C.c_size_t()
    check(load().tp_linear_workspace_size(lin.handle, int(N), int(op), C.byref(out)), "tp_linear_workspace_size")
    return out.value


def _ws(lin, N, op, ws, device):
    need = tp_linear_workspace_size(lin, N, op)
    if ws is None:
        return torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    if ws.numel() < need:
        raise ValueError(f"workspace needs {need} bytes, got {ws.numel()}")
    return ws


def tp_linear_fwd(lin: Linear, x, W, y=None, accumulate: bool = False, ws=None, stream=None):
    N = x.shape[0]
    if y is None:
        if accumulate:
            raise ValueError("accumulate needs y")
        y = torch.empty(N, lin.out_dim, dtype=torch.float32, device=x.device)
    ws = _ws(lin, N, TP_OP_FWD, ws, x.device)
    check(load().tp_linear_fwd(lin.handle, N, _ptr(x, torch.float32, "x"), _ptr(W, torch.float32, "W"),
                               _ptr(y, torch.float32, "y"), int(bool(accumulate)), _ptr(ws), ws.numel(),
                               _stream(stream)), "tp_linear_fwd")
    return y


def tp_linear_bwd(lin: Linear, x, W, gy, need_gx=True, need_gW=True, gx=None, gW=None, ws=None, stream=None):
    N = gy.shape[0]
    dev = gy.device
    if need_gx and gx is None:
        gx = torch.empty(N, lin.in_dim, dtype=torch.float32, device=dev)
    if need_gW and gW is None:
        gW = torch.empty(lin.n_weights, dtype=torch.float32, device=dev)
    ws = _ws(lin, N, TP_OP_BWD, ws, dev)
    check(load().tp_linear_bwd(lin.handle, N, _ptr(x, torch.float32, "x"), _ptr(W, torch.float32, "W"),
                               _ptr(gy, torch.float32, "gy"), _ptr(gx, torch.float32, "gx"),
                               _ptr(gW, torch.float32, "gW"), _ptr(ws), ws.numel(), _stream(stream)),
          "tp_linear_bwd")
    return gx, gW


class Gate:
    """Owns a tp_gate_t: [scalars | gates | gated] -> [act(scalars) | gated * sigmoid(gates)]."""

    def __init__(self, irreps_scalars: str, irreps_gates: str, irreps_gated: str):
        lib = load()
        self._lib = lib
        self.handle = C.c_void_p()
        check(lib.tp_gate_create(C.byref(self.handle), irreps_scalars.encode(), irreps_gates.encode(),
                                 irreps_gated.encode()), "tp_gate_create")
        a, b = C.c_int64(), C.c_int64()
        check(lib.tp_gate_query(self.handle, C.byref(a), C.byref(b)), "tp_gate_query")
        self.in_dim, self.out_dim = a.value, b.value

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            self._lib.tp_gate_destroy(h)
            self.handle = None


def tp_gate_fwd(gate: Gate, x, y=None, stream=None):
    if y is None:
        y = torch.empty(x.shape[0], gate.out_dim, dtype=torch.float32, device=x.device)
    check(load().tp_gate_fwd(gate.handle, x.shape[0], _ptr(x, torch.float32, "x"), _ptr(y, torch.float32, "y"),
                             _stream(stream)), "tp_gate_fwd")
    return y


def tp_gate_bwd(gate: Gate, x, gy, gx=None, stream=None):
    if gx is None:
        gx = torch.empty(x.shape[0], gate.in_dim, dtype=torch.float32, device=x.device)
    check(load().tp_gate_bwd(gate.handle, x.shape[0], _ptr(x, torch.float32, "x"), _ptr(gy, torch.float32, "gy"),
                             _ptr(gx, torch.float32, "gx"), _stream(stream)), "tp_gate_bwd")
    return gx


def tp_gate_dbwd(gate: Gate, x, gy, ggx, need_g_gy=True, need_g_x=True, stream=None):
    N = x.shape[0]
    g_gy = torch.empty(N, gate.out_dim, dtype=torch.float32, device=x.device) if need_g_gy else None
    g_x = torch.empty(N, gate.in_dim, dtype=torch.float32, device=x.device) if need_g_x else None
    check(load().tp_gate_dbwd(gate.handle, N, _ptr(x, torch.float32, "x"), _ptr(gy, torch.float32, "gy"),
                              _ptr(ggx, torch.float32, "ggx"), _ptr(g_gy, torch.float32, "g_gy"),
                              _ptr(g_x, torch.float32, "g_x"), _stream(stream)), "tp_gate_dbwd")
    return g_gy, g_x
