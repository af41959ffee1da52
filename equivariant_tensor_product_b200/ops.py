"""Python binding of the C ABI (include/tp.h): same names, argument marshalling only.

Every function takes torch CUDA tensors (or None for nullable arguments), checks dtype,
device and contiguity, allocates missing outputs and workspaces with torch's caching
allocator, and calls the library on the current torch stream.  All arithmetic runs in
libtp.so; there is no CPU path.
"""
from __future__ import annotations

import ctypes as C
from typing import Optional, Sequence

import torch

from . import _lib
from ._lib import TP_MODE_UVU, TP_MODE_UVW, TP_OP_BWD, TP_OP_DBWD, TP_OP_FWD, check, load

__all__ = ["Plan", "tp_plan_create", "tp_plan_query", "tp_workspace_size", "tp_csr_transpose_workspace_size", "tp_csr_transpose",
           "tp_conv_fwd", "tp_conv_bwd", "tp_conv_dbwd", "tp_radial_workspace_size", "tp_conv_fwd_radial",
           "tp_conv_bwd_radial", "tp_get_device_error", "tp_version"]


class Plan:
    """Owns a tp_plan_t (host memory only)."""

    def __init__(self, irreps_in: str, irreps_sh: str, irreps_out: str, paths: Sequence[Sequence[int]],
                 mode: str | int = "uvu", path_coeff: Optional[Sequence[float]] = None, flags: int = 0):
        lib = load()
        self._lib = lib
        self.handle = C.c_void_p()
        flat = [int(v) for p in paths for v in p]
        parr = (C.c_int32 * len(flat))(*flat)
        m = {"uvu": TP_MODE_UVU, "uvw": TP_MODE_UVW}.get(mode, mode)
        carr = (C.c_double * len(paths))(*path_coeff) if path_coeff is not None else None
        st = lib.tp_plan_create(C.byref(self.handle), irreps_in.encode(), irreps_sh.encode(),
                                irreps_out.encode(), C.cast(parr, C.c_void_p), len(paths), int(m),
                                C.cast(carr, C.c_void_p) if carr is not None else None, int(flags))
        check(st, "tp_plan_create")
        self.mode = int(m)
        self.n_paths = len(paths)
        self.in_dim, self.out_dim, self.n_edge_weights, self.n_shared_weights = tp_plan_query(self)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            self._lib.tp_plan_destroy(h)
            self.handle = None


def tp_version() -> str:
    return load().tp_version().decode()


def tp_plan_create(*args, **kw) -> Plan:
    return Plan(*args, **kw)


def tp_plan_query(plan: Plan):
    vals = [C.c_int64() for _ in range(4)]
    check(load().tp_plan_query(plan.handle, *[C.byref(v) for v in vals]), "tp_plan_query")
    return tuple(v.value for v in vals)


def tp_workspace_size(plan: Plan, N: int, E: int, op: int) -> int:
    out = C.c_size_t()
    check(load().tp_workspace_size(plan.handle, int(N), int(E), int(op), C.byref(out)), "tp_workspace_size")
    return out.value


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr() if t.numel() > 0 else None


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _workspace(plan, N, E, op, ws, device):
    need = tp_workspace_size(plan, N, E, op)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    elif ws.numel() < need:
        raise ValueError(f"workspace needs {need} bytes, got {ws.numel()}")
    return ws


def tp_csr_transpose_workspace_size(N: int, E: int) -> int:
    out = C.c_size_t()
    check(load().tp_csr_transpose_workspace_size(int(N), int(E), C.byref(out)), "tp_csr_transpose_workspace_size")
    return out.value


def tp_csr_transpose(rowptr: Optional[torch.Tensor], src: torch.Tensor, N: int, colptr=None, perm=None,
                     ws=None, stream=None):
    E = src.numel()
    dev = src.device
    colptr = torch.empty(N + 1, dtype=torch.int32, device=dev) if colptr is None else colptr
    perm = torch.empty(E, dtype=torch.int32, device=dev) if perm is None else perm
    need = tp_csr_transpose_workspace_size(N, E)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    st = load().tp_csr_transpose(N, E, _ptr(rowptr, torch.int32, "rowptr"), _ptr(src, torch.int32, "src"),
                                 _ptr(colptr, torch.int32, "colptr"), _ptr(perm, torch.int32, "perm"),
                                 _ptr(ws), ws.numel(), _stream(stream))
    check(st, "tp_csr_transpose")
    return colptr, perm


def tp_conv_fwd(plan: Plan, rowptr, src, x, vec, w, W=None, y=None, ws=None, stream=None):
    N = rowptr.numel() - 1
    E = src.numel()
    if y is None:
        y = torch.empty(N, plan.out_dim, dtype=torch.float32, device=x.device)
    ws = _workspace(plan, N, E, TP_OP_FWD, ws, x.device)
    st = load().tp_conv_fwd(plan.handle, N, E, _ptr(rowptr, torch.int32, "rowptr"), _ptr(src, torch.int32, "src"),
                            _ptr(x, torch.float32, "x"), _ptr(vec, torch.float32, "vec"),
                            _ptr(w, torch.float32, "w"), _ptr(W, torch.float32, "W"), _ptr(y, torch.float32, "y"),
                            _ptr(ws), ws.numel(), _stream(stream))
    check(st, "tp_conv_fwd")
    return y


def tp_conv_bwd(plan: Plan, rowptr, src, x, vec, w, gy, W=None, colptr=None, perm=None, need_gx=True,
                need_gw=True, need_gvec=False, need_gW=False, gx=None, gw=None, gvec=None, gW=None, ws=None,
                stream=None):
    N = rowptr.numel() - 1
    E = src.numel()
    dev = x.device
    if need_gx and gx is None:
        gx = torch.empty(N, plan.in_dim, dtype=torch.float32, device=dev)
    if need_gw and gw is None:
        gw = torch.empty(E, plan.n_edge_weights, dtype=torch.float32, device=dev)
    if need_gvec and gvec is None:
        gvec = torch.empty(E, 3, dtype=torch.float32, device=dev)
    if need_gW and gW is None and plan.n_shared_weights:
        gW = torch.empty(plan.n_shared_weights, dtype=torch.float32, device=dev)
    ws = _workspace(plan, N, E, TP_OP_BWD, ws, dev)
    st = load().tp_conv_bwd(plan.handle, N, E, _ptr(rowptr, torch.int32, "rowptr"), _ptr(src, torch.int32, "src"),
                            _ptr(colptr, torch.int32, "colptr"), _ptr(perm, torch.int32, "perm"),
                            _ptr(x, torch.float32, "x"), _ptr(vec, torch.float32, "vec"),
                            _ptr(w, torch.float32, "w"), _ptr(W, torch.float32, "W"), _ptr(gy, torch.float32, "gy"),
                            _ptr(gx, torch.float32, "gx"), _ptr(gw, torch.float32, "gw"),
                            _ptr(gvec, torch.float32, "gvec"), _ptr(gW, torch.float32, "gW"), _ptr(ws), ws.numel(),
                            _stream(stream))
    check(st, "tp_conv_bwd")
    return gx, gw, gvec, gW


def tp_radial_workspace_size(plan: Plan, N: int, E: int, H: int, op: int) -> int:
    out = C.c_size_t()
    check(load().tp_radial_workspace_size(plan.handle, int(N), int(E), int(H), int(op), C.byref(out)),
          "tp_radial_workspace_size")
    return out.value


def _radial_workspace(plan, N, E, H, op, ws, device):
    need = tp_radial_workspace_size(plan, N, E, H, op)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    elif ws.numel() < need:
        raise ValueError(f"workspace needs {need} bytes, got {ws.numel()}")
    return ws


def tp_conv_fwd_radial(plan: Plan, rowptr, src, x, vec, h, Wr, y=None, ws=None, stream=None):
    """uvu forward with the weights formed in the kernels as h[E, H] @ Wr[H, nw]."""
    N = rowptr.numel() - 1
    E = src.numel()
    H = Wr.shape[0]
    if y is None:
        y = torch.empty(N, plan.out_dim, dtype=torch.float32, device=x.device)
    ws = _radial_workspace(plan, N, E, H, TP_OP_FWD, ws, x.device)
    st = load().tp_conv_fwd_radial(plan.handle, N, E, H, _ptr(rowptr, torch.int32, "rowptr"),
                                   _ptr(src, torch.int32, "src"), _ptr(x, torch.float32, "x"),
                                   _ptr(vec, torch.float32, "vec"), _ptr(h, torch.float32, "h"),
                                   _ptr(Wr, torch.float32, "Wr"), _ptr(y, torch.float32, "y"), _ptr(ws), ws.numel(),
                                   _stream(stream))
    check(st, "tp_conv_fwd_radial")
    return y


def tp_conv_bwd_radial(plan: Plan, rowptr, src, x, vec, h, Wr, gy, colptr=None, perm=None, need_gx=True,
                       need_gh=True, need_gWr=True, need_gvec=False, gx=None, gh=None, gWr=None, gvec=None,
                       ws=None, stream=None):
    """VJP of tp_conv_fwd_radial: (gx, gh, gWr, gvec), each None when not requested."""
    N = rowptr.numel() - 1
    E = src.numel()
    H = Wr.shape[0]
    dev = x.device
    if need_gx and gx is None:
        gx = torch.empty(N, plan.in_dim, dtype=torch.float32, device=dev)
    if need_gh and gh is None:
        gh = torch.empty(E, H, dtype=torch.float32, device=dev)
    if need_gWr and gWr is None:
        gWr = torch.empty(H, plan.n_edge_weights, dtype=torch.float32, device=dev)
    if need_gvec and gvec is None:
        gvec = torch.empty(E, 3, dtype=torch.float32, device=dev)
    ws = _radial_workspace(plan, N, E, H, TP_OP_BWD, ws, dev)
    st = load().tp_conv_bwd_radial(plan.handle, N, E, H, _ptr(rowptr, torch.int32, "rowptr"),
                                   _ptr(src, torch.int32, "src"), _ptr(colptr, torch.int32, "colptr"),
                                   _ptr(perm, torch.int32, "perm"), _ptr(x, torch.float32, "x"),
                                   _ptr(vec, torch.float32, "vec"), _ptr(h, torch.float32, "h"),
                                   _ptr(Wr, torch.float32, "Wr"), _ptr(gy, torch.float32, "gy"),
                                   _ptr(gx, torch.float32, "gx"), _ptr(gh, torch.float32, "gh"),
                                   _ptr(gWr, torch.float32, "gWr"), _ptr(gvec, torch.float32, "gvec"), _ptr(ws),
                                   ws.numel(), _stream(stream))
    check(st, "tp_conv_bwd_radial")
    return gx, gh, gWr, gvec


def tp_conv_dbwd(plan: Plan, rowptr, src, x, vec, w, gy, ggx=None, ggw=None, ggvec=None, W=None, colptr=None,
                 perm=None, need=("g_gy", "g_x", "g_w", "g_vec"), ws=None, stream=None):
    N = rowptr.numel() - 1
    E = src.numel()
    dev = x.device
    g_gy = torch.empty(N, plan.out_dim, dtype=torch.float32, device=dev) if "g_gy" in need else None
    g_x = torch.empty(N, plan.in_dim, dtype=torch.float32, device=dev) if "g_x" in need else None
    g_w = torch.empty(E, plan.n_edge_weights, dtype=torch.float32, device=dev) if "g_w" in need else None
    g_vec = torch.empty(E, 3, dtype=torch.float32, device=dev) if "g_vec" in need else None
    ws = _workspace(plan, N, E, TP_OP_DBWD, ws, dev)
    st = load().tp_conv_dbwd(plan.handle, N, E, _ptr(rowptr, torch.int32, "rowptr"), _ptr(src, torch.int32, "src"),
                             _ptr(colptr, torch.int32, "colptr"), _ptr(perm, torch.int32, "perm"),
                             _ptr(x, torch.float32, "x"), _ptr(vec, torch.float32, "vec"),
                             _ptr(w, torch.float32, "w"), _ptr(W, torch.float32, "W"),
                             _ptr(gy, torch.float32, "gy"), _ptr(ggx, torch.float32, "ggx"),
                             _ptr(ggw, torch.float32, "ggw"), _ptr(ggvec, torch.float32, "ggvec"),
                             _ptr(g_gy, torch.float32, "g_gy"), _ptr(g_x, torch.float32, "g_x"),
                             _ptr(g_w, torch.float32, "g_w"), _ptr(g_vec, torch.float32, "g_vec"),
                             _ptr(ws), ws.numel(), _stream(stream))
    check(st, "tp_conv_dbwd")
    return g_gy, g_x, g_w, g_vec


def tp_get_device_error(plan: Optional[Plan], ws: Optional[torch.Tensor], stream=None) -> int:
    """Reads and clears the device error word (plan None: the per-device word)."""
    code = C.c_int32()
    check(load().tp_get_device_error(plan.handle if plan is not None else None, _ptr(ws), _stream(stream),
                                     C.byref(code)), "tp_get_device_error")
    return code.value
