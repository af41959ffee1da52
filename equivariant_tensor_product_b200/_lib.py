"""ctypes loader for libtp.so: symbol table and argument types.  No computation here."""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtp.so")

TP_OK, TP_ERR_INVALID_ARG, TP_ERR_UNSUPPORTED, TP_ERR_BAD_GRAPH, TP_ERR_WORKSPACE, TP_ERR_CUDA, \
    TP_ERR_TIMEOUT = range(7)
TP_MODE_UVU, TP_MODE_UVW = 0, 1
TP_FLAG_CHECK_INDICES = 1
TP_OP_FWD, TP_OP_BWD, TP_OP_DBWD = 0, 1, 2
TP_LINEAR_TENSOR_CORES, TP_LINEAR_CUDA_CORES = 1, 2

_p = C.c_void_p
_i64 = C.c_int64
_i32 = C.c_int32
_sz = C.c_size_t

SIGNATURES = {
    "tp_plan_create": (C.c_int, [C.POINTER(_p), C.c_char_p, C.c_char_p, C.c_char_p, _p, _i32, _i32, _p,
                                 C.c_uint32]),
    "tp_plan_destroy": (C.c_int, [_p]),
    "tp_plan_query": (C.c_int, [_p, C.POINTER(_i64), C.POINTER(_i64), C.POINTER(_i64), C.POINTER(_i64)]),
    "tp_workspace_size": (C.c_int, [_p, _i64, _i64, _i32, C.POINTER(_sz)]),
    "tp_csr_transpose_workspace_size": (C.c_int, [_i64, _i64, C.POINTER(_sz)]),
    "tp_csr_transpose": (C.c_int, [_i64, _i64, _p, _p, _p, _p, _p, _sz, _p]),
    "tp_conv_fwd": (C.c_int, [_p, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "tp_conv_bwd": (C.c_int, [_p, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz,
                              _p]),
    "tp_conv_dbwd": (C.c_int, [_p, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p,
                               _p, _p, _sz, _p]),
    "tp_radial_workspace_size": (C.c_int, [_p, _i64, _i64, _i32, _i32, C.POINTER(_sz)]),
    "tp_conv_fwd_radial": (C.c_int, [_p, _i64, _i64, _i32, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "tp_conv_bwd_radial": (C.c_int, [_p, _i64, _i64, _i32, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p,
                                     _p, _p, _sz, _p]),
    "tp_get_device_error": (C.c_int, [_p, _p, _p, C.POINTER(_i32)]),
    "tp_gather_rows": (C.c_int, [_p, _i64, _p, _i64, _p, _p]),
    "tp_add_rows": (C.c_int, [_p, _i64, _p, _i64, _p, _p]),
    "tp_status_string": (C.c_char_p, [C.c_int]),
    "tp_last_error_message": (C.c_char_p, []),
    "tp_version": (C.c_char_p, []),
    "tp_launch_count": (C.c_int64, []),
    "tp_check_bounded_waits": (C.c_int, [_i64, _p, C.POINTER(_i32)]),
    # the spherical-grid (Gaunt) convolution (include/tp_gaunt.h)
    "tp_gaunt_create": (C.c_int, [C.POINTER(_p), C.c_char_p, _i32, C.c_char_p]),
    "tp_gaunt_destroy": (C.c_int, [_p]),
    "tp_gaunt_query": (C.c_int, [_p, C.POINTER(_i64), C.POINTER(_i64), C.POINTER(_i64), C.POINTER(_i32)]),
    "tp_gaunt_workspace_size": (C.c_int, [_p, _i64, _i64, _i32, C.POINTER(_sz)]),
    "tp_gaunt_fwd": (C.c_int, [_p, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "tp_gaunt_bwd": (C.c_int, [_p, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    # node-side operators (include/tp_block.h)
    "tp_linear_create": (C.c_int, [C.POINTER(_p), C.c_char_p, C.c_char_p, _p, C.c_uint32]),
    "tp_linear_destroy": (C.c_int, [_p]),
    "tp_linear_query": (C.c_int, [_p, C.POINTER(_i64), C.POINTER(_i64), C.POINTER(_i64), C.POINTER(_i32)]),
    "tp_linear_workspace_size": (C.c_int, [_p, _i64, _i32, C.POINTER(_sz)]),
    "tp_linear_fwd": (C.c_int, [_p, _i64, _p, _p, _p, _i32, _p, _sz, _p]),
    "tp_linear_bwd": (C.c_int, [_p, _i64, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "tp_gate_create": (C.c_int, [C.POINTER(_p), C.c_char_p, C.c_char_p, C.c_char_p]),
    "tp_gate_destroy": (C.c_int, [_p]),
    "tp_gate_query": (C.c_int, [_p, C.POINTER(_i64), C.POINTER(_i64)]),
    "tp_gate_fwd": (C.c_int, [_p, _i64, _p, _p, _p]),
    "tp_gate_bwd": (C.c_int, [_p, _i64, _p, _p, _p, _p]),
    "tp_gate_dbwd": (C.c_int, [_p, _i64, _p, _p, _p, _p, _p, _p]),
}

_LIB = None


class TPError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: status {status}: {msg}")
        self.status = status


def load() -> C.CDLL:
    """Loads the in-tree libtp.so; raises if it has not been built (no fallback path)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m equivariant_tensor_product_b200.build`")
        lib = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _LIB = lib
    return _LIB


def check(status: int, where: str):
    if status != TP_OK:
        lib = load()
        msg = lib.tp_last_error_message().decode(errors="replace")
        raise TPError(status, where, msg or lib.tp_status_string(status).decode())
