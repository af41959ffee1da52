"""Host-side checks of the node-side operators' C ABI (include/tp_block.h), no GPU needed:
sizes agree with the oracle's reading, bad handles and bad calls are rejected with the
documented status before anything reaches the device, and a call that passes the checks
goes to CUDA (no CPU path)."""
import ctypes as C

import pytest

from oracle.block import GateSpec, linear_instructions, linear_weight_count
from oracle.irreps import Irreps


@pytest.fixture(scope="module")
def tp():
    from equivariant_tensor_product_b200 import build
    build.build()
    import equivariant_tensor_product_b200 as tp
    return tp


LINEARS = [
    ("32x0e+32x1o+32x2e", "32x0e+32x1o+32x2e"),
    ("32x0e+32x1e+32x1o+32x2e+32x2o", "32x0e+64x0e+32x1o+32x2e"),
    ("4x0e+12x0e+8x1o+20x3o", "36x0e+8x1o+4x1o+16x3o+8x2e"),
    ("128x0e+128x1o+128x2e", "128x0e+128x1e+128x1o+128x2e+128x2o"),
]


@pytest.mark.parametrize("ir_in,ir_out", LINEARS)
def test_linear_sizes_match_the_oracle(tp, ir_in, ir_out):
    lin = tp.Linear(ir_in, ir_out)
    assert lin.in_dim == Irreps(ir_in).dim and lin.out_dim == Irreps(ir_out).dim
    assert lin.n_weights == linear_weight_count(ir_in, ir_out)
    assert lin.n_instructions == len(linear_instructions(ir_in, ir_out))
    # workspace: node sized (regrouped rows) plus weight sized (split weights, split-K partials)
    N = 1000
    fwd = tp.tp_linear_workspace_size(lin, N, tp.TP_OP_FWD)
    bwd = tp.tp_linear_workspace_size(lin, N, tp.TP_OP_BWD)
    assert fwd <= 4 * N * lin.in_dim + 8 * lin.n_weights + 4096
    assert bwd <= 4 * N * (lin.in_dim + lin.out_dim) + (8 + 4 * 256) * lin.n_weights + 4096


@pytest.mark.parametrize("ir_in,ir_out,status", [
    ("6x0e", "4x0e", 2),            # multiplicity off the TMA pitch
    ("4x4e", "4x4e", 2),            # l > 3
    ("4x0e+", "4x0e", 1),           # syntax
    ("4x0e", "", 1),
])
def test_linear_validation(tp, ir_in, ir_out, status):
    with pytest.raises(tp.TPError) as e:
        tp.Linear(ir_in, ir_out)
    assert e.value.status == status


def test_linear_rejects_nonfinite_coefficients_and_bad_flags(tp):
    with pytest.raises(tp.TPError):
        tp.Linear("4x0e", "4x0e", coeff=[float("nan")])
    for flags in (3, 4):
        with pytest.raises(tp.TPError):
            tp.Linear("4x0e", "4x0e", flags=flags)


@pytest.mark.parametrize("args,status", [
    (("2x1o", "2x0e", "2x1o"), 1),      # scalar block with l > 0
    (("2x0e", "2x0o", "2x1o"), 1),      # odd gates
    (("2x0e", "3x0e", "2x1o"), 1),      # multiplicity mismatch
    (("2x0e", "2x0e", "2x4e"), 2),      # l > 3
])
def test_gate_validation(tp, args, status):
    with pytest.raises(tp.TPError) as e:
        tp.Gate(*args)
    assert e.value.status == status


def test_gate_sizes_match_the_oracle(tp):
    for args in (("32x0e", "32x0e+32x0e", "32x1o+32x2e"), ("3x0e+2x0o", "2x0e+3x0e", "2x1o+1x2e+2x1e"),
                 ("", "4x0e", "4x3o"), ("8x0e", "", "")):
        g = tp.Gate(*args)
        s = GateSpec(*args)
        assert (g.in_dim, g.out_dim) == (s.in_dim, s.out_dim)


def test_calls_reject_bad_arguments_before_the_device(tp):
    lib = tp.load()
    lin = tp.Linear("32x0e+32x1o", "32x0e+32x1o")
    h = lin.handle
    fake = C.c_void_p(0x10000)          # never dereferenced: every call below fails host checks
    odd = C.c_void_p(0x10002)
    big = 1 << 24
    assert lib.tp_linear_fwd(None, 4, fake, fake, fake, 0, fake, big, None) == 1
    assert lib.tp_linear_fwd(h, -1, fake, fake, fake, 0, fake, big, None) == 1
    assert lib.tp_linear_fwd(h, 4, None, fake, fake, 0, fake, big, None) == 1
    assert lib.tp_linear_fwd(h, 4, odd, fake, fake, 0, fake, big, None) == 1
    assert lib.tp_linear_fwd(h, 4, fake, fake, fake, 0, fake, 16, None) == 4           # workspace too small
    assert lib.tp_linear_fwd(h, 4, fake, fake, fake, 0, C.c_void_p(0x10040), big, None) == 4   # not 256-aligned
    assert lib.tp_linear_fwd(h, 0, None, None, None, 0, None, 0, None) == 0             # N = 0: no-op
    assert lib.tp_linear_fwd(h, 1 << 29, fake, fake, fake, 0, fake, big, None) == 2     # N (2l+1) >= 2^31
    assert lib.tp_linear_bwd(h, 4, fake, fake, None, fake, None, fake, big, None) == 1  # gy NULL
    assert lib.tp_linear_bwd(h, 4, None, fake, fake, None, fake, fake, big, None) == 1  # gW without x
    size = C.c_size_t()
    assert lib.tp_linear_workspace_size(h, 4, 2, C.byref(size)) == 1                    # no dbwd entry point
    g = tp.Gate("4x0e", "4x0e", "4x1o")
    assert lib.tp_gate_fwd(None, 4, fake, fake, None) == 1
    assert lib.tp_gate_fwd(g.handle, 4, fake, None, None) == 1
    assert lib.tp_gate_bwd(g.handle, 4, fake, None, fake, None) == 1
    assert lib.tp_gate_dbwd(g.handle, 4, fake, fake, None, fake, fake, None) == 1
    assert lib.tp_gate_fwd(g.handle, 4, odd, fake, None) == 1
    assert lib.tp_gate_fwd(g.handle, 0, None, None, None) == 0
    msg = lib.tp_last_error_message()
    assert msg


def test_no_cpu_fallback_without_device(tp):
    import torch
    if torch.cuda.is_available():
        pytest.skip("device present")
    lib = tp.load()
    g = tp.Gate("4x0e", "4x0e", "4x1o")
    fake = C.c_void_p(0x10000)
    assert lib.tp_gate_fwd(g.handle, 4, fake, fake, None) == 5
    for form in (tp.TP_LINEAR_TENSOR_CORES, tp.TP_LINEAR_CUDA_CORES):
        lin = tp.Linear("32x0e", "32x0e", flags=form)
        assert lib.tp_linear_fwd(lin.handle, 4, fake, fake, fake, 0, fake, 1 << 24, None) == 5
