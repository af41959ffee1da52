"""Failure detection and the memory contract on the GPU.

* Bounded waits: the two wait primitives of the pipelined kernels (copy-engine slot wait,
  tensor-core pipeline wait with abort flag) run against a barrier that nothing signals,
  with a 20 ms limit; both must give up and the context must stay usable.  No kernel is
  made to fault, trap or hang.
* Memory contract: with outputs and workspace supplied by the caller, a call allocates no
  device memory at all (the library never allocates; the workspace is node sized plus int
  edge indices).
* The per-device error word of plans without index checks (and of the linear maps, read
  without a plan) reads 0 after normal calls.
"""
import ctypes as C
import time

import numpy as np
import pytest
import torch

import synth
from gpu_util import assert_close, device_inputs, inputs, plans
from oracle import forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_tensor_product_b200 import build
    build.build()
    import equivariant_tensor_product_b200 as tp
    return tp


def test_waits_give_up_after_their_limit_and_the_context_survives(tp):
    lib = tp.load()
    gave_up = C.c_int32(0)
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    assert lib.tp_check_bounded_waits(20_000_000, stream, C.byref(gave_up)) == 0
    dt = time.perf_counter() - t0
    assert gave_up.value == 7, gave_up.value          # slot wait, pipeline wait, abort flag
    assert 0.04 <= dt < 2.0, dt                        # two 20 ms waits, then return
    # the context is still usable
    d = inputs("c1")
    plan, op = plans(d["spec"], tp)
    g = device_inputs(d)
    y = tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"])
    assert_close(y, forward(op, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"]), "c1 y after the check")


@pytest.mark.parametrize("name,n_atoms", [("c2", 512), ("c4", 400)])
def test_calls_allocate_no_device_memory(tp, name, n_atoms):
    d = inputs(name, n_atoms)
    spec = d["spec"]
    plan, _ = plans(spec, tp)
    g = device_inputs(d)
    N, E = len(d["rowptr"]) - 1, len(d["src"])
    uvw = spec.mode == "uvw"
    wkey = "s" if uvw else "w"
    W = g["W"] if uvw else None
    ws = torch.empty(max(tp.tp_workspace_size(plan, N, E, op) for op in
                         ((tp.TP_OP_FWD, tp.TP_OP_BWD) if uvw else (tp.TP_OP_FWD, tp.TP_OP_BWD, tp.TP_OP_DBWD))),
                     dtype=torch.uint8, device="cuda")
    y = torch.empty(N, plan.out_dim, device="cuda")
    gx = torch.empty(N, plan.in_dim, device="cuda")
    gw = torch.empty(E, plan.n_edge_weights, device="cuda")
    gvec = torch.empty(E, 3, device="cuda")
    gW = torch.empty(max(plan.n_shared_weights, 1), device="cuda") if uvw else None
    colptr, perm = tp.tp_csr_transpose(g["rowptr"], g["src"], N)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    before = torch.cuda.memory_allocated()
    tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g[wkey], W=W, y=y, ws=ws)
    tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g[wkey], g["gy"], W=W, colptr=colptr, perm=perm,
                   need_gvec=True, need_gW=uvw, gx=gx, gw=gw, gvec=gvec, gW=gW, ws=ws)
    torch.cuda.synchronize()
    assert torch.cuda.max_memory_allocated() == before
    # a workspace is at most node sized plus 8 bytes per edge beyond the node-sized uvw state
    node_bytes = 4 * N * (plan.in_dim + plan.out_dim)
    assert ws.numel() <= 8 * E + 64 * node_bytes + 68 * 4 * plan.n_shared_weights + (1 << 16)


def test_device_error_word_reads_zero_after_normal_calls(tp):
    d = inputs("c2", 256)
    plan, _ = plans(d["spec"], tp)
    g = device_inputs(d)
    tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"])
    tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"])
    assert tp.tp_get_device_error(plan, None) == 0
    # the linear maps' tensor-core GEMMs report to the same per-device word, read without a plan
    lin = tp.Linear("32x0e+32x1o", "32x0e+32x1o", flags=tp.TP_LINEAR_TENSOR_CORES)
    xl = torch.randn(300, lin.in_dim, device="cuda")
    Wl = torch.randn(lin.n_weights, device="cuda")
    tp.tp_linear_bwd(lin, xl, Wl, tp.tp_linear_fwd(lin, xl, Wl))
    assert tp.tp_get_device_error(None, None) == 0
