"""GPU parity of the node-side operators (include/tp_block.h) against the float64 oracle:
the irreps-wise linear map (forward, accumulate, backward, second order through the
autograd binding), the gate (forward, backward, double backward), and an interaction layer
linear -> convolution (1/average-degree coefficient) -> linear -> gate, differentiated
through the binding.  Per tensor max|gpu - ref| <= 1e-4 * max|ref|."""
import numpy as np
import pytest
import torch

import synth
from gpu_util import assert_close, dev
from oracle import OraclePlan, backward
from oracle.block import (GateSpec, gate, gate_backward, gate_double_backward, linear, linear_backward,
                          linear_double_backward, linear_instructions, linear_weight_count)
from oracle.irreps import Irreps

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_tensor_product_b200 import build
    build.build()
    import equivariant_tensor_product_b200 as tp
    return tp


# (irreps_in, irreps_out, N): ragged row counts (N (2l+1) not a multiple of the 128-row
# tile), several input blocks per irrep (concatenated K), several output blocks per irrep,
# inputs and outputs without a partner (zero blocks), K below one 32-wide K block, outputs
# wider than one 128-column tile, deep split-K reductions.
LINEARS = [
    ("32x0e+32x1o+32x2e", "32x0e+32x1o+32x2e", 300),
    ("32x0e+32x1e+32x1o+32x2e+32x2o", "32x0e+64x0e+32x1o+32x2e", 1536),
    ("4x0e+12x0e+8x1o+20x3o", "36x0e+8x1o+4x1o+16x3o+8x2e", 97),
    ("64x0e+64x1o", "192x0e+64x1o", 2000),
    ("128x0e+128x1o+128x2e", "128x0e+128x1o+128x2e", 4099),
]


FORMS = [0, 1, 2]     # chosen by size, tcgen05 GEMMs, CUDA cores


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("ir_in,ir_out,N", LINEARS)
def test_linear_forward_and_backward(tp, ir_in, ir_out, N, form):
    rng = np.random.default_rng(N)
    n_ins = len(linear_instructions(ir_in, ir_out))
    coeff = rng.uniform(0.5, 1.5, n_ins)
    lin = tp.Linear(ir_in, ir_out, coeff=list(coeff), flags=form)
    x = rng.standard_normal((N, Irreps(ir_in).dim)).astype(np.float32)
    W = rng.standard_normal(linear_weight_count(ir_in, ir_out)).astype(np.float32)
    gy = rng.standard_normal((N, Irreps(ir_out).dim)).astype(np.float32)
    y = tp.tp_linear_fwd(lin, dev(x), dev(W))
    assert_close(y, linear(ir_in, ir_out, x, W, coeff), f"{ir_out} y")
    gx, gW = tp.tp_linear_bwd(lin, dev(x), dev(W), dev(gy))
    ref = linear_backward(ir_in, ir_out, x, W, gy, coeff)
    assert_close(gx, ref["gx"], f"{ir_in} gx")
    assert_close(gW, ref["gW"], f"{ir_in} gW")
    # gx alone (x not needed) and gW alone (W not needed)
    gx2, _ = tp.tp_linear_bwd(lin, None, dev(W), dev(gy), need_gW=False)
    assert torch.equal(gx2, gx)
    _, gW2 = tp.tp_linear_bwd(lin, dev(x), None, dev(gy), need_gx=False)
    assert torch.equal(gW2, gW)


@pytest.mark.parametrize("form", [1, 2])
def test_linear_accumulate_and_empty(tp, form):
    ir_in, ir_out = "32x0e+32x1e+32x1o+32x2e+32x2o", "32x0e+64x0e+32x1o+32x2e+32x3o"
    rng = np.random.default_rng(5)
    lin = tp.Linear(ir_in, ir_out, flags=form)
    N = 200
    x = rng.standard_normal((N, lin.in_dim)).astype(np.float32)
    W = rng.standard_normal(lin.n_weights).astype(np.float32)
    y0 = rng.standard_normal((N, lin.out_dim)).astype(np.float32)
    y = dev(y0)
    tp.tp_linear_fwd(lin, dev(x), dev(W), y=y, accumulate=True)
    assert_close(y, torch.as_tensor(y0, dtype=torch.float64) + linear(ir_in, ir_out, x, W), "accumulated y")
    # the 3o output has no partner: accumulate leaves it, overwrite zeroes it
    off = Irreps(ir_out).offsets[-1]
    assert torch.equal(y[:, off:].cpu(), torch.as_tensor(y0[:, off:]))
    y2 = tp.tp_linear_fwd(lin, dev(x), dev(W), y=dev(y0))
    assert bool((y2[:, off:] == 0).all())
    # N = 0: nothing to do, and the weight gradient of no rows is zero
    e = torch.empty(0, lin.in_dim, device="cuda")
    ge = torch.empty(0, lin.out_dim, device="cuda")
    assert tp.tp_linear_fwd(lin, e, dev(W)).shape == (0, lin.out_dim)
    gx, gW = tp.tp_linear_bwd(lin, e, dev(W), ge)
    assert gx.shape == (0, lin.in_dim) and bool((gW == 0).all())


@pytest.mark.parametrize("form", [1, 2])
def test_linear_second_order_through_autograd(tp, form):
    ir_in, ir_out = "32x0e+32x1o+32x2e+32x1e", "64x0e+32x1o+32x2e+32x2o"
    rng = np.random.default_rng(6)
    lin = tp.Linear(ir_in, ir_out, flags=form)
    N = 333
    x = rng.standard_normal((N, lin.in_dim)).astype(np.float32)
    W = rng.standard_normal(lin.n_weights).astype(np.float32)
    gy = rng.standard_normal((N, lin.out_dim)).astype(np.float32)
    ggx = rng.standard_normal(x.shape).astype(np.float32)
    ggW = rng.standard_normal(W.shape).astype(np.float32)
    xt, Wt, gyt = (dev(a).requires_grad_(True) for a in (x, W, gy))
    y = tp.tp_linear(lin, xt, Wt)
    gx, gW = torch.autograd.grad(y, (xt, Wt), gyt, create_graph=True)
    s = (gx * dev(ggx)).sum() + (gW * dev(ggW)).sum()
    g_gy, g_x, g_W = torch.autograd.grad(s, (gyt, xt, Wt))
    ref = linear_double_backward(ir_in, ir_out, x, W, gy, ggx=ggx, ggW=ggW)
    assert_close(g_gy, ref["g_gy"], "linear g_gy")
    assert_close(g_x, ref["g_x"], "linear g_x")
    assert_close(g_W, ref["g_W"], "linear g_W")


GATES = [("32x0e", "32x0e+32x0e", "32x1o+32x2e"), ("3x0e+2x0o", "2x0e+3x0e", "2x1o+1x2e+2x1e"),
         ("", "8x0e", "8x3o"), ("16x0o", "", "")]


@pytest.mark.parametrize("args", GATES)
def test_gate_all_orders(tp, args):
    spec = GateSpec(*args)
    g = tp.Gate(*args)
    rng = np.random.default_rng(len(args[0]) + spec.in_dim)
    N = 1001
    x = (rng.standard_normal((N, spec.in_dim)) * 3).astype(np.float32)
    gy = rng.standard_normal((N, spec.out_dim)).astype(np.float32)
    ggx = rng.standard_normal((N, spec.in_dim)).astype(np.float32)
    assert_close(tp.tp_gate_fwd(g, dev(x)), gate(spec, x), "gate y")
    assert_close(tp.tp_gate_bwd(g, dev(x), dev(gy)), gate_backward(spec, x, gy), "gate gx")
    g_gy, g_x = tp.tp_gate_dbwd(g, dev(x), dev(gy), dev(ggx))
    ref = gate_double_backward(spec, x, gy, ggx)
    assert_close(g_gy, ref["g_gy"], "gate g_gy")
    assert_close(g_x, ref["g_x"], "gate g_x")
    # through the binding: second order by autograd
    xt, gyt = dev(x).requires_grad_(True), dev(gy).requires_grad_(True)
    (gx,) = torch.autograd.grad(tp.tp_gate(g, xt), xt, gyt, create_graph=True)
    a_gy, a_x = torch.autograd.grad((gx * dev(ggx)).sum(), (gyt, xt))
    assert torch.equal(a_gy, g_gy) and torch.equal(a_x, g_x)


def test_gate_extreme_inputs_stay_finite(tp):
    spec_args = ("2x0e+2x0o", "2x0e", "2x1o")
    g = tp.Gate(*spec_args)
    x = np.array([[-100.0, 100.0, -30.0, 30.0, -100.0, 100.0, 1, 2, 3, 4, 5, 6],
                  [0.0, 1e-6, -1e-6, 0.0, 0.0, -1e-6, 1, 2, 3, 4, 5, 6]], dtype=np.float32)
    gy = np.ones((2, 2 + 2 + 6), np.float32)
    spec = GateSpec(*spec_args)
    assert_close(tp.tp_gate_fwd(g, dev(x)), gate(spec, x), "extreme y")
    assert_close(tp.tp_gate_bwd(g, dev(x), dev(gy)), gate_backward(spec, x, gy), "extreme gx")


def test_interaction_layer_through_autograd(tp):
    """linear -> convolution (c_p = 1 / average degree) -> linear -> gate on the 1,536-atom
    graph, differentiated to x, both weight sets, the edge weights and the edge vectors; the
    oracle chains its own VJPs in float64."""
    spec = synth.CONFIGS["c2"]
    d = synth.make_inputs("c2", 400)
    rowptr, src, vec, w = d["rowptr"], d["src"], d["vec"], d["w"]
    N, E = len(rowptr) - 1, len(src)
    c_avg = [N / E] * len(spec.paths)
    h_in = spec.irreps_in
    gate_args = ("32x0e", "32x0e+32x0e", "32x1o+32x2e")
    mid = "+".join(gate_args)
    lin1, lin2 = tp.Linear(h_in, h_in), tp.Linear(spec.irreps_out, mid)
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvu", path_coeff=c_avg)
    op = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvu")
    gt = tp.Gate(*gate_args)
    rng = np.random.default_rng(11)
    W1 = (rng.standard_normal(lin1.n_weights) / np.sqrt(32)).astype(np.float32)
    W2 = (rng.standard_normal(lin2.n_weights) / np.sqrt(32)).astype(np.float32)
    x = d["x"]
    g_out = rng.standard_normal((N, gt.out_dim)).astype(np.float32)

    graph = tp.autograd.Graph(dev(rowptr), dev(src))
    xt, W1t, W2t, wt, vt = (dev(a).requires_grad_(True) for a in (x, W1, W2, w, vec))
    h1 = tp.tp_linear(lin1, xt, W1t)
    y = tp.tp_conv(plan, graph, h1, vt, wt)
    out = tp.tp_gate(gt, tp.tp_linear(lin2, y, W2t))
    grads = torch.autograd.grad(out, (xt, W1t, W2t, wt, vt), dev(g_out))

    # oracle: forward chain, then the VJPs in reverse
    from oracle import forward
    h1r = linear(h_in, h_in, x, W1)
    yr = forward(op, rowptr, src, h1r, vec, w=w) * (N / E)
    h2r = linear(spec.irreps_out, mid, yr, W2)
    gs = GateSpec(*gate_args)
    assert_close(out, gate(gs, h2r), "layer output")
    g_h2 = gate_backward(gs, h2r, g_out)
    b2 = linear_backward(spec.irreps_out, mid, yr, W2, g_h2)
    bc = backward(op, rowptr, src, h1r, vec, b2["gx"] * (N / E), w=w)
    b1 = linear_backward(h_in, h_in, x, W1, bc["gx"])
    for name, gpu, ref in zip(("x", "W1", "W2", "w", "vec"), grads,
                              (b1["gx"], b1["gW"], b2["gW"], bc["gw"], bc["gvec"])):
        assert_close(gpu, ref, f"layer d/d{name}")
