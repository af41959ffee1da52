"""GPU parity of the uvw mode (per-path 128 x 128 multiplicity mixing, the 100,000-atom
streaming workload and same-density replicas) against the float64 oracle's plain per-edge
form, per tensor max|gpu - ref| <= 1e-4 * max|ref|."""
import numpy as np
import pytest
import torch

from gpu_util import assert_close, dev, device_inputs, edges_from, edges_into, inputs, plans, sample_rows
from oracle import backward, forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_tensor_product_b200 import build
    build.build()
    import equivariant_tensor_product_b200 as tp
    return tp


def _fwd(tp, plan, g, W=None):
    return tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["s"], W=g["W"] if W is None else W)


def _bwd(tp, plan, g, gvec=True):
    return tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["s"], g["gy"], W=g["W"],
                          need_gvec=gvec, need_gW=True)


def test_c4_replica_forward_backward_complete(tp):
    d = inputs("c4", 240)
    plan, op = plans(d["spec"], tp)
    g = device_inputs(d)
    y = _fwd(tp, plan, g)
    ref = forward(op, d["rowptr"], d["src"], d["x"], d["vec"], s=d["s"], W=d["W"])
    assert_close(y, ref, "c4 replica y", irreps=d["spec"].irreps_out)
    gx, gs, gvec, gW = _bwd(tp, plan, g)
    r = backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], s=d["s"], W=d["W"])
    assert_close(gx, r["gx"], "c4 replica gx", irreps=d["spec"].irreps_in)
    assert_close(gs, r["gs"], "c4 replica gs")
    assert_close(gvec, r["gvec"], "c4 replica gvec")
    assert_close(gW.view(r["gW"].shape), r["gW"], "c4 replica gW")


def test_c4_replica_gW_through_promoted_accumulation(tp):
    """gW element by element against the float64 oracle at a size where every split-K partial
    of the gW GEMM reduces more than 16 K blocks of 32 rows for every input irrep, so the
    fp32 promotion of the tensor-core accumulator runs inside each split, as it does at full
    size (3,000 atoms: 2 splits of 1,500 * d1 rows, i.e. 47 to 235 K blocks each)."""
    d = inputs("c4", 3000)
    N = len(d["rowptr"]) - 1
    splits = min(64, max(1, (N + 1535) // 1536))
    assert splits >= 2 and (N // splits) // 32 > 16
    plan, op = plans(d["spec"], tp)
    g = device_inputs(d)
    gx, gs, _, gW = _bwd(tp, plan, g, gvec=False)
    r = backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], s=d["s"], W=d["W"])
    assert_close(gW.view(r["gW"].shape), r["gW"], "c4 3,000-atom gW")
    assert_close(gx, r["gx"], "c4 3,000-atom gx")
    assert_close(gs, r["gs"], "c4 3,000-atom gs")


def test_c4_full_size_sampled_and_adjoint(tp):
    d = inputs("c4")
    plan, op = plans(d["spec"], tp)
    g = device_inputs(d)
    y = _fwd(tp, plan, g)
    rows = sample_rows(d["rowptr"], k=24, seed=5)
    eids, rp = edges_into(d["rowptr"], rows)
    ref = forward(op, rp, d["src"][eids], d["x"], d["vec"][eids], s=d["s"][eids], W=d["W"])
    assert_close(y[torch.as_tensor(rows).cuda()], ref, "c4 y[sampled]")
    gx, gs, _, gW = _bwd(tp, plan, g, gvec=False)
    senders = sample_rows(d["rowptr"], k=12, seed=6)
    N = len(d["rowptr"]) - 1
    e2, rp2 = edges_from(d["src"], senders, d["dst"], N)
    r = backward(op, rp2, d["src"][e2], d["x"], d["vec"][e2], d["gy"], s=d["s"][e2], W=d["W"])
    assert_close(gx[torch.as_tensor(senders).cuda()], r["gx"][senders], "c4 gx[sampled]")
    assert_close(gs[torch.as_tensor(e2).cuda()], r["gs"], "c4 gs[sampled]")
    # gW at full size: y is linear in W, so <gW, dW> = <gy, y(dW)>
    dW = torch.randn(g["W"].shape, device="cuda", generator=torch.Generator(device="cuda").manual_seed(3))
    lhs = float((gW.double() * dW.view(-1).double()).sum())
    rhs = float((g["gy"].double() * _fwd(tp, plan, g, W=dW).double()).sum())
    assert abs(lhs - rhs) <= 1e-4 * max(abs(lhs), abs(rhs)), (lhs, rhs)


def test_uvw_deterministic(tp):
    d = inputs("c4", 400)
    plan, _ = plans(d["spec"], tp)
    g = device_inputs(d)
    assert torch.equal(_fwd(tp, plan, g), _fwd(tp, plan, g))
    a, b = _bwd(tp, plan, g), _bwd(tp, plan, g)
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_uvw_through_autograd(tp):
    """tp_conv in uvw mode: gradients to x, the edge vectors, the per-edge path scalars and the
    shared mixing weights W through torch autograd, against the float64 oracle."""
    d = inputs("c4", 240)
    plan, op = plans(d["spec"], tp)
    graph = tp.autograd.Graph(dev(d["rowptr"]), dev(d["src"]))
    x, vec, s, W = (dev(d[k]).requires_grad_() for k in ("x", "vec", "s", "W"))
    y = tp.tp_conv(plan, graph, x, vec, s, W)
    (y * dev(d["gy"])).sum().backward()
    r = backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], s=d["s"], W=d["W"])
    assert_close(x.grad, r["gx"], "autograd uvw gx")
    assert_close(vec.grad, r["gvec"], "autograd uvw gvec")
    assert_close(s.grad, r["gs"], "autograd uvw gs")
    assert_close(W.grad, r["gW"], "autograd uvw gW")
    with pytest.raises(ValueError):
        tp.tp_conv(plan, graph, x, vec, s)
