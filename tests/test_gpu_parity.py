"""GPU parity: the CUDA library (through the C ABI) against the float64 oracle on the same
seeded fp32 inputs, per tensor max|gpu - ref| <= 1e-4 * max|ref|; CSR transposes bit for
bit against numpy's stable argsort.

Reduced replicas (same irreps, same density, fewer atoms) are compared element by element;
the full-size workloads, in the launch configuration bench.py times, on sampled receivers,
senders and edges whose exact values the oracle computes from their own edges.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_util import (assert_close, dev, device_inputs, inputs, oracle_bwd_senders, oracle_dbwd_rows,
                      oracle_dbwd_senders, oracle_fwd_rows, plans, sample_rows)
from oracle import backward, double_backward, forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_tensor_product_b200 import build
    build.build()
    import equivariant_tensor_product_b200 as tp
    return tp


def _fwd(tp, plan, g):
    return tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"])


def _bwd(tp, plan, g, gvec=True):
    gx, gw, gv, _ = tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"],
                                   need_gvec=gvec)
    return gx, gw, gv


# ------------------------------------------------------------------------------------------
# Complete comparisons (oracle runs on every edge)
# ------------------------------------------------------------------------------------------

def test_c1_forward_complete(tp):
    d = inputs("c1")
    plan, op = plans(d["spec"], tp)
    g = device_inputs(d)
    y = _fwd(tp, plan, g)
    ref = forward(op, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"])
    assert_close(y, ref, "c1 y", irreps=d["spec"].irreps_out)


def test_c1_backward_and_double_backward_complete(tp):
    d = inputs("c1", with_gg=True)
    plan, op = plans(d["spec"], tp)
    g = device_inputs(d)
    gx, gw, gvec = _bwd(tp, plan, g)
    ref = backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], w=d["w"])
    assert_close(gx, ref["gx"], "c1 gx", irreps=d["spec"].irreps_in)
    assert_close(gw, ref["gw"], "c1 gw")
    assert_close(gvec, ref["gvec"], "c1 gvec")
    h = tp.tp_conv_dbwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"], g["ggx"], g["ggw"],
                        g["ggvec"])
    ref2 = double_backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], d["ggx"], d["ggw"], d["ggvec"],
                           w=d["w"])
    for k, name in enumerate(("g_gy", "g_x", "g_w", "g_vec")):
        assert_close(h[k], ref2[name], f"c1 {name}")


def test_c2_full_size_forward_backward_complete(tp):
    """The bench workload (1,536 atoms, 46,080 edges) compared on every output element."""
    d = inputs("c2")
    plan, op = plans(d["spec"], tp)
    g = device_inputs(d)
    y = _fwd(tp, plan, g)
    assert_close(y, forward(op, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"]), "c2 y",
                 irreps=d["spec"].irreps_out)
    gx, gw, gvec = _bwd(tp, plan, g)
    ref = backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], w=d["w"])
    assert_close(gx, ref["gx"], "c2 gx", irreps=d["spec"].irreps_in)
    assert_close(gw, ref["gw"], "c2 gw")
    assert_close(gvec, ref["gvec"], "c2 gvec")


@pytest.mark.parametrize("name,n_atoms", [("c3", 320), ("c5", 512)])
def test_replica_forward_backward_complete(tp, name, n_atoms):
    d = inputs(name, n_atoms)
    plan, op = plans(d["spec"], tp)
    g = device_inputs(d)
    y = _fwd(tp, plan, g)
    assert_close(y, forward(op, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"]), f"{name} y",
                 irreps=d["spec"].irreps_out)
    gx, gw, gvec = _bwd(tp, plan, g)
    ref = backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], w=d["w"])
    assert_close(gx, ref["gx"], f"{name} gx", irreps=d["spec"].irreps_in)
    assert_close(gw, ref["gw"], f"{name} gw")
    assert_close(gvec, ref["gvec"], f"{name} gvec")


def test_c5_replica_double_backward_complete(tp):
    d = inputs("c5", 320, with_gg=True)
    plan, op = plans(d["spec"], tp)
    g = device_inputs(d)
    h = tp.tp_conv_dbwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"], g["ggx"], g["ggw"],
                        g["ggvec"])
    ref = double_backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], d["ggx"], d["ggw"], d["ggvec"],
                          w=d["w"])
    lay = {"g_gy": d["spec"].irreps_out, "g_x": d["spec"].irreps_in}
    for k, name in enumerate(("g_gy", "g_x", "g_w", "g_vec")):
        assert_close(h[k], ref[name], f"c5 replica {name}", irreps=lay.get(name))


def test_force_training_special_case(tp):
    """ggx = ggw = 0 (passed as NULL), ggvec != 0."""
    d = inputs("c5", 320, with_gg=True)
    plan, op = plans(d["spec"], tp)
    g = device_inputs(d)
    h = tp.tp_conv_dbwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"], None, None, g["ggvec"])
    ref = double_backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], None, None, d["ggvec"], w=d["w"])
    for k, name in enumerate(("g_gy", "g_x", "g_w", "g_vec")):
        assert_close(h[k], ref[name], f"force-training {name}")


# ------------------------------------------------------------------------------------------
# Full-size workloads, sampled outputs
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["c3", "c5"])
def test_full_size_sampled(tp, name):
    d = inputs(name)
    plan, op = plans(d["spec"], tp)
    g = device_inputs(d)
    y = _fwd(tp, plan, g)
    rows = sample_rows(d["rowptr"], k=40, seed=1)
    ref = oracle_fwd_rows(op, d, rows)
    assert_close(y[torch.as_tensor(rows).cuda()], ref, f"{name} y[sampled]")
    gx, gw, gvec = _bwd(tp, plan, g)
    senders = sample_rows(d["rowptr"], k=24, seed=2)
    refb, eids = oracle_bwd_senders(op, d, senders)
    sel = torch.as_tensor(senders).cuda()
    assert_close(gx[sel], refb["gx"][senders], f"{name} gx[sampled]")
    e = torch.as_tensor(eids).cuda()
    assert_close(gw[e], refb["gw"], f"{name} gw[sampled]")
    assert_close(gvec[e], refb["gvec"], f"{name} gvec[sampled]")


def test_c5_full_size_double_backward_sampled(tp):
    d = inputs("c5", with_gg=True)
    plan, op = plans(d["spec"], tp)
    g = device_inputs(d)
    h = tp.tp_conv_dbwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"], g["ggx"], g["ggw"],
                        g["ggvec"])
    rows = sample_rows(d["rowptr"], k=12, seed=3)
    ref, eids = oracle_dbwd_rows(op, d, rows)
    assert_close(h[0][torch.as_tensor(rows).cuda()], ref["g_gy"], "c5 g_gy[sampled]")
    e = torch.as_tensor(eids).cuda()
    assert_close(h[2][e], ref["g_w"], "c5 g_w[sampled]")
    assert_close(h[3][e], ref["g_vec"], "c5 g_vec[sampled]")
    senders = sample_rows(d["rowptr"], k=8, seed=4)
    ref2, _ = oracle_dbwd_senders(op, d, senders)
    assert_close(h[1][torch.as_tensor(senders).cuda()], ref2["g_x"][senders], "c5 g_x[sampled]")


# ------------------------------------------------------------------------------------------
# CSR transpose: bit exact
# ------------------------------------------------------------------------------------------

def _check_transpose(tp, rowptr, src, N):
    colptr, perm = tp.tp_csr_transpose(dev(rowptr), dev(src), N)
    src = np.asarray(src)
    ref_perm = np.argsort(src, kind="stable").astype(np.int32)
    ref_col = np.concatenate([[0], np.cumsum(np.bincount(src, minlength=N))]).astype(np.int32)
    np.testing.assert_array_equal(colptr.cpu().numpy(), ref_col)
    np.testing.assert_array_equal(perm.cpu().numpy(), ref_perm)


@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c4", "c5"])
def test_transpose_bit_exact_configs(tp, name):
    d = inputs(name)
    _check_transpose(tp, d["rowptr"], d["src"], len(d["rowptr"]) - 1)


def test_transpose_adversarial(tp):
    rng = np.random.default_rng(0)
    # every edge from one sender
    N, E = 100, 5000
    rowptr = np.concatenate([[0], np.cumsum(np.bincount(rng.integers(0, N, E), minlength=N))]).astype(np.int32)
    _check_transpose(tp, rowptr, np.full(E, 7, np.int32), N)
    # many empty rows and empty sender segments
    N = 1000
    deg = np.where(rng.random(N) < 0.8, 0, rng.integers(1, 50, N))
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int32)
    src = rng.integers(0, 20, int(rowptr[-1])).astype(np.int32)
    _check_transpose(tp, rowptr, src, N)
    # no edges at all
    _check_transpose(tp, np.zeros(6, np.int32), np.zeros(0, np.int32), 5)
    # no nodes, no edges
    _check_transpose(tp, np.zeros(1, np.int32), np.zeros(0, np.int32), 0)
    # a ragged last tile, node counts at the one-pass / two-pass boundary of the digit width
    for N in (2047, 2048, 4095):
        E = 2048 * 3 + 17
        src = rng.integers(0, N, E).astype(np.int32)
        rowptr = np.concatenate([[0], np.cumsum(np.bincount(rng.integers(0, N, E), minlength=N))]).astype(np.int32)
        _check_transpose(tp, rowptr, src, N)
    # many nodes and few edges: long runs of senders without edges in colptr
    N, E = 300_000, 64
    src = rng.integers(0, N, E).astype(np.int32)
    src[:8] = N - 1
    rowptr = np.concatenate([[0], np.cumsum(np.bincount(rng.integers(0, N, E), minlength=N))]).astype(np.int32)
    _check_transpose(tp, rowptr, src, N)


def test_transpose_hub_sender_is_linear_time(tp):
    """One sender with 1.2M out-edges among 1.25M: a radix sort does O(E) work whatever the
    degree distribution; the call takes well under 1 ms on a B200."""
    rng = np.random.default_rng(11)
    N, E = 2000, 1_250_000
    src = rng.integers(0, N, E).astype(np.int32)
    src[rng.random(E) < 0.96] = 1234
    assert (src == 1234).sum() >= 1_000_000
    rowptr = np.concatenate([[0], np.cumsum(np.bincount(rng.integers(0, N, E), minlength=N))]).astype(np.int32)
    _check_transpose(tp, rowptr, src, N)
    r, s_ = dev(rowptr), dev(src)
    colptr = torch.empty(N + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(E, dtype=torch.int32, device="cuda")
    ws = torch.empty(tp.tp_csr_transpose_workspace_size(N, E), dtype=torch.uint8, device="cuda")
    for _ in range(3):
        tp.tp_csr_transpose(r, s_, N, colptr=colptr, perm=perm, ws=ws)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(10):
        tp.tp_csr_transpose(r, s_, N, colptr=colptr, perm=perm, ws=ws)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / 10
    assert ms < 1.0, f"transpose of a 1.2M-edge hub took {ms:.3f} ms"


def test_transpose_senders_out_of_range_go_last(tp):
    """Edges whose sender lies outside [0, N) are not counted in colptr and follow every valid
    edge in perm, in increasing edge order."""
    rng = np.random.default_rng(5)
    N, E = 700, 9000
    src = rng.integers(0, N, E).astype(np.int32)
    bad = rng.random(E) < 0.05
    src[bad] = rng.choice(np.array([-1, -5, N, N + 3, 2**31 - 1], np.int32), bad.sum())
    rowptr = np.concatenate([[0], np.cumsum(np.bincount(rng.integers(0, N, E), minlength=N))]).astype(np.int32)
    colptr, perm = tp.tp_csr_transpose(dev(rowptr), dev(src), N)
    valid = ~bad
    key = np.where(valid, src, N)
    np.testing.assert_array_equal(perm.cpu().numpy(), np.argsort(key, kind="stable"))
    ref_col = np.concatenate([[0], np.cumsum(np.bincount(src[valid], minlength=N))])
    np.testing.assert_array_equal(colptr.cpu().numpy(), ref_col)
    assert colptr[-1].item() == int(valid.sum())


# ------------------------------------------------------------------------------------------
# Edge cases and properties
# ------------------------------------------------------------------------------------------

def test_empty_rows_zero_length_edges_and_no_edges(tp):
    spec = synth.CONFIGS["c2"]
    plan, op = plans(spec, tp)
    rng = np.random.default_rng(5)
    N = 40
    deg = rng.integers(0, 4, N)
    deg[:5] = 0
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int32)
    E = int(rowptr[-1])
    src = rng.integers(0, N, E).astype(np.int32)
    vec = rng.standard_normal((E, 3)).astype(np.float32)
    vec[::7] = 0.0                                         # zero-length edges: Y_0 = 1, Y_l>0 = 0
    x = rng.standard_normal((N, plan.in_dim)).astype(np.float32)
    w = rng.standard_normal((E, plan.n_edge_weights)).astype(np.float32)
    gy = rng.standard_normal((N, plan.out_dim)).astype(np.float32)
    g = dict(rowptr=dev(rowptr), src=dev(src), x=dev(x), vec=dev(vec), w=dev(w), gy=dev(gy))
    y = _fwd(tp, plan, g)
    assert_close(y, forward(op, rowptr, src, x, vec, w=w), "edge-case y")
    assert float(y[:5].abs().max()) == 0.0
    gx, gw, gvec = _bwd(tp, plan, g)
    ref = backward(op, rowptr, src, x, vec, gy, w=w)
    assert_close(gx, ref["gx"], "edge-case gx")
    assert_close(gw, ref["gw"], "edge-case gw")
    assert_close(gvec, ref["gvec"], "edge-case gvec")
    assert float(gvec[::7].abs().max()) == 0.0
    # graph without edges: zero outputs
    z = dict(rowptr=dev(np.zeros(N + 1, np.int32)), src=dev(np.zeros(0, np.int32)), x=g["x"],
             vec=dev(np.zeros((0, 3), np.float32)), w=dev(np.zeros((0, plan.n_edge_weights), np.float32)),
             gy=g["gy"])
    assert float(_fwd(tp, plan, z).abs().max()) == 0.0
    gx0, _, _ = _bwd(tp, plan, z)
    assert float(gx0.abs().max()) == 0.0


def test_path_coefficients(tp):
    d = inputs("c2", 256)
    spec = d["spec"]
    coeff = np.linspace(0.5, 2.0, len(spec.paths))
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvu", path_coeff=coeff)
    from oracle import OraclePlan
    op = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvu", path_coeff=coeff)
    g = device_inputs(d)
    assert_close(_fwd(tp, plan, g), forward(op, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"]), "coeff y")
    gx, gw, gvec = _bwd(tp, plan, g)
    ref = backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], w=d["w"])
    assert_close(gx, ref["gx"], "coeff gx")
    assert_close(gw, ref["gw"], "coeff gw")
    assert_close(gvec, ref["gvec"], "coeff gvec")


def test_deterministic_run_to_run(tp):
    d = inputs("c5", 512)
    plan, _ = plans(d["spec"], tp)
    g = device_inputs(d)
    a, b = _fwd(tp, plan, g), _fwd(tp, plan, g)
    assert torch.equal(a, b)
    ga, gb = _bwd(tp, plan, g), _bwd(tp, plan, g)
    for u, v in zip(ga, gb):
        assert torch.equal(u, v)


def test_user_supplied_transpose_and_streams(tp):
    d = inputs("c2", 512)
    plan, _ = plans(d["spec"], tp)
    g = device_inputs(d)
    colptr, perm = tp.tp_csr_transpose(g["rowptr"], g["src"], len(d["rowptr"]) - 1)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        gx1, gw1, _, _ = tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"],
                                        colptr=colptr, perm=perm)
    s.synchronize()
    gx2, gw2, _ = _bwd(tp, plan, g, gvec=False)
    assert torch.equal(gx1, gx2) and torch.equal(gw1, gw2)


def test_index_check_reports_bad_sender(tp):
    d = inputs("c1")
    spec = d["spec"]
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, flags=tp.TP_FLAG_CHECK_INDICES)
    g = device_inputs(d)
    bad = g["src"].clone()
    bad[5] = 10_000
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    y = tp.tp_conv_fwd(plan, g["rowptr"], bad, g["x"], g["vec"], g["w"], ws=ws)
    assert tp.tp_get_device_error(plan, ws) == 2
    assert torch.isfinite(y).all()
    y = tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], ws=ws)
    assert tp.tp_get_device_error(plan, ws) == 0
    # decreasing rowptr (values stay within [0, E])
    rp = g["rowptr"].clone()
    rp[3] = rp[5]
    tp.tp_conv_fwd(plan, rp, g["src"], g["x"], g["vec"], g["w"], ws=ws)
    assert tp.tp_get_device_error(plan, ws) == 1
    torch.cuda.synchronize()


def test_autograd_first_and_second_derivatives(tp):
    from equivariant_tensor_product_b200.autograd import Graph, tp_conv
    d = inputs("c5", 256, with_gg=True)
    plan, op = plans(d["spec"], tp)
    graph = Graph(dev(d["rowptr"]), dev(d["src"]))
    x = dev(d["x"]).requires_grad_(True)
    vec = dev(d["vec"]).requires_grad_(True)
    w = dev(d["w"]).requires_grad_(True)
    y = tp_conv(plan, graph, x, vec, w)
    gy = dev(d["gy"])
    gx, gvec, gw = torch.autograd.grad(y, [x, vec, w], gy, create_graph=True)
    ref = backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], w=d["w"])
    assert_close(gx, ref["gx"], "autograd gx")
    assert_close(gvec, ref["gvec"], "autograd gvec")
    L = (gvec * dev(d["ggvec"])).sum()                   # force-training style loss
    g2 = torch.autograd.grad(L, [x, vec, w])
    ref2 = double_backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], None, None, d["ggvec"], w=d["w"])
    assert_close(g2[0], ref2["g_x"], "autograd g_x")
    assert_close(g2[1], ref2["g_vec"], "autograd g_vec")
    assert_close(g2[2], ref2["g_w"], "autograd g_w")
