"""Pins for the oracle convolution (forward, backward, double backward).

Checks that hold by mathematics, not by re-running the oracle's formula: rotation
equivariance, inversion parity, the l=0 case against scipy.sparse SpMV, linearity,
node relabelling, central finite differences, the adjoint identity, a pure-Python loop,
chunk independence, the uvw reassociation identity and hand-derived single-edge values.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.sparse as sp
import torch

import synth
from oracle import OraclePlan, backward, double_backward, forward, forward_uvw_reassociated
from oracle.brute import forward_loops
from oracle.so3 import random_rotation, wigner_D

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _graph(rng, n, deg_lo=0, deg_hi=5):
    deg = rng.integers(deg_lo, deg_hi + 1, size=n)
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int32)
    src = rng.integers(0, n, size=int(rowptr[-1])).astype(np.int32)
    vec = rng.standard_normal((len(src), 3)) * 2.0
    return rowptr, src, vec


def _case(irreps_in, irreps_sh, irreps_out, paths, mode="uvu", n=7, seed=0, deg_hi=5):
    rng = np.random.default_rng(seed)
    plan = OraclePlan(irreps_in, irreps_sh, irreps_out, paths, mode)
    rowptr, src, vec = _graph(rng, n, 0, deg_hi)
    E = len(src)
    x = rng.standard_normal((n, plan.irr_in.dim))
    w = rng.standard_normal((E, plan.n_weights))
    W = rng.standard_normal(plan.W_shape) / 4 if mode == "uvw" else None
    gy = rng.standard_normal((n, plan.irr_out.dim))
    return plan, rowptr, src, vec, x, w, W, gy


L2_CASE = ("2x0e+2x1o+2x2e", "1x0e+1x1o+1x2e", "2x0e+2x1e+2x1o+2x2e+2x2o", synth.L2_PATHS)
L3_CASE = ("2x0e+2x1o+2x2e+2x3o", "1x0e+1x1o+1x2e+1x3o", "2x0e+2x1e+2x1o+2x2e+2x2o+2x3e+2x3o",
           synth.L3_PATHS)


def _fwd(plan, rowptr, src, vec, x, w, W):
    if plan.mode == "uvu":
        return forward(plan, rowptr, src, x, vec, w=w).numpy()
    return forward(plan, rowptr, src, x, vec, s=w, W=W).numpy()


def _block_D(irreps, R, with_parity=False):
    """Block-diagonal representation matrix on a feature row ([u][m] layout)."""
    mats = []
    for mul, l, p in irreps.blocks:
        D = wigner_D(l, R) * (p if with_parity else 1)
        mats.append(np.kron(np.eye(mul), D))
    from scipy.linalg import block_diag
    return block_diag(*mats)


@pytest.mark.parametrize("case,mode", [(L2_CASE, "uvu"), (L3_CASE, "uvu"), (L2_CASE, "uvw")])
def test_rotation_equivariance(case, mode):
    plan, rowptr, src, vec, x, w, W, _ = _case(*case, mode=mode, seed=1)
    if mode == "uvw":
        w = w[:, :len(plan.paths)]
    rng = np.random.default_rng(5)
    y = _fwd(plan, rowptr, src, vec, x, w, W)
    for _ in range(3):
        R = random_rotation(rng)
        Din, Dout = _block_D(plan.irr_in, R), _block_D(plan.irr_out, R)
        yr = _fwd(plan, rowptr, src, vec @ R.T, x @ Din.T, w, W)
        np.testing.assert_allclose(yr, y @ Dout.T, atol=1e-11)


def test_inversion_parity():
    plan, rowptr, src, vec, x, w, W, _ = _case(*L3_CASE, seed=2)
    Pin = _block_D(plan.irr_in, np.eye(3), with_parity=True)
    Pout = _block_D(plan.irr_out, np.eye(3), with_parity=True)
    y = _fwd(plan, rowptr, src, vec, x, w, None)
    yi = _fwd(plan, rowptr, src, -vec, x @ Pin.T, w, None)
    np.testing.assert_allclose(yi, y @ Pout.T, atol=1e-12)


@pytest.mark.parametrize("paths,msg", [([(1, 1, 1)], "parity"), ([(0, 2, 0)], "triangle"),
                                       ([(0, 1, 0)], "triangle")])
def test_selection_rules_rejected(paths, msg):
    with pytest.raises(ValueError, match=msg):
        OraclePlan("4x0e+4x1o", "1x0e+1x1o+1x2e", "4x0e+4x1o", paths)


def test_rejects_bad_sh_and_multiplicity():
    with pytest.raises(ValueError):
        OraclePlan("4x0e", "1x1e", "4x1e", [(0, 0, 0)])
    with pytest.raises(ValueError):
        OraclePlan("4x0e", "1x0e", "8x0e", [(0, 0, 0)], "uvu")


def test_l0_is_weighted_spmv():
    rng = np.random.default_rng(3)
    n, mul = 50, 6
    rowptr, src, vec = _graph(rng, n, 0, 9)
    plan = OraclePlan(f"{mul}x0e", "1x0e", f"{mul}x0e", [(0, 0, 0)])
    x = rng.standard_normal((n, mul))
    w = rng.standard_normal((len(src), mul))
    y = _fwd(plan, rowptr, src, vec, x, w, None)
    for u in range(mul):
        A = sp.csr_matrix((w[:, u], src, rowptr), shape=(n, n))
        np.testing.assert_allclose(y[:, u], A @ x[:, u], atol=1e-12)


def test_linearity_in_x_and_w():
    plan, rowptr, src, vec, x, w, _, _ = _case(*L2_CASE, seed=4)
    rng = np.random.default_rng(9)
    x2, w2 = rng.standard_normal(x.shape), rng.standard_normal(w.shape)
    f = lambda xx, ww: _fwd(plan, rowptr, src, vec, xx, ww, None)
    np.testing.assert_allclose(f(2 * x - 3 * x2, w), 2 * f(x, w) - 3 * f(x2, w), atol=1e-11)
    np.testing.assert_allclose(f(x, 2 * w + w2), 2 * f(x, w) + f(x, w2), atol=1e-11)


def test_node_relabelling():
    plan, rowptr, src, vec, x, w, _, _ = _case(*L2_CASE, seed=6, n=9)
    n = len(rowptr) - 1
    y = _fwd(plan, rowptr, src, vec, x, w, None)
    perm = np.random.default_rng(1).permutation(n)          # new label of old node i
    dst = np.repeat(np.arange(n), np.diff(rowptr))
    nd, ns = perm[dst], perm[src]
    order = np.lexsort((ns, nd))
    rp = np.concatenate([[0], np.cumsum(np.bincount(nd, minlength=n))])
    xn = np.empty_like(x)
    xn[perm] = x
    yn = _fwd(plan, rp, ns[order], vec[order], xn, w[order], None)
    np.testing.assert_allclose(yn[perm], y, atol=1e-12)


def _dirderiv(f, theta, d, h=1e-6):
    return (f(theta + h * d) - f(theta - h * d)) / (2 * h)


@pytest.mark.parametrize("case", [L2_CASE, L3_CASE])
def test_backward_finite_differences(case):
    plan, rowptr, src, vec, x, w, _, gy = _case(*case, seed=7)
    g = backward(plan, rowptr, src, x, vec, gy, w=w)
    rng = np.random.default_rng(11)
    L = lambda xx, vv, ww: float((gy * _fwd(plan, rowptr, src, vv, xx, ww, None)).sum())
    for name, arr in [("gx", x), ("gw", w), ("gvec", vec)]:
        d = rng.standard_normal(arr.shape)
        if name == "gx":
            fd = _dirderiv(lambda t: L(t, vec, w), x, d)
        elif name == "gw":
            fd = _dirderiv(lambda t: L(x, vec, t), w, d)
        else:
            fd = _dirderiv(lambda t: L(x, t, w), vec, d)
        an = float((g[name].numpy() * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_backward_uvw_finite_differences():
    plan, rowptr, src, vec, x, w, W, gy = _case(*L2_CASE, mode="uvw", seed=8)
    s = w[:, :len(plan.paths)]
    g = backward(plan, rowptr, src, x, vec, gy, s=s, W=W)
    rng = np.random.default_rng(12)
    L = lambda xx, vv, ss, WW: float((gy * forward(plan, rowptr, src, xx, vv, s=ss, W=WW).numpy()).sum())
    for name, arr, fn in [("gx", x, lambda t: L(t, vec, s, W)), ("gs", s, lambda t: L(x, vec, t, W)),
                          ("gW", W, lambda t: L(x, vec, s, t)), ("gvec", vec, lambda t: L(x, t, s, W))]:
        d = rng.standard_normal(arr.shape)
        fd = _dirderiv(fn, arr, d)
        an = float((g[name].numpy() * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


@pytest.mark.parametrize("case", [L2_CASE, L3_CASE])
def test_double_backward_finite_differences(case):
    """d/dt <gg, bwd(theta + t d)> equals <g_theta, d> for theta in (x, vec, w, gy)."""
    plan, rowptr, src, vec, x, w, _, gy = _case(*case, seed=9, n=6, deg_hi=4)
    rng = np.random.default_rng(13)
    ggx, ggw, ggvec = (rng.standard_normal(a.shape) for a in (x, w, vec))
    h = double_backward(plan, rowptr, src, x, vec, gy, ggx, ggw, ggvec, w=w)

    def S(xx, vv, ww, gg):
        b = backward(plan, rowptr, src, xx, vv, gg, w=ww)
        return float((ggx * b["gx"].numpy()).sum() + (ggw * b["gw"].numpy()).sum()
                     + (ggvec * b["gvec"].numpy()).sum())

    for name, arr, fn in [("g_x", x, lambda t: S(t, vec, w, gy)), ("g_vec", vec, lambda t: S(x, t, w, gy)),
                          ("g_w", w, lambda t: S(x, vec, t, gy)), ("g_gy", gy, lambda t: S(x, vec, w, t))]:
        d = rng.standard_normal(arr.shape)
        fd = _dirderiv(fn, arr, d)
        an = float((h[name].numpy() * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_double_backward_force_training_case():
    """ggx = ggw = 0, ggvec != 0: g_gy equals the directional derivative of y along ggvec."""
    plan, rowptr, src, vec, x, w, _, gy = _case(*L3_CASE, seed=10, n=6, deg_hi=4)
    rng = np.random.default_rng(14)
    ggvec = rng.standard_normal(vec.shape)
    h = double_backward(plan, rowptr, src, x, vec, gy, None, None, ggvec, w=w)
    fd = _dirderiv(lambda t: _fwd(plan, rowptr, src, t, x, w, None), vec, ggvec)
    np.testing.assert_allclose(h["g_gy"].numpy(), fd, atol=1e-7)


def test_adjoint_identity():
    plan, rowptr, src, vec, x, w, _, gy = _case(*L3_CASE, seed=15)
    g = backward(plan, rowptr, src, x, vec, gy, w=w)
    rng = np.random.default_rng(16)
    dx = rng.standard_normal(x.shape)
    dw = rng.standard_normal(w.shape)
    # forward is linear in x and in w separately
    lhs_x = float((gy * _fwd(plan, rowptr, src, vec, dx, w, None)).sum())
    lhs_w = float((gy * _fwd(plan, rowptr, src, vec, x, dw, None)).sum())
    assert abs(lhs_x - float((g["gx"].numpy() * dx).sum())) < 1e-10 * max(1, abs(lhs_x))
    assert abs(lhs_w - float((g["gw"].numpy() * dw).sum())) < 1e-10 * max(1, abs(lhs_w))


def test_brute_force_matches_vectorised_c1():
    d = synth.make_inputs("c1")
    spec = d["spec"]
    plan = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths)
    yv = forward(plan, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"]).numpy()
    yb = forward_loops(plan, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"])
    np.testing.assert_allclose(yv, yb, atol=1e-12)


@pytest.mark.parametrize("case,mode", [(L3_CASE, "uvu"), (L2_CASE, "uvw")])
def test_brute_force_matches_vectorised_small(case, mode):
    plan, rowptr, src, vec, x, w, W, _ = _case(*case, mode=mode, seed=17, n=6, deg_hi=3)
    if mode == "uvw":
        w = w[:, :len(plan.paths)]
        yv = forward(plan, rowptr, src, x, vec, s=w, W=W).numpy()
        yb = forward_loops(plan, rowptr, src, x, vec, s=w, W=W)
    else:
        yv = forward(plan, rowptr, src, x, vec, w=w).numpy()
        yb = forward_loops(plan, rowptr, src, x, vec, w=w)
    np.testing.assert_allclose(yv, yb, atol=1e-12)


def test_chunked_equals_unchunked_c2():
    d = synth.make_inputs("c2")
    spec = d["spec"]
    plan = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths)
    y1 = forward(plan, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"], max_edges=1 << 20)
    y2 = forward(plan, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"], max_edges=997)
    np.testing.assert_allclose(y1.numpy(), y2.numpy(), atol=1e-11)


def test_uvw_plain_equals_reassociated():
    d = synth.make_inputs("c4", n_atoms=150)
    spec = d["spec"]
    plan = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvw")
    y1 = forward(plan, d["rowptr"], d["src"], d["x"], d["vec"], s=d["s"], W=d["W"]).numpy()
    y2 = forward_uvw_reassociated(plan, d["rowptr"], d["src"], d["x"], d["vec"], d["s"], d["W"]).numpy()
    np.testing.assert_allclose(y1, y2, atol=1e-10 * np.abs(y1).max())


def test_zero_degree_rows_and_empty_graph():
    plan = OraclePlan(*L2_CASE[:3], L2_CASE[3])
    rowptr = np.zeros(5, dtype=np.int32)
    x = np.ones((4, plan.irr_in.dim))
    y = forward(plan, rowptr, np.zeros(0, np.int32), x, np.zeros((0, 3)), w=np.zeros((0, plan.n_weights)))
    assert y.shape == (4, plan.irr_out.dim) and float(y.abs().max()) == 0.0


def test_single_edge_closed_forms():
    """Hand-derived single-edge values (tests/golden/single_edge_closed_forms.json)."""
    with open(os.path.join(GOLDEN, "single_edge_closed_forms.json")) as f:
        cases = json.load(f)["cases"]
    env = {"sqrt": math.sqrt, "pi": math.pi}
    for c in cases:
        plan = OraclePlan(c["irreps_in"], c["irreps_sh"], c["irreps_out"], c["paths"])
        y = forward(plan, [0, 1], [0], np.array([c["x"]]), np.array([c["vec"]]),
                    w=np.array([c["w"]])).numpy()[0]
        expect = [eval(e, env) for e in c["expected"]]
        np.testing.assert_allclose(y, expect, atol=1e-13, err_msg=c["name"])


@pytest.mark.parametrize("mutation", ["transpose_m1_m2", "flip_one_path", "drop_one_path", "y_not_x"])
def test_planted_mistakes_are_caught(mutation, monkeypatch):
    """Plant a plausible mistake in the oracle (CPU only) and check a pin catches it."""
    import oracle.conv as oc
    from oracle.so3 import cg_real as good_cg, real_sh as good_sh

    if mutation == "transpose_m1_m2":
        monkeypatch.setattr(oc, "cg_real", lambda a, b, c: good_cg(b, a, c).transpose(1, 0, 2)
                            if a == b else good_cg(a, b, c))
    elif mutation == "flip_one_path":
        monkeypatch.setattr(oc, "cg_real", lambda a, b, c: -good_cg(a, b, c) if (a, b, c) == (1, 1, 0)
                            else good_cg(a, b, c))
    elif mutation == "drop_one_path":
        monkeypatch.setattr(oc, "cg_real", lambda a, b, c: 0 * good_cg(a, b, c) if (a, b, c) == (0, 1, 1)
                            else good_cg(a, b, c))
    elif mutation == "y_not_x":
        # SH evaluated with x and y swapped: still unit-norm, so only a pin on values catches it
        monkeypatch.setattr(oc, "real_sh", lambda l, v: good_sh(l, v[:, [1, 0, 2]]))
    caught = False
    try:
        test_single_edge_closed_forms()
    except AssertionError:
        caught = True
    if not caught:
        try:
            test_rotation_equivariance(L2_CASE, "uvu")
        except AssertionError:
            caught = True
    assert caught, mutation
