"""Pins for the float64 oracle of the convolution with the radial projection fused in.

w = h @ W_r is checked against an explicit triple loop feeding the pure-Python per-edge
forward (no matmul, no einsum), the map's bilinearity in (h, W_r), the rank-one case that
factors into a per-edge scalar times a per-weight row, and central finite differences of
<gy, y> in every input (independent of autograd).  A planted mistake in the projection
(a dropped hidden unit, the matrix read transposed, half of the gradient lost) must fail
one of them.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import OraclePlan, forward
from oracle.brute import forward_loops
from oracle.radial import backward_radial, forward_radial

L2_CASE = ("2x0e+2x1o+2x2e", "1x0e+1x1o+1x2e", "2x0e+2x1e+2x1o+2x2e+2x2o", synth.L2_PATHS)
MIXED_CASE = ("3x0e+2x1o", "1x0e+1x1o", "3x0e+3x1o+2x1o+2x1e+2x0e",
              [(0, 0, 0), (0, 1, 1), (1, 0, 2), (1, 1, 3), (1, 1, 4)])


def _case(spec, n=6, H=5, seed=0, deg_hi=4):
    rng = np.random.default_rng(seed)
    plan = OraclePlan(*spec, "uvu")
    deg = rng.integers(0, deg_hi + 1, size=n)
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int32)
    E = int(rowptr[-1])
    src = rng.integers(0, n, size=E).astype(np.int32)
    vec = rng.standard_normal((E, 3)) * 2.0
    x = rng.standard_normal((n, plan.irr_in.dim))
    h = rng.standard_normal((E, H))
    Wr = rng.standard_normal((H, plan.n_weights)) / np.sqrt(H)
    gy = rng.standard_normal((n, plan.irr_out.dim))
    return plan, rowptr, src, vec, x, h, Wr, gy


def _loops_projection(h, Wr):
    E, H = len(h), len(Wr)
    nw = len(Wr[0])
    w = [[0.0] * nw for _ in range(E)]
    for e in range(E):
        for c in range(nw):
            acc = 0.0
            for k in range(H):
                acc += float(h[e][k]) * float(Wr[k][c])
            w[e][c] = acc
    return np.array(w)


@pytest.mark.parametrize("spec", [L2_CASE, MIXED_CASE])
def test_forward_matches_loops(spec):
    plan, rowptr, src, vec, x, h, Wr, _ = _case(spec, seed=3)
    y = forward_radial(plan, rowptr, src, x, vec, h, Wr).numpy()
    ref = forward_loops(plan, rowptr, src, x, vec, w=_loops_projection(h, Wr))
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-11)


def test_bilinear_in_h_and_Wr():
    plan, rowptr, src, vec, x, h, Wr, _ = _case(L2_CASE, seed=4)
    rng = np.random.default_rng(5)
    h2, Wr2 = rng.standard_normal(h.shape), rng.standard_normal(Wr.shape)
    f = lambda hh, WW: forward_radial(plan, rowptr, src, x, vec, hh, WW).numpy()
    np.testing.assert_allclose(f(h + 2.5 * h2, Wr), f(h, Wr) + 2.5 * f(h2, Wr), rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(f(h, Wr - 0.5 * Wr2), f(h, Wr) - 0.5 * f(h, Wr2), rtol=1e-10, atol=1e-10)


def test_rank_one_factorises():
    """W_r = a b^T gives w[e, :] = (h[e] . a) b: the projection is a per-edge scalar times a row."""
    plan, rowptr, src, vec, x, h, _, _ = _case(L2_CASE, seed=6, H=4)
    rng = np.random.default_rng(7)
    a, b = rng.standard_normal(4), rng.standard_normal(plan.n_weights)
    y = forward_radial(plan, rowptr, src, x, vec, h, np.outer(a, b)).numpy()
    ref = forward(plan, rowptr, src, x, vec, w=(h @ a)[:, None] * b[None, :]).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-11)


def _dirderiv(f, theta, d, eps=1e-6):
    return (f(theta + eps * d) - f(theta - eps * d)) / (2 * eps)


@pytest.mark.parametrize("spec", [L2_CASE, MIXED_CASE])
def test_backward_finite_differences(spec):
    plan, rowptr, src, vec, x, h, Wr, gy = _case(spec, seed=8)
    g = backward_radial(plan, rowptr, src, x, vec, h, Wr, gy)
    L = lambda xx, vv, hh, WW: float((gy * forward_radial(plan, rowptr, src, xx, vv, hh, WW).numpy()).sum())
    rng = np.random.default_rng(9)
    for name, arr in [("gx", x), ("gvec", vec), ("gh", h), ("gWr", Wr)]:
        d = rng.standard_normal(arr.shape)
        if name == "gx":
            fd = _dirderiv(lambda t: L(t, vec, h, Wr), x, d)
        elif name == "gvec":
            fd = _dirderiv(lambda t: L(x, t, h, Wr), vec, d)
        elif name == "gh":
            fd = _dirderiv(lambda t: L(x, vec, t, Wr), h, d)
        else:
            fd = _dirderiv(lambda t: L(x, vec, h, t), Wr, d)
        an = float((g[name].numpy() * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_empty_graph_and_rows():
    plan, _, _, _, x, _, Wr, gy = _case(L2_CASE, seed=10)
    n = len(x)
    rowptr = np.zeros(n + 1, np.int32)
    src = np.zeros(0, np.int32)
    vec, h = np.zeros((0, 3)), np.zeros((0, Wr.shape[0]))
    assert not forward_radial(plan, rowptr, src, x, vec, h, Wr).abs().max() > 0
    g = backward_radial(plan, rowptr, src, x, vec, h, Wr, gy)
    assert g["gh"].shape == (0, Wr.shape[0]) and not g["gWr"].abs().max() > 0 and not g["gx"].abs().max() > 0


@pytest.mark.parametrize("mutation", ["drop_hidden_unit", "transposed_read", "half_weight_gradient"])
def test_planted_mistakes_are_caught(mutation, monkeypatch):
    """Plant a plausible mistake in the projection (CPU only) and check a pin catches it."""
    import oracle.radial as orad

    good = orad.radial_weights
    if mutation == "drop_hidden_unit":
        monkeypatch.setattr(orad, "radial_weights", lambda h, Wr: good(np.asarray(h)[:, :-1], np.asarray(Wr)[:-1]))
    elif mutation == "transposed_read":
        # reads W_r[k, c] as the flat (c, k) entry of the same storage: same shape, wrong layout
        monkeypatch.setattr(orad, "radial_weights",
                            lambda h, Wr: good(h, np.asarray(Wr).reshape(-1).reshape(np.asarray(Wr).shape[1], -1).T))
    else:
        real_messages = orad._edge_messages

        def half_gradient(plan, xs, vec, wts, W):
            # same values, but only half of the weights' gradient flows back to h and W_r
            return real_messages(plan, xs, vec, 0.5 * wts + (0.5 * wts).detach(), W)
        monkeypatch.setattr(orad, "_edge_messages", half_gradient)
    caught = False
    for pin in (lambda: test_forward_matches_loops(L2_CASE), lambda: test_backward_finite_differences(L2_CASE)):
        try:
            pin()
        except AssertionError:
            caught = True
            break
    assert caught, mutation
