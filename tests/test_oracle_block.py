"""Pins of the float64 node-side oracle (irreps-wise linear map and gate) against facts that
do not come from the oracle itself: special cases that reduce to a matrix product or to
scipy's logistic function, rotation equivariance with the oracle's Wigner-D (fitted
independently of these operators), inversion parity, finite differences, the adjoint
identity and gradgradcheck."""
import numpy as np
import pytest
import scipy.special
import torch

from oracle.block import (GateSpec, gate, gate_backward, gate_double_backward, linear, linear_backward,
                          linear_double_backward, linear_instructions, linear_weight_count)
from oracle.irreps import Irreps
from oracle.so3 import random_rotation, wigner_D


def _rotate(irreps: str, x: np.ndarray, R: np.ndarray, inversion: bool = False) -> np.ndarray:
    ir = Irreps(irreps)
    out = np.empty_like(x)
    for (mul, l, p), off in zip(ir.blocks, ir.offsets):
        d = 2 * l + 1
        D = wigner_D(l, R)
        if inversion:
            D = D * p
        blk = x[:, off:off + mul * d].reshape(len(x), mul, d)
        out[:, off:off + mul * d] = np.einsum("ab,nub->nua", D, blk).reshape(len(x), mul * d)
    return out


# ---------------------------------------------------------------- linear


def test_instructions_pair_equal_irreps_in_lexicographic_order():
    assert linear_instructions("2x0e+3x1o+1x1e+2x0e", "4x1o+5x0e+1x0o") == [(0, 1), (1, 0), (3, 1)]
    assert linear_weight_count("2x0e+3x1o+1x1e+2x0e", "4x1o+5x0e+1x0o") == 2 * 5 + 3 * 4 + 2 * 5


def test_scalar_linear_is_a_matrix_product():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((7, 3))
    W = rng.standard_normal((3, 5))                      # W[u, w], row-major
    y = linear("3x0e", "5x0e", x, W.ravel()).numpy()
    np.testing.assert_allclose(y, x @ W, rtol=1e-13, atol=1e-13)


def test_inputs_of_one_irrep_sum_into_the_output_with_their_coefficients():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((6, 5))
    W1, W2 = rng.standard_normal((3, 4)), rng.standard_normal((2, 4))
    W = np.concatenate([W1.ravel(), W2.ravel()])
    y = linear("3x0e+2x0e", "4x0e", x, W, coeff=[2.0, -0.5]).numpy()
    np.testing.assert_allclose(y, 2.0 * x[:, :3] @ W1 - 0.5 * x[:, 3:] @ W2, rtol=1e-13, atol=1e-13)


def test_vector_block_mixes_channels_and_keeps_m():
    # one l = 1 block: every m component is the same matrix product over channels
    rng = np.random.default_rng(2)
    x = rng.standard_normal((4, 3 * 3))
    W = rng.standard_normal((3, 2))
    y = linear("3x1o", "2x1o", x, W.ravel()).numpy().reshape(4, 2, 3)
    xb = x.reshape(4, 3, 3)
    for m in range(3):
        np.testing.assert_allclose(y[:, :, m], xb[:, :, m] @ W, rtol=1e-13, atol=1e-13)


def test_blocks_without_instruction_are_zero():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 2 + 9))
    W = rng.standard_normal(linear_weight_count("2x0e+3x1o", "2x2o+4x1o+2x1e"))
    y = linear("2x0e+3x1o", "2x2o+4x1o+2x1e", x, W).numpy()
    assert np.all(y[:, :10] == 0) and np.all(y[:, 22:] == 0)
    assert np.abs(y[:, 10:22]).max() > 0


IR_IN = "4x0e+3x1o+2x1o+2x2e+1x0o+2x3o"
IR_OUT = "3x1o+2x0e+2x2e+1x0o+3x3o+2x1e"


@pytest.mark.parametrize("inversion", [False, True])
def test_linear_commutes_with_rotations_and_inversion(inversion):
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, Irreps(IR_IN).dim))
    W = rng.standard_normal(linear_weight_count(IR_IN, IR_OUT))
    for _ in range(3):
        R = random_rotation(rng)
        lhs = linear(IR_IN, IR_OUT, _rotate(IR_IN, x, R, inversion), W).numpy()
        rhs = _rotate(IR_OUT, linear(IR_IN, IR_OUT, x, W).numpy(), R, inversion)
        np.testing.assert_allclose(lhs, rhs, rtol=1e-10, atol=1e-10)


def test_linear_backward_matches_finite_differences_and_the_adjoint_identity():
    rng = np.random.default_rng(5)
    N = 3
    x = rng.standard_normal((N, Irreps(IR_IN).dim))
    W = rng.standard_normal(linear_weight_count(IR_IN, IR_OUT))
    gy = rng.standard_normal((N, Irreps(IR_OUT).dim))
    coeff = rng.uniform(0.5, 2.0, len(linear_instructions(IR_IN, IR_OUT)))
    g = linear_backward(IR_IN, IR_OUT, x, W, gy, coeff)
    f = lambda xx, WW: float((linear(IR_IN, IR_OUT, xx, WW, coeff).numpy() * gy).sum())
    h = 1e-6
    for arr, key in ((x, "gx"), (W, "gW")):
        flat = arr.reshape(-1)
        for idx in rng.choice(flat.size, 12, replace=False):
            p, m = flat.copy(), flat.copy()
            p[idx] += h
            m[idx] -= h
            args_p = (p.reshape(arr.shape), W) if key == "gx" else (x, p)
            args_m = (m.reshape(arr.shape), W) if key == "gx" else (x, m)
            fd = (f(*args_p) - f(*args_m)) / (2 * h)
            assert abs(fd - g[key].reshape(-1)[idx].item()) <= 1e-6 * max(1.0, abs(fd))
    dx = rng.standard_normal(x.shape)
    lhs = (gy * linear(IR_IN, IR_OUT, dx, W, coeff).numpy()).sum()
    np.testing.assert_allclose(lhs, (g["gx"].numpy() * dx).sum(), rtol=1e-12)


def test_linear_double_backward_is_the_composition_of_forward_and_backward():
    # gx is linear in (gy, W) and gW bilinear in (x, gy): the second-order terms are again
    # applications of the map and of its adjoint
    rng = np.random.default_rng(6)
    N = 4
    x = rng.standard_normal((N, Irreps(IR_IN).dim))
    W = rng.standard_normal(linear_weight_count(IR_IN, IR_OUT))
    gy = rng.standard_normal((N, Irreps(IR_OUT).dim))
    ggx = rng.standard_normal(x.shape)
    ggW = rng.standard_normal(W.shape)
    r = linear_double_backward(IR_IN, IR_OUT, x, W, gy, ggx=ggx, ggW=ggW)
    np.testing.assert_allclose(r["g_gy"].numpy(), (linear(IR_IN, IR_OUT, ggx, W) + linear(IR_IN, IR_OUT, x, ggW)).numpy(),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["g_x"].numpy(), linear_backward(IR_IN, IR_OUT, x, ggW, gy)["gx"].numpy(),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["g_W"].numpy(), linear_backward(IR_IN, IR_OUT, ggx, W, gy)["gW"].numpy(),
                               rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- gate

G_SC, G_GT, G_GD = "3x0e+2x0o", "2x0e+3x0e", "2x1o+1x2e+2x1e"


def test_gate_validation():
    with pytest.raises(ValueError):
        GateSpec("2x1o", "2x0e", "2x1o")          # scalar block with l > 0
    with pytest.raises(ValueError):
        GateSpec("2x0e", "2x0o", "2x1o")          # odd gates
    with pytest.raises(ValueError):
        GateSpec("2x0e", "3x0e", "2x1o")          # multiplicity mismatch
    s = GateSpec(G_SC, G_GT, G_GD)
    assert (s.in_dim, s.out_dim) == (5 + 5 + 6 + 5 + 6, 5 + 6 + 5 + 6)


def test_gate_matches_the_logistic_function():
    rng = np.random.default_rng(7)
    s = GateSpec(G_SC, G_GT, G_GD)
    x = rng.standard_normal((6, s.in_dim)) * 3
    y = gate(s, x).numpy()
    np.testing.assert_allclose(y[:, :3], x[:, :3] * scipy.special.expit(x[:, :3]), rtol=1e-13)
    np.testing.assert_allclose(y[:, 3:5], np.tanh(x[:, 3:5]), rtol=1e-13)
    sig = scipy.special.expit(x[:, 5:10])
    v = x[:, 10:]
    ref = np.concatenate([(v[:, :6].reshape(6, 2, 3) * sig[:, 0:2, None]).reshape(6, 6),
                          v[:, 6:11] * sig[:, 2:3],
                          (v[:, 11:17].reshape(6, 2, 3) * sig[:, 3:5, None]).reshape(6, 6)], axis=1)
    np.testing.assert_allclose(y[:, 5:], ref, rtol=1e-13)


@pytest.mark.parametrize("inversion", [False, True])
def test_gate_commutes_with_rotations_and_inversion(inversion):
    rng = np.random.default_rng(8)
    s = GateSpec(G_SC, G_GT, G_GD)
    ir_in = "+".join([G_SC, G_GT, G_GD])
    ir_out = "+".join([G_SC, G_GD])
    x = rng.standard_normal((5, s.in_dim))
    R = random_rotation(rng)
    lhs = gate(s, _rotate(ir_in, x, R, inversion)).numpy()
    rhs = _rotate(ir_out, gate(s, x).numpy(), R, inversion)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-10, atol=1e-10)


def test_gate_derivatives_at_zero():
    # closed forms: silu'(0) = 1/2, tanh'(0) = 1, d/dg [v sigmoid(g)] at g = 0 is v/4
    s = GateSpec("1x0e+1x0o", "1x0e", "1x1o")
    x = np.array([[0.0, 0.0, 0.0, 1.0, -2.0, 3.0]])
    gy = np.array([[1.0, 1.0, 1.0, 1.0, 1.0]])
    gx = gate_backward(s, x, gy).numpy()
    np.testing.assert_allclose(gx[0, :3], [0.5, 1.0, 0.25 * (1.0 - 2.0 + 3.0)], rtol=1e-14)
    np.testing.assert_allclose(gx[0, 3:], [0.5, 0.5, 0.5], rtol=1e-14)


def test_gate_backward_matches_finite_differences():
    rng = np.random.default_rng(9)
    s = GateSpec(G_SC, G_GT, G_GD)
    x = rng.standard_normal((3, s.in_dim))
    gy = rng.standard_normal((3, s.out_dim))
    gx = gate_backward(s, x, gy).numpy().reshape(-1)
    f = lambda xx: float((gate(s, xx).numpy() * gy).sum())
    h = 1e-6
    flat = x.reshape(-1)
    for idx in range(flat.size):
        p, m = flat.copy(), flat.copy()
        p[idx] += h
        m[idx] -= h
        fd = (f(p.reshape(x.shape)) - f(m.reshape(x.shape))) / (2 * h)
        assert abs(fd - gx[idx]) <= 1e-6 * max(1.0, abs(fd))


def test_gate_double_backward_gradgradcheck():
    rng = np.random.default_rng(10)
    s = GateSpec("2x0e+1x0o", "2x0e", "1x1o+1x2e")
    x = torch.tensor(rng.standard_normal((2, s.in_dim)), requires_grad=True)
    from oracle.block import _gate_t
    assert torch.autograd.gradgradcheck(lambda t: _gate_t(s, t), (x,), eps=1e-6, atol=1e-6)
    gy = rng.standard_normal((2, s.out_dim))
    ggx = rng.standard_normal(x.shape)
    r = gate_double_backward(s, x.detach(), gy, ggx)
    # g_gy is the forward Jacobian applied to ggx: a finite difference of the forward map
    h = 1e-6
    xd = x.detach().numpy()
    jv = (gate(s, xd + h * ggx).numpy() - gate(s, xd - h * ggx).numpy()) / (2 * h)
    np.testing.assert_allclose(r["g_gy"].numpy(), jv, rtol=1e-6, atol=1e-8)


# ---------------------------------------------------------------- planted mistakes

def _permute_blocks(irreps: str, x, to_mu: bool):
    """[u][m] <-> [m][u] inside every block of a feature row."""
    ir = Irreps(irreps)
    out = x.clone()
    for (mul, l, _), off in zip(ir.blocks, ir.offsets):
        d = 2 * l + 1
        blk = x[:, off:off + mul * d]
        out[:, off:off + mul * d] = (blk.reshape(-1, mul, d).transpose(1, 2) if to_mu
                                     else blk.reshape(-1, d, mul).transpose(1, 2)).reshape(-1, mul * d)
    return out


@pytest.mark.parametrize("mutation", ["w_transposed", "m_u_swapped", "dropped_instruction", "coeff_ignored"])
def test_planted_linear_mistakes_are_caught(mutation, monkeypatch):
    """Plant a plausible mistake in the oracle's linear map (CPU only); a pin must fail."""
    import oracle.block as ob
    good = ob._linear_t

    def bad(ir_in, ir_out, x, W, coeff):
        ins = linear_instructions(ir_in, ir_out)
        a, b = Irreps(ir_in), Irreps(ir_out)
        if mutation == "w_transposed":          # W_k read as [mul_out][mul_in]
            parts, off = [], 0
            for i, o in ins:
                mi, mo = a.blocks[i][0], b.blocks[o][0]
                parts.append(W[off:off + mi * mo].reshape(mo, mi).T.reshape(-1))
                off += mi * mo
            return good(ir_in, ir_out, x, torch.cat(parts), coeff)
        if mutation == "m_u_swapped":           # blocks read as [m][u]
            return good(ir_in, ir_out, _permute_blocks(ir_in, x, True), W, coeff)
        if mutation == "dropped_instruction":   # the last instruction left out
            mi, mo = a.blocks[ins[-1][0]][0], b.blocks[ins[-1][1]][0]
            W2 = W.clone()
            W2[len(W) - mi * mo:] = 0
            return good(ir_in, ir_out, x, W2, coeff)
        return good(ir_in, ir_out, x, W, None)   # coefficients ignored

    monkeypatch.setattr(ob, "_linear_t", bad)
    pins = [test_scalar_linear_is_a_matrix_product, test_inputs_of_one_irrep_sum_into_the_output_with_their_coefficients,
            test_vector_block_mixes_channels_and_keeps_m,
            lambda: test_linear_commutes_with_rotations_and_inversion(False)]
    caught = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught, mutation


@pytest.mark.parametrize("mutation", ["sigmoid_on_scalars", "tanh_on_even", "gate_shifted", "gate_unsquashed"])
def test_planted_gate_mistakes_are_caught(mutation, monkeypatch):
    """Plant a plausible mistake in the oracle's gate (CPU only); a pin must fail."""
    import oracle.block as ob

    def bad(spec, x):
        N = x.shape[0]
        cols, off = [], 0
        for m, _, p in spec.scalar_blocks:
            s = x[:, off:off + m]
            if mutation == "sigmoid_on_scalars":
                cols.append(torch.sigmoid(s))
            elif mutation == "tanh_on_even":
                cols.append(torch.tanh(s))
            else:
                cols.append(torch.nn.functional.silu(s) if p == 1 else torch.tanh(s))
            off += m
        g = x[:, off:off + spec.n_gate]
        if mutation == "gate_shifted":
            g = torch.roll(g, 1, dims=1)
        gates = g if mutation == "gate_unsquashed" else torch.sigmoid(g)
        off += spec.n_gate
        c = 0
        for m, l, _ in spec.gated_blocks:
            d = 2 * l + 1
            v = x[:, off:off + m * d].reshape(N, m, d)
            cols.append((v * gates[:, c:c + m, None]).reshape(N, m * d))
            off += m * d
            c += m
        return torch.cat(cols, dim=1)

    monkeypatch.setattr(ob, "_gate_t", bad)
    caught = False
    try:
        test_gate_matches_the_logistic_function()
    except AssertionError:
        caught = True
    assert caught, mutation
