"""GPU parity of the spherical-grid (Gaunt) convolution (include/tp_gaunt.h) against the
float64 oracle (oracle/gaunt.py): forward y, backward gx, gw and gvec, per tensor
max|gpu - ref| <= 1e-4 * max|ref|, on the c2 graph shape (lmax 2, 28-point grid) and on
lmax-3 cases (50-point grid) with 48 channels (a ragged second slice), a subset of degrees
and zero-length edges."""
import numpy as np
import pytest
import torch

from gpu_util import assert_close, dev, inputs
from oracle.gaunt import GauntPlan, gaunt_backward, gaunt_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_tensor_product_b200 import build
    build.build()
    import equivariant_tensor_product_b200 as tp
    return tp


def _check(tp, ir_in, L, ir_out, rowptr, src, vec, seed, tag):
    g = tp.Gaunt(ir_in, L, ir_out)
    op = GauntPlan(ir_in, L, ir_out)
    assert (g.in_dim, g.out_dim, g.n_edge_weights) == (op.in_dim, op.out_dim, op.nw)
    N, E = len(rowptr) - 1, len(src)
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((N, g.in_dim)).astype(np.float32)
    w = rng.standard_normal((E, g.n_edge_weights)).astype(np.float32)
    gy = rng.standard_normal((N, g.out_dim)).astype(np.float32)
    t = {k: dev(v) for k, v in dict(rowptr=rowptr, src=src, vec=vec, x=x, w=w, gy=gy).items()}
    y = tp.tp_gaunt_fwd(g, t["rowptr"], t["src"], t["x"], t["vec"], t["w"])
    assert_close(y, gaunt_forward(op, rowptr, src, x, vec, w), f"{tag} y", irreps=ir_out)
    gx, gw, gvec = tp.tp_gaunt_bwd(g, t["rowptr"], t["src"], t["x"], t["vec"], t["w"], t["gy"], need_gvec=True)
    r = gaunt_backward(op, rowptr, src, x, vec, w, gy)
    assert_close(gx, r["gx"], f"{tag} gx", irreps=ir_in)
    assert_close(gw, r["gw"], f"{tag} gw")
    assert_close(gvec, r["gvec"], f"{tag} gvec")
    return g


def test_gaunt_c2_graph(tp):
    d = inputs("c2", 400)
    g = _check(tp, "32x0e+32x1o+32x2e", 2, "32x0e+32x1o+32x2e", d["rowptr"], d["src"], d["vec"], 1, "gaunt c2")
    assert g.grid_points == 28


def test_gaunt_lmax3_ragged_channels_subset_and_zero_length_edges(tp):
    rng = np.random.default_rng(4)
    N = 90
    deg = rng.integers(0, 20, N)
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int32)
    E = int(rowptr[-1])
    src = rng.integers(0, N, E).astype(np.int32)
    vec = (rng.standard_normal((E, 3)) * rng.uniform(0.5, 4, (E, 1))).astype(np.float32)
    vec[::17] = 0.0                                   # zero-length edges
    g = _check(tp, "48x0e+48x1o+48x2e+48x3o", 3, "48x0e+48x2e+48x3o", rowptr, src, vec, 2, "gaunt l3")
    assert g.grid_points == 50
    _check(tp, "16x1o+16x3o", 2, "16x0e+16x2e", rowptr, src, vec, 3, "gaunt odd in")


def test_gaunt_given_transpose_and_determinism(tp):
    d = inputs("c2", 300)
    g = tp.Gaunt("8x0e+8x1o", 1, "8x0e+8x1o")
    rng = np.random.default_rng(5)
    N, E = len(d["rowptr"]) - 1, len(d["src"])
    x = dev(rng.standard_normal((N, g.in_dim)).astype(np.float32))
    w = dev(rng.standard_normal((E, g.n_edge_weights)).astype(np.float32))
    gy = dev(rng.standard_normal((N, g.out_dim)).astype(np.float32))
    r, s, v = dev(d["rowptr"]), dev(d["src"]), dev(d["vec"])
    colptr, perm = tp.tp_csr_transpose(r, s, N)
    a = tp.tp_gaunt_bwd(g, r, s, x, v, w, gy, colptr=colptr, perm=perm, need_gvec=True)
    b = tp.tp_gaunt_bwd(g, r, s, x, v, w, gy, need_gvec=True)
    for u, t in zip(a, b):
        assert torch.equal(u, t)
    assert torch.equal(tp.tp_gaunt_fwd(g, r, s, x, v, w), tp.tp_gaunt_fwd(g, r, s, x, v, w))
