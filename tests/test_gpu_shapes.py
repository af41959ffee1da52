"""GPU parity on shapes the workload configurations do not reach: other channel counts (the
general kernels; ragged 32-channel slices; uvw GEMM tiles narrower than 128), rows whose
degree spans several 32-edge batches of every warp (the staged-row rings refill across
batches), and rows that start off a 16-byte boundary (the staged kernels must step aside).
Per tensor max|gpu - ref| <= 1e-4 * max|ref| against the float64 oracle."""
import numpy as np
import pytest
import torch

import synth
from gpu_util import assert_close, dev
from oracle import OraclePlan, backward, double_backward, forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_tensor_product_b200 import build
    build.build()
    import equivariant_tensor_product_b200 as tp
    return tp


def _irreps(template: str, mul: int) -> str:
    return "+".join(f"{mul}x{b.split('x')[1]}" for b in template.split("+"))


def _graph(rng, N, degrees):
    """CSR with the given receiver degrees (padded with zero-degree rows) and random senders."""
    deg = np.zeros(N, np.int64)
    deg[: len(degrees)] = degrees
    rng.shuffle(deg)
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int32)
    E = int(rowptr[-1])
    src = rng.integers(0, N, E).astype(np.int32)
    vec = (rng.standard_normal((E, 3)) * rng.uniform(1.0, 5.0, (E, 1))).astype(np.float32)
    return rowptr, src, vec


# degrees around the batch sizes: one warp takes 32 edges per batch, four warps split a row
DEGREES = [0, 1, 2, 3, 31, 32, 33, 64, 127, 128, 129, 200, 300]


@pytest.mark.parametrize("mul", [32, 16, 48])
def test_uvu_channel_counts_and_long_rows(tp, mul):
    spec = synth.CONFIGS["c2"]
    ins, outs = _irreps(spec.irreps_in, mul), _irreps(spec.irreps_out, mul)
    plan = tp.Plan(ins, spec.irreps_sh, outs, spec.paths, "uvu")
    op = OraclePlan(ins, spec.irreps_sh, outs, spec.paths, "uvu")
    rng = np.random.default_rng(100 + mul)
    N = 64
    rowptr, src, vec = _graph(rng, N, DEGREES)
    E = len(src)
    x = rng.standard_normal((N, plan.in_dim)).astype(np.float32)
    w = rng.standard_normal((E, plan.n_edge_weights)).astype(np.float32)
    gy = rng.standard_normal((N, plan.out_dim)).astype(np.float32)
    g = dict(rowptr=dev(rowptr), src=dev(src), x=dev(x), vec=dev(vec), w=dev(w), gy=dev(gy))
    y = tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"])
    assert_close(y, forward(op, rowptr, src, x, vec, w=w), f"mul {mul} y")
    for gvec in (False, True):
        gx, gw, gv, _ = tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"],
                                       need_gvec=gvec)
        ref = backward(op, rowptr, src, x, vec, gy, w=w)
        assert_close(gx, ref["gx"], f"mul {mul} gx")
        assert_close(gw, ref["gw"], f"mul {mul} gw")
        if gvec:
            assert_close(gv, ref["gvec"], f"mul {mul} gvec")
    ggx = rng.standard_normal(x.shape).astype(np.float32)
    ggw = rng.standard_normal(w.shape).astype(np.float32)
    ggvec = rng.standard_normal(vec.shape).astype(np.float32)
    out = dict(zip(("g_gy", "g_x", "g_w", "g_vec"),
                   tp.tp_conv_dbwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"], ggx=dev(ggx),
                                   ggw=dev(ggw), ggvec=dev(ggvec))))
    ref = double_backward(op, rowptr, src, x, vec, gy, ggx=ggx, ggw=ggw, ggvec=ggvec, w=w)
    for k in ("g_gy", "g_x", "g_w", "g_vec"):
        assert_close(out[k], ref[k], f"mul {mul} {k}")


# (128, 128): the receiver pass with per-edge coupling matrices, two warps; (64, 32): one warp;
# (96, 64): the second warp's upper 32 channels idle; (32, 96): the general receiver pass
@pytest.mark.parametrize("mul_in,mul_out,cfg", [(128, 128, "c4"), (64, 32, "c4"), (96, 64, "c4"), (32, 96, "c4"),
                                                (64, 64, "c1"), (128, 32, "c1")])
def test_uvw_channel_counts_and_long_rows(tp, mul_in, mul_out, cfg):
    spec = synth.CONFIGS[cfg]
    ins, outs = _irreps(spec.irreps_in, mul_in), _irreps(spec.irreps_out, mul_out)
    plan = tp.Plan(ins, spec.irreps_sh, outs, spec.paths, "uvw")
    op = OraclePlan(ins, spec.irreps_sh, outs, spec.paths, "uvw")
    rng = np.random.default_rng(7 + mul_in + mul_out)
    N = 48
    rowptr, src, vec = _graph(rng, N, DEGREES[:12])
    E = len(src)
    P = len(spec.paths)
    x = rng.standard_normal((N, plan.in_dim)).astype(np.float32)
    s = rng.standard_normal((E, P)).astype(np.float32)
    W = (rng.standard_normal((P, mul_in, mul_out)) / np.sqrt(mul_in)).astype(np.float32)
    gy = rng.standard_normal((N, plan.out_dim)).astype(np.float32)
    g = dict(rowptr=dev(rowptr), src=dev(src), x=dev(x), vec=dev(vec), s=dev(s), W=dev(W), gy=dev(gy))
    y = tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["s"], W=g["W"])
    assert_close(y, forward(op, rowptr, src, x, vec, s=s, W=W), f"uvw {mul_in}/{mul_out} y")
    gx, gs, gvec, gW = tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["s"], g["gy"], W=g["W"],
                                      need_gvec=True, need_gW=True)
    ref = backward(op, rowptr, src, x, vec, gy, s=s, W=W)
    assert_close(gx, ref["gx"], f"uvw {mul_in}/{mul_out} gx")
    assert_close(gs, ref["gs"], f"uvw {mul_in}/{mul_out} gs")
    assert_close(gvec, ref["gvec"], f"uvw {mul_in}/{mul_out} gvec")
    assert_close(gW.view(ref["gW"].shape), ref["gW"], f"uvw {mul_in}/{mul_out} gW")
    # without the direction gradient the sender pass takes its coupling-matrix form
    gx2, gs2, _, gW2 = tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["s"], g["gy"], W=g["W"],
                                      need_gvec=False, need_gW=True)
    assert_close(gx2, ref["gx"], f"uvw {mul_in}/{mul_out} gx (no gvec)")
    assert_close(gs2, ref["gs"], f"uvw {mul_in}/{mul_out} gs (no gvec)")
    assert_close(gW2.view(ref["gW"].shape), ref["gW"], f"uvw {mul_in}/{mul_out} gW (no gvec)")


def test_uvw_path_coefficients(tp):
    """Non-unit path coefficients through the uvw edge passes (the coupling matrices fold c_p
    in with s[e, p] in the receiver pass and into K_e in the sender pass)."""
    spec = synth.CONFIGS["c4"]
    ins, outs = _irreps(spec.irreps_in, 128), _irreps(spec.irreps_out, 64)
    coeff = np.linspace(-1.5, 2.0, len(spec.paths))
    plan = tp.Plan(ins, spec.irreps_sh, outs, spec.paths, "uvw", path_coeff=coeff)
    op = OraclePlan(ins, spec.irreps_sh, outs, spec.paths, "uvw", path_coeff=coeff)
    rng = np.random.default_rng(11)
    N = 40
    rowptr, src, vec = _graph(rng, N, DEGREES[:10])
    E = len(src)
    P = len(spec.paths)
    x = rng.standard_normal((N, plan.in_dim)).astype(np.float32)
    s = rng.standard_normal((E, P)).astype(np.float32)
    W = (rng.standard_normal((P, 128, 64)) / np.sqrt(128)).astype(np.float32)
    gy = rng.standard_normal((N, plan.out_dim)).astype(np.float32)
    g = dict(rowptr=dev(rowptr), src=dev(src), x=dev(x), vec=dev(vec), s=dev(s), W=dev(W), gy=dev(gy))
    y = tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["s"], W=g["W"])
    assert_close(y, forward(op, rowptr, src, x, vec, s=s, W=W), "uvw coeff y")
    ref = backward(op, rowptr, src, x, vec, gy, s=s, W=W)
    for need_gvec in (False, True):
        gx, gs, gvec, gW = tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["s"], g["gy"], W=g["W"],
                                          need_gvec=need_gvec, need_gW=True)
        assert_close(gx, ref["gx"], f"uvw coeff gx ({need_gvec})")
        assert_close(gs, ref["gs"], f"uvw coeff gs ({need_gvec})")
        assert_close(gW.view(ref["gW"].shape), ref["gW"], f"uvw coeff gW ({need_gvec})")
        if need_gvec:
            assert_close(gvec, ref["gvec"], "uvw coeff gvec")


def test_rows_off_16_byte_boundaries_take_the_general_path(tp):
    spec = synth.CONFIGS["c2"]
    d = synth.make_inputs("c2", 192)
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvu")
    op = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvu")

    def shifted(a):   # same values, base address 4 bytes past a 16-byte boundary
        t = torch.as_tensor(np.ascontiguousarray(a))
        buf = torch.empty(t.numel() + 1, dtype=t.dtype, device="cuda")
        v = buf[1:].view(t.shape)
        v.copy_(t.cuda())
        assert v.data_ptr() % 16 == 4
        return v

    rowptr, src = dev(d["rowptr"]), dev(d["src"])
    x, vec, w, gy = shifted(d["x"]), shifted(d["vec"]), shifted(d["w"]), shifted(d["gy"])
    y = tp.tp_conv_fwd(plan, rowptr, src, x, vec, w)
    assert_close(y, forward(op, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"]), "shifted y")
    gx, gw, _, _ = tp.tp_conv_bwd(plan, rowptr, src, x, vec, w, gy)
    ref = backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], w=d["w"])
    assert_close(gx, ref["gx"], "shifted gx")
    assert_close(gw, ref["gw"], "shifted gw")
    # uvw: x and gy off the boundary, so both edge passes and the mixing GEMM's operands
    # take their unstaged forms
    s4 = synth.CONFIGS["c4"]
    d4 = synth.make_inputs("c4", 200)
    p4 = tp.Plan(s4.irreps_in, s4.irreps_sh, s4.irreps_out, s4.paths, "uvw")
    o4 = OraclePlan(s4.irreps_in, s4.irreps_sh, s4.irreps_out, s4.paths, "uvw")
    r4, sr4 = dev(d4["rowptr"]), dev(d4["src"])
    x4, gy4 = shifted(d4["x"]), shifted(d4["gy"])
    y4 = tp.tp_conv_fwd(p4, r4, sr4, x4, dev(d4["vec"]), dev(d4["s"]), W=dev(d4["W"]))
    assert_close(y4, forward(o4, d4["rowptr"], d4["src"], d4["x"], d4["vec"], s=d4["s"], W=d4["W"]), "shifted uvw y")
    gx4, gs4, _, gW4 = tp.tp_conv_bwd(p4, r4, sr4, x4, dev(d4["vec"]), dev(d4["s"]), gy4, W=dev(d4["W"]),
                                      need_gW=True)
    ref4 = backward(o4, d4["rowptr"], d4["src"], d4["x"], d4["vec"], d4["gy"], s=d4["s"], W=d4["W"])
    assert_close(gx4, ref4["gx"], "shifted uvw gx")
    assert_close(gs4, ref4["gs"], "shifted uvw gs")
    assert_close(gW4.view(ref4["gW"].shape), ref4["gW"], "shifted uvw gW")
