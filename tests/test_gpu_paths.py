"""GPU parity of plans without a compiled specialisation (the runtime path table): random
subsets and orders of the allowed (l1, l2, l3) paths at lmax 2 and 3, blocks of different
multiplicities (ragged 32-channel slices), repeated paths, output blocks no path reaches and
non-unit path coefficients -- forward, backward and double backward against the float64
oracle, per tensor max|gpu - ref| <= 1e-4 * max|ref|."""
import numpy as np
import pytest
import torch

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


def _irreps(blocks):
    return "+".join(f"{m}x{l}{'e' if p > 0 else 'o'}" for m, l, p in blocks)


def random_spec(seed, lmax, muls, n_keep, shuffle=True, repeat=0):
    """Input blocks (mul, l, parity), SH 0..lmax, output blocks that each path may reach: every
    parity-allowed (l3, p3) once per input multiplicity.  A random subset of the allowed paths,
    optionally shuffled, with `repeat` paths listed twice."""
    rng = np.random.default_rng(seed)
    ins = [(int(muls[k % len(muls)]), l, (-1) ** l if rng.random() < 0.7 else -((-1) ** l))
           for k, l in enumerate(rng.permutation(np.arange(lmax + 1)))]
    outs = sorted({(m, l3, p) for m in {b[0] for b in ins} for l3 in range(lmax + 1) for p in (1, -1)},
                  key=lambda t: (t[1], -t[2], t[0]))
    allowed = []
    for a, (ma, la, pa) in enumerate(ins):
        for b in range(lmax + 1):
            for o, (mo, lo, po) in enumerate(outs):
                if mo == ma and abs(la - b) <= lo <= la + b and po == pa * (-1) ** b:
                    allowed.append((a, b, o))
    keep = sorted(rng.choice(len(allowed), size=min(n_keep, len(allowed)), replace=False))
    paths = [allowed[k] for k in keep]
    if shuffle:
        paths = [paths[k] for k in rng.permutation(len(paths))]
    for k in range(repeat):
        paths.append(paths[k])
    sh = "+".join(f"1x{l}{'e' if l % 2 == 0 else 'o'}" for l in range(lmax + 1))
    return _irreps(ins), sh, _irreps(outs), paths


def random_graph(seed, N, max_deg):
    rng = np.random.default_rng(seed)
    deg = rng.integers(0, max_deg + 1, N)
    rowptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int32)
    E = int(rowptr[-1])
    src = rng.integers(0, N, E).astype(np.int32)
    v = rng.standard_normal((E, 3))
    vec = (v / np.linalg.norm(v, axis=1, keepdims=True) * rng.uniform(1, 5, (E, 1))).astype(np.float32)
    return rowptr, src, vec, rng


def _arrays(plan, N, E, rng):
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    return dict(x=f(N, plan.in_dim), w=f(E, plan.n_edge_weights), gy=f(N, plan.out_dim),
                ggx=f(N, plan.in_dim), ggw=f(E, plan.n_edge_weights), ggvec=f(E, 3))


def _check_all(tp, spec, N=160, max_deg=24, seed=0, coeff=None, tag=""):
    ir_in, ir_sh, ir_out, paths = spec
    plan = tp.Plan(ir_in, ir_sh, ir_out, paths, "uvu", path_coeff=coeff)
    op = OraclePlan(ir_in, ir_sh, ir_out, paths, "uvu", path_coeff=coeff)
    rowptr, src, vec, rng = random_graph(seed, N, max_deg)
    d = _arrays(plan, N, len(src), rng)
    g = {k: dev(v) for k, v in dict(rowptr=rowptr, src=src, vec=vec, **d).items()}
    y = tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"])
    assert_close(y, forward(op, rowptr, src, d["x"], vec, w=d["w"]), f"{tag} y", irreps=ir_out)
    gx, gw, gvec, _ = tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"],
                                     need_gvec=True)
    r = backward(op, rowptr, src, d["x"], vec, d["gy"], w=d["w"])
    assert_close(gx, r["gx"], f"{tag} gx", irreps=ir_in)
    assert_close(gw, r["gw"], f"{tag} gw")
    assert_close(gvec, r["gvec"], f"{tag} gvec")
    h = tp.tp_conv_dbwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"], g["ggx"], g["ggw"],
                        g["ggvec"])
    r2 = double_backward(op, rowptr, src, d["x"], vec, d["gy"], d["ggx"], d["ggw"], d["ggvec"], w=d["w"])
    for k, name in enumerate(("g_gy", "g_x", "g_w", "g_vec")):
        assert_close(h[k], r2[name], f"{tag} {name}")
    return plan


@pytest.mark.parametrize("lmax,muls,n_keep,seed", [(2, (32,), 9, 1), (2, (16, 48), 12, 2), (3, (32,), 20, 3),
                                                   (3, (8, 40), 16, 4), (1, (5,), 5, 5)])
def test_random_path_subsets(tp, lmax, muls, n_keep, seed):
    spec = random_spec(seed, lmax, muls, n_keep)
    _check_all(tp, spec, seed=seed, tag=f"lmax {lmax} muls {muls} seed {seed}")


def test_repeated_paths_and_coefficients(tp):
    spec = random_spec(7, 2, (32,), 8, repeat=2)
    coeff = list(np.random.default_rng(7).uniform(-2, 2, len(spec[3])))
    _check_all(tp, spec, seed=7, coeff=coeff, tag="repeated + coeff")


def test_reordered_config_list_matches_compiled_kernels(tp):
    """The c2 path list in reverse order has no compiled specialisation; its results equal the
    compiled kernels' on the same inputs (weights permuted with the paths), both within the
    oracle tolerance."""
    import synth
    d = synth.make_inputs("c2", 160, with_gy=True)
    spec = d["spec"]
    P, mul = len(spec.paths), 32
    order = list(range(P))[::-1]
    rev = [spec.paths[k] for k in order]
    fast = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths)
    slow = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, rev)
    w = d["w"].reshape(-1, P, mul)
    w_rev = np.ascontiguousarray(w[:, order, :].reshape(len(w), -1))
    g = {k: dev(d[k]) for k in ("rowptr", "src", "x", "vec", "w", "gy")}
    y1 = tp.tp_conv_fwd(fast, g["rowptr"], g["src"], g["x"], g["vec"], g["w"])
    y2 = tp.tp_conv_fwd(slow, g["rowptr"], g["src"], g["x"], g["vec"], dev(w_rev))
    op = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvu")
    ref = forward(op, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"])
    assert_close(y1, ref, "compiled y")
    assert_close(y2, ref, "path table y")
    _, gw2, _, _ = tp.tp_conv_bwd(slow, g["rowptr"], g["src"], g["x"], g["vec"], dev(w_rev), g["gy"])
    _, gw1, _, _ = tp.tp_conv_bwd(fast, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"])
    gw2 = gw2.view(-1, P, mul)[:, np.argsort(order), :].reshape(gw1.shape)
    assert_close(gw2, gw1.double(), "path table gw vs compiled", tol=1e-5)


def test_output_block_without_paths_is_zero(tp):
    ir_in, ir_sh = "16x0e+16x1o", "1x0e+1x1o"
    ir_out = "16x0e+16x1o+16x2e"           # no path reaches 2e
    paths = [(0, 0, 0), (1, 1, 0), (0, 1, 1)]
    plan = _check_all(tp, (ir_in, ir_sh, ir_out, paths), N=50, seed=9, tag="unreached block")
    assert plan.out_dim == 16 + 48 + 80


def test_path_table_deterministic_and_index_check(tp):
    spec = random_spec(11, 2, (24,), 10)
    plan = tp.Plan(*spec, "uvu")
    rowptr, src, vec, rng = random_graph(11, 300, 30)
    d = _arrays(plan, 300, len(src), rng)
    g = {k: dev(v) for k, v in dict(rowptr=rowptr, src=src, vec=vec, **d).items()}
    a = tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"])
    b = tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"])
    assert torch.equal(a, b)
    r1 = tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"], need_gvec=True)
    r2 = tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["w"], g["gy"], need_gvec=True)
    for u, v in zip(r1[:3], r2[:3]):
        assert torch.equal(u, v)
    # a sender outside [0, N) is reported by a check-mode plan, never read
    chk = tp.Plan(*spec, "uvu", flags=tp.TP_FLAG_CHECK_INDICES)
    bad = src.copy()
    bad[3] = 10_000
    ws = torch.zeros(tp.tp_workspace_size(chk, 300, len(src), tp.TP_OP_FWD), dtype=torch.uint8, device="cuda")
    tp.tp_conv_fwd(chk, g["rowptr"], dev(bad), g["x"], g["vec"], g["w"], ws=ws)
    assert tp.tp_get_device_error(chk, ws) == 2


def _check_uvw(tp, spec, N=120, max_deg=16, seed=0, coeff=None, tag=""):
    ir_in, ir_sh, ir_out, paths = spec
    plan = tp.Plan(ir_in, ir_sh, ir_out, paths, "uvw", path_coeff=coeff)
    op = OraclePlan(ir_in, ir_sh, ir_out, paths, "uvw", path_coeff=coeff)
    rowptr, src, vec, rng = random_graph(seed, N, max_deg)
    E = len(src)
    mi, mo = int(ir_in.split("x")[0]), int(ir_out.split("x")[0])
    x = rng.standard_normal((N, plan.in_dim)).astype(np.float32)
    s_ = rng.standard_normal((E, len(paths))).astype(np.float32)
    W = (rng.standard_normal((len(paths), mi, mo)) / np.sqrt(mi)).astype(np.float32)
    gy = rng.standard_normal((N, plan.out_dim)).astype(np.float32)
    g = {k: dev(v) for k, v in dict(rowptr=rowptr, src=src, vec=vec, x=x, s=s_, W=W, gy=gy).items()}
    y = tp.tp_conv_fwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["s"], W=g["W"])
    assert_close(y, forward(op, rowptr, src, x, vec, s=s_, W=W), f"{tag} y", irreps=ir_out)
    gx, gs, gvec, gW = tp.tp_conv_bwd(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["s"], g["gy"], W=g["W"],
                                      need_gvec=True, need_gW=True)
    r = backward(op, rowptr, src, x, vec, gy, s=s_, W=W)
    assert_close(gx, r["gx"], f"{tag} gx", irreps=ir_in)
    assert_close(gs, r["gs"], f"{tag} gs")
    assert_close(gvec, r["gvec"], f"{tag} gvec")
    assert_close(gW.view(r["gW"].shape), r["gW"], f"{tag} gW")


def _uniform(spec, mi, mo):
    ir_in, ir_sh, ir_out, paths = spec
    relabel = lambda irr, m: "+".join(f"{m}x{b.split('x')[1]}" for b in irr.split("+"))
    return relabel(ir_in, mi), ir_sh, relabel(ir_out, mo), paths


@pytest.mark.parametrize("lmax,mi,mo,n_keep,seed", [(2, 16, 24, 8, 21), (3, 8, 40, 14, 22), (1, 5, 7, 4, 23)])
def test_uvw_random_path_subsets(tp, lmax, mi, mo, n_keep, seed):
    spec = _uniform(random_spec(seed, lmax, (8,), n_keep), mi, mo)
    coeff = list(np.random.default_rng(seed).uniform(0.5, 1.5, len(spec[3])))
    _check_uvw(tp, spec, seed=seed, coeff=coeff, tag=f"uvw lmax {lmax} {mi}->{mo}")


def test_uvw_config_list_off_the_tma_pitch(tp):
    """The c4 path list with 30 input channels (not a multiple of 4): the path table."""
    import synth
    c4 = synth.CONFIGS["c4"]
    spec = _uniform((c4.irreps_in, c4.irreps_sh, c4.irreps_out, c4.paths), 30, 20)
    _check_uvw(tp, spec, N=60, seed=24, tag="uvw c4 list 30->20")
