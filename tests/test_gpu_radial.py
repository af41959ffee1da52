"""GPU parity of the convolution with the radial projection fused in (tp_conv_fwd_radial /
tp_conv_bwd_radial): the weights are formed in the kernels as h @ W_r from the radial
network's last hidden layer.  Compared with the float64 oracle (oracle.radial) per tensor,
max|gpu - ref| <= 1e-4 * max|ref|: the c2 workload at full size (forward on sampled rows, gW_r
complete, gx/gh/gvec on sampled senders), a c2 replica and an lmax-3 64-channel replica
completely (weight rows too wide for more than a few edges per on-chip chunk), path-table
plans with mixed multiplicities and path coefficients, hidden widths 4 and 64, hub rows longer
than a chunk, rows without edges and a graph without edges."""
import numpy as np
import pytest
import torch

import synth
from gpu_util import assert_close, dev, edges_from, edges_into, sample_rows
from oracle import OraclePlan
from oracle.radial import backward_radial, forward_radial
from test_gpu_paths import random_graph, random_spec

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_tensor_product_b200 import build
    build.build()
    import equivariant_tensor_product_b200 as tp
    return tp


def _run(tp, plan, g, need_gvec=True):
    y = tp.tp_conv_fwd_radial(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["h"], g["Wr"])
    gx, gh, gWr, gvec = tp.tp_conv_bwd_radial(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["h"], g["Wr"],
                                              g["gy"], need_gvec=need_gvec)
    torch.cuda.synchronize()
    return y, gx, gh, gWr, gvec


def _check_complete(tp, ir_in, ir_sh, ir_out, paths, rowptr, src, vec, x, h, Wr, gy, tag, coeff=None):
    plan = tp.Plan(ir_in, ir_sh, ir_out, paths, "uvu", path_coeff=coeff)
    op = OraclePlan(ir_in, ir_sh, ir_out, paths, "uvu", path_coeff=coeff)
    g = {k: dev(v) for k, v in dict(rowptr=rowptr, src=src, vec=vec, x=x, h=h, Wr=Wr, gy=gy).items()}
    y, gx, gh, gWr, gvec = _run(tp, plan, g)
    assert_close(y, forward_radial(op, rowptr, src, x, vec, h, Wr), f"{tag} y", irreps=ir_out)
    r = backward_radial(op, rowptr, src, x, vec, h, Wr, gy)
    assert_close(gx, r["gx"], f"{tag} gx", irreps=ir_in)
    assert_close(gh, r["gh"], f"{tag} gh")
    assert_close(gWr, r["gWr"], f"{tag} gWr")
    assert_close(gvec, r["gvec"], f"{tag} gvec")


@pytest.mark.parametrize("name,n_atoms", [("c2", 256), ("c3", 160)])
def test_replicas_complete(tp, name, n_atoms):
    d = synth.make_inputs(name, n_atoms, with_gy=True)
    h, Wr = synth.radial_hidden(d)
    s = d["spec"]
    _check_complete(tp, s.irreps_in, s.irreps_sh, s.irreps_out, s.paths, d["rowptr"], d["src"], d["vec"], d["x"],
                    h, Wr, d["gy"], f"{name} replica")


@pytest.mark.parametrize("lmax,muls,n_keep,seed,H", [(2, (16, 48), 10, 2, 64), (3, (8, 40), 14, 4, 4),
                                                      (1, (5,), 5, 5, 12)])
def test_path_table_plans(tp, lmax, muls, n_keep, seed, H):
    ir_in, ir_sh, ir_out, paths = random_spec(seed, lmax, muls, n_keep)
    rowptr, src, vec, rng = random_graph(seed, 120, 40)       # hub rows longer than a 32-edge chunk
    op = OraclePlan(ir_in, ir_sh, ir_out, paths, "uvu")
    coeff = list(rng.uniform(-2, 2, len(paths)))
    f = lambda *shape: rng.standard_normal(shape).astype(np.float32)
    _check_complete(tp, ir_in, ir_sh, ir_out, paths, rowptr, src, vec, f(120, op.irr_in.dim), f(len(src), H),
                    (f(H, op.n_weights) / np.sqrt(H)).astype(np.float32), f(120, op.irr_out.dim),
                    f"lmax {lmax} muls {muls} H {H}", coeff=coeff)


def test_c2_full_size(tp):
    """The c2 workload (1,536 atoms, 46,080 edges) at full size: y on sampled receivers, gx and
    gh / gvec on sampled senders and their edges, gW_r (a sum over every edge) completely."""
    d = synth.make_inputs("c2", with_gy=True)
    h, Wr = synth.radial_hidden(d)
    s = d["spec"]
    plan = tp.Plan(s.irreps_in, s.irreps_sh, s.irreps_out, s.paths)
    op = OraclePlan(s.irreps_in, s.irreps_sh, s.irreps_out, s.paths, "uvu")
    g = {k: dev(v) for k, v in dict(rowptr=d["rowptr"], src=d["src"], vec=d["vec"], x=d["x"], h=h, Wr=Wr,
                                    gy=d["gy"]).items()}
    y, gx, gh, gWr, gvec = _run(tp, plan, g)
    rows = sample_rows(d["rowptr"], k=64, seed=1)
    eids, rp = edges_into(d["rowptr"], rows)
    ref = forward_radial(op, rp, d["src"][eids], d["x"], d["vec"][eids], h[eids], Wr)
    assert_close(y[torch.as_tensor(rows).cuda()], ref, "c2 y (sampled rows)", irreps=s.irreps_out)
    N = len(d["rowptr"]) - 1
    colptr = np.concatenate([[0], np.cumsum(np.bincount(d["src"], minlength=N))])
    senders = sample_rows(colptr, k=48, seed=2)
    eids, rp = edges_from(d["src"], senders, d["dst"], N)
    r = backward_radial(op, rp, d["src"][eids], d["x"], d["vec"][eids], h[eids], Wr, d["gy"])
    assert_close(gx[torch.as_tensor(senders).cuda()], r["gx"][torch.as_tensor(senders)], "c2 gx (sampled senders)")
    assert_close(gh[torch.as_tensor(eids).cuda()], r["gh"], "c2 gh (edges of the sampled senders)")
    assert_close(gvec[torch.as_tensor(eids).cuda()], r["gvec"], "c2 gvec (edges of the sampled senders)")
    full = backward_radial(op, d["rowptr"], d["src"], d["x"], d["vec"], h, Wr, d["gy"])
    assert_close(gWr, full["gWr"], "c2 gWr (complete)")


def test_no_edges_and_empty_rows(tp):
    ir_in, ir_sh, ir_out = "8x0e+8x1o", "1x0e+1x1o", "8x0e+8x1o+8x1e"
    paths = [(0, 0, 0), (0, 1, 1), (1, 0, 1), (1, 1, 2), (1, 1, 0)]
    plan = tp.Plan(ir_in, ir_sh, ir_out, paths)
    rng = np.random.default_rng(11)
    N, H = 9, 8
    x = dev(rng.standard_normal((N, plan.in_dim)).astype(np.float32))
    gy = dev(rng.standard_normal((N, plan.out_dim)).astype(np.float32))
    Wr = dev(rng.standard_normal((H, plan.n_edge_weights)).astype(np.float32))
    rowptr = dev(np.zeros(N + 1, np.int32))
    src = torch.zeros(0, dtype=torch.int32, device="cuda")
    vec = torch.zeros(0, 3, dtype=torch.float32, device="cuda")
    h = torch.zeros(0, H, dtype=torch.float32, device="cuda")
    y = tp.tp_conv_fwd_radial(plan, rowptr, src, x, vec, h, Wr)
    gx, gh, gWr, gvec = tp.tp_conv_bwd_radial(plan, rowptr, src, x, vec, h, Wr, gy, need_gvec=True)
    torch.cuda.synchronize()
    assert float(y.abs().max()) == 0 and float(gx.abs().max()) == 0 and float(gWr.abs().max()) == 0
    assert gh.shape == (0, H) and gvec.shape == (0, 3)
    # rows without edges between rows with edges
    rowptr_np = np.array([0, 0, 3, 3, 3, 7, 7, 8, 8, 8], np.int32)
    src_np = rng.integers(0, N, 8).astype(np.int32)
    vec_np = rng.standard_normal((8, 3)).astype(np.float32)
    h_np = rng.standard_normal((8, H)).astype(np.float32)
    _check_complete(tp, ir_in, ir_sh, ir_out, paths, rowptr_np, src_np, vec_np, x.cpu().numpy(), h_np,
                    Wr.cpu().numpy(), gy.cpu().numpy(), "empty rows")


def test_autograd_first_derivatives(tp):
    """tp_conv_radial through torch autograd: gradients to x, vec, h and W_r against the oracle."""
    from equivariant_tensor_product_b200.autograd import Graph, tp_conv_radial
    d = synth.make_inputs("c2", 128, with_gy=True)
    h, Wr = synth.radial_hidden(d)
    s = d["spec"]
    plan = tp.Plan(s.irreps_in, s.irreps_sh, s.irreps_out, s.paths)
    op = OraclePlan(s.irreps_in, s.irreps_sh, s.irreps_out, s.paths, "uvu")
    graph = Graph(dev(d["rowptr"]), dev(d["src"]))
    leaves = [dev(a).requires_grad_(True) for a in (d["x"], d["vec"], h, Wr)]
    y = tp_conv_radial(plan, graph, *leaves)
    (y * dev(d["gy"])).sum().backward()
    r = backward_radial(op, d["rowptr"], d["src"], d["x"], d["vec"], h, Wr, d["gy"])
    assert_close(y, forward_radial(op, d["rowptr"], d["src"], d["x"], d["vec"], h, Wr), "autograd y")
    for t, name in zip(leaves, ("gx", "gvec", "gh", "gWr")):
        assert_close(t.grad, r[name], f"autograd {name}")


def test_index_check_reports_bad_sender(tp):
    d = synth.make_inputs("c1", with_gy=True)
    h, Wr = synth.radial_hidden(d)
    s = d["spec"]
    plan = tp.Plan(s.irreps_in, s.irreps_sh, s.irreps_out, s.paths, flags=tp.TP_FLAG_CHECK_INDICES)
    g = {k: dev(v) for k, v in dict(rowptr=d["rowptr"], src=d["src"], vec=d["vec"], x=d["x"], h=h, Wr=Wr,
                                    gy=d["gy"]).items()}
    bad = g["src"].clone()
    bad[5] = 10_000
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    y = tp.tp_conv_fwd_radial(plan, g["rowptr"], bad, g["x"], g["vec"], g["h"], g["Wr"], ws=ws)
    assert tp.tp_get_device_error(plan, ws) == 2
    assert torch.isfinite(y).all()
    tp.tp_conv_fwd_radial(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["h"], g["Wr"], ws=ws)
    assert tp.tp_get_device_error(plan, ws) == 0
    N, E, H = len(d["rowptr"]) - 1, len(d["src"]), h.shape[1]
    wsb = torch.zeros(tp.tp_radial_workspace_size(plan, N, E, H, tp.TP_OP_BWD), dtype=torch.uint8, device="cuda")
    tp.tp_conv_bwd_radial(plan, g["rowptr"], bad, g["x"], g["vec"], g["h"], g["Wr"], g["gy"], ws=wsb)
    assert tp.tp_get_device_error(plan, wsb) == 2
    torch.cuda.synchronize()


@pytest.mark.parametrize("lmax,mul", [(2, 64), (2, 128), (3, 32), (3, 48)])
def test_compiled_lists_at_other_channel_counts(tp, lmax, mul):
    """All paths of lmax 2 or 3 at other multiplicities: wider weight rows change the chunk size
    (and with it the kernel: the compiled-list instances or the path-table ones), ragged slices."""
    ls = range(lmax + 1)
    ir_in = "+".join(f"{mul}x{l}{'e' if l % 2 == 0 else 'o'}" for l in ls)
    ir_sh = "+".join(f"1x{l}{'e' if l % 2 == 0 else 'o'}" for l in ls)
    spec = synth.CONFIGS["c2" if lmax == 2 else "c3"]
    ir_out = "+".join(f"{mul}x{b.split('x')[1]}" for b in spec.irreps_out.split("+"))
    paths = synth.L2_PATHS if lmax == 2 else synth.L3_PATHS
    rowptr, src, vec, rng = random_graph(20 + mul, 40, 12)
    op = OraclePlan(ir_in, ir_sh, ir_out, paths, "uvu")
    f = lambda *shape: rng.standard_normal(shape).astype(np.float32)
    _check_complete(tp, ir_in, ir_sh, ir_out, paths, rowptr, src, vec, f(40, op.irr_in.dim), f(len(src), 64),
                    (f(64, op.n_weights) / 8).astype(np.float32), f(40, op.irr_out.dim), f"lmax {lmax} mul {mul}")


def test_calls_allocate_no_device_memory(tp):
    """With caller-supplied outputs and workspace, the fused-radial calls allocate nothing: no
    torch allocation and no change of the device's free memory; the backward workspace holds
    W_r-sized regions beyond the transpose's, nothing edge x feature sized."""
    d = synth.make_inputs("c2", 512, with_gy=True)
    h, Wr = synth.radial_hidden(d)
    s = d["spec"]
    plan = tp.Plan(s.irreps_in, s.irreps_sh, s.irreps_out, s.paths)
    g = {k: dev(v) for k, v in dict(rowptr=d["rowptr"], src=d["src"], vec=d["vec"], x=d["x"], h=h, Wr=Wr,
                                    gy=d["gy"]).items()}
    N, E, H = len(d["rowptr"]) - 1, len(d["src"]), h.shape[1]
    ws = torch.empty(tp.tp_radial_workspace_size(plan, N, E, H, tp.TP_OP_BWD), dtype=torch.uint8, device="cuda")
    y = torch.empty(N, plan.out_dim, device="cuda")
    gx = torch.empty(N, plan.in_dim, device="cuda")
    gh = torch.empty(E, H, device="cuda")
    gWr = torch.empty(H, plan.n_edge_weights, device="cuda")
    gvec = torch.empty(E, 3, device="cuda")
    colptr, perm = tp.tp_csr_transpose(g["rowptr"], g["src"], N)
    # first calls outside the measurement (kernel attributes, module load)
    tp.tp_conv_fwd_radial(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["h"], g["Wr"], y=y, ws=ws)
    tp.tp_conv_bwd_radial(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["h"], g["Wr"], g["gy"], colptr=colptr,
                          perm=perm, need_gvec=True, gx=gx, gh=gh, gWr=gWr, gvec=gvec, ws=ws)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    before = torch.cuda.memory_allocated()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        tp.tp_conv_fwd_radial(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["h"], g["Wr"], y=y, ws=ws)
        tp.tp_conv_bwd_radial(plan, g["rowptr"], g["src"], g["x"], g["vec"], g["h"], g["Wr"], g["gy"],
                              colptr=colptr, perm=perm, need_gvec=True, gx=gx, gh=gh, gWr=gWr, gvec=gvec, ws=ws)
    torch.cuda.synchronize()
    assert torch.cuda.max_memory_allocated() == before
    assert torch.cuda.mem_get_info()[0] == free0
    base = tp.tp_workspace_size(plan, N, E, tp.TP_OP_BWD)
    assert ws.numel() - base <= 4 * H * plan.n_edge_weights * 257 + 512
