"""Receiver-range sharding (equivariant_tensor_product_b200/shard.py) on the CPU: the row
planning, and the sharded forward and backward with the real exchanges between gloo ranks
(world size 2 and 3), the convolution of every shard computed by the float64 oracle in place
of the CUDA kernels.  Every rank's rows and edges must equal the unsharded oracle's."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _graph(seed=3, N=90, max_deg=14):
    rng = np.random.default_rng(seed)
    deg = rng.integers(0, max_deg + 1, N)
    deg[5] = 40                                   # one long row
    deg[10:14] = 0                                # empty rows
    rowptr = np.concatenate([[0], np.cumsum(deg)])
    E = int(rowptr[-1])
    src = rng.integers(0, N, E)
    src[:30] = 7                                  # a hub sender
    return rowptr, src


def test_row_bounds_balance_edges_and_rows():
    from equivariant_tensor_product_b200.shard import row_bounds
    rowptr, _ = _graph()
    for world in (1, 2, 3, 5, 8):
        b = row_bounds(rowptr, world)
        assert b[0] == 0 and b[-1] == len(rowptr) - 1 and np.all(np.diff(b) >= 0)
        cost = rowptr[b[1:]] + b[1:] - rowptr[b[:-1]] - b[:-1]
        total = rowptr[-1] + len(rowptr) - 1
        assert cost.max() <= total / world + 41 + 1       # off by at most one row (the longest)


def test_shard_plans_are_consistent():
    from equivariant_tensor_product_b200.shard import ShardPlan
    rowptr, src = _graph()
    N = len(rowptr) - 1
    for world in (1, 2, 4):
        plans = [ShardPlan(rowptr, src, world, r) for r in range(world)]
        assert sum(p.n_own for p in plans) == N and sum(p.e1 - p.e0 for p in plans) == rowptr[-1]
        for r, p in enumerate(plans):
            # local edges map back to the global senders
            halo = np.concatenate([p.halo, [-1]])       # a pad entry for the world-size-1 case
            glob = np.where(p.src_local < p.n_own, p.src_local + p.r0, halo[np.maximum(p.src_local - p.n_own, 0)])
            np.testing.assert_array_equal(glob, src[p.e0:p.e1])
            assert p.rowptr_local[-1] == p.e1 - p.e0 and len(p.rowptr_local) == p.n_ext + 1
            assert np.all(np.isin(p.halo, np.arange(p.r0, p.r1), invert=True))
            for q in range(world):        # what q sends r equals what r expects from q
                sent = plans[q].send_idx[plans[q].send_offsets[r]:plans[q].send_offsets[r + 1]] + plans[q].r0
                lo = plans[r].recv_counts[:q].sum()
                np.testing.assert_array_equal(sent, plans[r].halo[lo:lo + plans[r].recv_counts[q]])


class _OracleOps:
    """Row movement with torch CPU indexing and the convolution by the float64 oracle."""

    def gather_rows(self, src, idx):
        return src[idx.long()]

    def add_rows(self, dst, idx, src):
        dst.index_add_(0, idx.long(), src)

    def fwd(self, plan, graph, x, vec, w, W):
        from oracle import forward
        return forward(plan, graph.rowptr.numpy(), graph.src.numpy(), x, vec, w=w)

    def bwd(self, plan, graph, x, vec, w, W, gy, need_gvec, need_gW):
        from oracle import backward
        r = backward(plan, graph.rowptr.numpy(), graph.src.numpy(), x, vec, gy, w=w)
        return r["gx"], r["gw"], r["gvec"], None


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import synth
    from equivariant_tensor_product_b200.shard import ShardedConv
    from oracle import OraclePlan, backward, forward
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = synth.make_inputs("c2", 120, with_gy=True)
        spec = d["spec"]
        op = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, spec.mode)
        sc = ShardedConv(op, d["rowptr"], d["src"], world, rank, "cpu", ops=_OracleOps())
        r0, r1 = sc.row_range()
        e0, e1 = sc.edge_range()
        t = lambda a: torch.as_tensor(np.asarray(a), dtype=torch.float64)
        x_own, vec, w, gy_own = t(d["x"][r0:r1]), t(d["vec"][e0:e1]), t(d["w"][e0:e1]), t(d["gy"][r0:r1])
        y = sc.forward(x_own, vec, w)
        gx, gw, gvec, _ = sc.backward(x_own, vec, w, gy_own, need_gvec=True)
        ref_y = forward(op, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"])
        ref = backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], w=d["w"])
        errs = [float((y - ref_y[r0:r1]).abs().max()) if r1 > r0 else 0.0,
                float((gx - ref["gx"][r0:r1]).abs().max()) if r1 > r0 else 0.0,
                float((gw - ref["gw"][e0:e1]).abs().max()) if e1 > e0 else 0.0,
                float((gvec - ref["gvec"][e0:e1]).abs().max()) if e1 > e0 else 0.0]
        q.put((rank, errs, sc.sp.n_halo, float(ref["gx"].abs().max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_forward_backward_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + world * 10 + os.getpid() % 500
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert sum(r[2] for r in res) > 0                         # the shards did exchange halo rows
    for rank, errs, n_halo, scale in res:
        assert max(errs) <= 1e-10 * max(scale, 1.0), (rank, errs)
