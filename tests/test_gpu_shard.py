"""Receiver-range sharding with the CUDA kernels on one GPU: every rank of a world of 2 or 3
runs in its own host thread with its own shard (owned rows, their edges, the halo), and the
collectives are emulated by an in-process exchange between the threads (a host barrier, then
copies; no kernel waits on another).  The sharded forward and backward must match the float64
oracle on the whole graph, rank by rank, within 1e-4 * max|ref| (uvu and uvw)."""
import threading

import numpy as np
import pytest
import torch

from gpu_util import assert_close, inputs, plans
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


class ThreadExchange:
    """all_to_all / all_reduce between host threads of one process (one per emulated rank)."""

    def __init__(self, world):
        self.world = world
        self.box = [[None] * world for _ in range(world)]
        self.red = [None] * world
        self.bar = threading.Barrier(world, timeout=120)

    def for_rank(self, rank):
        ex = self

        class _View:
            def all_to_all(self, out, inp, out_rows, in_rows):
                torch.cuda.synchronize()
                off = np.concatenate([[0], np.cumsum(in_rows)])
                for q in range(ex.world):
                    ex.box[rank][q] = inp[off[q]:off[q + 1]].clone()
                torch.cuda.synchronize()
                ex.bar.wait()
                oo = np.concatenate([[0], np.cumsum(out_rows)])
                for q in range(ex.world):
                    out[oo[q]:oo[q + 1]].copy_(ex.box[q][rank])
                torch.cuda.synchronize()
                ex.bar.wait()

            def all_reduce(self, t):
                torch.cuda.synchronize()
                ex.red[rank] = t.clone()
                ex.bar.wait()
                acc = ex.red[0].clone()
                for q in range(1, ex.world):
                    acc += ex.red[q]
                t.copy_(acc)
                torch.cuda.synchronize()
                ex.bar.wait()

        return _View()


def _run(tp, d, world, uvw):
    from equivariant_tensor_product_b200.shard import ShardedConv
    spec = d["spec"]
    plan, _ = plans(spec, tp)
    ex = ThreadExchange(world)
    wkey = "s" if uvw else "w"
    out, errors = [None] * world, []

    def rank_main(r):
        try:
            torch.cuda.set_device(0)
            sc = ShardedConv(plan, d["rowptr"], d["src"], world, r, torch.device("cuda"), exchange=ex.for_rank(r))
            r0, r1 = sc.row_range()
            e0, e1 = sc.edge_range()
            cu = lambda a: torch.as_tensor(np.ascontiguousarray(a)).cuda()
            x, vec, w, gy = cu(d["x"][r0:r1]), cu(d["vec"][e0:e1]), cu(d[wkey][e0:e1]), cu(d["gy"][r0:r1])
            W = cu(d["W"]) if uvw else None
            y = sc.forward(x, vec, w, W=W)
            gx, gw, gvec, gW = sc.backward(x, vec, w, gy, W=W, need_gvec=True, need_gW=uvw)
            torch.cuda.synchronize()
            out[r] = dict(r=(r0, r1), e=(e0, e1), y=y.cpu(), gx=gx.cpu(), gw=gw.cpu(), gvec=gvec.cpu(),
                          gW=None if gW is None else gW.cpu(), halo=sc.sp.n_halo)
        except Exception as exc:  # noqa: BLE001
            errors.append(exc)
            ex.bar.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(300)
    if errors:
        raise errors[0]
    return out


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_uvu_matches_oracle(tp, world):
    d = inputs("c2", 400)
    _, op = plans(d["spec"], tp)
    out = _run(tp, d, world, False)
    assert sum(o["halo"] for o in out) > 0
    ref_y = forward(op, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"])
    ref = backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], w=d["w"])
    y = torch.cat([o["y"] for o in out])
    gx = torch.cat([o["gx"] for o in out])
    gw = torch.cat([o["gw"] for o in out])
    gvec = torch.cat([o["gvec"] for o in out])
    assert_close(y, ref_y, f"sharded y (world {world})")
    assert_close(gx, ref["gx"], f"sharded gx (world {world})")
    assert_close(gw, ref["gw"], f"sharded gw (world {world})")
    assert_close(gvec, ref["gvec"], f"sharded gvec (world {world})")


def test_sharded_uvw_matches_oracle(tp):
    d = inputs("c4", 240)
    _, op = plans(d["spec"], tp)
    out = _run(tp, d, 2, True)
    ref_y = forward(op, d["rowptr"], d["src"], d["x"], d["vec"], s=d["s"], W=d["W"])
    ref = backward(op, d["rowptr"], d["src"], d["x"], d["vec"], d["gy"], s=d["s"], W=d["W"])
    assert_close(torch.cat([o["y"] for o in out]), ref_y, "sharded uvw y")
    assert_close(torch.cat([o["gx"] for o in out]), ref["gx"], "sharded uvw gx")
    assert_close(torch.cat([o["gw"] for o in out]), ref["gs"], "sharded uvw gs")
    for o in out:                                     # every rank holds the summed gW
        assert_close(o["gW"].view(ref["gW"].shape), ref["gW"], "sharded uvw gW")
