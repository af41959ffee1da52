"""Helpers shared by the GPU parity tests: move synthetic inputs to the device, build the
oracle's answers on edge subsets (every output is a sum of per-edge terms, so the exact
value of a sampled row needs only that row's edges), and the per-tensor tolerance
max|gpu - ref| <= 1e-4 * max|ref| stated for fp32 results."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import OraclePlan, backward, double_backward, forward

TOL = 1e-4

# (tensor name, irreps block, max|err| / max|ref| of the tensor, max|err| / max|ref| of the block)
BLOCK_RECORDS = []


def irreps_blocks(irreps):
    """Column ranges of the blocks of an irreps string: [(label, start, stop)]."""
    out, start = [], 0
    for term in irreps.split("+"):
        mul, ir = term.split("x")
        width = int(mul) * (2 * int(ir[:-1]) + 1)
        out.append((term, start, start + width))
        start += width
    return out


def block_error_ratios(g, r, irreps):
    """Per irreps block of the last axis: max|err| over the tensor's max|ref| and over the
    block's own max|ref|."""
    scale = float(r.abs().max()) if r.numel() else 0.0
    rows = []
    for label, a, b in irreps_blocks(irreps):
        err = float((g[..., a:b] - r[..., a:b]).abs().max()) if g.numel() else 0.0
        bscale = float(r[..., a:b].abs().max()) if r.numel() else 0.0
        rows.append((label, err / scale if scale else 0.0, err / bscale if bscale else 0.0))
    return rows


def assert_close(gpu, ref, name, tol=TOL, irreps=None):
    """Per tensor max|gpu - ref| <= tol * max|ref|.  With `irreps` (the layout of the last axis)
    the error of every irreps block is recorded too (reported in the pytest summary)."""
    g = gpu.detach().double().cpu() if isinstance(gpu, torch.Tensor) else torch.as_tensor(gpu, dtype=torch.float64)
    r = ref.detach().double().cpu() if isinstance(ref, torch.Tensor) else torch.as_tensor(ref, dtype=torch.float64)
    assert g.shape == r.shape, (name, g.shape, r.shape)
    assert torch.isfinite(g).all(), f"{name}: non-finite values"
    err = float((g - r).abs().max()) if g.numel() else 0.0
    scale = float(r.abs().max()) if r.numel() else 0.0
    blocks = ""
    if irreps is not None:
        rows = block_error_ratios(g, r, irreps)
        BLOCK_RECORDS.extend((name, lab, a, b) for lab, a, b in rows)
        blocks = "; per block " + ", ".join(f"{lab}: {a:.1e}" for lab, a, _ in rows)
    assert err <= tol * scale or (scale == 0.0 and err == 0.0), \
        f"{name}: max|err| = {err:.3e} > {tol} * max|ref| = {tol * scale:.3e}{blocks}"
    return err / scale if scale else 0.0


def dev(a, dtype=None):
    t = torch.as_tensor(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def plans(spec, tp, flags=0):
    p = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, spec.mode, flags=flags)
    o = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, spec.mode)
    return p, o


def device_inputs(d):
    out = {k: dev(d[k]) for k in ("rowptr", "src", "vec", "x") if k in d}
    for k in ("w", "s", "W", "gy", "ggx", "ggw", "ggvec"):
        if k in d:
            out[k] = dev(d[k])
    return out


def sample_rows(rowptr, k=48, seed=0):
    deg = np.diff(np.asarray(rowptr))
    n = len(deg)
    rng = np.random.default_rng(seed)
    pick = {int(np.argmax(deg)), int(np.argmin(deg)), 0, n - 1}
    pick |= set(rng.choice(n, size=min(k, n), replace=False).tolist())
    return np.array(sorted(pick))


def edges_into(rowptr, rows):
    rowptr = np.asarray(rowptr, dtype=np.int64)
    eids = np.concatenate([np.arange(rowptr[i], rowptr[i + 1]) for i in rows]) if len(rows) else np.zeros(0, int)
    rp = np.concatenate([[0], np.cumsum(rowptr[rows + 1] - rowptr[rows])])
    return eids.astype(np.int64), rp


def edges_from(src, senders, dst, N):
    mask = np.isin(np.asarray(src), senders)
    eids = np.nonzero(mask)[0]                    # receiver order kept (edge ids are receiver sorted)
    rp = np.concatenate([[0], np.cumsum(np.bincount(dst[eids], minlength=N))])
    return eids, rp


def oracle_fwd_rows(oplan, d, rows):
    eids, rp = edges_into(d["rowptr"], rows)
    if oplan.mode == "uvu":
        return forward(oplan, rp, d["src"][eids], d["x"], d["vec"][eids], w=d["w"][eids])
    return forward(oplan, rp, d["src"][eids], d["x"], d["vec"][eids], s=d["s"][eids], W=d["W"])


def oracle_bwd_senders(oplan, d, senders):
    """Exact gx rows of `senders`, and gw/gvec of every edge leaving them (edge ids returned)."""
    N = len(d["rowptr"]) - 1
    eids, rp = edges_from(d["src"], senders, d["dst"], N)
    kw = dict(w=d["w"][eids]) if oplan.mode == "uvu" else dict(s=d["s"][eids], W=d["W"])
    g = backward(oplan, rp, d["src"][eids], d["x"], d["vec"][eids], d["gy"], **kw)
    return g, eids


def oracle_dbwd_rows(oplan, d, rows):
    """Exact g_gy rows of `rows` and g_w / g_vec of their incoming edges."""
    eids, rp = edges_into(d["rowptr"], rows)
    h = double_backward(oplan, rp, d["src"][eids], d["x"], d["vec"][eids], d["gy"][rows],
                        d["ggx"], d["ggw"][eids], d["ggvec"][eids], w=d["w"][eids])
    return h, eids


def oracle_dbwd_senders(oplan, d, senders):
    N = len(d["rowptr"]) - 1
    eids, rp = edges_from(d["src"], senders, d["dst"], N)
    h = double_backward(oplan, rp, d["src"][eids], d["x"], d["vec"][eids], d["gy"],
                        d["ggx"], d["ggw"][eids], d["ggvec"][eids], w=d["w"][eids])
    return h, eids


_CACHE = {}


def inputs(name, n_atoms=None, with_gg=False):
    key = (name, n_atoms, with_gg)
    if key not in _CACHE:
        _CACHE.clear() if len(_CACHE) > 3 else None
        _CACHE[key] = synth.make_inputs(name, n_atoms, with_gy=True, with_gg=with_gg)
    return _CACHE[key]
