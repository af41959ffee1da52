"""Seeded synthetic inputs for the edge-conditioned tensor-product convolution.

This module is shared by the float64 oracle (test side) and the CUDA path
(product side).  It holds no tensor-product arithmetic: it draws atom
positions, builds the receiver-sorted CSR neighbour graph, draws node features
and upstream gradients, and evaluates a small radial MLP (Bessel basis ->
linear/SiLU layers) that produces the per-edge radial weights, exactly as an
interatomic-potential model would hand them to the convolution.

Workloads follow the graph shapes the source pages describe:
  * "Accelerating Tensor Products in E(3)-Equivariant GNNs" (abstract): a
    1,536-atom molecular graph with 46,080 directed edges;
  * "The GPU Workload That Rewrites Molecular Physics" (section "Variable-degree
    graphs"): degree spread between ~5 and ~30 neighbours, here widened to 3-120;
  * "Sobek: Streaming Equivariant TP Convolutions" (abstract): large graphs
    where edge-sized intermediates must not exist (100,000 atoms, ~3M edges).

Draw order per config (numpy ``default_rng(1000 + k)``):
positions -> edges -> vec -> x -> radial-MLP weights -> W (uvw only) -> gy ->
ggx, ggw, ggvec.  Later draws never change earlier ones, so a caller may stop
after any stage.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Tuple

import numpy as np

__all__ = ["CONFIGS", "ConfigSpec", "make_inputs", "irreps_dim", "n_edge_weights",
           "csr_from_edges", "L3_PATHS", "L2_PATHS"]

# ---------------------------------------------------------------------------
# Config data.  Path lists are (i_in, i_sh, i_out) index triples into the
# irreps lists, written out literally in (l1, l2, l3) lexicographic order.
# ---------------------------------------------------------------------------

# (l1, l2, l3) for lmax 2 inputs / SH / outputs; the output irreps list is
# 0e, 1e, 1o, 2e, 2o (ordered by l, then e before o).
L2_TRIPLES = [(0, 0, 0), (0, 1, 1), (0, 2, 2), (1, 0, 1), (1, 1, 0), (1, 1, 1), (1, 1, 2),
              (1, 2, 1), (1, 2, 2), (2, 0, 2), (2, 1, 1), (2, 1, 2), (2, 2, 0), (2, 2, 1),
              (2, 2, 2)]
# output index for (l3, parity) in the list 0e,1e,1o,2e,2o
_OUT2 = {(0, 1): 0, (1, 1): 1, (1, -1): 2, (2, 1): 3, (2, -1): 4}
L2_PATHS = [(l1, l2, _OUT2[(l3, (-1) ** (l1 + l2))]) for (l1, l2, l3) in L2_TRIPLES]

L3_TRIPLES = [(0, 0, 0), (0, 1, 1), (0, 2, 2), (0, 3, 3),
              (1, 0, 1), (1, 1, 0), (1, 1, 1), (1, 1, 2), (1, 2, 1), (1, 2, 2), (1, 2, 3),
              (1, 3, 2), (1, 3, 3),
              (2, 0, 2), (2, 1, 1), (2, 1, 2), (2, 1, 3), (2, 2, 0), (2, 2, 1), (2, 2, 2),
              (2, 2, 3), (2, 3, 1), (2, 3, 2), (2, 3, 3),
              (3, 0, 3), (3, 1, 2), (3, 1, 3), (3, 2, 1), (3, 2, 2), (3, 2, 3), (3, 3, 0),
              (3, 3, 1), (3, 3, 2), (3, 3, 3)]
# output list 0e,1e,1o,2e,2o,3e,3o
_OUT3 = {(0, 1): 0, (1, 1): 1, (1, -1): 2, (2, 1): 3, (2, -1): 4, (3, 1): 5, (3, -1): 6}
L3_PATHS = [(l1, l2, _OUT3[(l3, (-1) ** (l1 + l2))]) for (l1, l2, l3) in L3_TRIPLES]

C1_PATHS = [(0, 0, 0), (0, 1, 1), (1, 0, 1), (1, 1, 0)]


@dataclasses.dataclass(frozen=True)
class ConfigSpec:
    name: str
    irreps_in: str
    irreps_sh: str
    irreps_out: str
    paths: Tuple[Tuple[int, int, int], ...]
    mode: str                    # "uvu" or "uvw"
    n_atoms: int
    graph: str                   # graph recipe name
    box: float                   # periodic box edge (Angstrom); 0 for "c1"
    cutoff: float
    mlp_hidden: Tuple[int, ...]
    passes: Tuple[str, ...]
    seed: int
    description: str = ""


def _mk(name, k, irreps_in, irreps_sh, irreps_out, paths, mode, n_atoms, graph, box, cutoff,
        hidden, passes, desc):
    return ConfigSpec(name, irreps_in, irreps_sh, irreps_out, tuple(map(tuple, paths)), mode,
                      n_atoms, graph, box, cutoff, tuple(hidden), tuple(passes), 1000 + k, desc)


CONFIGS: Dict[str, ConfigSpec] = {
    "c1": _mk("c1", 1, "4x0e+4x1o", "1x0e+1x1o", "4x0e+4x1o", C1_PATHS, "uvu", 24, "fixed8",
              0.0, 5.0, (16,), ("fwd",),
              "tiny correctness graph: 24 nodes x 8 incoming edges, lmax 1"),
    "c2": _mk("c2", 2, "32x0e+32x1o+32x2e", "1x0e+1x1o+1x2e", "32x0e+32x1e+32x1o+32x2e+32x2o",
              L2_PATHS, "uvu", 1536, "exact46080", 29.929, 5.0, (64, 64), ("fwd", "bwd"),
              "NequIP-like: 1,536 atoms, exactly 46,080 directed edges, lmax 2, uvu"),
    "c3": _mk("c3", 3, "64x0e+64x1o+64x2e+64x3o", "1x0e+1x1o+1x2e+1x3o",
              "64x0e+64x1e+64x1o+64x2e+64x2o+64x3e+64x3o", L3_PATHS, "uvu", 4096, "uniform",
              37.708, 5.0, (64, 64), ("fwd", "bwd"),
              "SevenNet/MACE-like l=3: 4,096 atoms, mean degree ~40, uvu path-aggregated"),
    "c4": _mk("c4", 4, "128x0e+128x1o+128x2e", "1x0e+1x1o+1x2e",
              "128x0e+128x1e+128x1o+128x2e+128x2o", L2_PATHS, "uvw", 100000, "uniform",
              120.400, 5.0, (64, 64), ("fwd", "bwd"),
              "large streaming uvw: 100,000 atoms, ~3.0M edges, per-path 128x128 mixing"),
    "c5": _mk("c5", 5, "32x0e+32x1o+32x2e+32x3o", "1x0e+1x1o+1x2e+1x3o",
              "32x0e+32x1e+32x1o+32x2e+32x2o+32x3e+32x3o", L3_PATHS, "uvu", 8192, "clusters",
              80.0, 5.0, (64, 64), ("fwd", "bwd", "dbwd"),
              "skewed degree 3-120: 64 Gaussian clusters + uniform background, double backward"),
}


# ---------------------------------------------------------------------------
# Layout helpers (sizes only)
# ---------------------------------------------------------------------------

def _blocks(irreps: str) -> List[Tuple[int, int]]:
    out = []
    for term in irreps.replace(" ", "").split("+"):
        mul, ir = term.split("x")
        out.append((int(mul), int(ir[:-1])))
    return out


def irreps_dim(irreps: str) -> int:
    return sum(m * (2 * l + 1) for m, l in _blocks(irreps))


def n_edge_weights(spec: ConfigSpec) -> int:
    """Per-edge radial weights: uvu -> sum over paths of mul_in; uvw -> one scalar per path."""
    if spec.mode == "uvw":
        return len(spec.paths)
    bl = _blocks(spec.irreps_in)
    return sum(bl[p[0]][0] for p in spec.paths)


def shared_weight_shape(spec: ConfigSpec):
    bi, bo = _blocks(spec.irreps_in), _blocks(spec.irreps_out)
    p0 = spec.paths[0]
    return (len(spec.paths), bi[p0[0]][0], bo[p0[2]][0])


# ---------------------------------------------------------------------------
# Graphs
# ---------------------------------------------------------------------------

def _min_image(d: np.ndarray, box: float) -> np.ndarray:
    return d - box * np.round(d / box)


def csr_from_edges(dst: np.ndarray, src: np.ndarray, n: int):
    """Sort directed edges by (receiver, sender) and return (rowptr, src, dst, order)."""
    order = np.lexsort((src, dst))
    dst_s, src_s = dst[order], src[order]
    counts = np.bincount(dst_s, minlength=n)
    rowptr = np.zeros(n + 1, dtype=np.int64)
    np.cumsum(counts, out=rowptr[1:])
    return rowptr.astype(np.int32), src_s.astype(np.int32), dst_s.astype(np.int32), order


def _pairs_within(pos: np.ndarray, box: float, r: float):
    from scipy.spatial import cKDTree
    tree = cKDTree(pos, boxsize=box)
    pairs = tree.query_pairs(r, output_type="ndarray")
    d = _min_image(pos[pairs[:, 1]] - pos[pairs[:, 0]], box)
    dist = np.sqrt((d * d).sum(1))
    return pairs, dist


def _graph_fixed8(rng, n):
    """Each receiver gets 8 distinct senders from the other n-1 nodes; vec drawn directly."""
    dst, src = [], []
    for i in range(n):
        others = np.array([j for j in range(n) if j != i])
        pick = rng.choice(others, size=8, replace=False)
        dst.extend([i] * 8)
        src.extend(pick.tolist())
    return np.array(dst), np.array(src)


def _graph_exact(pos, box, n_directed):
    n_pairs = n_directed // 2
    pairs, dist = _pairs_within(pos, box, 5.5)
    if len(dist) <= n_pairs:
        raise RuntimeError("search radius too small for the requested edge count")
    srt = np.sort(dist)
    rc = 0.5 * (srt[n_pairs - 1] + srt[n_pairs])
    keep = dist < rc
    pairs = pairs[keep]
    dst = np.concatenate([pairs[:, 0], pairs[:, 1]])
    src = np.concatenate([pairs[:, 1], pairs[:, 0]])
    return dst, src, rc


def _graph_cutoff(pos, box, rc):
    pairs, _ = _pairs_within(pos, box, rc)
    dst = np.concatenate([pairs[:, 0], pairs[:, 1]])
    src = np.concatenate([pairs[:, 1], pairs[:, 0]])
    return dst, src


def _graph_clamped(pos, box, rc, max_deg=120, min_deg=3):
    """Cutoff graph, each receiver keeps at most its max_deg nearest senders; receivers with
    fewer than min_deg in-cutoff senders take their min_deg nearest regardless of cutoff."""
    from scipy.spatial import cKDTree
    n = len(pos)
    pairs, dist = _pairs_within(pos, box, rc)
    dst = np.concatenate([pairs[:, 0], pairs[:, 1]])
    src = np.concatenate([pairs[:, 1], pairs[:, 0]])
    dd = np.concatenate([dist, dist])
    order = np.lexsort((src, dd, dst))          # by receiver, then distance
    dst, src, dd = dst[order], src[order], dd[order]
    counts = np.bincount(dst, minlength=n)
    start = np.concatenate([[0], np.cumsum(counts)[:-1]])
    rank = np.arange(len(dst)) - start[dst]
    keep = rank < max_deg
    dst, src = dst[keep], src[keep]
    counts = np.bincount(dst, minlength=n)
    low = np.nonzero(counts < min_deg)[0]
    if len(low):
        tree = cKDTree(pos, boxsize=box)
        _, nn = tree.query(pos[low], k=min_deg + 1)
        ex_dst, ex_src = [], []
        for i, row in zip(low, nn):
            row = [j for j in row if j != i][:min_deg]
            have = set(src[dst == i].tolist())
            for j in row:
                if j not in have:
                    ex_dst.append(i)
                    ex_src.append(j)
        dst = np.concatenate([dst, np.array(ex_dst, dtype=dst.dtype)])
        src = np.concatenate([src, np.array(ex_src, dtype=src.dtype)])
    return dst, src


# ---------------------------------------------------------------------------
# Radial MLP (input generation only)
# ---------------------------------------------------------------------------

def _silu(z):
    return z / (1.0 + np.exp(-z))


def _radial_weights(rng, r: np.ndarray, cutoff: float, hidden, n_out: int,
                    chunk: int = 65536) -> np.ndarray:
    """Bessel basis sqrt(2/rc) sin(n pi r/rc)/r (n=1..8) -> bias-free linear layers with
    N(0, 1/fan_in) weights and SiLU between hidden layers -> n_out weights, float64 -> float32."""
    sizes = [8] + list(hidden) + [n_out]
    mats = [rng.normal(0.0, 1.0 / math.sqrt(a), size=(a, b)) for a, b in zip(sizes[:-1], sizes[1:])]
    out = np.empty((len(r), n_out), dtype=np.float32)
    nb = np.arange(1, 9, dtype=np.float64)
    for s in range(0, len(r), chunk):
        rr = r[s:s + chunk].astype(np.float64)[:, None]
        h = math.sqrt(2.0 / cutoff) * np.sin(nb * math.pi * rr / cutoff) / rr
        for k, m in enumerate(mats):
            h = h @ m
            if k < len(mats) - 1:
                h = _silu(h)
        out[s:s + chunk] = h
    return out


def radial_hidden(d: dict, seed: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Inputs of the convolution with the radial projection fused in, for workload ``d``:
    the radial network's last hidden layer h[E, H] (the Bessel basis of |vec| through the
    workload's bias-free hidden layers with SiLU, N(0, 1/fan_in) weights) and its output
    layer W_r[H, nw] (N(0, 1/H)), both float64 -> float32.  Its own seed, so the workload's
    other arrays are unchanged."""
    spec = d["spec"]
    rng = np.random.default_rng(spec.seed + 7919 if seed is None else seed)
    sizes = [8] + list(spec.mlp_hidden)
    mats = [rng.normal(0.0, 1.0 / math.sqrt(a), size=(a, b)) for a, b in zip(sizes[:-1], sizes[1:])]
    H, nw = sizes[-1], n_edge_weights(spec)
    Wr = rng.normal(0.0, 1.0 / math.sqrt(H), size=(H, nw)).astype(np.float32)
    r = np.linalg.norm(np.asarray(d["vec"], dtype=np.float64), axis=1)
    h = np.empty((len(r), H), dtype=np.float32)
    nb = np.arange(1, 9, dtype=np.float64)
    for s in range(0, len(r), 65536):
        rr = np.maximum(r[s:s + 65536], 1e-9)[:, None]
        z = math.sqrt(2.0 / spec.cutoff) * np.sin(nb * math.pi * rr / spec.cutoff) / rr
        for m in mats:
            z = _silu(z @ m)
        h[s:s + 65536] = z
    return h, Wr


# ---------------------------------------------------------------------------
# Public generator
# ---------------------------------------------------------------------------

def make_inputs(name: str, n_atoms: Optional[int] = None, *, with_gy: bool = True,
                with_gg: bool = False, seed: Optional[int] = None) -> dict:
    """Build one workload.

    ``n_atoms`` shrinks the system at constant density (box scaled by the cube root; for
    "clusters" the cluster count scales too) to give a same-shaped replica the float64
    oracle finishes in seconds.  Returns numpy arrays: rowptr[N+1] int32, src[E] int32,
    dst[E] int32, vec[E,3] f32, x[N,in] f32, w[E,nw] f32 (uvu) or s[E,P] f32 + W[P,u,w]
    f32 (uvw), gy[N,out] f32, and optionally ggx, ggw, ggvec.
    """
    spec = CONFIGS[name]
    rng = np.random.default_rng(spec.seed if seed is None else seed)
    n = spec.n_atoms if n_atoms is None else int(n_atoms)
    scale = (n / spec.n_atoms) ** (1.0 / 3.0)
    box = spec.box * scale
    info = {"name": name, "n_atoms": n, "box": box}

    # positions -> edges -> vec
    if spec.graph == "fixed8":
        dst, src = _graph_fixed8(rng, n)
        rowptr, src, dst, _ = csr_from_edges(dst, src, n)
        u = rng.standard_normal((len(src), 3))
        u /= np.linalg.norm(u, axis=1, keepdims=True)
        length = rng.uniform(1.0, 5.0, size=(len(src), 1))
        vec = (u * length).astype(np.float32)
        r = np.linalg.norm(vec.astype(np.float64), axis=1)
    else:
        if spec.graph == "clusters":
            n_cl = max(1, round(64 * n / spec.n_atoms))
            n_bg = n - 64 * n_cl
            centres = rng.uniform(0.0, box, size=(n_cl, 3))
            offs = rng.normal(0.0, 1.5, size=(n_cl, 64, 3))
            bg = rng.uniform(0.0, box, size=(n_bg, 3))
            pos = np.concatenate([(centres[:, None, :] + offs).reshape(-1, 3), bg]) % box
        else:
            pos = rng.uniform(0.0, box, size=(n, 3))
        if spec.graph == "exact46080":
            n_dir = int(round(46080 * n / spec.n_atoms))
            n_dir -= n_dir % 2
            dst, src, rc = _graph_exact(pos, box, n_dir)
            info["cutoff"] = rc
        elif spec.graph == "clusters":
            dst, src = _graph_clamped(pos, box, spec.cutoff)
        else:
            dst, src = _graph_cutoff(pos, box, spec.cutoff)
        rowptr, src, dst, _ = csr_from_edges(dst, src, n)
        d = _min_image(pos[src] - pos[dst], box)          # points receiver -> sender
        vec = d.astype(np.float32)
        r = np.linalg.norm(d, axis=1)
        info["pos"] = pos

    in_dim, out_dim = irreps_dim(spec.irreps_in), irreps_dim(spec.irreps_out)
    x = rng.standard_normal((n, in_dim), dtype=np.float32)
    nw = n_edge_weights(spec)
    w = _radial_weights(rng, r, spec.cutoff, spec.mlp_hidden, nw)
    out = dict(rowptr=rowptr, src=src, dst=dst, vec=vec, x=x, info=info, spec=spec)
    if spec.mode == "uvw":
        P, U, V = shared_weight_shape(spec)
        out["s"] = w
        out["W"] = (rng.standard_normal((P, U, V)) / math.sqrt(U)).astype(np.float32)
    else:
        out["w"] = w
    if with_gy or with_gg:
        out["gy"] = rng.standard_normal((n, out_dim), dtype=np.float32)
    if with_gg:
        E = len(src)
        out["ggx"] = rng.standard_normal((n, in_dim), dtype=np.float32)
        out["ggw"] = rng.standard_normal((E, nw), dtype=np.float32)
        out["ggvec"] = rng.standard_normal((E, 3), dtype=np.float32)
    return out


def cell_sorted(d: dict, cell: float = 5.0) -> dict:
    """The same workload with atoms relabelled in spatial-cell order (cells of ``cell`` Å,
    lexicographic in (z, y, x) cell index, stable), so that the senders of consecutive
    receivers sit close together in memory.  Every per-node and per-edge value is carried
    over unchanged; only the labels, and with them the CSR order of the edges, change."""
    pos = d["info"].get("pos")
    if pos is None:
        raise ValueError("cell order needs generated positions")
    box = d["info"]["box"]
    nc = max(1, int(box // cell))
    c = np.minimum((pos / box * nc).astype(np.int64), nc - 1)
    key = (c[:, 2] * nc + c[:, 1]) * nc + c[:, 0]
    perm = np.argsort(key, kind="stable")              # new label k -> old atom perm[k]
    inv = np.empty_like(perm)
    inv[perm] = np.arange(len(perm))
    n = len(perm)
    dst = inv[d["dst"]]
    src = inv[d["src"]]
    order = np.lexsort((src, dst))                       # receiver-major, then sender
    counts = np.bincount(dst, minlength=n)
    out = dict(d)
    out["rowptr"] = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    out["src"] = src[order].astype(np.int32)
    out["dst"] = dst[order].astype(np.int32)
    for k in ("vec", "w", "s", "ggw", "ggvec"):
        if k in d:
            out[k] = np.ascontiguousarray(d[k][order])
    for k in ("x", "gy", "ggx"):
        if k in d:
            out[k] = np.ascontiguousarray(d[k][perm])
    info = dict(d["info"])
    info["order"] = "cell-sorted"
    info["pos"] = pos[perm]
    out["info"] = info
    return out
