"""Pure-Python per-edge loop (no einsum, no autograd) for tiny graphs.

TEST INFRASTRUCTURE ONLY.  Cross-checks the vectorised oracle's indexing: every sum of
the definition in oracle/__init__.py is an explicit loop here, with the CG tensor
indexed as C[m1][m2][m3] (m1 -> sender feature, m2 -> spherical harmonic, m3 -> output).
"""
from __future__ import annotations

import numpy as np

from .irreps import OraclePlan
from .so3 import cg_real, real_sh_np


def forward_loops(plan: OraclePlan, rowptr, src, x, vec, w=None, s=None, W=None):
    rowptr = [int(v) for v in rowptr]
    N = len(rowptr) - 1
    x = np.asarray(x, dtype=np.float64).tolist()
    vec = np.asarray(vec, dtype=np.float64)
    wt = np.asarray(w if plan.mode == "uvu" else s, dtype=np.float64).tolist()
    Wl = np.asarray(W, dtype=np.float64).tolist() if plan.mode == "uvw" else None
    y = [[0.0] * plan.irr_out.dim for _ in range(N)]
    cg = {t: cg_real(*t).tolist() for t in set(plan.triples)}
    for i in range(N):
        for e in range(rowptr[i], rowptr[i + 1]):
            j = int(src[e])
            Ys = [real_sh_np(l, vec[e:e + 1])[0].tolist() for _, l, _ in plan.irr_sh.blocks]
            for p, (a, b, o) in enumerate(plan.paths):
                ma, la, _ = plan.irr_in.blocks[a]
                mo, lo, _ = plan.irr_out.blocks[o]
                lb = plan.irr_sh.blocks[b][1]
                C = cg[(la, lb, lo)]
                d1, d2, d3 = 2 * la + 1, 2 * lb + 1, 2 * lo + 1
                ioff, ooff = plan.irr_in.offsets[a], plan.irr_out.offsets[o]
                for wo in range(mo):
                    for m3 in range(d3):
                        acc = 0.0
                        for m1 in range(d1):
                            if plan.mode == "uvu":
                                xin = wt[e][plan.w_off[p] + wo] * x[j][ioff + wo * d1 + m1]
                            else:
                                xin = 0.0
                                for u in range(ma):
                                    xin += Wl[p][u][wo] * x[j][ioff + u * d1 + m1]
                                xin *= wt[e][p]
                            for m2 in range(d2):
                                acc += C[m1][m2][m3] * Ys[b][m2] * xin
                        y[i][ooff + wo * d3 + m3] += plan.coeff[p] * acc
    return np.array(y)
