"""Float64 CPU oracle for the edge-conditioned E(3)-equivariant tensor-product convolution.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package: only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may use it.  It shares no code, tables or helpers with the CUDA
library; it builds its own real spherical harmonics (Legendre-derivative route), its own
Wigner-D matrices (least squares) and its own Clebsch-Gordan tables (null space of the
rotation-equivariance constraint).

What it computes (plain form; see ``oracle.conv``): for receiver i and every incoming
edge e = (src j -> dst i) with edge vector v_e,

    y[i, o, w, m3] = sum_e sum_{p: out(p)=o} c_p sum_{m1,m2} C_p[m1,m2,m3] Y_l2(v_e)[m2] X_pe[w,m1]
        uvu: X_pe[u, m1] = w[e,p,u] x[j, in(p), u, m1]
        uvw: X_pe[w, m1] = s[e,p] sum_u W_p[u,w] x[j, in(p), u, m1]

as described by "Sobek: Streaming Equivariant Tensor Product Convolutions" (abstract:
edge-conditioned tensor-product convolution, radial projection, spherical-harmonic
coupling, graph aggregation) and "The GPU Workload That Rewrites Molecular Physics"
(section "Equivariant feature transforms": spherical harmonics and Clebsch-Gordan
products).  Backward and double backward are the vector-Jacobian products of this map
("Sobek", abstract: forward, backward and double backward), taken by torch autograd.

``oracle.radial`` composes the same map with the radial projection fused in: the uvu
weights formed as w = h @ W_r from the radial network's last hidden layer ("Sobek",
abstract: the radial projection reordered so that edge-specific weights are never
materialised), with its backward to (x, vec, h, W_r) by autograd.

``oracle.gaunt`` holds the second operator, the spherical-grid (Gaunt) tensor-product
convolution ("The Price of Freedom: Exploring Expressivity and Runtime Tradeoffs in
Equivariant Tensor Products", abstract), with its Gaunt coefficients integrated on an exact
quadrature grid and pinned against sympy's closed form.

Pins (tests/test_oracle_*.py): SH against scipy's complex spherical harmonics and the
addition theorem; Wigner-D group law; CG against sympy's Clebsch-Gordan coefficients,
orthogonality and equivariance; operator equivariance, parity, the l=0 case against
scipy.sparse SpMV, finite differences, gradgradcheck and a pure-Python brute-force loop.
"""
from .irreps import Irreps, OraclePlan  # noqa: F401
from .so3 import real_sh, wigner_D, cg_real, random_rotation  # noqa: F401
from .conv import forward, backward, double_backward, forward_uvw_reassociated  # noqa: F401
from .radial import forward_radial, backward_radial  # noqa: F401
