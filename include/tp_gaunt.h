/* The spherical-grid (Gaunt) tensor-product convolution on B200 (sm_100a).
 *
 * "The Price of Freedom: Exploring Expressivity and Runtime Tradeoffs in Equivariant Tensor
 * Products" (abstract) names the Gaunt tensor product and computes it directly on a
 * spherical grid.  As a convolution over the receiver-sorted CSR of include/tp.h:
 *
 *   y[i, u, l3, m3] = sum_{e: dst(e) = i} integral f_{src(e),u}(r) g_{e,u}(r) Y_l3m3(r) dOmega / (4 pi)
 *     f_{j,u}(r) = sum_{l1,m1} x[j, u, l1, m1] Y_l1m1(r)              (the node feature as a function)
 *     g_{e,u}(r) = sum_{l2 <= lmax_sh} w[e, l2, u] sum_m2 Y_l2m2(v_e) Y_l2m2(r)   (the edge filter)
 *
 * i.e. the real Gaunt coefficients applied to x, the edge's spherical harmonics and per-degree
 * radial weights.  The library evaluates f and the adjoint of the projection on an exact
 * quadrature grid per node (node-sized workspaces) and the filter per edge from the Legendre
 * polynomials of r_hat . r_g, so the per-edge work is pointwise on the grid.
 *
 * Layouts: irreps "u x 0e + u x 1o + ..." -- natural parity (-1)^l, one multiplicity u <= 128
 * for every block, degrees <= 3, each degree at most once, increasing; [u][m] inside a
 * block (as include/tp.h).  w[E, lmax_sh + 1, u] (degree outer, channel inner).  All
 * pointers device memory, 4-byte aligned; outputs are fully overwritten; calls are
 * asynchronous on `stream`.  Errors: TP_ERR_INVALID_ARG (syntax, parity, multiplicities,
 * NULL or misaligned pointers), TP_ERR_UNSUPPORTED (l > 3, u > 128), TP_ERR_WORKSPACE,
 * TP_ERR_CUDA. */
#ifndef TP_GAUNT_H_
#define TP_GAUNT_H_

#include "tp.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tp_gaunt_s* tp_gaunt_t;

/* Plan: input and output irreps as above, filter degrees 0..lmax_sh (<= 3).  The grid
 * integrates degree 3 L exactly, L = the largest degree of the three. */
tp_status_t tp_gaunt_create(tp_gaunt_t* plan, const char* irreps_in, int32_t lmax_sh, const char* irreps_out);
tp_status_t tp_gaunt_destroy(tp_gaunt_t plan);

/* Widths, per-edge weights (lmax_sh + 1) * u and the number of grid points. */
tp_status_t tp_gaunt_query(tp_gaunt_t plan, int64_t* in_dim, int64_t* out_dim, int64_t* n_edge_weights,
                           int32_t* grid_points);

/* Workspace bytes: forward N x grid x 32 ceil(u / 32) floats (the node features on the grid, in
 * 32-channel slices); backward twice that (also the receivers' adjoint on the grid) plus room
 * to build the transpose (int32) when colptr / perm are not given. */
tp_status_t tp_gaunt_workspace_size(tp_gaunt_t plan, int64_t N, int64_t E, int32_t op, size_t* bytes);

/* Forward: y[N, out_dim]. */
tp_status_t tp_gaunt_fwd(tp_gaunt_t plan, int64_t N, int64_t E, const int32_t* rowptr, const int32_t* src,
                         const float* x, const float* vec, const float* w, float* y, void* ws, size_t ws_bytes,
                         tp_stream_t stream);

/* Backward against gy[N, out_dim]: gx[N, in_dim], gw[E, lmax_sh + 1, u], gvec[E, 3], each NULL
 * = skipped.  colptr / perm: a transpose from tp_csr_transpose, or both NULL to build it in ws. */
tp_status_t tp_gaunt_bwd(tp_gaunt_t plan, int64_t N, int64_t E, const int32_t* rowptr, const int32_t* src,
                         const int32_t* colptr, const int32_t* perm, const float* x, const float* vec,
                         const float* w, const float* gy, float* gx, float* gw, float* gvec, void* ws,
                         size_t ws_bytes, tp_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* TP_GAUNT_H_ */
