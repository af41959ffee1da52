// The convolution for any path list with l <= 3: kernels driven by a runtime path table.
//
// A plan whose irreps and path list match no compiled specialisation (a subset or another
// order of paths, other irreps, blocks of different multiplicities) carries a GenTable: per
// path its degrees, the id of its (l1, l2, l3) triple, its block offsets, channel count,
// weight offset and coefficient.  Every kernel below walks the paths of its task and hands
// each to the generated contractions of its triple (gen::with_triple: a switch over the 34
// triples of generic_cg.h, each an unrolled chain over the non-zero Clebsch-Gordan entries;
// "FlashTP", abstract: sparsity-aware, path-aggregated execution).  The arithmetic per edge,
// path and channel is that of the compiled kernels; what changes is the schedule:
//   k_gen_recv   one warp per (receiver, output block, 32-channel slice), lane = channel: the
//                block's paths one after another, each over the receiver's edges, summed in
//                registers (forward y; double-backward g_gy);
//   k_gen_send   one warp per (sender, input block, slice), edges in the stable sender order of
//                the transpose: gx (g_x) in registers, gw (g_w) written per edge;
//   k_gen_edge   one warp per edge: the direction gradient gvec (g_vec), a sum over paths and
//                channels reduced across the warp.
// Every output element is written by exactly one warp, in a fixed order: deterministic, no
// float atomics, no edge-sized intermediate.
#include <algorithm>

#include "generic_cg.h"
#include "tp_common.h"
#include "tp_kernels.cuh"

namespace tp {
namespace {

constexpr int kGenWarps = 4;   // warps per CTA

// dY/dv . d for one degree: (grad P(r) . d - l Y (r . d)) / |v|
template <int L>
__device__ __forceinline__ void sh_dir(float rx, float ry, float rz, float ir, float dx, float dy, float dz,
                                       const float (&Y)[2 * L + 1], float (&Yp)[2 * L + 1]) {
  float G[2 * L + 1][3];
  gen::ShBlock<L>::grad(rx, ry, rz, G);
  const float rd = fmaf(rx, dx, fmaf(ry, dy, rz * dz));
#pragma unroll
  for (int m = 0; m < 2 * L + 1; ++m)
    Yp[m] = ir * (fmaf(G[m][0], dx, fmaf(G[m][1], dy, G[m][2] * dz)) - (float)L * Y[m] * rd);
}

template <int D>
__device__ __forceinline__ void load_row(const float* __restrict__ p, float (&v)[D]) {
#pragma unroll
  for (int m = 0; m < D; ++m) v[m] = __ldg(p + m);
}

template <int D>
__device__ __forceinline__ void zero(float (&v)[D]) {
#pragma unroll
  for (int m = 0; m < D; ++m) v[m] = 0.f;
}

// ---------------------------------------------------------------------------------------
// Receiver pass.  MODE 0: y = sum_p c_p w_p C_p(x[src], Y).  MODE 1 (double backward):
// g_gy = sum_p c_p (ggw_p C_p(x, Y) + w_p (C_p(ggx, Y) + C_p(x, dY[ggvec]))).
// UVW: the input rows are x W per path (a.x, row a.in_dim) and the weight is the per-edge
// scalar s[e, p].
// ---------------------------------------------------------------------------------------
template <int MODE, bool UVW>
__global__ void __launch_bounds__(32 * kGenWarps) k_gen_recv(const __grid_constant__ LaunchArgs a,
                                                             const __grid_constant__ GenTable T) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * kGenWarps + (threadIdx.x >> 5);
  if (wid >= (int64_t)a.N * T.n_rtask) return;
  const int row = (int)(wid / T.n_rtask), task = (int)(wid - (int64_t)row * T.n_rtask);
  const int o = T.rtask_block[task];
  const int c = T.rtask_slice[task] * 32 + lane;
  const bool act = c < T.out_mul[o];
  int e0 = __ldg(a.rowptr + row), e1 = __ldg(a.rowptr + row + 1);
  if (a.check) {
    e0 = max(0, min(e0, a.E));
    e1 = max(e0, min(e1, a.E));
  }
  float acc[7];
  zero(acc);
  for (int pi = T.out_first[o]; pi < T.out_first[o + 1]; ++pi) {
    const int p = T.out_paths[pi];
    const GenPath P = T.path[p];
    gen::with_triple(P.tid, [&](auto cg) {
      using Cg = decltype(cg);
      for (int base = e0; base < e1; base += 32) {
        const int my_e = base + lane;
        int my_j = -1;
        float vx = 0.f, vy = 0.f, vz = 0.f, dx = 0.f, dy = 0.f, dz = 0.f;
        if (my_e < e1) {
          my_j = __ldg(a.src + my_e);
          vx = __ldg(a.vec + 3 * (int64_t)my_e);
          vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
          vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
          if (MODE == 1 && a.ggvec) {
            dx = __ldg(a.ggvec + 3 * (int64_t)my_e);
            dy = __ldg(a.ggvec + 3 * (int64_t)my_e + 1);
            dz = __ldg(a.ggvec + 3 * (int64_t)my_e + 2);
          }
          if (a.check && (unsigned)my_j >= (unsigned)a.N) {
            report(a, kDevBadSrc);
            my_j = -1;
          }
        }
        const int ne = min(32, e1 - base);
        for (int k = 0; k < ne; ++k) {
          const int j = __shfl_sync(kFull, my_j, k);
          const float ux = __shfl_sync(kFull, vx, k), uy = __shfl_sync(kFull, vy, k), uz = __shfl_sync(kFull, vz, k);
          const float ex = __shfl_sync(kFull, dx, k), ey = __shfl_sync(kFull, dy, k), ez = __shfl_sync(kFull, dz, k);
          if (j < 0 || !act) continue;
          const int e = base + k;
          float rx, ry, rz, ir;
          edge_geometry(ux, uy, uz, rx, ry, rz, ir);
          float Y[Cg::D2];
          gen::ShBlock<Cg::L2>::sh(rx, ry, rz, Y);
          float xv[Cg::D1];
          load_row(a.x + (int64_t)j * a.in_dim + P.in_off + (int64_t)c * Cg::D1, xv);
          const int64_t widx = (int64_t)e * a.nw + (UVW ? p : P.w_off + c);
          const float w = P.coeff * __ldg(a.w + widx);
          float t[Cg::D3];
          Cg::fwd(xv, Y, t);
          if constexpr (MODE == 0) {
#pragma unroll
            for (int m = 0; m < Cg::D3; ++m) acc[m] = fmaf(w, t[m], acc[m]);
          } else {
            const float gw = a.ggw ? P.coeff * __ldg(a.ggw + widx) : 0.f;
            float gxv[Cg::D1], Yp[Cg::D2], t2[Cg::D3], t3[Cg::D3];
            if (a.ggx) load_row(a.ggx + (int64_t)j * a.in_dim + P.in_off + (int64_t)c * Cg::D1, gxv);
            else zero(gxv);
            sh_dir<Cg::L2>(rx, ry, rz, ir, ex, ey, ez, Y, Yp);
            Cg::fwd(gxv, Y, t2);
            Cg::fwd(xv, Yp, t3);
#pragma unroll
            for (int m = 0; m < Cg::D3; ++m) acc[m] = fmaf(gw, t[m], fmaf(w, t2[m] + t3[m], acc[m]));
          }
        }
      }
    });
  }
  if (act) {
    const int d3 = 2 * T.out_l[o] + 1;
    float* yr = a.y + (int64_t)row * a.out_dim + T.out_off[o] + (int64_t)c * d3;
#pragma unroll
    for (int m = 0; m < 7; ++m)
      if (m < d3) yr[m] = acc[m];
  }
}

// ---------------------------------------------------------------------------------------
// Sender pass (uvu).  MODE 0: gx[j] = sum_p c_p w_p C_p^T(Y, gy[i]) and gw[e, p, u] = c_p
// <x[j], C_p^T(Y, gy[i])>.  MODE 1 (double backward): g_x[j] = sum_p c_p (ggw_p z + w_p z')
// and g_w[e, p, u] = c_p (<ggx[j], z> + <x[j], z'>), z = C_p^T(Y, gy[i]), z' = C_p^T(dY[ggvec], gy[i]).
// ---------------------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(32 * kGenWarps) k_gen_send(const __grid_constant__ LaunchArgs a,
                                                             const __grid_constant__ GenTable T) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * kGenWarps + (threadIdx.x >> 5);
  if (wid >= (int64_t)a.N * T.n_stask) return;
  const int node = (int)(wid / T.n_stask), task = (int)(wid - (int64_t)node * T.n_stask);
  const int ib = T.stask_block[task];
  const int c = T.stask_slice[task] * 32 + lane;
  const bool act = c < T.in_mul[ib];
  int q0 = __ldg(a.colptr + node), q1 = __ldg(a.colptr + node + 1);
  if (a.check) {
    q0 = max(0, min(q0, a.E));
    q1 = max(q0, min(q1, a.E));
  }
  float gx[7];
  zero(gx);
  for (int pi = T.in_first[ib]; pi < T.in_first[ib + 1]; ++pi) {
    const int p = T.in_paths[pi];
    const GenPath P = T.path[p];
    gen::with_triple(P.tid, [&](auto cg) {
      using Cg = decltype(cg);
      float xv[Cg::D1], gxv[Cg::D1];
      zero(xv);
      zero(gxv);
      if (act) {
        load_row(a.x + (int64_t)node * a.in_dim + P.in_off + (int64_t)c * Cg::D1, xv);
        if (MODE == 1 && a.ggx) load_row(a.ggx + (int64_t)node * a.in_dim + P.in_off + (int64_t)c * Cg::D1, gxv);
      }
      for (int base = q0; base < q1; base += 32) {
        const int my_q = base + lane;
        int my_e = -1, my_i = 0;
        float vx = 0.f, vy = 0.f, vz = 0.f, dx = 0.f, dy = 0.f, dz = 0.f;
        if (my_q < q1) {
          my_e = __ldg(a.perm + my_q);
          if (a.check && (unsigned)my_e >= (unsigned)a.E) {
            report(a, kDevBadPerm);
            my_e = -1;
          } else {
            my_i = find_row(a.rowptr, a.N, my_e);
            vx = __ldg(a.vec + 3 * (int64_t)my_e);
            vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
            vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
            if (MODE == 1 && a.ggvec) {
              dx = __ldg(a.ggvec + 3 * (int64_t)my_e);
              dy = __ldg(a.ggvec + 3 * (int64_t)my_e + 1);
              dz = __ldg(a.ggvec + 3 * (int64_t)my_e + 2);
            }
          }
        }
        const int ne = min(32, q1 - base);
        for (int k = 0; k < ne; ++k) {
          const int e = __shfl_sync(kFull, my_e, k), i = __shfl_sync(kFull, my_i, k);
          const float ux = __shfl_sync(kFull, vx, k), uy = __shfl_sync(kFull, vy, k), uz = __shfl_sync(kFull, vz, k);
          const float ex = __shfl_sync(kFull, dx, k), ey = __shfl_sync(kFull, dy, k), ez = __shfl_sync(kFull, dz, k);
          if (e < 0 || !act) continue;
          float rx, ry, rz, ir;
          edge_geometry(ux, uy, uz, rx, ry, rz, ir);
          float Y[Cg::D2];
          gen::ShBlock<Cg::L2>::sh(rx, ry, rz, Y);
          float gyv[Cg::D3];
          load_row(a.gy + (int64_t)i * a.out_dim + P.out_off + (int64_t)c * Cg::D3, gyv);
          const int64_t widx = (int64_t)e * a.nw + P.w_off + c;
          const float w = P.coeff * __ldg(a.w + widx);
          float z[Cg::D1];
          Cg::tx(Y, gyv, z);
          if constexpr (MODE == 0) {
            float s = 0.f;
#pragma unroll
            for (int m = 0; m < Cg::D1; ++m) {
              gx[m] = fmaf(w, z[m], gx[m]);
              s = fmaf(xv[m], z[m], s);
            }
            if (a.gw) a.gw[widx] = P.coeff * s;
          } else {
            const float gw = a.ggw ? P.coeff * __ldg(a.ggw + widx) : 0.f;
            float Yp[Cg::D2], zp[Cg::D1];
            sh_dir<Cg::L2>(rx, ry, rz, ir, ex, ey, ez, Y, Yp);
            Cg::tx(Yp, gyv, zp);
            float s = 0.f;
#pragma unroll
            for (int m = 0; m < Cg::D1; ++m) {
              gx[m] = fmaf(gw, z[m], fmaf(w, zp[m], gx[m]));
              s = fmaf(gxv[m], z[m], fmaf(xv[m], zp[m], s));
            }
            if (a.gw) a.gw[widx] = P.coeff * s;
          }
        }
      }
    });
  }
  if (act && a.gx) {
    const int d1 = 2 * T.in_l[ib] + 1;
    float* gr = a.gx + (int64_t)node * a.in_dim + T.in_off[ib] + (int64_t)c * d1;
#pragma unroll
    for (int m = 0; m < 7; ++m)
      if (m < d1) gr[m] = gx[m];
  }
}

// ---------------------------------------------------------------------------------------
// Direction gradient per edge.  MODE 0: gvec[e] = sum_m gY_m dY_m/dv with
// gY = sum_{p, u} c_p w_p Q_p(x[src], gy[dst]), Q(x, g)[m2] = sum C x[m1] g[m3].
// MODE 1: g_vec[e] = sum_m G1_m dY_m/dv + G2_m (d^2 Y_m / dv^2) ggvec with
// G1 = sum c_p (ggw_p Q_p(x, gy) + w_p Q_p(ggx, gy)), G2 = sum c_p w_p Q_p(x, gy).
// UVW (MODE 0): x is x W per path and w the per-edge path scalar s[e, p].
// ---------------------------------------------------------------------------------------
template <int MODE, bool UVW = false>
__global__ void __launch_bounds__(32 * kGenWarps) k_gen_edge(const __grid_constant__ LaunchArgs a,
                                                             const __grid_constant__ GenTable T) {
  const int lane = threadIdx.x & 31;
  const int64_t e64 = (int64_t)blockIdx.x * kGenWarps + (threadIdx.x >> 5);
  if (e64 >= a.E) return;
  const int e = (int)e64;
  const int j = __ldg(a.src + e);
  if ((unsigned)j >= (unsigned)a.N) {     // outside the graph: nothing to differentiate
    if (a.check) report(a, kDevBadSrc);
    if (lane == 0) {
      float* g = a.gvec + 3 * (int64_t)e;
      g[0] = g[1] = g[2] = 0.f;
    }
    return;
  }
  const int i = find_row(a.rowptr, a.N, e);
  float rx, ry, rz, ir;
  edge_geometry(__ldg(a.vec + 3 * (int64_t)e), __ldg(a.vec + 3 * (int64_t)e + 1), __ldg(a.vec + 3 * (int64_t)e + 2),
                rx, ry, rz, ir);
  float G1[16], G2[16];
  zero(G1);
  zero(G2);
  for (int p = 0; p < T.n_paths; ++p) {
    const GenPath P = T.path[p];
    if (P.l2 == 0) continue;               // Y_0 is constant
    gen::with_triple(P.tid, [&](auto cg) {
      using Cg = decltype(cg);
      constexpr int base = Cg::L2 * Cg::L2;   // first component of degree L2 in the 16 SH values
      for (int c = lane; c < P.mul; c += 32) {
        float xv[Cg::D1], gyv[Cg::D3], qa[Cg::D2];
        load_row(a.x + (int64_t)j * a.in_dim + P.in_off + (int64_t)c * Cg::D1, xv);
        load_row(a.gy + (int64_t)i * a.out_dim + P.out_off + (int64_t)c * Cg::D3, gyv);
        const int64_t widx = (int64_t)e * a.nw + (UVW ? p : P.w_off + c);
        const float w = P.coeff * __ldg(a.w + widx);
        Cg::ty(xv, gyv, qa);
        if constexpr (MODE == 0) {
#pragma unroll
          for (int m = 0; m < Cg::D2; ++m) G1[base + m] = fmaf(w, qa[m], G1[base + m]);
        } else {
          const float gw = a.ggw ? P.coeff * __ldg(a.ggw + widx) : 0.f;
          float gxv[Cg::D1], qb[Cg::D2];
          if (a.ggx) load_row(a.ggx + (int64_t)j * a.in_dim + P.in_off + (int64_t)c * Cg::D1, gxv);
          else zero(gxv);
          Cg::ty(gxv, gyv, qb);
#pragma unroll
          for (int m = 0; m < Cg::D2; ++m) {
            G1[base + m] = fmaf(gw, qa[m], fmaf(w, qb[m], G1[base + m]));
            G2[base + m] = fmaf(w, qa[m], G2[base + m]);
          }
        }
      }
    });
  }
  float Y[16], G[16][3];
  gen::ShAll::sh(rx, ry, rz, Y);
  gen::ShAll::sh_grad(rx, ry, rz, G);
  float g0 = 0.f, g1 = 0.f, g2 = 0.f;
  if constexpr (MODE == 0) {
    float sdeg = 0.f;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      g0 = fmaf(G1[m], G[m][0], g0);
      g1 = fmaf(G1[m], G[m][1], g1);
      g2 = fmaf(G1[m], G[m][2], g2);
      sdeg = fmaf(gen::ShAll::sh_degree(m) * G1[m], Y[m], sdeg);
    }
    g0 = ir * (g0 - rx * sdeg);
    g1 = ir * (g1 - ry * sdeg);
    g2 = ir * (g2 - rz * sdeg);
  } else {
    float ddx = 0.f, ddy = 0.f, ddz = 0.f;
    if (a.ggvec) {
      ddx = __ldg(a.ggvec + 3 * (int64_t)e);
      ddy = __ldg(a.ggvec + 3 * (int64_t)e + 1);
      ddz = __ldg(a.ggvec + 3 * (int64_t)e + 2);
    }
    float HD[16][3];
    gen::ShAll::sh_hess_dot(rx, ry, rz, ddx, ddy, ddz, HD);
    const float rd = fmaf(rx, ddx, fmaf(ry, ddy, rz * ddz));
    const float ir2 = ir * ir;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const float l = gen::ShAll::sh_degree(m);
      const float gdm = fmaf(G[m][0], ddx, fmaf(G[m][1], ddy, G[m][2] * ddz));
      const float cJ = G1[m] * ir;                   // first-derivative coefficient
      const float cK = G2[m] * ir2;                  // second-derivative coefficient
      const float lY = l * Y[m];
      const float rcoef = -cJ * lY + cK * (-l * gdm + l * (l + 2.f) * Y[m] * rd);
      const float gcoef = cJ - cK * l * rd;
      const float dcoef = -cK * lY;
      g0 += gcoef * G[m][0] + cK * HD[m][0] + rcoef * rx + dcoef * ddx;
      g1 += gcoef * G[m][1] + cK * HD[m][1] + rcoef * ry + dcoef * ddy;
      g2 += gcoef * G[m][2] + cK * HD[m][2] + rcoef * rz + dcoef * ddz;
    }
  }
  g0 = warp_sum(g0);
  g1 = warp_sum(g1);
  g2 = warp_sum(g2);
  if (lane == 0) {
    float* g = a.gvec + 3 * (int64_t)e;
    g[0] = g0;
    g[1] = g1;
    g[2] = g2;
  }
}

// ---------------------------------------------------------------------------------------
// uvw through the path table ("Sobek", abstract: the shared multiplicity mixing W_p kept,
// applied on node state instead of per edge).  Forward: xt_p[j] = W_p^T x_a[j] per path and
// node, then the receiver pass with xt_p as the path's input rows and s[e, p] as its weight.
// Backward: B_p[j] = sum_{e: src=j} c_p s_p C_p^T(Y, gy[dst]) (sender pass, which also gives
// gs[e, p] = c_p <xt_p[j], C_p^T(Y, gy[dst])>), gx_a[j] = sum_{p: in=a} W_p B_p[j],
// gW_p = sum_j x_a[j] B_p[j]^T (node chunks, summed in chunk order).  Layout of a row of xt
// and of B: path after path, [w][m1] inside a path.
// ---------------------------------------------------------------------------------------

// xt[j, off_p + w d1 + m1] = sum_u W[p, u, w] x[j, in_a + u d1 + m1]: one thread per (j, p, w)
__global__ void __launch_bounds__(256) k_gen_xw(const __grid_constant__ LaunchArgs a,
                                                const __grid_constant__ GenTable T) {
  const int64_t per_node = (int64_t)T.n_paths * T.mul_out;
  const int64_t total = (int64_t)a.N * per_node;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = t / per_node;
    const int r = (int)(t - j * per_node);
    const int p = r / T.mul_out, w = r - p * T.mul_out;
    const GenPath P = T.path[p];
    const int d1 = 2 * P.l1 + 1;
    const float* xr = a.x + j * a.in_dim + T.in_off[P.in_block];
    const float* Wp = a.W + (int64_t)p * T.mul_in * T.mul_out + w;
    float acc[7];
    zero(acc);
    for (int u = 0; u < T.mul_in; ++u) {
      const float wv = __ldg(Wp + (int64_t)u * T.mul_out);
#pragma unroll
      for (int m = 0; m < 7; ++m)
        if (m < d1) acc[m] = fmaf(wv, __ldg(xr + u * d1 + m), acc[m]);
    }
    float* o = a.A + j * T.xt_dim + P.in_off + (int64_t)w * d1;
#pragma unroll
    for (int m = 0; m < 7; ++m)
      if (m < d1) o[m] = acc[m];
  }
}

// One warp per (sender, path): B_p[j] (all output channels, in groups of four 32-channel
// slices kept in registers) and gs[e, p] (a warp sum per edge; later groups add to it).
__global__ void __launch_bounds__(32 * kGenWarps) k_gen_send_uvw(const __grid_constant__ LaunchArgs a,
                                                                 const __grid_constant__ GenTable T) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * kGenWarps + (threadIdx.x >> 5);
  if (wid >= (int64_t)a.N * T.n_paths) return;
  const int node = (int)(wid / T.n_paths), p = (int)(wid - (int64_t)node * T.n_paths);
  const GenPath P = T.path[p];
  const int q0 = __ldg(a.colptr + node), q1 = __ldg(a.colptr + node + 1);
  const int n_sl = (T.mul_out + 31) / 32;
  gen::with_triple(P.tid, [&](auto cg) {
    using Cg = decltype(cg);
    for (int g0 = 0; g0 < n_sl; g0 += 4) {
      float B[4][Cg::D1], xt[4][Cg::D1];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        zero(B[k]);
        zero(xt[k]);
        const int c = (g0 + k) * 32 + lane;
        if (g0 + k < n_sl && c < T.mul_out) load_row(a.A + (int64_t)node * T.xt_dim + P.in_off + (int64_t)c * Cg::D1, xt[k]);
      }
      for (int base = q0; base < q1; base += 32) {
        const int my_q = base + lane;
        int my_e = -1, my_i = 0;
        float vx = 0.f, vy = 0.f, vz = 0.f;
        if (my_q < q1) {
          my_e = __ldg(a.perm + my_q);
          my_i = find_row(a.rowptr, a.N, my_e);
          vx = __ldg(a.vec + 3 * (int64_t)my_e);
          vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
          vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
        }
        const int ne = min(32, q1 - base);
        for (int k = 0; k < ne; ++k) {
          const int e = __shfl_sync(kFull, my_e, k), i = __shfl_sync(kFull, my_i, k);
          const float ux = __shfl_sync(kFull, vx, k), uy = __shfl_sync(kFull, vy, k), uz = __shfl_sync(kFull, vz, k);
          float rx, ry, rz, ir;
          edge_geometry(ux, uy, uz, rx, ry, rz, ir);
          float Y[Cg::D2];
          gen::ShBlock<Cg::L2>::sh(rx, ry, rz, Y);
          const float sc = P.coeff * __ldg(a.w + (int64_t)e * a.nw + p);
          float part = 0.f;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int c = (g0 + kk) * 32 + lane;
            if (g0 + kk < n_sl && c < T.mul_out) {
              float gyv[Cg::D3], z[Cg::D1];
              load_row(a.gy + (int64_t)i * a.out_dim + P.out_off + (int64_t)c * Cg::D3, gyv);
              Cg::tx(Y, gyv, z);
#pragma unroll
              for (int m = 0; m < Cg::D1; ++m) {
                B[kk][m] = fmaf(sc, z[m], B[kk][m]);
                part = fmaf(xt[kk][m], z[m], part);
              }
            }
          }
          part = warp_sum(part);
          if (lane == 0 && a.gw) {
            float* gs = a.gw + (int64_t)e * a.nw + p;
            *gs = g0 == 0 ? P.coeff * part : *gs + P.coeff * part;
          }
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = (g0 + k) * 32 + lane;
        if (g0 + k < n_sl && c < T.mul_out) {
          float* o = a.G + (int64_t)node * T.xt_dim + P.in_off + (int64_t)c * Cg::D1;
#pragma unroll
          for (int m = 0; m < Cg::D1; ++m) o[m] = B[k][m];
        }
      }
    }
  });
}

// gx[j, in_a + u d1 + m1] = sum_{p: in(p) = a} sum_w W[p, u, w] B[j, off_p + w d1 + m1]:
// one thread per (j, input block, u)
__global__ void __launch_bounds__(256) k_gen_bw(const __grid_constant__ LaunchArgs a,
                                                const __grid_constant__ GenTable T) {
  const int64_t per_node = (int64_t)T.n_in * T.mul_in;
  const int64_t total = (int64_t)a.N * per_node;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = t / per_node;
    const int r = (int)(t - j * per_node);
    const int ib = r / T.mul_in, u = r - ib * T.mul_in;
    const int d1 = 2 * T.in_l[ib] + 1;
    float acc[7];
    zero(acc);
    for (int pi = T.in_first[ib]; pi < T.in_first[ib + 1]; ++pi) {
      const int p = T.in_paths[pi];
      const float* Wr = a.W + ((int64_t)p * T.mul_in + u) * T.mul_out;
      const float* Br = a.G + j * T.xt_dim + T.path[p].in_off;
      for (int w = 0; w < T.mul_out; ++w) {
        const float wv = __ldg(Wr + w);
#pragma unroll
        for (int m = 0; m < 7; ++m)
          if (m < d1) acc[m] = fmaf(wv, Br[w * d1 + m], acc[m]);
      }
    }
    float* o = a.gx + j * a.in_dim + T.in_off[ib] + (int64_t)u * d1;
#pragma unroll
    for (int m = 0; m < 7; ++m)
      if (m < d1) o[m] = acc[m];
  }
}

// part[z, p, u, w] = sum over the nodes j of chunk z and m1 of x[j, in_a + u d1 + m1] B[j, off_p + w d1 + m1]
__global__ void __launch_bounds__(256) k_gen_gw_part(const __grid_constant__ LaunchArgs a,
                                                     const __grid_constant__ GenTable T) {
  const int64_t n_sh = (int64_t)T.n_paths * T.mul_in * T.mul_out;
  const int z = blockIdx.y;
  const int64_t chunk = ((int64_t)a.N + a.splits - 1) / a.splits;
  const int64_t j0 = z * chunk, j1 = min((int64_t)a.N, j0 + chunk);
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n_sh; t += (int64_t)gridDim.x * blockDim.x) {
    const int p = (int)(t / ((int64_t)T.mul_in * T.mul_out));
    const int r = (int)(t - (int64_t)p * T.mul_in * T.mul_out);
    const int u = r / T.mul_out, w = r - u * T.mul_out;
    const GenPath P = T.path[p];
    const int d1 = 2 * P.l1 + 1;
    float acc = 0.f;
    for (int64_t j = j0; j < j1; ++j) {
      const float* xr = a.x + j * a.in_dim + T.in_off[P.in_block] + (int64_t)u * d1;
      const float* Br = a.G + j * T.xt_dim + P.in_off + (int64_t)w * d1;
      for (int m = 0; m < d1; ++m) acc = fmaf(__ldg(xr + m), Br[m], acc);
    }
    a.part[(int64_t)z * n_sh + t] = acc;
  }
}

__global__ void __launch_bounds__(256) k_gen_gw_reduce(const __grid_constant__ LaunchArgs a, int64_t n_sh) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n_sh; t += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int z = 0; z < a.splits; ++z) s += a.part[(int64_t)z * n_sh + t];
    a.gW[t] = s;
  }
}

unsigned flat_grid(int64_t n) {
  int64_t g = (n + 255) / 256;
  if (g > 148 * 32) g = 148 * 32;
  return (unsigned)(g < 1 ? 1 : g);
}

unsigned warps_grid(int64_t warps) { return (unsigned)((warps + kGenWarps - 1) / kGenWarps); }

}  // namespace

int gen_triple_id(int l1, int l2, int l3) { return gen::triple_id(l1, l2, l3); }

cudaError_t launch_gen_fwd(const LaunchArgs& a, const GenTable& T, cudaStream_t s) {
  if (a.N == 0 || T.n_rtask == 0) return cudaSuccess;
  k_gen_recv<0, false><<<warps_grid((int64_t)a.N * T.n_rtask), 32 * kGenWarps, 0, s>>>(a, T);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_gen_bwd(const LaunchArgs& a, const GenTable& T, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  if ((a.gx || a.gw) && T.n_stask > 0) {
    k_gen_send<0><<<warps_grid((int64_t)a.N * T.n_stask), 32 * kGenWarps, 0, s>>>(a, T);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.gvec && a.E > 0) {
    k_gen_edge<0><<<warps_grid(a.E), 32 * kGenWarps, 0, s>>>(a, T);
    count_launches(1);
  }
  return cudaGetLastError();
}

// recv: g_gy into a.y; send: g_x (a.gx), g_w (a.gw) and g_vec (a.gvec), each skipped when NULL.
cudaError_t launch_gen_dbwd(const LaunchArgs& a, const GenTable& T, bool recv, bool send, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  if (recv && T.n_rtask > 0) {
    k_gen_recv<1, false><<<warps_grid((int64_t)a.N * T.n_rtask), 32 * kGenWarps, 0, s>>>(a, T);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (send && (a.gx || a.gw) && T.n_stask > 0) {
    k_gen_send<1><<<warps_grid((int64_t)a.N * T.n_stask), 32 * kGenWarps, 0, s>>>(a, T);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (send && a.gvec && a.E > 0) {
    k_gen_edge<1><<<warps_grid(a.E), 32 * kGenWarps, 0, s>>>(a, T);
    count_launches(1);
  }
  return cudaGetLastError();
}

cudaError_t launch_gen_uvw_fwd(const LaunchArgs& a, const GenTable& T, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  k_gen_xw<<<flat_grid((int64_t)a.N * T.n_paths * T.mul_out), 256, 0, s>>>(a, T);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || T.n_rtask == 0) return e;
  LaunchArgs b = a;                 // the receiver pass reads x W per path
  b.x = a.A;
  b.in_dim = T.xt_dim;
  b.nw = T.n_paths;
  k_gen_recv<0, true><<<warps_grid((int64_t)a.N * T.n_rtask), 32 * kGenWarps, 0, s>>>(b, T);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_gen_uvw_bwd(const LaunchArgs& a, const GenTable& T, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  k_gen_xw<<<flat_grid((int64_t)a.N * T.n_paths * T.mul_out), 256, 0, s>>>(a, T);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.gw || a.gx || a.gW) {
    LaunchArgs b = a;
    b.nw = T.n_paths;
    k_gen_send_uvw<<<warps_grid((int64_t)a.N * T.n_paths), 32 * kGenWarps, 0, s>>>(b, T);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.gvec && a.E > 0) {
    LaunchArgs b = a;
    b.x = a.A;
    b.in_dim = T.xt_dim;
    b.nw = T.n_paths;
    k_gen_edge<0, true><<<warps_grid(a.E), 32 * kGenWarps, 0, s>>>(b, T);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.gx) {
    k_gen_bw<<<flat_grid((int64_t)a.N * T.n_in * T.mul_in), 256, 0, s>>>(a, T);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.gW) {
    const int64_t n_sh = (int64_t)T.n_paths * T.mul_in * T.mul_out;
    const dim3 grid((unsigned)std::min<int64_t>((n_sh + 255) / 256, 1024), (unsigned)a.splits);
    k_gen_gw_part<<<grid, 256, 0, s>>>(a, T);
    k_gen_gw_reduce<<<flat_grid(n_sh), 256, 0, s>>>(a, n_sh);
    count_launches(2);
  }
  return cudaGetLastError();
}

}  // namespace tp
