// The spherical-grid (Gaunt) tensor-product convolution (include/tp_gaunt.h).
//
// "The Price of Freedom: Exploring Expressivity and Runtime Tradeoffs in Equivariant Tensor
// Products" (abstract): the Gaunt product of two spherical functions, computed directly on a
// spherical grid.  Per channel u the sender's feature is f(r) = sum x_lm Y_lm(r); the edge
// filter is g(r) = sum_l2 w_l2 sum_m2 Y_l2m2(v_hat) Y_l2m2(r) = sum_l2 w_l2 (2 l2 + 1)
// P_l2(v_hat . r) (addition theorem, component normalisation); the message is the projection
// of f g onto the output harmonics.  On a grid that integrates degree 3 L exactly:
//
//   k_gaunt_to_grid<L, 0>  F[j][g][u] = sum_lm x[j, u, lm] Y_lm(r_g)                 (per node)
//   k_gaunt_fwd<L>         acc[g] = sum_{e into i} F[src][g][u] S_e(g),  S_e(g) = sum_l2 w_l2 (2l2+1) P_l2(t_g),
//                          t_g = v_hat . r_g; y[i, u, lm] = sum_g q_g Y_lm(r_g) acc[g]   (per receiver)
//   k_gaunt_to_grid<L, 1>  Gq[i][g][u] = q_g sum_lm Y_lm(r_g) gy[i, u, lm]           (per node)
//   k_gaunt_bwd<L>         per sender j and out-edge e (stable transpose order):
//                          gF[g] += S_e(g) Gq[dst][g][u];  gw[e, l2, u] = sum_g (2l2+1) P_l2(t_g) F_j(g) Gq(g);
//                          gvec[e] = |v|^-1 sum_{g,u} F_j Gq S_e'(t_g) (r_g - t_g v_hat);
//                          gx[j, u, lm] = sum_g Y_lm(r_g) gF[g]
// Grid rows are node sized ([node][32-channel slice][pairs of grid points][lane]), nothing per
// edge is stored; the pointwise work runs on two grid points per FFMA2, the filter by Horner's
// rule of the plan's filter degree, and the backward computes the weight moments and the
// direction terms only when their outputs are requested.  Warps per node: (slice, phase), the
// phases splitting the node's edges; sums in fixed order.
#include <algorithm>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "../../include/tp_gaunt.h"
#include "gaunt_grid.h"
#include "tp_common.h"
#include "tp_host.h"
#include "tp_kernels.cuh"

namespace tp {
namespace {

struct GauntArgs {
  int N, E, mul, lmax_sh, nw, in_dim, out_dim, nsl;
  int split;                   // warps that split a node's edges (nsl * split <= 4)
  int in_off[4], out_off[4];   // offset of the block of degree l in a row, -1 when absent
  const int32_t *rowptr, *src, *colptr, *perm;
  const float *x, *vec, *w, *gy;
  float2 *F, *Gq;              // [N][nsl][NG / 2][32 lanes] pairs of grid points
  float *y, *gx, *gw, *gvec;
};

// The filter sum_l w_l (2l+1) P_l(t) as a cubic in t: a0 + a1 t + a2 t^2 + a3 t^3
// (3 P_1 = 3t, 5 P_2 = 7.5 t^2 - 2.5, 7 P_3 = 17.5 t^3 - 10.5 t).
__device__ __forceinline__ void filter_cubic(const float (&wl)[4], float (&c)[4]) {
  c[0] = fmaf(-2.5f, wl[2], wl[0]);
  c[1] = fmaf(-10.5f, wl[3], 3.f * wl[1]);
  c[2] = 7.5f * wl[2];
  c[3] = 17.5f * wl[3];
}

__device__ __forceinline__ float2 dup2(float v) { return make_float2(v, v); }

// t_g = r_hat . r_g for every grid point, in pairs of points, from the grid's product structure:
// r_g has cos(theta) = ct(k), sin(theta) = st(k) and azimuth phi_j, so
// t = rz ct(k) + st(k) (rx cos phi_j + ry sin phi_j).
template <class Gr>
__device__ __forceinline__ void grid_dots2(float rx, float ry, float rz, float2 (&t)[Gr::NG / 2]) {
  float c[Gr::NP], z[Gr::NT];
#pragma unroll
  for (int j = 0; j < Gr::NP; ++j) c[j] = fmaf(rx, Gr::cp(j), ry * Gr::sp(j));
#pragma unroll
  for (int k = 0; k < Gr::NT; ++k) z[k] = rz * Gr::ct(k);
#pragma unroll
  for (int g2 = 0; g2 < Gr::NG / 2; ++g2) {
    const int g0 = 2 * g2, g1 = 2 * g2 + 1;
    t[g2] = make_float2(fmaf(Gr::st(g0 / Gr::NP), c[g0 % Gr::NP], z[g0 / Gr::NP]),
                        fmaf(Gr::st(g1 / Gr::NP), c[g1 % Gr::NP], z[g1 / Gr::NP]));
  }
}

// Horner of degree D in pairs: sum_{d <= D} c_d t^d
template <int D>
__device__ __forceinline__ float2 horner2(const float (&c)[4], float2 t) {
  float2 s = dup2(c[D]);
#pragma unroll
  for (int d = D - 1; d >= 0; --d) s = __ffma2_rn(s, t, dup2(c[d]));
  return s;
}

// MODE 0: F from x (input blocks); MODE 1: Gq from gy (output blocks, times q_g).  One thread
// per (node, slice, lane); lanes past the channel count write zeros.
template <int L, int MODE>
__global__ void __launch_bounds__(256) k_gaunt_to_grid(const __grid_constant__ GauntArgs a) {
  using Gr = gaunt::Grid<L>;
  const int64_t total = (int64_t)a.N * a.nsl * 32;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t js = t >> 5;            // node * nsl + slice
    const int lane = (int)(t & 31);
    const int64_t j = js / a.nsl;
    const int u = (int)(js - j * a.nsl) * 32 + lane;
    const bool act = u < a.mul;
    const float* row = MODE == 0 ? a.x + j * a.in_dim : a.gy + j * a.out_dim;
    const int* off = MODE == 0 ? a.in_off : a.out_off;
    float c[Gr::NSH];
#pragma unroll
    for (int l = 0; l <= L; ++l) {
#pragma unroll
      for (int m = 0; m < 2 * l + 1; ++m)
        c[l * l + m] = (act && off[l] >= 0) ? __ldg(row + off[l] + u * (2 * l + 1) + m) : 0.f;
    }
    float2* out = (MODE == 0 ? a.F : a.Gq) + js * (Gr::NG / 2) * 32 + lane;
#pragma unroll
    for (int g2 = 0; g2 < Gr::NG / 2; ++g2) {
      float v0 = 0.f, v1 = 0.f;
#pragma unroll
      for (int k = 0; k < Gr::NSH; ++k) {
        v0 = fmaf(c[k], Gr::Y(2 * g2, k), v0);
        v1 = fmaf(c[k], Gr::Y(2 * g2 + 1, k), v1);
      }
      out[g2 * 32] = MODE == 1 ? make_float2(Gr::q(2 * g2) * v0, Gr::q(2 * g2 + 1) * v1) : make_float2(v0, v1);
    }
  }
}

// w_l2 (2l2+1 folded into the cubic) of edge e for channel u; filter degrees above LSH read as
// 0, degrees above 0 of a zero-length edge too (its harmonics are Y_0 = 1, Y_l>0 = 0)
template <int LSH>
__device__ __forceinline__ void edge_weights(const GauntArgs& a, int e, int u, bool act, float ir, float (&wl)[4]) {
#pragma unroll
  for (int l = 0; l < 4; ++l)
    wl[l] = (act && l <= LSH && (l == 0 || ir > 0.f)) ? __ldg(a.w + (int64_t)e * a.nw + l * a.mul + u) : 0.f;
}

// Forward: CTA = one receiver; warp w = (slice w / split, phase w % split); the phases take
// interleaved edges of the row and their grid accumulators are added through shared memory in
// phase order.  Per edge and lane (channel): the sender's grid row (pairs of points), the
// filter by Horner's rule, acc += F S, all two points per FFMA2.  On grids of <= 32 points
// the next edge's row is loaded while the current one is computed.
template <int L, int LSH>
__global__ void __launch_bounds__(128) k_gaunt_fwd(const __grid_constant__ GauntArgs a) {
  using Gr = gaunt::Grid<L>;
  constexpr int NGP = Gr::NG / 2;
  constexpr bool PF = Gr::NG <= 32;
  extern __shared__ float2 red2[];            // [(split-1) * nsl][NGP][32]
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int st = a.split, sl = wid / st, phase = wid - sl * st;
  const int i = blockIdx.x;
  const int u = sl * 32 + lane;
  const bool act = u < a.mul;
  const int e0 = __ldg(a.rowptr + i), e1 = __ldg(a.rowptr + i + 1);
  float2 acc[NGP];
#pragma unroll
  for (int g = 0; g < NGP; ++g) acc[g] = make_float2(0.f, 0.f);
  auto row_of = [&](int j) { return a.F + ((int64_t)j * a.nsl + sl) * NGP * 32 + lane; };
  auto edge = [&](int e, float vx, float vy, float vz, const float2 (&f)[NGP]) {
    float rx, ry, rz, ir;
    edge_geometry(vx, vy, vz, rx, ry, rz, ir);
    float wl[4], cf[4];
    edge_weights<LSH>(a, e, u, act, ir, wl);
    filter_cubic(wl, cf);
    float2 t[NGP];
    grid_dots2<Gr>(rx, ry, rz, t);
#pragma unroll
    for (int g = 0; g < NGP; ++g) acc[g] = __ffma2_rn(f[g], horner2<LSH>(cf, t[g]), acc[g]);
  };
  for (int base = e0 + phase; base < e1; base += 32 * st) {
    const int my_e = base + lane * st;
    int my_j = 0;
    float vx = 0.f, vy = 0.f, vz = 0.f;
    if (my_e < e1) {
      my_j = __ldg(a.src + my_e);
      vx = __ldg(a.vec + 3 * (int64_t)my_e);
      vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
      vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
    }
    const int ne = min(32, (e1 - base + st - 1) / st);
    if constexpr (PF) {
      // two row buffers: the row of edge k + 1 is loaded while edge k is computed
      float2 fa[NGP], fb[NGP];
      {
        const float2* r = row_of(__shfl_sync(kFull, my_j, 0));
#pragma unroll
        for (int g = 0; g < NGP; ++g) fa[g] = r[g * 32];
      }
      for (int k = 0; k < ne; k += 2) {
        const bool two = k + 1 < ne;
        {
          const float2* r = row_of(__shfl_sync(kFull, my_j, min(k + 1, 31)));
          if (two) {
#pragma unroll
            for (int g = 0; g < NGP; ++g) fb[g] = r[g * 32];
          }
        }
        edge(base + k * st, __shfl_sync(kFull, vx, k), __shfl_sync(kFull, vy, k), __shfl_sync(kFull, vz, k), fa);
        if (!two) break;
        {
          const float2* r = row_of(__shfl_sync(kFull, my_j, min(k + 2, 31)));
          if (k + 2 < ne) {
#pragma unroll
            for (int g = 0; g < NGP; ++g) fa[g] = r[g * 32];
          }
        }
        edge(base + (k + 1) * st, __shfl_sync(kFull, vx, k + 1), __shfl_sync(kFull, vy, k + 1),
             __shfl_sync(kFull, vz, k + 1), fb);
      }
    } else {
      for (int k = 0; k < ne; ++k) {
        const float2* r = row_of(__shfl_sync(kFull, my_j, k));
        float2 f[NGP];
#pragma unroll
        for (int g = 0; g < NGP; ++g) f[g] = r[g * 32];
        edge(base + k * st, __shfl_sync(kFull, vx, k), __shfl_sync(kFull, vy, k), __shfl_sync(kFull, vz, k), f);
      }
    }
  }
  if (st > 1) {
    if (phase > 0) {
      float2* dst = red2 + (((size_t)(phase - 1) * a.nsl + sl) * NGP) * 32 + lane;
#pragma unroll
      for (int g = 0; g < NGP; ++g) dst[g * 32] = acc[g];
    }
    __syncthreads();
    if (phase == 0) {
      for (int ph = 1; ph < st; ++ph) {
        const float2* srcp = red2 + (((size_t)(ph - 1) * a.nsl + sl) * NGP) * 32 + lane;
#pragma unroll
        for (int g = 0; g < NGP; ++g) acc[g] = __fadd2_rn(acc[g], srcp[g * 32]);
      }
    }
  }
  if (!act || phase != 0) return;
  float* yr = a.y + (int64_t)i * a.out_dim;
#pragma unroll
  for (int l = 0; l <= L; ++l) {
    if (a.out_off[l] < 0) continue;
#pragma unroll
    for (int m = 0; m < 2 * l + 1; ++m) {
      float v = 0.f;
#pragma unroll
      for (int g = 0; g < NGP; ++g) {
        v = fmaf(Gr::q(2 * g) * Gr::Y(2 * g, l * l + m), acc[g].x, v);
        v = fmaf(Gr::q(2 * g + 1) * Gr::Y(2 * g + 1, l * l + m), acc[g].y, v);
      }
      yr[a.out_off[l] + u * (2 * l + 1) + m] = v;
    }
  }
}

// Backward: CTA = one sender, warps as in the forward, out-edges in the stable transpose order.
// Per edge and lane: the receiver's grid row Gq (pairs), the filter S, gF += S Gq; with GW the
// moments sum_g h t^n (n <= LSH) of h = F Gq give the weight gradient, (2l+1) P_l being a
// polynomial in t; with GVEC the direction terms h S'(t) (r_g - t r_hat).
template <int L, int LSH, bool GW, bool GVEC>
__global__ void __launch_bounds__(128) k_gaunt_bwd(const __grid_constant__ GauntArgs a) {
  using Gr = gaunt::Grid<L>;
  constexpr int NGP = Gr::NG / 2;
  extern __shared__ float2 red2[];            // [(split-1) * nsl][NGP][32]
  __shared__ float part[4][32][4][4];         // [phase][edge of the batch][slice][4]: gvec partials
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int st = a.split, sl = wid / st, phase = wid - sl * st;
  const int j = blockIdx.x;
  const int u = sl * 32 + lane;
  const bool act = u < a.mul;
  const int q0 = __ldg(a.colptr + j), q1 = __ldg(a.colptr + j + 1);
  float2 Fj[NGP], gF[NGP];
  {
    const float2* Fr = a.F + ((int64_t)j * a.nsl + sl) * NGP * 32 + lane;
#pragma unroll
    for (int g = 0; g < NGP; ++g) {
      Fj[g] = Fr[g * 32];
      gF[g] = make_float2(0.f, 0.f);
    }
  }
  for (int base = q0 + phase; base < q1; base += 32 * st) {
    const int my_q = base + lane * st;
    int my_e = 0, my_i = 0;
    float vx = 0.f, vy = 0.f, vz = 0.f;
    if (my_q < q1) {
      my_e = __ldg(a.perm + my_q);
      my_i = find_row(a.rowptr, a.N, my_e);
      vx = __ldg(a.vec + 3 * (int64_t)my_e);
      vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
      vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
    }
    const int ne = min(32, (q1 - base + st - 1) / st);
    for (int k = 0; k < ne; ++k) {
      const int e = __shfl_sync(kFull, my_e, k), i = __shfl_sync(kFull, my_i, k);
      float rx, ry, rz, ir;
      edge_geometry(__shfl_sync(kFull, vx, k), __shfl_sync(kFull, vy, k), __shfl_sync(kFull, vz, k), rx, ry, rz, ir);
      float wl[4];
      edge_weights<LSH>(a, e, u, act, ir, wl);
      float hx = 0.f, hy = 0.f, hz = 0.f, hs = 0.f;
      {
        const float2* Gp = a.Gq + ((int64_t)i * a.nsl + sl) * NGP * 32 + lane;
        float2 gq[NGP], t[NGP];
        float cf[4];
#pragma unroll
        for (int g = 0; g < NGP; ++g) gq[g] = Gp[g * 32];
        filter_cubic(wl, cf);
        grid_dots2<Gr>(rx, ry, rz, t);
        float2 M[LSH + 1];
#pragma unroll
        for (int n = 0; n <= LSH; ++n) M[n] = make_float2(0.f, 0.f);
        const float dc[4] = {cf[1], 2.f * cf[2], 3.f * cf[3], 0.f};   // S'(t)
#pragma unroll
        for (int g = 0; g < NGP; ++g) {
          gF[g] = __ffma2_rn(horner2<LSH>(cf, t[g]), gq[g], gF[g]);
          if constexpr (GW || GVEC) {
            const float2 h = __fmul2_rn(Fj[g], gq[g]);
            if constexpr (GW) {
              float2 ht = h;
              M[0] = __fadd2_rn(M[0], ht);
#pragma unroll
              for (int n = 1; n <= LSH; ++n) {
                ht = __fmul2_rn(ht, t[g]);
                M[n] = __fadd2_rn(M[n], ht);
              }
            }
            if constexpr (GVEC && LSH > 0) {
              const float2 c2 = __fmul2_rn(h, horner2<LSH - 1>(dc, t[g]));   // h S'(t)
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                const int gg = 2 * g + hh;
                const float c = hh ? c2.y : c2.x;
                hx = fmaf(c, Gr::st(gg / Gr::NP) * Gr::cp(gg % Gr::NP), hx);
                hy = fmaf(c, Gr::st(gg / Gr::NP) * Gr::sp(gg % Gr::NP), hy);
                hz = fmaf(c, Gr::ct(gg / Gr::NP), hz);
                hs = fmaf(c, hh ? t[g].y : t[g].x, hs);
              }
            }
          }
        }
        if constexpr (GW) {
          float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int n = 0; n <= LSH; ++n) m[n] = M[n].x + M[n].y;
          // (2l+1) P_l(t) = 1, 3t, 7.5t^2 - 2.5, 17.5t^3 - 10.5t
          const float gw[4] = {m[0], 3.f * m[1], fmaf(7.5f, m[2], -2.5f * m[0]), fmaf(17.5f, m[3], -10.5f * m[1])};
          if (act) {
#pragma unroll
            for (int l = 0; l <= LSH; ++l)
              a.gw[(int64_t)e * a.nw + l * a.mul + u] = (l == 0 || ir > 0.f) ? gw[l] : 0.f;
          }
        }
      }
      if constexpr (GVEC) {
        hx = warp_sum(hx);
        hy = warp_sum(hy);
        hz = warp_sum(hz);
        hs = warp_sum(hs);
        if (a.nsl == 1) {
          if (lane == 0) {
            float* gv = a.gvec + 3 * (int64_t)e;
            gv[0] = ir * (hx - rx * hs);
            gv[1] = ir * (hy - ry * hs);
            gv[2] = ir * (hz - rz * hs);
          }
        } else if (lane == 0) {
          part[phase][k][sl][0] = hx;
          part[phase][k][sl][1] = hy;
          part[phase][k][sl][2] = hz;
          part[phase][k][sl][3] = hs;
        }
      }
    }
    if (GVEC && a.nsl > 1) {
      // the slices of this phase have written their partials of the batch's edges
      named_barrier(1 + phase, 32 * a.nsl);
      if (sl == 0 && lane < ne) {
        float h0 = 0.f, h1 = 0.f, h2 = 0.f, h3 = 0.f;
        for (int s2 = 0; s2 < a.nsl; ++s2) {
          h0 += part[phase][lane][s2][0];
          h1 += part[phase][lane][s2][1];
          h2 += part[phase][lane][s2][2];
          h3 += part[phase][lane][s2][3];
        }
        float rx, ry, rz, ir;
        edge_geometry(vx, vy, vz, rx, ry, rz, ir);
        float* gv = a.gvec + 3 * (int64_t)my_e;
        gv[0] = ir * (h0 - rx * h3);
        gv[1] = ir * (h1 - ry * h3);
        gv[2] = ir * (h2 - rz * h3);
      }
      named_barrier(1 + phase, 32 * a.nsl);
    }
  }
  if (st > 1) {
    if (phase > 0) {
      float2* dst = red2 + (((size_t)(phase - 1) * a.nsl + sl) * NGP) * 32 + lane;
#pragma unroll
      for (int g = 0; g < NGP; ++g) dst[g * 32] = gF[g];
    }
    __syncthreads();
    if (phase == 0) {
      for (int ph = 1; ph < st; ++ph) {
        const float2* srcp = red2 + (((size_t)(ph - 1) * a.nsl + sl) * NGP) * 32 + lane;
#pragma unroll
        for (int g = 0; g < NGP; ++g) gF[g] = __fadd2_rn(gF[g], srcp[g * 32]);
      }
    }
  }
  if (!act || !a.gx || phase != 0) return;
  float* gr = a.gx + (int64_t)j * a.in_dim;
#pragma unroll
  for (int l = 0; l <= L; ++l) {
    if (a.in_off[l] < 0) continue;
#pragma unroll
    for (int m = 0; m < 2 * l + 1; ++m) {
      float v = 0.f;
#pragma unroll
      for (int g = 0; g < NGP; ++g) {
        v = fmaf(Gr::Y(2 * g, l * l + m), gF[g].x, v);
        v = fmaf(Gr::Y(2 * g + 1, l * l + m), gF[g].y, v);
      }
      gr[a.in_off[l] + u * (2 * l + 1) + m] = v;
    }
  }
}

unsigned node_grid(int64_t n) {
  int64_t g = (n + 255) / 256;
  if (g > 148 * 32) g = 148 * 32;
  return (unsigned)(g < 1 ? 1 : g);
}

template <int L>
size_t red_bytes(const GauntArgs& a) {
  return sizeof(float2) * (size_t)(a.split - 1) * a.nsl * (gaunt::Grid<L>::NG / 2) * 32;
}

template <int L, int LSH>
cudaError_t gaunt_fwd_seq(const GauntArgs& a, cudaStream_t s) {
  k_gaunt_to_grid<L, 0><<<node_grid((int64_t)a.N * a.nsl * 32), 256, 0, s>>>(a);
  k_gaunt_fwd<L, LSH><<<(unsigned)a.N, 32 * a.nsl * a.split, red_bytes<L>(a), s>>>(a);
  count_launches(2);
  return cudaGetLastError();
}

template <int L, int LSH>
cudaError_t gaunt_bwd_seq(const GauntArgs& a, cudaStream_t s) {
  k_gaunt_to_grid<L, 0><<<node_grid((int64_t)a.N * a.nsl * 32), 256, 0, s>>>(a);
  k_gaunt_to_grid<L, 1><<<node_grid((int64_t)a.N * a.nsl * 32), 256, 0, s>>>(a);
  const unsigned grid = (unsigned)a.N, threads = 32 * a.nsl * a.split;
  const size_t rb = red_bytes<L>(a);
  if (a.gvec) {
    if (a.gw) k_gaunt_bwd<L, LSH, true, true><<<grid, threads, rb, s>>>(a);
    else k_gaunt_bwd<L, LSH, false, true><<<grid, threads, rb, s>>>(a);
  } else {
    if (a.gw) k_gaunt_bwd<L, LSH, true, false><<<grid, threads, rb, s>>>(a);
    else k_gaunt_bwd<L, LSH, false, false><<<grid, threads, rb, s>>>(a);
  }
  count_launches(3);
  return cudaGetLastError();
}

// dispatch over (grid degree L, filter degree LSH <= L)
template <bool FWD>
cudaError_t gaunt_seq(int L, int LSH, const GauntArgs& a, cudaStream_t s) {
#define TP_GAUNT_CASE(LL, SS) \
  if (L == LL && LSH == SS) return FWD ? gaunt_fwd_seq<LL, SS>(a, s) : gaunt_bwd_seq<LL, SS>(a, s);
  TP_GAUNT_CASE(1, 0)
  TP_GAUNT_CASE(1, 1)
  TP_GAUNT_CASE(2, 0)
  TP_GAUNT_CASE(2, 1)
  TP_GAUNT_CASE(2, 2)
  TP_GAUNT_CASE(3, 0)
  TP_GAUNT_CASE(3, 1)
  TP_GAUNT_CASE(3, 2)
  TP_GAUNT_CASE(3, 3)
#undef TP_GAUNT_CASE
  return cudaErrorInvalidValue;
}

size_t al256(size_t v) { return (v + 255) & ~size_t(255); }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace
}  // namespace tp

struct tp_gaunt_s {
  int L, lmax_sh, mul, ng;
  int in_off[4], out_off[4];
  int64_t in_dim, out_dim, nw;
};

namespace {

bool gaunt_irreps(const char* s, int& mul, int (&off)[4], int64_t& dim, std::string& why) {
  std::vector<tp::IrrepTerm> t;
  if (!tp::parse_irreps_terms(s, t, why)) return false;
  for (int& o : off) o = -1;
  mul = t[0].mul;
  dim = 0;
  int last = -1;
  for (const auto& b : t) {
    if (b.l > 3) {
      why = "l > 3";
      return false;
    }
    if (b.parity != ((b.l & 1) ? -1 : 1)) {
      why = "the Gaunt product needs natural parity (-1)^l";
      return false;
    }
    if (b.mul != mul || b.l <= last) {
      why = "one multiplicity and increasing degrees, each at most once";
      return false;
    }
    off[b.l] = (int)dim;
    dim += (int64_t)b.mul * (2 * b.l + 1);
    last = b.l;
  }
  return true;
}

int grid_points(int L) { return L == 1 ? tp::gaunt::Grid<1>::NG : L == 2 ? tp::gaunt::Grid<2>::NG : tp::gaunt::Grid<3>::NG; }

size_t grid_bytes(const tp_gaunt_s* p, int64_t N) {
  return tp::al256(sizeof(float) * (size_t)(N > 0 ? N : 1) * p->ng * 32 * (size_t)((p->mul + 31) / 32));
}

// header 256 | colptr[N+1] | perm[E] | transpose scratch  (the transpose region of the backward)
size_t transpose_bytes(int64_t N, int64_t E) {
  return 256 + tp::al256(sizeof(int32_t) * (size_t)(N + 1)) + tp::al256(sizeof(int32_t) * (size_t)(E > 0 ? E : 1)) +
         tp::al256(sizeof(int32_t) * (size_t)tp::transpose_scratch_ints(N, E));
}

tp::GauntArgs base(const tp_gaunt_s* p, int64_t N, int64_t E) {
  tp::GauntArgs a;
  std::memset(&a, 0, sizeof(a));
  a.N = (int)N;
  a.E = (int)E;
  a.mul = p->mul;
  a.lmax_sh = p->lmax_sh;
  a.nw = (int)p->nw;
  a.in_dim = (int)p->in_dim;
  a.out_dim = (int)p->out_dim;
  a.nsl = (p->mul + 31) / 32;
  // warps per node: up to 4 over the slices and the phases that split the node's edges
  const double avg = N > 0 ? (double)E / (double)N : 0.0;
  a.split = std::max(1, std::min(4 / a.nsl, avg >= 24.0 ? 4 : avg >= 8.0 ? 2 : 1));
  std::memcpy(a.in_off, p->in_off, sizeof(a.in_off));
  std::memcpy(a.out_off, p->out_off, sizeof(a.out_off));
  return a;
}

tp_status_t check_nE(int64_t N, int64_t E) {
  if (N < 0 || E < 0 || N >= (int64_t)1 << 31 || E >= (int64_t)1 << 31)
    return tp::set_failure(TP_ERR_INVALID_ARG, "N and E must be in [0, 2^31)");
  return TP_OK;
}

}  // namespace

extern "C" {

tp_status_t tp_gaunt_create(tp_gaunt_t* plan, const char* irreps_in, int32_t lmax_sh, const char* irreps_out) {
  if (!plan) return tp::set_failure(TP_ERR_INVALID_ARG, "plan out-pointer is NULL");
  *plan = nullptr;
  tp_gaunt_s p;
  std::memset(&p, 0, sizeof(p));
  std::string why;
  int mo = 0;
  if (!gaunt_irreps(irreps_in, p.mul, p.in_off, p.in_dim, why) ||
      !gaunt_irreps(irreps_out, mo, p.out_off, p.out_dim, why))
    return tp::set_failure(why == "l > 3" ? TP_ERR_UNSUPPORTED : TP_ERR_INVALID_ARG, "gaunt irreps: " + why);
  if (mo != p.mul) return tp::set_failure(TP_ERR_INVALID_ARG, "input and output multiplicities differ");
  if (lmax_sh < 0) return tp::set_failure(TP_ERR_INVALID_ARG, "lmax_sh must be >= 0");
  if (lmax_sh > 3) return tp::set_failure(TP_ERR_UNSUPPORTED, "lmax_sh > 3");
  if (p.mul > 128) return tp::set_failure(TP_ERR_UNSUPPORTED, "at most 128 channels");
  int L = lmax_sh;
  for (int l = 0; l < 4; ++l)
    if (p.in_off[l] >= 0 || p.out_off[l] >= 0) L = std::max(L, l);
  p.L = std::max(1, L);
  p.lmax_sh = lmax_sh;
  p.ng = grid_points(p.L);
  p.nw = (int64_t)(lmax_sh + 1) * p.mul;
  tp_gaunt_s* out = new (std::nothrow) tp_gaunt_s(p);
  if (!out) return tp::set_failure(TP_ERR_INVALID_ARG, "out of host memory");
  *plan = out;
  return TP_OK;
}

tp_status_t tp_gaunt_destroy(tp_gaunt_t plan) {
  delete plan;
  return TP_OK;
}

tp_status_t tp_gaunt_query(tp_gaunt_t plan, int64_t* in_dim, int64_t* out_dim, int64_t* n_edge_weights,
                           int32_t* grid_pts) {
  if (!plan) return tp::set_failure(TP_ERR_INVALID_ARG, "plan is NULL");
  if (in_dim) *in_dim = plan->in_dim;
  if (out_dim) *out_dim = plan->out_dim;
  if (n_edge_weights) *n_edge_weights = plan->nw;
  if (grid_pts) *grid_pts = plan->ng;
  return TP_OK;
}

tp_status_t tp_gaunt_workspace_size(tp_gaunt_t plan, int64_t N, int64_t E, int32_t op, size_t* bytes) {
  if (!plan || !bytes) return tp::set_failure(TP_ERR_INVALID_ARG, "plan and bytes must not be NULL");
  tp_status_t st = check_nE(N, E);
  if (st != TP_OK) return st;
  if (op == TP_OP_FWD) *bytes = grid_bytes(plan, N);
  else if (op == TP_OP_BWD) *bytes = 2 * grid_bytes(plan, N) + transpose_bytes(N, E);
  else return tp::set_failure(TP_ERR_UNSUPPORTED, "the Gaunt convolution has forward and backward");
  return TP_OK;
}

tp_status_t tp_gaunt_fwd(tp_gaunt_t plan, int64_t N, int64_t E, const int32_t* rowptr, const int32_t* src,
                         const float* x, const float* vec, const float* w, float* y, void* ws, size_t ws_bytes,
                         tp_stream_t stream) {
  if (!plan) return tp::set_failure(TP_ERR_INVALID_ARG, "plan is NULL");
  tp_status_t st = check_nE(N, E);
  if (st != TP_OK) return st;
  if (N == 0) return TP_OK;
  if (!rowptr || !y || !x || (E > 0 && (!src || !vec || !w)))
    return tp::set_failure(TP_ERR_INVALID_ARG, "NULL input or output");
  for (const void* p : {(const void*)rowptr, (const void*)src, (const void*)x, (const void*)vec, (const void*)w,
                        (const void*)y, (const void*)ws})
    if (!tp::aligned4(p)) return tp::set_failure(TP_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  if (!ws || ws_bytes < grid_bytes(plan, N)) return tp::set_failure(TP_ERR_WORKSPACE, "workspace too small");
  tp::GauntArgs a = base(plan, N, E);
  a.rowptr = rowptr;
  a.src = src;
  a.x = x;
  a.vec = vec;
  a.w = w;
  a.y = y;
  a.F = static_cast<float2*>(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = tp::gaunt_seq<true>(plan->L, plan->lmax_sh, a, s);
  if (e != cudaSuccess) return tp::set_failure(TP_ERR_CUDA, std::string("tp_gaunt_fwd: ") + cudaGetErrorString(e));
  return TP_OK;
}

tp_status_t tp_gaunt_bwd(tp_gaunt_t plan, int64_t N, int64_t E, const int32_t* rowptr, const int32_t* src,
                         const int32_t* colptr, const int32_t* perm, const float* x, const float* vec,
                         const float* w, const float* gy, float* gx, float* gw, float* gvec, void* ws,
                         size_t ws_bytes, tp_stream_t stream) {
  if (!plan) return tp::set_failure(TP_ERR_INVALID_ARG, "plan is NULL");
  tp_status_t st = check_nE(N, E);
  if (st != TP_OK) return st;
  if (N == 0 || (!gx && !gw && !gvec)) return TP_OK;
  if (!rowptr || !x || !gy || (E > 0 && (!src || !vec || !w)))
    return tp::set_failure(TP_ERR_INVALID_ARG, "NULL input");
  if ((colptr == nullptr) != (perm == nullptr))
    return tp::set_failure(TP_ERR_INVALID_ARG, "colptr and perm must both be given or both be NULL");
  for (const void* p : {(const void*)rowptr, (const void*)src, (const void*)colptr, (const void*)perm, (const void*)x,
                        (const void*)vec, (const void*)w, (const void*)gy, (const void*)gx, (const void*)gw,
                        (const void*)gvec, (const void*)ws})
    if (!tp::aligned4(p)) return tp::set_failure(TP_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  size_t need = 0;
  tp_gaunt_workspace_size(plan, N, E, TP_OP_BWD, &need);
  if (!ws || ws_bytes < need) return tp::set_failure(TP_ERR_WORKSPACE, "workspace too small");
  char* wsb = static_cast<char*>(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t gb = grid_bytes(plan, N);
  if (!colptr) {
    char* t = wsb + 2 * gb;
    int32_t* cp = reinterpret_cast<int32_t*>(t + 256);
    int32_t* pm = reinterpret_cast<int32_t*>(t + 256 + tp::al256(sizeof(int32_t) * (size_t)(N + 1)));
    int32_t* sc = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(pm) + tp::al256(sizeof(int32_t) * (size_t)(E > 0 ? E : 1)));
    cudaError_t e = tp::launch_csr_transpose((int)N, (int)E, src, cp, pm, sc, s);
    if (e != cudaSuccess) return tp::set_failure(TP_ERR_CUDA, std::string("transpose: ") + cudaGetErrorString(e));
    colptr = cp;
    perm = pm;
  }
  tp::GauntArgs a = base(plan, N, E);
  a.rowptr = rowptr;
  a.src = src;
  a.colptr = colptr;
  a.perm = perm;
  a.x = x;
  a.vec = vec;
  a.w = w;
  a.gy = gy;
  a.gx = gx;
  a.gw = gw;
  a.gvec = gvec;
  a.F = reinterpret_cast<float2*>(wsb);
  a.Gq = reinterpret_cast<float2*>(wsb + gb);
  cudaError_t e = tp::gaunt_seq<false>(plan->L, plan->lmax_sh, a, s);
  if (e != cudaSuccess) return tp::set_failure(TP_ERR_CUDA, std::string("tp_gaunt_bwd: ") + cudaGetErrorString(e));
  return TP_OK;
}

}  // extern "C"
