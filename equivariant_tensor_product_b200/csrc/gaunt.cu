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
// Grid rows are node sized; nothing per edge is stored.  One warp per 32-channel slice of a
// node, every warp of a CTA walking the node's edges in order; sums in fixed order.
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
  float *F, *Gq;               // [N][NG][mul]
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

// t_g = r_hat . r_g for every grid point, from the grid's product structure: r_g has
// cos(theta) = ct(k), sin(theta) = st(k) and azimuth phi_j, so t = rz ct(k) + st(k) (rx cos phi_j + ry sin phi_j).
template <class Gr>
__device__ __forceinline__ void grid_dots(float rx, float ry, float rz, float (&t)[Gr::NG]) {
  float c[Gr::NP];
#pragma unroll
  for (int j = 0; j < Gr::NP; ++j) c[j] = fmaf(rx, Gr::cp(j), ry * Gr::sp(j));
#pragma unroll
  for (int k = 0; k < Gr::NT; ++k) {
    const float z = rz * Gr::ct(k);
#pragma unroll
    for (int j = 0; j < Gr::NP; ++j) t[k * Gr::NP + j] = fmaf(Gr::st(k), c[j], z);
  }
}

// MODE 0: F from x (input blocks); MODE 1: Gq from gy (output blocks, times q_g).  One thread
// per (node, channel).
template <int L, int MODE>
__global__ void __launch_bounds__(256) k_gaunt_to_grid(const __grid_constant__ GauntArgs a) {
  using Gr = gaunt::Grid<L>;
  const int64_t total = (int64_t)a.N * a.mul;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = t / a.mul;
    const int u = (int)(t - j * a.mul);
    const float* row = MODE == 0 ? a.x + j * a.in_dim : a.gy + j * a.out_dim;
    const int* off = MODE == 0 ? a.in_off : a.out_off;
    float c[Gr::NSH];
#pragma unroll
    for (int l = 0; l <= L; ++l) {
#pragma unroll
      for (int m = 0; m < 2 * l + 1; ++m)
        c[l * l + m] = off[l] >= 0 ? __ldg(row + off[l] + u * (2 * l + 1) + m) : 0.f;
    }
    float* out = (MODE == 0 ? a.F : a.Gq) + j * (int64_t)Gr::NG * a.mul + u;
#pragma unroll
    for (int g = 0; g < Gr::NG; ++g) {
      float v = 0.f;
#pragma unroll
      for (int k = 0; k < Gr::NSH; ++k) v = fmaf(c[k], Gr::Y(g, k), v);
      out[(int64_t)g * a.mul] = MODE == 1 ? Gr::q(g) * v : v;
    }
  }
}

// w_l2 (2l2+1 folded into E) of edge e for channel u; filter degrees above lmax_sh read as 0,
// degrees above 0 of a zero-length edge too (its harmonics are Y_0 = 1, Y_l>0 = 0)
__device__ __forceinline__ void edge_weights(const GauntArgs& a, int e, int u, bool act, float ir, float (&wl)[4]) {
#pragma unroll
  for (int l = 0; l < 4; ++l)
    wl[l] = (act && l <= a.lmax_sh && (l == 0 || ir > 0.f)) ? __ldg(a.w + (int64_t)e * a.nw + l * a.mul + u) : 0.f;
}

// Forward: CTA = one receiver; warp w = (slice w / split, phase w % split); the phases take
// interleaved edges of the row and their grid accumulators are added through shared memory in
// phase order.  Each edge's grid row F[src][.][u] is loaded in one batch before the pointwise
// math.
template <int L>
__global__ void __launch_bounds__(128) k_gaunt_fwd(const __grid_constant__ GauntArgs a) {
  using Gr = gaunt::Grid<L>;
  extern __shared__ float red[];             // [(split-1) * nsl][NG][32]
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int st = a.split, sl = wid / st, phase = wid - sl * st;
  const int i = blockIdx.x;
  const int u = sl * 32 + lane;
  const bool act = u < a.mul;
  const int e0 = __ldg(a.rowptr + i), e1 = __ldg(a.rowptr + i + 1);
  float acc[Gr::NG];
#pragma unroll
  for (int g = 0; g < Gr::NG; ++g) acc[g] = 0.f;
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
    if constexpr (Gr::NG <= 32) {
      // small grids: the row of edge k + 1 is loaded while edge k is computed (a larger grid
      // would not fit two rows in registers)
      float fn[Gr::NG];
      {
        const int j0 = __shfl_sync(kFull, my_j, 0);
#pragma unroll
        for (int g = 0; g < Gr::NG; ++g) fn[g] = act ? __ldg(a.F + ((int64_t)j0 * Gr::NG + g) * a.mul + u) : 0.f;
      }
      for (int k = 0; k < ne; ++k) {
        float f[Gr::NG];
#pragma unroll
        for (int g = 0; g < Gr::NG; ++g) f[g] = fn[g];
        const int jn = __shfl_sync(kFull, my_j, min(k + 1, 31));
        if (act && k + 1 < ne) {
#pragma unroll
          for (int g = 0; g < Gr::NG; ++g) fn[g] = __ldg(a.F + ((int64_t)jn * Gr::NG + g) * a.mul + u);
        }
        float rx, ry, rz, ir;
        edge_geometry(__shfl_sync(kFull, vx, k), __shfl_sync(kFull, vy, k), __shfl_sync(kFull, vz, k), rx, ry, rz, ir);
        if (!act) continue;
        float wl[4], cf[4], tg[Gr::NG];
        edge_weights(a, base + k * st, u, act, ir, wl);
        filter_cubic(wl, cf);
        grid_dots<Gr>(rx, ry, rz, tg);
#pragma unroll
        for (int g = 0; g < Gr::NG; ++g) {
          const float s = fmaf(fmaf(fmaf(cf[3], tg[g], cf[2]), tg[g], cf[1]), tg[g], cf[0]);
          acc[g] = fmaf(f[g], s, acc[g]);
        }
      }
    } else {
      for (int k = 0; k < ne; ++k) {
        const int j = __shfl_sync(kFull, my_j, k);
        float rx, ry, rz, ir;
        edge_geometry(__shfl_sync(kFull, vx, k), __shfl_sync(kFull, vy, k), __shfl_sync(kFull, vz, k), rx, ry, rz, ir);
        if (!act) continue;
        float wl[4], cf[4], tg[Gr::NG];
        edge_weights(a, base + k * st, u, act, ir, wl);
        filter_cubic(wl, cf);
        const float* Fr = a.F + (int64_t)j * Gr::NG * a.mul + u;
        float f[Gr::NG];
#pragma unroll
        for (int g = 0; g < Gr::NG; ++g) f[g] = __ldg(Fr + (int64_t)g * a.mul);
        grid_dots<Gr>(rx, ry, rz, tg);
#pragma unroll
        for (int g = 0; g < Gr::NG; ++g) {
          const float s = fmaf(fmaf(fmaf(cf[3], tg[g], cf[2]), tg[g], cf[1]), tg[g], cf[0]);
          acc[g] = fmaf(f[g], s, acc[g]);
        }
      }
    }
  }
  if (st > 1) {
    if (phase > 0) {
      float* dst = red + (((size_t)(phase - 1) * a.nsl + sl) * Gr::NG) * 32 + lane;
#pragma unroll
      for (int g = 0; g < Gr::NG; ++g) dst[g * 32] = acc[g];
    }
    __syncthreads();
    if (phase == 0) {
      for (int ph = 1; ph < st; ++ph) {
        const float* srcp = red + (((size_t)(ph - 1) * a.nsl + sl) * Gr::NG) * 32 + lane;
#pragma unroll
        for (int g = 0; g < Gr::NG; ++g) acc[g] += srcp[g * 32];
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
      for (int g = 0; g < Gr::NG; ++g) v = fmaf(Gr::q(g) * Gr::Y(g, l * l + m), acc[g], v);
      yr[a.out_off[l] + u * (2 * l + 1) + m] = v;
    }
  }
}

// Backward: CTA = one sender, warps as in the forward, out-edges in the stable transpose order.
template <int L>
__global__ void __launch_bounds__(128) k_gaunt_bwd(const __grid_constant__ GauntArgs a) {
  using Gr = gaunt::Grid<L>;
  extern __shared__ float red[];             // [(split-1) * nsl][NG][32]
  __shared__ float part[4][32][4][4];        // [phase][edge of the batch][slice][4]: gvec partials
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int st = a.split, sl = wid / st, phase = wid - sl * st;
  const int j = blockIdx.x;
  const int u = sl * 32 + lane;
  const bool act = u < a.mul;
  const int q0 = __ldg(a.colptr + j), q1 = __ldg(a.colptr + j + 1);
  float Fj[Gr::NG], gF[Gr::NG];
  const float* Fr = a.F + (int64_t)j * Gr::NG * a.mul + u;
#pragma unroll
  for (int g = 0; g < Gr::NG; ++g) {
    Fj[g] = act ? __ldg(Fr + (int64_t)g * a.mul) : 0.f;
    gF[g] = 0.f;
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
      edge_weights(a, e, u, act, ir, wl);
      float gw[4] = {0.f, 0.f, 0.f, 0.f};
      float hx = 0.f, hy = 0.f, hz = 0.f, hs = 0.f;
      if (act) {
        const float* Gp = a.Gq + (int64_t)i * Gr::NG * a.mul + u;
        float gq[Gr::NG], tg[Gr::NG], cf[4];
#pragma unroll
        for (int g = 0; g < Gr::NG; ++g) gq[g] = __ldg(Gp + (int64_t)g * a.mul);
        filter_cubic(wl, cf);
        grid_dots<Gr>(rx, ry, rz, tg);
        // moments sum_g h t^n give the weight gradient: (2l+1) P_l(t) is a cubic in t
        float M0 = 0.f, M1 = 0.f, M2 = 0.f, M3 = 0.f;
#pragma unroll
        for (int g = 0; g < Gr::NG; ++g) {
          const float t = tg[g];
          const float s = fmaf(fmaf(fmaf(cf[3], t, cf[2]), t, cf[1]), t, cf[0]);
          gF[g] = fmaf(s, gq[g], gF[g]);
          const float h = Fj[g] * gq[g];
          const float ht = h * t, ht2 = ht * t;
          M0 += h;
          M1 += ht;
          M2 += ht2;
          M3 = fmaf(ht2, t, M3);
          const float c = h * fmaf(fmaf(3.f * cf[3], t, 2.f * cf[2]), t, cf[1]);   // h s'(t)
          hx = fmaf(c, Gr::st(g / Gr::NP) * Gr::cp(g % Gr::NP), hx);
          hy = fmaf(c, Gr::st(g / Gr::NP) * Gr::sp(g % Gr::NP), hy);
          hz = fmaf(c, Gr::ct(g / Gr::NP), hz);
          hs = fmaf(c, t, hs);
        }
        gw[0] = M0;
        gw[1] = 3.f * M1;
        gw[2] = fmaf(7.5f, M2, -2.5f * M0);
        gw[3] = fmaf(17.5f, M3, -10.5f * M1);
        if (a.gw) {
          for (int l = 0; l <= a.lmax_sh; ++l)
            a.gw[(int64_t)e * a.nw + l * a.mul + u] = (l == 0 || ir > 0.f) ? gw[l] : 0.f;
        }
      }
      if (a.gvec) {
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
    if (a.gvec && a.nsl > 1) {
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
      float* dst = red + (((size_t)(phase - 1) * a.nsl + sl) * Gr::NG) * 32 + lane;
#pragma unroll
      for (int g = 0; g < Gr::NG; ++g) dst[g * 32] = gF[g];
    }
    __syncthreads();
    if (phase == 0) {
      for (int ph = 1; ph < st; ++ph) {
        const float* srcp = red + (((size_t)(ph - 1) * a.nsl + sl) * Gr::NG) * 32 + lane;
#pragma unroll
        for (int g = 0; g < Gr::NG; ++g) gF[g] += srcp[g * 32];
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
      for (int g = 0; g < Gr::NG; ++g) v = fmaf(Gr::Y(g, l * l + m), gF[g], v);
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
  return sizeof(float) * (size_t)(a.split - 1) * a.nsl * gaunt::Grid<L>::NG * 32;
}

template <int L>
cudaError_t gaunt_fwd_seq(const GauntArgs& a, cudaStream_t s) {
  k_gaunt_to_grid<L, 0><<<node_grid((int64_t)a.N * a.mul), 256, 0, s>>>(a);
  k_gaunt_fwd<L><<<(unsigned)a.N, 32 * a.nsl * a.split, red_bytes<L>(a), s>>>(a);
  count_launches(2);
  return cudaGetLastError();
}

template <int L>
cudaError_t gaunt_bwd_seq(const GauntArgs& a, cudaStream_t s) {
  k_gaunt_to_grid<L, 0><<<node_grid((int64_t)a.N * a.mul), 256, 0, s>>>(a);
  k_gaunt_to_grid<L, 1><<<node_grid((int64_t)a.N * a.mul), 256, 0, s>>>(a);
  k_gaunt_bwd<L><<<(unsigned)a.N, 32 * a.nsl * a.split, red_bytes<L>(a), s>>>(a);
  count_launches(3);
  return cudaGetLastError();
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

size_t grid_bytes(const tp_gaunt_s* p, int64_t N) { return tp::al256(sizeof(float) * (size_t)(N > 0 ? N : 1) * p->ng * p->mul); }

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
  a.F = static_cast<float*>(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = plan->L == 1 ? tp::gaunt_fwd_seq<1>(a, s) : plan->L == 2 ? tp::gaunt_fwd_seq<2>(a, s)
                                                                            : tp::gaunt_fwd_seq<3>(a, s);
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
  a.F = reinterpret_cast<float*>(wsb);
  a.Gq = reinterpret_cast<float*>(wsb + gb);
  cudaError_t e = plan->L == 1 ? tp::gaunt_bwd_seq<1>(a, s) : plan->L == 2 ? tp::gaunt_bwd_seq<2>(a, s)
                                                                            : tp::gaunt_bwd_seq<3>(a, s);
  if (e != cudaSuccess) return tp::set_failure(TP_ERR_CUDA, std::string("tp_gaunt_bwd: ") + cudaGetErrorString(e));
  return TP_OK;
}

}  // extern "C"
