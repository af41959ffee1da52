// Fused-radial-projection passes for plans that run a compiled whole path list (all paths of
// lmax 2 or 3, one multiplicity): the chunk schedule of radial.cu (project the chunk's weights
// w = h W_r into shared memory, stage the per-edge rows) with the coupling of the compiled
// kernels -- every path of an edge in one generated chain over the non-zero Clebsch-Gordan
// entries, the x (x) Y products shared by the paths of each (l1, l2) pair ("FlashTP", abstract:
// path-aggregated execution) -- instead of the path table's chain per path.
//   k_rad_fwd_spec   one CTA per receiver: warp = (32-channel slice, edge phase); the senders'
//                    x rows read from L2; each warp keeps its row sums in registers across
//                    chunks; phases are summed through shared memory in phase order at the end.
//   k_rad_send_spec  one CTA per sender: the same warps; gx in registers, the receivers' gy
//                    rows read from L2, the chunk's gw written over its w in shared memory (then
//                    gh as in radial.cu), gvec per edge from the generated SH-gradient sums,
//                    reduced over lanes and then over slices in slice order.
#include "radial.cuh"
#include "spec_full_l2.h"
#include "spec_full_l3.h"

namespace tp {
namespace {

using namespace rad;

// Shared memory of the compiled-list forward: hs [H][CE + 4] | ws [CE][nwp] | Ys [CE][16] |
// es, ns [CE]; the senders' x rows are read from L2 by the coupling.
__host__ __device__ inline size_t fwd_smem_floats(int H, int CE, int nwp) {
  return (size_t)H * (CE + 4) + (size_t)CE * nwp + 16 * (size_t)CE + 2 * round4(CE);
}

template <int CE>
__device__ __forceinline__ RadSmem fwd_smem(float* base, const RadArgs& a) {
  RadSmem s;
  s.hs = base;
  s.ws = s.hs + a.H * (CE + 4);
  s.gs = s.vs = s.xn = s.rs = nullptr;
  s.Ys = s.ws + CE * a.nwp;
  s.es = reinterpret_cast<int*>(s.Ys + CE * 16);
  s.ns = s.es + round4(CE);
  return s;
}

template <class S, int CE>
__global__ void __launch_bounds__(kRadThreads, 2) k_rad_fwd_spec(const __grid_constant__ RadArgs a,
                                                                 const __grid_constant__ GenTable T) {
  extern __shared__ float4 rad_smem_raw[];
  const RadSmem s = fwd_smem<CE>(reinterpret_cast<float*>(rad_smem_raw), a);
  const int row = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nsl = (a.mul + 31) >> 5, phases = kRadWarps / nsl;
  const int sl = warp % nsl, ph = warp / nsl;
  const bool busy = ph < phases;
  const int c = sl * 32 + lane;
  const bool act = busy && c < a.mul;
  int e0 = __ldg(a.rowptr + row), e1 = __ldg(a.rowptr + row + 1);
  if (a.check) {
    e0 = max(0, min(e0, a.E));
    e1 = max(e0, min(e1, a.E));
  }
  float acc[S::OUT_PC];
#pragma unroll
  for (int k = 0; k < S::OUT_PC; ++k) acc[k] = 0.f;
  for (int c0 = e0; c0 < e1; c0 += CE) {
    const int ne = min(CE, e1 - c0);
    __syncthreads();
    if (threadIdx.x < CE) {
      const int r = threadIdx.x;
      int e = -1, j = -1;
      float Y[S::NSH];
#pragma unroll
      for (int m = 0; m < S::NSH; ++m) Y[m] = 0.f;
      if (r < ne) {
        e = c0 + r;
        j = __ldg(a.src + e);
        if (a.check && (unsigned)j >= (unsigned)a.N) {
          rad_report(a, kDevBadSrc);
          e = j = -1;
        } else {
          float rx, ry, rz, ir;
          edge_geometry(__ldg(a.vec + 3 * (int64_t)e), __ldg(a.vec + 3 * (int64_t)e + 1),
                        __ldg(a.vec + 3 * (int64_t)e + 2), rx, ry, rz, ir);
          S::sh(rx, ry, rz, Y);
        }
      }
      s.es[r] = e;
      s.ns[r] = j;
#pragma unroll
      for (int m = 0; m < S::NSH; ++m) s.Ys[r * 16 + m] = Y[m];
    }
    __syncthreads();
    stage_chunk<CE>(a, s, ne, a.x, 0);     // the hidden rows only; x rows are read from L2
    __syncthreads();
    project<CE>(a, s);
    __syncthreads();
    if (act) {
      for (int r = ph; r < ne; r += phases) {
        if (s.es[r] < 0) continue;
        float xa[S::IN_PC], wa[S::P], Y[S::NSH];
        S::load_in(a.x + (int64_t)s.ns[r] * a.in_dim, a.mul, c, xa);
        const float* wr = s.ws + r * a.nwp + c;
#pragma unroll
        for (int p = 0; p < S::P; ++p) wa[p] = T.path[p].coeff * wr[p * a.mul];
#pragma unroll
        for (int m = 0; m < S::NSH; ++m) Y[m] = s.Ys[r * 16 + m];
        S::fwd(xa, Y, wa, acc);
      }
    }
  }
  // phase sums through the weight tile (free now), added in phase order
  __syncthreads();
  float* red = s.ws;
  if (busy && ph > 0) {
    float* dst = red + ((size_t)((ph - 1) * nsl + sl) * S::OUT_PC) * 32 + lane;
#pragma unroll
    for (int k = 0; k < S::OUT_PC; ++k) dst[k * 32] = acc[k];
  }
  __syncthreads();
  if (busy && ph == 0) {
    for (int q = 1; q < phases; ++q) {
      const float* src = red + ((size_t)((q - 1) * nsl + sl) * S::OUT_PC) * 32 + lane;
#pragma unroll
      for (int k = 0; k < S::OUT_PC; ++k) acc[k] += src[k * 32];
    }
    if (c < a.mul) S::store_out(a.y + (int64_t)row * a.out_dim, a.mul, c, acc);
  }
}

// Shared memory of the compiled-list sender pass: hs [H][CE + 4] | ws [CE][nwp] (the chunk's w,
// overwritten in place by its gw) | gvec partials [CE][8][4] | Ys [CE][16] | es, ns [CE].  The
// receivers' gy rows are read from L2 by the coupling, so one weight tile of 32 edges fits
// two CTAs per SM.
__host__ __device__ inline size_t send_smem_floats(int H, int CE, int nwp) {
  return (size_t)H * (CE + 4) + (size_t)CE * nwp + 32 * (size_t)CE + 16 * (size_t)CE + 2 * round4(CE) +
         32 * (size_t)H;
}

template <int CE>
__device__ __forceinline__ RadSmem send_smem(float* base, const RadArgs& a) {
  RadSmem s;
  s.hs = base;
  s.ws = s.hs + a.H * (CE + 4);
  s.gs = s.ws;
  s.vs = s.xn = nullptr;
  s.rs = s.ws + CE * a.nwp;
  s.Ys = s.rs + 32 * CE;
  s.es = reinterpret_cast<int*>(s.Ys + CE * 16);
  s.ns = s.es + round4(CE);
  s.xn = reinterpret_cast<float*>(s.ns + round4(CE));   // gh column-part sums [32 H]
  return s;
}

template <class S, int CE, bool GVEC>
__global__ void __launch_bounds__(kRadThreads, 2) k_rad_send_spec(const __grid_constant__ RadArgs a,
                                                                  const __grid_constant__ GenTable T) {
  extern __shared__ float4 rad_smem_raw[];
  const RadSmem s = send_smem<CE>(reinterpret_cast<float*>(rad_smem_raw), a);
  const int node = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nsl = (a.mul + 31) >> 5, phases = kRadWarps / nsl;
  const int sl = warp % nsl, ph = warp / nsl;
  const bool busy = ph < phases;
  const int c = sl * 32 + lane;
  const bool act = busy && c < a.mul;
  int q0 = __ldg(a.colptr + node), q1 = __ldg(a.colptr + node + 1);
  if (a.check) {
    q0 = max(0, min(q0, a.E));
    q1 = max(q0, min(q1, a.E));
  }
  float xr[S::IN_PC], gx[S::IN_PC];
#pragma unroll
  for (int k = 0; k < S::IN_PC; ++k) gx[k] = xr[k] = 0.f;
  if (act) S::load_in(a.x + (int64_t)node * a.in_dim, a.mul, c, xr);
  float* gvp = s.rs;                       // gvec partials [CE][nsl][4] (gx lives in registers)
  for (int c0 = q0; c0 < q1; c0 += CE) {
    const int ne = min(CE, q1 - c0);
    __syncthreads();
    if (threadIdx.x < CE) {
      const int r = threadIdx.x;
      int e = -1, i = 0;
      float Y[S::NSH];
#pragma unroll
      for (int m = 0; m < S::NSH; ++m) Y[m] = 0.f;
      if (r < ne) {
        e = __ldg(a.perm + c0 + r);
        if (a.check && (unsigned)e >= (unsigned)a.E) {
          rad_report(a, kDevBadPerm);
          e = -1;
        } else {
          i = find_row(a.rowptr, a.N, e);
          float rx, ry, rz, ir;
          edge_geometry(__ldg(a.vec + 3 * (int64_t)e), __ldg(a.vec + 3 * (int64_t)e + 1),
                        __ldg(a.vec + 3 * (int64_t)e + 2), rx, ry, rz, ir);
          S::sh(rx, ry, rz, Y);
        }
      }
      s.es[r] = e;
      s.ns[r] = i;
#pragma unroll
      for (int m = 0; m < S::NSH; ++m) s.Ys[r * 16 + m] = Y[m];
    }
    __syncthreads();
    stage_chunk<CE>(a, s, ne, a.gy, 0);    // the hidden rows only; gy rows are read from L2
    __syncthreads();
    project<CE>(a, s);
    __syncthreads();
    if (busy) {
      for (int r = ph; r < ne; r += phases) {
        const int e = s.es[r];
        if (e < 0) continue;               // warp-uniform
        float Y[S::NSH], gY[S::NSH];
#pragma unroll
        for (int m = 0; m < S::NSH; ++m) {
          Y[m] = s.Ys[r * 16 + m];
          gY[m] = 0.f;
        }
        if (act) {
          float gya[S::OUT_PC], wa[S::P], gw[S::P];
          S::load_out(a.gy + (int64_t)s.ns[r] * a.out_dim, a.mul, c, gya);
          const float* wr = s.ws + r * a.nwp + c;
#pragma unroll
          for (int p = 0; p < S::P; ++p) wa[p] = T.path[p].coeff * wr[p * a.mul];
          S::template bwd<GVEC>(xr, Y, wa, gya, gx, gw, gY);
          // gw overwrites w in place: this lane's entries of edge r are read above and by nobody else
          float* gr = s.gs + r * a.nwp + c;
#pragma unroll
          for (int p = 0; p < S::P; ++p) gr[p * a.mul] = T.path[p].coeff * gw[p];
        }
        if constexpr (GVEC) {
          float rx, ry, rz, ir;
          edge_geometry(__ldg(a.vec + 3 * (int64_t)e), __ldg(a.vec + 3 * (int64_t)e + 1),
                        __ldg(a.vec + 3 * (int64_t)e + 2), rx, ry, rz, ir);
          float G[S::NSH][3];
          S::sh_grad(rx, ry, rz, G);
          float h0 = 0.f, h1 = 0.f, h2 = 0.f, sdeg = 0.f;
#pragma unroll
          for (int m = 0; m < S::NSH; ++m) {
            h0 = fmaf(gY[m], G[m][0], h0);
            h1 = fmaf(gY[m], G[m][1], h1);
            h2 = fmaf(gY[m], G[m][2], h2);
            sdeg = fmaf(S::sh_degree(m) * gY[m], Y[m], sdeg);
          }
          h0 = warp_sum(h0);
          h1 = warp_sum(h1);
          h2 = warp_sum(h2);
          sdeg = warp_sum(sdeg);
          if (lane == 0) {
            float* g = gvp + (r * nsl + sl) * 4;
            g[0] = h0;
            g[1] = h1;
            g[2] = h2;
            g[3] = sdeg;
          }
        }
      }
    }
    __syncthreads();
    if (GVEC && a.gvec && threadIdx.x < ne) {
      const int r = threadIdx.x, e = s.es[r];
      if (e >= 0) {
        float h0 = 0.f, h1 = 0.f, h2 = 0.f, sdeg = 0.f;
        for (int q = 0; q < nsl; ++q) {
          const float* g = gvp + (r * nsl + q) * 4;
          h0 += g[0];
          h1 += g[1];
          h2 += g[2];
          sdeg += g[3];
        }
        float rx, ry, rz, ir;
        edge_geometry(__ldg(a.vec + 3 * (int64_t)e), __ldg(a.vec + 3 * (int64_t)e + 1),
                      __ldg(a.vec + 3 * (int64_t)e + 2), rx, ry, rz, ir);
        float* g = a.gvec + 3 * (int64_t)e;
        g[0] = ir * (h0 - rx * sdeg);
        g[1] = ir * (h1 - ry * sdeg);
        g[2] = ir * (h2 - rz * sdeg);
      }
    }
    if (a.gh) {
      if (CE < 4 * kRadWarps && ((reinterpret_cast<uintptr_t>(a.WrT) | reinterpret_cast<uintptr_t>(a.gh)) & 7u) == 0)
        gh_chunk_split<CE>(a, s, ne, s.xn);
      else
        gh_chunk<CE>(a, s, ne);
    }
  }
  // phase sums of gx through the weight tile, added in phase order
  __syncthreads();
  float* red = s.ws;
  if (busy && ph > 0) {
    float* dst = red + ((size_t)((ph - 1) * nsl + sl) * S::IN_PC) * 32 + lane;
#pragma unroll
    for (int k = 0; k < S::IN_PC; ++k) dst[k * 32] = gx[k];
  }
  __syncthreads();
  if (busy && ph == 0) {
    for (int q = 1; q < phases; ++q) {
      const float* src = red + ((size_t)((q - 1) * nsl + sl) * S::IN_PC) * 32 + lane;
#pragma unroll
      for (int k = 0; k < S::IN_PC; ++k) gx[k] += src[k * 32];
    }
    if (a.gx && c < a.mul) S::store_in(a.gx + (int64_t)node * a.in_dim, a.mul, c, gx);
  }
}

template <class K>
cudaError_t spec_launch(K kern, size_t smem, cudaStream_t s, const RadArgs& a, const GenTable& T) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)a.N, kRadThreads, smem, s>>>(a, T);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rad_fwd_spec(const RadArgs& a, const GenTable& T, int ce, size_t smem, cudaStream_t s,
                                bool* handled) {
  (void)ce;
  (void)smem;
  *handled = false;
  if (a.spec != 2 && a.spec != 3) return cudaSuccess;
  // this pass's own chunk: the largest instantiated size whose weight tile fits the tile budget
  const int sizes[2][3] = {{32, 16, 16}, {16, 8, 4}};
  int c2 = 0;
  for (int q = 0; q < 3 && !c2; ++q) {
    const int v = sizes[a.spec - 2][q];
    if ((size_t)v * a.nwp * 4 <= (size_t)kRadTileBudget || q == 2) c2 = v;
  }
  const size_t sm = sizeof(float) * fwd_smem_floats(a.H, c2, a.nwp);
  const int nsl = (a.mul + 31) / 32;
  if (sm > (size_t)kRadSmemBudget || nsl < 1 || nsl > kRadWarps) return cudaSuccess;
  const int phases = kRadWarps / nsl;
  const size_t red = (size_t)(phases - 1) * nsl * (a.spec == 2 ? Spec_full_l2::OUT_PC : Spec_full_l3::OUT_PC) * 32;
  if (red > (size_t)c2 * a.nwp) return cudaSuccess;
  *handled = true;
  if (a.spec == 2) {
    if (c2 == 32) return spec_launch(k_rad_fwd_spec<Spec_full_l2, 32>, sm, s, a, T);
    return spec_launch(k_rad_fwd_spec<Spec_full_l2, 16>, sm, s, a, T);
  }
  if (c2 == 16) return spec_launch(k_rad_fwd_spec<Spec_full_l3, 16>, sm, s, a, T);
  if (c2 == 8) return spec_launch(k_rad_fwd_spec<Spec_full_l3, 8>, sm, s, a, T);
  return spec_launch(k_rad_fwd_spec<Spec_full_l3, 4>, sm, s, a, T);
}

cudaError_t launch_rad_send_spec(const RadArgs& a, const GenTable& T, int ce, size_t smem, cudaStream_t s,
                                 bool* handled) {
  (void)ce;
  (void)smem;
  *handled = false;
  if (a.spec != 2 && a.spec != 3) return cudaSuccess;
  // this pass's own chunk: the largest instantiated size whose weight tile fits the tile budget
  const int sizes[2][2] = {{32, 16}, {8, 4}};
  int c2 = 0;
  for (int q = 0; q < 2 && !c2; ++q) {
    const int v = sizes[a.spec - 2][q];
    if ((size_t)v * a.nwp * 4 <= (size_t)kRadTileBudget || q == 1) c2 = v;
  }
  const size_t sm = sizeof(float) * send_smem_floats(a.H, c2, a.nwp);
  const int nsl = (a.mul + 31) / 32;
  if (sm > (size_t)kRadSmemBudget || nsl < 1 || nsl > kRadWarps) return cudaSuccess;
  const int phases = kRadWarps / nsl;
  const size_t red = (size_t)(phases - 1) * nsl * (a.spec == 2 ? Spec_full_l2::IN_PC : Spec_full_l3::IN_PC) * 32;
  if (red > (size_t)c2 * a.nwp) return cudaSuccess;
  *handled = true;
  if (a.spec == 2) {
    if (c2 == 32) return a.gvec ? spec_launch(k_rad_send_spec<Spec_full_l2, 32, true>, sm, s, a, T)
                                : spec_launch(k_rad_send_spec<Spec_full_l2, 32, false>, sm, s, a, T);
    return a.gvec ? spec_launch(k_rad_send_spec<Spec_full_l2, 16, true>, sm, s, a, T)
                  : spec_launch(k_rad_send_spec<Spec_full_l2, 16, false>, sm, s, a, T);
  }
  if (c2 == 8) return a.gvec ? spec_launch(k_rad_send_spec<Spec_full_l3, 8, true>, sm, s, a, T)
                             : spec_launch(k_rad_send_spec<Spec_full_l3, 8, false>, sm, s, a, T);
  return a.gvec ? spec_launch(k_rad_send_spec<Spec_full_l3, 4, true>, sm, s, a, T)
                : spec_launch(k_rad_send_spec<Spec_full_l3, 4, false>, sm, s, a, T);
}

}  // namespace tp
