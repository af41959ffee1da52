// The uvu convolution with the radial projection fused in ("Sobek: Streaming Equivariant Tensor
// Product Convolutions", abstract: the radial projection reordered so that edge-specific
// weights are never materialised).
//
// The caller passes the radial network's last hidden layer h[E, H] and its bias-free output
// layer W_r[H, nw] instead of the weights w[E, nw].  Every pass forms the weights of a chunk of
// edges in shared memory, w[e, c] = sum_k h[e, k] W_r[k, c] (k ascending, fp32, packed
// FFMA2 over pairs of edges), and uses them there: no edge-sized float tensor exists in HBM,
// in the workspace or between kernels.  The coupling is the path table's (per-triple unrolled
// Clebsch-Gordan chains, lane = channel):
//   k_rad_fwd      one CTA per receiver, its edges in chunks: project the chunk, then one warp
//                  per (output block, 32-channel slice) sums its paths into a shared-memory row;
//                  the row is written once.
//   k_rad_send     one CTA per sender, its edges in the stable sender order of the transpose:
//                  project the chunk; one warp per (input block, slice) accumulates gx and
//                  writes the chunk's weight gradient gw into shared memory; gh = gw W_r^T from
//                  there; gvec by one warp per edge.
//   k_rad_gwr      gW_r = sum_e h[e]^T gw[e]: one warp per (path, slice) recomputes its gw from
//                  x, gy and Y (gw needs no w), edges in receiver order split over the grid's y
//                  dimension; k_rad_gwr_reduce sums the partials in split order.
// Every output element is written by one thread in a fixed order: deterministic, no float
// atomics.  The projection costs 2 H flops per weight on the CUDA cores; the edge stream is H
// floats per edge instead of nw.
#include "radial.cuh"

namespace tp {
namespace {

using namespace rad;

// ---------------------------------------------------------------------------------------
// Forward: y[i] = sum_{e into i} sum_p c_p w[e, p, u] C_p(x[src e], Y(e)), w projected per chunk.
// ---------------------------------------------------------------------------------------
template <int CE>
__global__ void __launch_bounds__(kRadThreads) k_rad_fwd(const __grid_constant__ RadArgs a,
                                                         const __grid_constant__ GenTable T) {
  extern __shared__ float4 rad_smem_raw[];
  const RadSmem s = rad_smem<CE>(reinterpret_cast<float*>(rad_smem_raw), a, false);
  const int row = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int e0 = __ldg(a.rowptr + row), e1 = __ldg(a.rowptr + row + 1);
  if (a.check) {
    e0 = max(0, min(e0, a.E));
    e1 = max(e0, min(e1, a.E));
  }
  for (int t = threadIdx.x; t < a.out_dim; t += blockDim.x) s.rs[t] = 0.f;
  for (int c0 = e0; c0 < e1; c0 += CE) {
    const int ne = min(CE, e1 - c0);
    __syncthreads();                       // readers of the previous chunk are done
    if (threadIdx.x < CE) {
      const int r = threadIdx.x;
      int e = -1, j = -1;
      float Y[16], rx, ry, rz, ir;
#pragma unroll
      for (int m = 0; m < 16; ++m) Y[m] = 0.f;
      if (r < ne) {
        e = c0 + r;
        j = __ldg(a.src + e);
        if (a.check && (unsigned)j >= (unsigned)a.N) {
          rad_report(a, kDevBadSrc);
          e = j = -1;
        } else {
          sh16(a.vec, e, Y, rx, ry, rz, ir);
        }
      }
      s.es[r] = e;
      s.ns[r] = j;
#pragma unroll
      for (int m = 0; m < 16; ++m) s.Ys[r * 16 + m] = Y[m];
    }
    __syncthreads();
    stage_chunk<CE>(a, s, ne, a.x, a.in_dim);
    __syncthreads();
    project<CE>(a, s);
    __syncthreads();
    const int xp = round4(a.in_dim);
    for (int task = warp; task < T.n_rtask; task += kRadWarps) {
      const int o = T.rtask_block[task];
      const int c = T.rtask_slice[task] * 32 + lane;
      if (c >= T.out_mul[o]) continue;     // no warp-level operation below
      const int d3 = 2 * T.out_l[o] + 1;
      float* yr = s.rs + T.out_off[o] + c * d3;
      float acc[7];
#pragma unroll
      for (int m = 0; m < 7; ++m) acc[m] = m < d3 ? yr[m] : 0.f;
      for (int pi = T.out_first[o]; pi < T.out_first[o + 1]; ++pi) {
        const GenPath P = T.path[T.out_paths[pi]];
        gen::with_triple(P.tid, [&](auto cg) {
          using Cg = decltype(cg);
          constexpr int sb = Cg::L2 * Cg::L2;
          for (int r = 0; r < ne; ++r) {
            if (s.es[r] < 0) continue;
            float Y[Cg::D2], xv[Cg::D1], t[Cg::D3];
#pragma unroll
            for (int m = 0; m < Cg::D2; ++m) Y[m] = s.Ys[r * 16 + sb + m];
            const float* xr = s.vs + r * xp + P.in_off + c * Cg::D1;
#pragma unroll
            for (int m = 0; m < Cg::D1; ++m) xv[m] = xr[m];
            const float w = P.coeff * s.ws[r * a.nwp + P.w_off + c];
            Cg::fwd(xv, Y, t);
#pragma unroll
            for (int m = 0; m < Cg::D3; ++m) acc[m] = fmaf(w, t[m], acc[m]);
          }
        });
      }
#pragma unroll
      for (int m = 0; m < 7; ++m)
        if (m < d3) yr[m] = acc[m];
    }
  }
  __syncthreads();
  float* yrow = a.y + (int64_t)row * a.out_dim;
  for (int t = threadIdx.x; t < a.out_dim; t += blockDim.x) yrow[t] = s.rs[t];
}

// gvec of one edge from G1[m] = sum_{p, u} c_p w Q_p(x, gy)[m] over the 16 SH components:
// (grad Y . G1 - r_hat (sum_m l_m G1_m Y_m)) / |v|, summed across the warp.
__device__ __forceinline__ void rad_gvec_store(float* g, float rx, float ry, float rz, float ir,
                                               const float (&G1)[16], int lane) {
  float Y[16], G[16][3];
  gen::ShAll::sh(rx, ry, rz, Y);
  gen::ShAll::sh_grad(rx, ry, rz, G);
  float g0 = 0.f, g1 = 0.f, g2 = 0.f, sdeg = 0.f;
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    g0 = fmaf(G1[m], G[m][0], g0);
    g1 = fmaf(G1[m], G[m][1], g1);
    g2 = fmaf(G1[m], G[m][2], g2);
    sdeg = fmaf(gen::ShAll::sh_degree(m) * G1[m], Y[m], sdeg);
  }
  g0 = warp_sum(ir * (g0 - rx * sdeg));
  g1 = warp_sum(ir * (g1 - ry * sdeg));
  g2 = warp_sum(ir * (g2 - rz * sdeg));
  if (lane == 0) {
    g[0] = g0;
    g[1] = g1;
    g[2] = g2;
  }
}

// ---------------------------------------------------------------------------------------
// Sender pass: gx[j] = sum_{e out of j} sum_p c_p w[e, p, u] C_p^T(Y, gy[dst e]),
// gw[e, p, u] = c_p <x[j], C_p^T(Y, gy[dst e])> (shared memory only), gh[e] = gw[e] W_r^T,
// gvec[e] through the SH derivatives.
// ---------------------------------------------------------------------------------------
template <int CE>
__global__ void __launch_bounds__(kRadThreads) k_rad_send(const __grid_constant__ RadArgs a,
                                                          const __grid_constant__ GenTable T) {
  extern __shared__ float4 rad_smem_raw[];
  const RadSmem s = rad_smem<CE>(reinterpret_cast<float*>(rad_smem_raw), a, true);
  const int node = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int q0 = __ldg(a.colptr + node), q1 = __ldg(a.colptr + node + 1);
  if (a.check) {
    q0 = max(0, min(q0, a.E));
    q1 = max(q0, min(q1, a.E));
  }
  for (int t = threadIdx.x; t < a.in_dim; t += blockDim.x) {
    s.rs[t] = 0.f;
    s.xn[t] = __ldg(a.x + (int64_t)node * a.in_dim + t);
  }
  const int gp = round4(a.out_dim);
  for (int c0 = q0; c0 < q1; c0 += CE) {
    const int ne = min(CE, q1 - c0);
    __syncthreads();
    if (threadIdx.x < CE) {
      const int r = threadIdx.x;
      int e = -1, i = 0;
      float Y[16], rx, ry, rz, ir;
#pragma unroll
      for (int m = 0; m < 16; ++m) Y[m] = 0.f;
      if (r < ne) {
        e = __ldg(a.perm + c0 + r);
        if (a.check && (unsigned)e >= (unsigned)a.E) {
          rad_report(a, kDevBadPerm);
          e = -1;
        } else {
          i = find_row(a.rowptr, a.N, e);
          sh16(a.vec, e, Y, rx, ry, rz, ir);
        }
      }
      s.es[r] = e;
      s.ns[r] = i;
#pragma unroll
      for (int m = 0; m < 16; ++m) s.Ys[r * 16 + m] = Y[m];
    }
    __syncthreads();
    stage_chunk<CE>(a, s, ne, a.gy, a.out_dim);
    __syncthreads();
    project<CE>(a, s);
    __syncthreads();
    // gx (accumulated over chunks in rs) and the chunk's gw
    for (int task = warp; task < T.n_stask; task += kRadWarps) {
      const int ib = T.stask_block[task];
      const int c = T.stask_slice[task] * 32 + lane;
      if (c >= T.in_mul[ib]) continue;
      const int d1 = 2 * T.in_l[ib] + 1;
      float* gr = s.rs + T.in_off[ib] + c * d1;
      float gacc[7];
#pragma unroll
      for (int m = 0; m < 7; ++m) gacc[m] = m < d1 ? gr[m] : 0.f;
      for (int pi = T.in_first[ib]; pi < T.in_first[ib + 1]; ++pi) {
        const GenPath P = T.path[T.in_paths[pi]];
        gen::with_triple(P.tid, [&](auto cg) {
          using Cg = decltype(cg);
          constexpr int sb = Cg::L2 * Cg::L2;
          float xv[Cg::D1];
#pragma unroll
          for (int m = 0; m < Cg::D1; ++m) xv[m] = s.xn[P.in_off + c * Cg::D1 + m];
          for (int r = 0; r < ne; ++r) {
            if (s.es[r] < 0) continue;
            float Y[Cg::D2], gyv[Cg::D3], z[Cg::D1];
#pragma unroll
            for (int m = 0; m < Cg::D2; ++m) Y[m] = s.Ys[r * 16 + sb + m];
            const float* gr2 = s.vs + r * gp + P.out_off + c * Cg::D3;
#pragma unroll
            for (int m = 0; m < Cg::D3; ++m) gyv[m] = gr2[m];
            Cg::tx(Y, gyv, z);
            const int widx = r * a.nwp + P.w_off + c;
            const float w = P.coeff * s.ws[widx];
            float d = 0.f;
#pragma unroll
            for (int m = 0; m < Cg::D1; ++m) {
              gacc[m] = fmaf(w, z[m], gacc[m]);
              d = fmaf(xv[m], z[m], d);
            }
            s.gs[widx] = P.coeff * d;
          }
        });
      }
#pragma unroll
      for (int m = 0; m < 7; ++m)
        if (m < d1) gr[m] = gacc[m];
    }
    __syncthreads();
    if (a.gh) gh_chunk<CE>(a, s, ne);
    // gvec: a warp per edge, lanes over channels, all paths with l2 > 0
    if (a.gvec) {
      for (int r = warp; r < ne; r += kRadWarps) {
        const int e = s.es[r];
        if (e < 0) continue;               // warp-uniform
        float rx, ry, rz, ir;
        edge_geometry(__ldg(a.vec + 3 * (int64_t)e), __ldg(a.vec + 3 * (int64_t)e + 1),
                      __ldg(a.vec + 3 * (int64_t)e + 2), rx, ry, rz, ir);
        float G1[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) G1[m] = 0.f;
        for (int p = 0; p < T.n_paths; ++p) {
          const GenPath P = T.path[p];
          if (P.l2 == 0) continue;           // Y_0 is constant
          gen::with_triple(P.tid, [&](auto cg) {
            using Cg = decltype(cg);
            constexpr int sb = Cg::L2 * Cg::L2;
            for (int c = lane; c < P.mul; c += 32) {
              float xv[Cg::D1], gyv[Cg::D3], q[Cg::D2];
#pragma unroll
              for (int m = 0; m < Cg::D1; ++m) xv[m] = s.xn[P.in_off + c * Cg::D1 + m];
#pragma unroll
              for (int m = 0; m < Cg::D3; ++m) gyv[m] = s.vs[r * gp + P.out_off + c * Cg::D3 + m];
              const float w = P.coeff * s.ws[r * a.nwp + P.w_off + c];
              Cg::ty(xv, gyv, q);
#pragma unroll
              for (int m = 0; m < Cg::D2; ++m) G1[sb + m] = fmaf(w, q[m], G1[sb + m]);
            }
          });
        }
        rad_gvec_store(a.gvec + 3 * (int64_t)e, rx, ry, rz, ir, G1, lane);
      }
    }
  }
  __syncthreads();
  if (a.gx) {
    float* grow = a.gx + (int64_t)node * a.in_dim;
    for (int t = threadIdx.x; t < a.in_dim; t += blockDim.x) grow[t] = s.rs[t];
  }
}

// ---------------------------------------------------------------------------------------
// gW_r partials: part[s][k][w_off(p) + u] = sum over split s's edges of h[e, k] gw[e, p, u],
// gw recomputed as c_p <x[src e], C_p^T(Y, gy[dst e])>.  A CTA per ((path, 32-channel slice)
// unit, edge split): its warps take interleaved batches of two edges of each staged chunk (all
// warps of a CTA run the same triple's code), load the x and gy slices of a batch before using
// them, and are summed in warp order at the end; 128 registers, four CTAs per SM.
// ---------------------------------------------------------------------------------------
constexpr int kGwrChunk = 64;
constexpr int kGwrBatch = 2;

template <int HC>
__global__ void __launch_bounds__(kGwrThreads, 4) k_rad_gwr(const __grid_constant__ RadArgs a,
                                                         const __grid_constant__ GenTable T) {
  const int H = HC ? HC : a.H;          // hidden width (a compile-time 64 in the common case)
  __shared__ __align__(16) float hs[kGwrChunk * kRadMaxHidden];
  __shared__ float Ys[kGwrChunk * 16];
  __shared__ int js[kGwrChunk], is[kGwrChunk];
  __shared__ float2 red[(kGwrWarps - 1) * (kRadMaxHidden / 2) * 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // this CTA's (path, slice) unit
  int unit = blockIdx.x, p = -1, sl = 0;
  for (int q = 0; q < T.n_paths; ++q) {
    const int ns = (T.path[q].mul + 31) >> 5;
    if (unit < ns) {
      p = q;
      sl = unit;
      break;
    }
    unit -= ns;
  }
  const int64_t lo = (int64_t)a.E * blockIdx.y / a.splits, hi = (int64_t)a.E * (blockIdx.y + 1) / a.splits;
  float2 acc[kRadMaxHidden / 2];            // hidden units (2k, 2k + 1)
#pragma unroll
  for (int k = 0; k < kRadMaxHidden / 2; ++k) acc[k] = make_float2(0.f, 0.f);
  const GenPath P = T.path[p < 0 ? 0 : p];
  const int c = sl * 32 + lane;
  const bool act = p >= 0 && c < P.mul;
  for (int64_t c0 = lo; c0 < hi; c0 += kGwrChunk) {
    const int ne = (int)(hi - c0 < kGwrChunk ? hi - c0 : kGwrChunk);
    __syncthreads();
    for (int t = threadIdx.x; t < ne * H; t += blockDim.x) hs[t] = __ldg(a.h + c0 * H + t);
    if (threadIdx.x < ne) {
      const int r = threadIdx.x, e = (int)c0 + r;
      int j = __ldg(a.src + e);
      if (a.check && (unsigned)j >= (unsigned)a.N) {
        rad_report(a, kDevBadSrc);
        j = -1;
      }
      float Y[16], rx, ry, rz, ir;
      sh16(a.vec, e, Y, rx, ry, rz, ir);
      js[r] = j;
      is[r] = find_row(a.rowptr, a.N, e);
#pragma unroll
      for (int m = 0; m < 16; ++m) Ys[r * 16 + m] = Y[m];
    }
    __syncthreads();
    if (!act) continue;
    for (int r0 = warp * kGwrBatch; r0 < ne; r0 += kGwrWarps * kGwrBatch) {
      // gw of four edges (the per-triple part of the code stays small), then h[e]^T gw[e]
      float g[kGwrBatch];
      gen::with_triple(P.tid, [&](auto cg) {
        using Cg = decltype(cg);
        constexpr int sb = Cg::L2 * Cg::L2;
        float xv[kGwrBatch][Cg::D1], gyv[kGwrBatch][Cg::D3];
#pragma unroll
        for (int b = 0; b < kGwrBatch; ++b) {
          const int r = r0 + b;
          const bool ok = r < ne && js[r] >= 0;
          const float* xr = a.x + (int64_t)(ok ? js[r] : 0) * a.in_dim + P.in_off + (int64_t)c * Cg::D1;
          const float* gr = a.gy + (int64_t)(ok ? is[r] : 0) * a.out_dim + P.out_off + (int64_t)c * Cg::D3;
#pragma unroll
          for (int m = 0; m < Cg::D1; ++m) xv[b][m] = ok ? __ldg(xr + m) : 0.f;
#pragma unroll
          for (int m = 0; m < Cg::D3; ++m) gyv[b][m] = ok ? __ldg(gr + m) : 0.f;
        }
#pragma unroll
        for (int b = 0; b < kGwrBatch; ++b) {
          const int r = min(r0 + b, ne - 1);
          float Y[Cg::D2], z[Cg::D1];
#pragma unroll
          for (int m = 0; m < Cg::D2; ++m) Y[m] = Ys[r * 16 + sb + m];
          Cg::tx(Y, gyv[b], z);
          float d = 0.f;
#pragma unroll
          for (int m = 0; m < Cg::D1; ++m) d = fmaf(xv[b][m], z[m], d);
          g[b] = P.coeff * d;                // zero for the batch's padding and skipped edges
        }
      });
      const int nb = min(kGwrBatch, ne - r0);
#pragma unroll
      for (int b = 0; b < kGwrBatch; ++b) {
        if (b >= nb) break;
        // k pairs: one FFMA2 per two hidden units
        const float4* hr = reinterpret_cast<const float4*>(hs + (r0 + b) * H);
        const float2 gb = make_float2(g[b], g[b]);
#pragma unroll
        for (int k4 = 0; k4 < kRadMaxHidden / 4; ++k4) {
          if (4 * k4 < H) {
            const float4 hv = hr[k4];
            acc[2 * k4] = __ffma2_rn(make_float2(hv.x, hv.y), gb, acc[2 * k4]);
            acc[2 * k4 + 1] = __ffma2_rn(make_float2(hv.z, hv.w), gb, acc[2 * k4 + 1]);
          }
        }
      }
    }
  }
  // warps 1.. hand their sums to warp 0, which adds them in warp order
  if (act && warp > 0) {
#pragma unroll
    for (int k = 0; k < kRadMaxHidden / 2; ++k)
      if (2 * k < H) red[((warp - 1) * (kRadMaxHidden / 2) + k) * 32 + lane] = acc[k];
  }
  __syncthreads();
  if (!act || warp > 0) return;
  for (int w = 1; w < kGwrWarps; ++w) {
#pragma unroll
    for (int k = 0; k < kRadMaxHidden / 2; ++k)
      if (2 * k < H) {
        const float2 v = red[((w - 1) * (kRadMaxHidden / 2) + k) * 32 + lane];
        acc[k].x += v.x;
        acc[k].y += v.y;
      }
  }
  float* out = a.part + (int64_t)blockIdx.y * H * a.nw + P.w_off + c;
#pragma unroll
  for (int k = 0; k < kRadMaxHidden / 2; ++k)
    if (2 * k < H) {
      out[(int64_t)(2 * k) * a.nw] = acc[k].x;
      out[(int64_t)(2 * k + 1) * a.nw] = acc[k].y;
    }
}

__global__ void __launch_bounds__(256) k_rad_gwr_reduce(const __grid_constant__ RadArgs a) {
  const int64_t n = (int64_t)a.H * a.nw;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n; t += (int64_t)gridDim.x * blockDim.x) {
    float v = 0.f;
    for (int sp = 0; sp < a.splits; ++sp) v += a.part[sp * n + t];
    a.gWr[t] = v;
  }
}

// WrT[c, k] = W_r[k, c] (the layout the gh loop reads with consecutive k across a warp)
__global__ void __launch_bounds__(256) k_rad_transpose(const __grid_constant__ RadArgs a) {
  const int64_t n = (int64_t)a.H * a.nw;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = t / a.H, k = t - c * a.H;
    a.WrT[t] = __ldg(a.Wr + k * a.nw + c);
  }
}

unsigned rad_flat_grid(int64_t n) {
  int64_t g = (n + 255) / 256;
  if (g > 148 * 8) g = 148 * 8;
  return (unsigned)(g < 1 ? 1 : g);
}

int rad_units(const GenTable& T) {
  int n = 0;
  for (int p = 0; p < T.n_paths; ++p) n += (T.path[p].mul + 31) / 32;
  return n;
}

template <class K>
cudaError_t rad_launch(K kern, unsigned grid, size_t smem, cudaStream_t s, const RadArgs& a, const GenTable& T) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kRadThreads, smem, s>>>(a, T);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

int rad_chunk(const RadArgs& a, bool bwd, size_t* smem_bytes) {
  const int vdim = bwd ? a.out_dim : a.in_dim;
  for (int ce = 32; ce >= 4; ce >>= 1) {
    const size_t b = sizeof(float) * rad_smem_floats(a.H, ce, a.nwp, a.in_dim, a.out_dim, bwd);
    const size_t tile = sizeof(float) * rad_tile_floats(ce, a.nwp, vdim, bwd);
    if (b <= (size_t)kRadSmemBudget && (tile <= (size_t)kRadTileBudget || ce == 4)) {
      if (smem_bytes) *smem_bytes = b;
      return ce;
    }
  }
  if (smem_bytes) *smem_bytes = 0;
  return 0;
}

int rad_splits(const GenTable& T, int64_t E) {
  // one wave: the gW_r pass keeps four CTAs per SM resident (128 registers), so
  // units x splits <= 4 x 148 avoids a partly filled second wave
  const int ctas = rad_units(T);
  int64_t sp = (4 * 148) / ctas;
  sp = std::min<int64_t>(sp, std::max<int64_t>(1, (E + kGwrChunk - 1) / kGwrChunk));
  return (int)std::max<int64_t>(1, std::min<int64_t>(sp, 256));
}

cudaError_t launch_rad_fwd(const RadArgs& a, const GenTable& T, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  size_t smem = 0;
  const int ce = rad_chunk(a, false, &smem);
  bool handled = false;
  cudaError_t e = launch_rad_fwd_spec(a, T, ce, smem, s, &handled);
  if (handled) return e;
  switch (ce) {
    case 32: return rad_launch(k_rad_fwd<32>, (unsigned)a.N, smem, s, a, T);
    case 16: return rad_launch(k_rad_fwd<16>, (unsigned)a.N, smem, s, a, T);
    case 8: return rad_launch(k_rad_fwd<8>, (unsigned)a.N, smem, s, a, T);
    case 4: return rad_launch(k_rad_fwd<4>, (unsigned)a.N, smem, s, a, T);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_rad_bwd(const RadArgs& a, const GenTable& T, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  if (a.gh) {
    k_rad_transpose<<<rad_flat_grid((int64_t)a.H * a.nw), 256, 0, s>>>(a);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.gx || a.gh || a.gvec) {
    size_t smem = 0;
    const int ce = rad_chunk(a, true, &smem);
    bool handled = false;
    e = launch_rad_send_spec(a, T, ce, smem, s, &handled);
    if (handled && e != cudaSuccess) return e;
    if (!handled) switch (ce) {
      case 32: e = rad_launch(k_rad_send<32>, (unsigned)a.N, smem, s, a, T); break;
      case 16: e = rad_launch(k_rad_send<16>, (unsigned)a.N, smem, s, a, T); break;
      case 8: e = rad_launch(k_rad_send<8>, (unsigned)a.N, smem, s, a, T); break;
      case 4: e = rad_launch(k_rad_send<4>, (unsigned)a.N, smem, s, a, T); break;
      default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
  }
  if (a.gWr) {
    if (a.E == 0) return cudaMemsetAsync(a.gWr, 0, sizeof(float) * (size_t)a.H * a.nw, s);
    const dim3 grid((unsigned)rad_units(T), (unsigned)a.splits);
    if (a.H == kRadMaxHidden) k_rad_gwr<kRadMaxHidden><<<grid, kGwrThreads, 0, s>>>(a, T);
    else k_rad_gwr<0><<<grid, kGwrThreads, 0, s>>>(a, T);
    k_rad_gwr_reduce<<<rad_flat_grid((int64_t)a.H * a.nw), 256, 0, s>>>(a);
    count_launches(2);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace tp
