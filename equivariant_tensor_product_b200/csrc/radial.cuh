// Shared pieces of the fused-radial-projection passes (radial.cu: path-table kernels;
// radial_spec.cu: kernels of the compiled whole path lists): shared-memory layout, staging of
// a chunk's hidden rows and per-edge rows, and the projection w = h W_r of a chunk.
#pragma once
#include "generic_cg.h"
#include "tp_common.h"
#include "tp_kernels.cuh"

namespace tp {
namespace rad {

constexpr int kRadThreads = 256;              // the edge passes
constexpr int kRadWarps = kRadThreads / 32;
constexpr int kGwrThreads = 128;              // the gW_r pass: a warp per (path, slice) unit
constexpr int kGwrWarps = kGwrThreads / 32;
constexpr int kRadSmemBudget = 200 * 1024;    // dynamic shared memory of one pass at most
constexpr int kRadTileBudget = 104 * 1024;    // the per-edge tiles of a chunk: two CTAs per SM

__device__ __forceinline__ void rad_report(const RadArgs& a, int code) {
  if (a.err) atomicCAS(a.err, 0, code);
}

template <int D>
__device__ __forceinline__ void rad_load(const float* __restrict__ p, float (&v)[D]) {
#pragma unroll
  for (int m = 0; m < D; ++m) v[m] = __ldg(p + m);
}

__host__ __device__ constexpr int round4(int v) { return (v + 3) & ~3; }

// Shared-memory layout of both passes (floats; every region a multiple of 16 bytes):
//   hs [H][CE + 4]  hidden rows of the chunk, k-major (rows past the chunk are zero)
//   ws [CE][nwp]    the chunk's weights
//   gs [CE][nwp]    sender pass: the chunk's weight gradient
//   vs [CE][vdim]   the rows the coupling reads per edge: forward x[src], sender pass gy[dst]
//   xn [in_dim]     sender pass: x of the CTA's sender
//   rs [row]        the CTA's output row (forward: y; sender pass: gx)
//   Ys [CE][16]     real spherical harmonics of degrees 0..3 per edge
//   es, ns [CE]     edge ids (-1: skipped) and the other endpoint of each edge
struct RadSmem {
  float *hs, *ws, *gs, *vs, *xn, *rs, *Ys;
  int *es, *ns;
};

__host__ __device__ inline size_t rad_tile_floats(int CE, int nwp, int vdim, bool bwd) {
  return (size_t)CE * (nwp * (bwd ? 2 : 1) + round4(vdim));
}

__host__ __device__ inline size_t rad_smem_floats(int H, int CE, int nwp, int in_dim, int out_dim, bool bwd) {
  const int vdim = bwd ? out_dim : in_dim, row = bwd ? in_dim : out_dim;
  return (size_t)H * (CE + 4) + rad_tile_floats(CE, nwp, vdim, bwd) + (bwd ? round4(in_dim) : 0) + round4(row) +
         (size_t)CE * 16 + 2 * round4(CE);
}

template <int CE>
__device__ __forceinline__ RadSmem rad_smem(float* base, const RadArgs& a, bool bwd) {
  RadSmem s;
  const int vdim = bwd ? a.out_dim : a.in_dim, row = bwd ? a.in_dim : a.out_dim;
  s.hs = base;
  s.ws = s.hs + a.H * (CE + 4);
  s.gs = s.ws + CE * a.nwp;
  s.vs = s.gs + (bwd ? CE * a.nwp : 0);
  s.xn = s.vs + CE * round4(vdim);
  s.rs = s.xn + (bwd ? round4(a.in_dim) : 0);
  s.Ys = s.rs + round4(row);
  s.es = reinterpret_cast<int*>(s.Ys + CE * 16);
  s.ns = s.es + round4(CE);
  return s;
}

// Hidden rows of the chunk's edges into hs (k-major, transposed on the way in) and the rows
// the coupling reads per edge into vs (row ns[r] of `src_rows`, width vdim): every load of
// the chunk is independent, so they are all in flight together.
template <int CE>
__device__ __forceinline__ void stage_chunk(const RadArgs& a, const RadSmem& s, int ne, const float* src_rows,
                                            int vdim) {
  const int n = a.H * CE;
  for (int t = threadIdx.x; t < n; t += blockDim.x) {
    const int r = t / a.H, k = t - r * a.H;
    const int e = r < ne ? s.es[r] : -1;
    s.hs[k * (CE + 4) + r] = e >= 0 ? __ldg(a.h + (int64_t)e * a.H + k) : 0.f;
  }
  const int vp = round4(vdim), nv = ne * vdim;
  for (int t = threadIdx.x; t < nv; t += blockDim.x) {
    const int r = t / vdim, m = t - r * vdim;
    s.vs[r * vp + m] = s.es[r] >= 0 ? __ldg(src_rows + (int64_t)s.ns[r] * vdim + m) : 0.f;
  }
}

// ws[r][c] = sum_k hs[k][r] W_r[k, c]: a thread per pair of weight columns (c, c + blockDim.x),
// the chunk's edges in registers as pairs (one FFMA2 per edge pair, column and k), so that
// each broadcast read of hs feeds four FFMA2; W_r read in batches of 8 k of both columns;
// each W_r element is read once per chunk.
template <int CE, int HC>
__device__ __forceinline__ void project_h(const RadArgs& a, const RadSmem& s) {
  const int H = HC ? HC : a.H;
  constexpr int KB = 8;
  const int stride = 2 * blockDim.x;
  for (int c = threadIdx.x; c < a.nw; c += stride) {
    const int c2 = c + blockDim.x;
    const bool two = c2 < a.nw;
    float2 acc[CE / 2], acd[CE / 2];
#pragma unroll
    for (int q = 0; q < CE / 2; ++q) acc[q] = acd[q] = make_float2(0.f, 0.f);
    // a constant width that is a multiple of the batch needs no per-k guard
    constexpr bool kExact = HC > 0 && HC % KB == 0;
#pragma unroll 1
    for (int k0 = 0; k0 < H; k0 += KB) {
      float v[KB], u2[KB];
#pragma unroll
      for (int u = 0; u < KB; ++u) {
        const bool ok = kExact || k0 + u < H;
        const float* wk = a.Wr + (int64_t)(ok ? k0 + u : 0) * a.nw;
        v[u] = ok ? __ldg(wk + c) : 0.f;
        u2[u] = ok && two ? __ldg(wk + c2) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < KB; ++u) {
        if (kExact || k0 + u < H) {
          const float2 va = make_float2(v[u], v[u]), vb = make_float2(u2[u], u2[u]);
          const float4* hk = reinterpret_cast<const float4*>(s.hs + (k0 + u) * (CE + 4));
#pragma unroll
          for (int q = 0; q < CE / 4; ++q) {
            const float4 hv = hk[q];
            const float2 lo = make_float2(hv.x, hv.y), hi = make_float2(hv.z, hv.w);
            acc[2 * q] = __ffma2_rn(lo, va, acc[2 * q]);
            acc[2 * q + 1] = __ffma2_rn(hi, va, acc[2 * q + 1]);
            acd[2 * q] = __ffma2_rn(lo, vb, acd[2 * q]);
            acd[2 * q + 1] = __ffma2_rn(hi, vb, acd[2 * q + 1]);
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < CE / 2; ++q) {
      s.ws[(2 * q) * a.nwp + c] = acc[q].x;
      s.ws[(2 * q + 1) * a.nwp + c] = acc[q].y;
      if (two) {
        s.ws[(2 * q) * a.nwp + c2] = acd[q].x;
        s.ws[(2 * q + 1) * a.nwp + c2] = acd[q].y;
      }
    }
  }
}

// The projection with the hidden width a compile-time constant when it is 64 and the chunk has
// at most 16 edges (no per-k guards; measured faster there: c3 forward 3.96 -> 3.11 ms, c5 3.95 ->
// 3.63 ms); the 32-edge chunks keep the runtime width, whose smaller live range spills less.
template <int CE>
__device__ __forceinline__ void project(const RadArgs& a, const RadSmem& s) {
  if (CE <= 16 && a.H == kRadMaxHidden) project_h<CE, kRadMaxHidden>(a, s);
  else project_h<CE, 0>(a, s);
}

// gh[e, k] = sum_c gw[e, c] W_r[k, c] for the chunk's edges, gw in gs: thread (k, quarter)
// over every fourth edge of the chunk, W_r read transposed (WrT) so that a warp's loads of one
// column are contiguous.  Call after the chunk's gs is complete (a barrier after its writes).
template <int CE>
__device__ __forceinline__ void gh_chunk_pairs(const RadArgs& a, const RadSmem& s, int ne);

template <int CE>
__device__ __forceinline__ void gh_chunk(const RadArgs& a, const RadSmem& s, int ne) {
  if constexpr (CE == 4 * kRadWarps) {
    // the pair form uses 8-byte accesses to W_r^T and gh (the ABI promises 4-byte alignment)
    if (((reinterpret_cast<uintptr_t>(a.WrT) | reinterpret_cast<uintptr_t>(a.gh)) & 7u) == 0) {
      gh_chunk_pairs<CE>(a, s, ne);
      return;
    }
  }
  constexpr int NQ = kRadThreads / 64, RQ = CE / NQ > 0 ? CE / NQ : 1;
  const int k = threadIdx.x & 63, quarter = threadIdx.x >> 6;
  if (k < a.H && quarter < CE) {
    float acc[RQ];
#pragma unroll
    for (int q = 0; q < RQ; ++q) acc[q] = 0.f;
    const int nw4 = a.nw & ~3;
    for (int c = 0; c < nw4; c += 4) {
      const float w0 = __ldg(a.WrT + (int64_t)c * a.H + k), w1 = __ldg(a.WrT + (int64_t)(c + 1) * a.H + k);
      const float w2 = __ldg(a.WrT + (int64_t)(c + 2) * a.H + k), w3 = __ldg(a.WrT + (int64_t)(c + 3) * a.H + k);
#pragma unroll
      for (int q = 0; q < RQ; ++q) {
        const float4 g = *reinterpret_cast<const float4*>(s.gs + (quarter + NQ * q) * a.nwp + c);
        acc[q] = fmaf(g.x, w0, fmaf(g.y, w1, fmaf(g.z, w2, fmaf(g.w, w3, acc[q]))));
      }
    }
    for (int c = nw4; c < a.nw; ++c) {
      const float wv = __ldg(a.WrT + (int64_t)c * a.H + k);
#pragma unroll
      for (int q = 0; q < RQ; ++q) acc[q] = fmaf(s.gs[(quarter + NQ * q) * a.nwp + c], wv, acc[q]);
    }
#pragma unroll
    for (int q = 0; q < RQ; ++q) {
      const int r = quarter + NQ * q;
      if (r < ne && s.es[r] >= 0) a.gh[(int64_t)s.es[r] * a.H + k] = acc[q];
    }
  }
}

// gh for chunks of 4 edges per warp: lane = pair of hidden units (k, k + 1), warp = four edges
// of the chunk.  A lane's W_r^T loads of one column are one 8-byte load (contiguous across the
// warp), each gw value is a broadcast shared-memory read, and one FFMA2 updates both hidden
// units of an edge.
template <int CE>
__device__ __forceinline__ void gh_chunk_pairs(const RadArgs& a, const RadSmem& s, int ne) {
  const int kp = threadIdx.x & 31, r0 = 4 * (threadIdx.x >> 5);
  if (2 * kp >= a.H) return;
  float2 acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
  const int nw4 = a.nw & ~3;
  const float2* wt = reinterpret_cast<const float2*>(a.WrT) + kp;   // WrT[c][2 kp .. 2 kp + 1]
  const int hp = a.H >> 1;
  for (int c = 0; c < nw4; c += 4) {
    float2 w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) w[u] = __ldg(wt + (int64_t)(c + u) * hp);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 g = *reinterpret_cast<const float4*>(s.gs + (r0 + q) * a.nwp + c);
      acc[q] = __ffma2_rn(make_float2(g.x, g.x), w[0], acc[q]);
      acc[q] = __ffma2_rn(make_float2(g.y, g.y), w[1], acc[q]);
      acc[q] = __ffma2_rn(make_float2(g.z, g.z), w[2], acc[q]);
      acc[q] = __ffma2_rn(make_float2(g.w, g.w), w[3], acc[q]);
    }
  }
  for (int c = nw4; c < a.nw; ++c) {
    const float2 wv = __ldg(wt + (int64_t)c * hp);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float g = s.gs[(r0 + q) * a.nwp + c];
      acc[q] = __ffma2_rn(make_float2(g, g), wv, acc[q]);
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int r = r0 + q;
    if (r < ne && s.es[r] >= 0) *reinterpret_cast<float2*>(a.gh + (int64_t)s.es[r] * a.H + 2 * kp) = acc[q];
  }
}

// gh for chunks of fewer than 32 edges, pair form: warp = (group of four edges, part of the
// columns), lane = pair of hidden units; the column parts' sums go through `red` (32 H floats)
// and are added in part order.  Every thread of the CTA must call it (it has barriers).
template <int CE>
__device__ __forceinline__ void gh_chunk_split(const RadArgs& a, const RadSmem& s, int ne, float* red) {
  constexpr int G = CE / 4, NP = kRadWarps / G;
  const int kp = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = warp % G, part = warp / G, r0 = 4 * g;
  const int hp = a.H >> 1, nw4 = a.nw & ~3;
  const int c_lo = ((nw4 >> 2) * part / NP) << 2, c_hi = ((nw4 >> 2) * (part + 1) / NP) << 2;
  if (kp < hp) {
    float2 acc[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
    const float2* wt = reinterpret_cast<const float2*>(a.WrT) + kp;
    for (int c = c_lo; c < c_hi; c += 4) {
      float2 w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) w[u] = __ldg(wt + (int64_t)(c + u) * hp);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(s.gs + (r0 + q) * a.nwp + c);
        acc[q] = __ffma2_rn(make_float2(v.x, v.x), w[0], acc[q]);
        acc[q] = __ffma2_rn(make_float2(v.y, v.y), w[1], acc[q]);
        acc[q] = __ffma2_rn(make_float2(v.z, v.z), w[2], acc[q]);
        acc[q] = __ffma2_rn(make_float2(v.w, v.w), w[3], acc[q]);
      }
    }
    if (part == NP - 1) {
      for (int c = nw4; c < a.nw; ++c) {
        const float2 wv = __ldg(wt + (int64_t)c * hp);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float v = s.gs[(r0 + q) * a.nwp + c];
          acc[q] = __ffma2_rn(make_float2(v, v), wv, acc[q]);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
      reinterpret_cast<float2*>(red)[(part * CE + r0 + q) * hp + kp] = acc[q];
  }
  __syncthreads();
  for (int t = threadIdx.x; t < CE * hp; t += blockDim.x) {
    const int r = t / hp, k2 = t - r * hp;
    float2 v = reinterpret_cast<const float2*>(red)[r * hp + k2];
    for (int q = 1; q < NP; ++q) {
      const float2 u = reinterpret_cast<const float2*>(red)[(q * CE + r) * hp + k2];
      v.x += u.x;
      v.y += u.y;
    }
    if (r < ne && s.es[r] >= 0) *reinterpret_cast<float2*>(a.gh + (int64_t)s.es[r] * a.H + 2 * k2) = v;
  }
}

__device__ __forceinline__ void sh16(const float* __restrict__ vec, int e, float (&Y)[16], float& rx, float& ry,
                                     float& rz, float& ir) {
  edge_geometry(__ldg(vec + 3 * (int64_t)e), __ldg(vec + 3 * (int64_t)e + 1), __ldg(vec + 3 * (int64_t)e + 2), rx,
                ry, rz, ir);
  gen::ShAll::sh(rx, ry, rz, Y);
}

}  // namespace rad

// Spec-specialised passes (radial_spec.cu): launch when the plan runs a compiled whole path list
// and the chunk size has an instance; *handled = false otherwise (nothing launched).
cudaError_t launch_rad_fwd_spec(const RadArgs& a, const GenTable& T, int ce, size_t smem, cudaStream_t s,
                                bool* handled);
cudaError_t launch_rad_send_spec(const RadArgs& a, const GenTable& T, int ce, size_t smem, cudaStream_t s,
                                 bool* handled);

}  // namespace tp
