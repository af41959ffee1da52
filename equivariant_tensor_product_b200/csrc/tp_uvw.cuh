// uvw mode: fully connected multiplicity mixing per path, reassociated so that no edge-sized
// tensor exists ("Sobek: Streaming Equivariant Tensor Product Convolutions", abstract: the
// streaming formulation keeps fully connected multiplicity mixing; edge-sized intermediates
// are artifacts of the schedule).
//
//   y[i, o, w, m3] = sum_{p into o} sum_u W_p[u, w] A_p[i, u, m3]
//   A_p[i, u, m3]  = sum_{e into i} c_p s[e, p] sum_{m1,m2} C_p[m1,m2,m3] x[j, in(p), u, m1] Y(v_e)[m2]
//
// Forward: A is node-sized state (N x sum_p mul (2 l3 + 1) floats), aggregated by the
// receiver-order edge pass below (which gathers the narrow x rows) and mixed by a tcgen05
// GEMM per output irrep.  Backward, re-associated on the sender side so that the per-edge
// gather is the gy row (sum_o mul_out (2 l3 + 1) floats) rather than a per-path gradient
// state:
//   xt_p[j, w, m1] = sum_u x[j, in(p), u, m1] W_p[u, w]                       (GEMM)
//   B_p[j, w, m1]  = sum_{e from j} c_p s[e,p] sum_{m2,m3} C Y[m2] gy[i, o(p), w, m3]   (sender pass)
//   gs[e, p]       = c_p sum_{w,m1,m2,m3} C xt_p[j,w,m1] Y[m2] gy[i,o(p),w,m3]        (sender pass)
//   gx[j, a, u, m1] = sum_{p: in(p)=a} sum_w B_p[j, w, m1] W_p[u, w]          (GEMM)
//   gW_p[u, w]     = sum_j sum_m1 x[j, in(p), u, m1] B_p[j, w, m1]           (split-K GEMM)
// All sums run in a fixed order: the results are deterministic.
#pragma once
#include <algorithm>
#include <type_traits>

#include "tp_kernels.cuh"
#include "tp_mma.cuh"

namespace tp {

// ---------------------------------------------------------------------------------------
// Edge pass: A (receiver order).  grid = N * n_slices, block = 32 * split.
// ---------------------------------------------------------------------------------------
template <class S>
__global__ void __launch_bounds__(kMaxThreads) k_uvw_edge(const __grid_constant__ LaunchArgs a) {
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31;
  const int phase = threadIdx.x >> 5;
  const int row = blockIdx.x / a.n_slices;
  const int sl = blockIdx.x - row * a.n_slices;
  const int c = sl * 32 + lane;
  const bool act = c < a.mul;
  int e0 = __ldg(a.rowptr + row), e1 = __ldg(a.rowptr + row + 1);
  if (a.check) {
    e0 = max(0, min(e0, a.E));
    e1 = max(e0, min(e1, a.E));
  }
  const int st = a.split;
  float acc[S::A_PC];
#pragma unroll
  for (int k = 0; k < S::A_PC; ++k) acc[k] = 0.f;
  for (int base = e0 + phase; base < e1; base += 32 * st) {
    const int my_e = base + lane * st;
    int my_j = 0;
    float vx = 0.f, vy = 0.f, vz = 0.f;
    if (my_e < e1) {
      my_j = __ldg(a.src + my_e);
      vx = __ldg(a.vec + 3 * (int64_t)my_e);
      vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
      vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
      if (a.check && (unsigned)my_j >= (unsigned)a.N) {
        report(a, kDevBadSrc);
        my_j = -1;
      }
    }
    const int ne = min(32, (e1 - base + st - 1) / st);
#pragma unroll 1
    for (int k = 0; k < ne; ++k) {
      const int e = base + k * st;
      const int j = __shfl_sync(kFull, my_j, k);
      const float ux = __shfl_sync(kFull, vx, k);
      const float uy = __shfl_sync(kFull, vy, k);
      const float uz = __shfl_sync(kFull, vz, k);
      if (j < 0) continue;
      float x[S::IN_PC], s[S::P];
      if (act) S::load_in(a.x + (int64_t)j * a.in_dim, a.mul, c, x);
      const float* srow = a.w + (int64_t)e * S::P;
#pragma unroll
      for (int p = 0; p < S::P; ++p) s[p] = __ldg(srow + p) * (a.has_coeff ? a.coeff[p] : 1.f);
      float rx, ry, rz, ir;
      edge_geometry(ux, uy, uz, rx, ry, rz, ir);
      float Y[S::NSH];
      S::sh(rx, ry, rz, Y);
      if (act) S::uvw_edge(x, Y, s, acc);
    }
  }
  reduce_phases(acc, smem, phase, st, lane, 0, 1);
  if (phase == 0 && act) S::store_uvw(a.A, a.N, a.mul, row, c, acc);
}

// Split of one shared weight into its TF32 hi part (at dst) and lo part (at dst + n).
__device__ __forceinline__ void put_split(float* dst, int64_t n, float v) {
  const float h = tf32_hi(v);
  dst[0] = h;
  dst[n] = v - h;
}

// Receiver pass with the senders' x rows staged whole by cp.async.bulk into a ring of
// kEdgeSlots shared-memory slots read by all NSL slice warps of the CTA (one CTA per
// receiver, warp = 32-channel slice, every warp walks all edges of the row); the last warp
// to finish with a slot refills it with the row kEdgeSlots edges ahead.  Same arithmetic
// as k_uvw_edge.  Needs no index checks, a CTA that covers every input channel and 16-byte
// aligned rows (the launcher checks).
constexpr int kEdgeSlots = 4;

template <class S, int NSL>
__global__ void __launch_bounds__(kMaxThreads) k_uvw_edge_staged(const __grid_constant__ LaunchArgs a) {
  extern __shared__ __align__(128) unsigned char esm[];
  __shared__ __align__(8) uint64_t full_bar[kEdgeSlots];
  __shared__ float sbat[32 * S::P];
  __shared__ uint32_t read_cnt[kEdgeSlots];
  __shared__ int last_fill[kEdgeSlots];
  __shared__ volatile int gather_failed;
  const int lane = threadIdx.x & 31;
  const int sl = threadIdx.x >> 5;
  const int row = blockIdx.x;
  const int c = sl * 32 + lane;
  const bool act = c < a.mul;
  const int e0 = __ldg(a.rowptr + row), e1 = __ldg(a.rowptr + row + 1);
  const uint32_t row_bytes = (uint32_t)a.in_dim * 4u;
  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < kEdgeSlots; ++s2) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sm_addr(&full_bar[s2])) : "memory");
      read_cnt[s2] = 0;
      last_fill[s2] = -1;
    }
    gather_failed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  auto fill = [&](int f, int j) {
    const int s2 = f % kEdgeSlots;
    const uint32_t mb = sm_addr(&full_bar[s2]);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mb), "r"(row_bytes) : "memory");
    bulk_g2s(sm_addr(esm + (size_t)s2 * row_bytes), a.x + (int64_t)j * a.in_dim, row_bytes, mb);
    last_fill[s2] = f;
  };
  float acc[S::A_PC];
#pragma unroll
  for (int k = 0; k < S::A_PC; ++k) acc[k] = 0.f;
  int first = 0;
  for (int base = e0; base < e1; base += 32) {
    const int my_e = base + lane;
    int my_j = 0;
    float vx = 0.f, vy = 0.f, vz = 0.f;
    if (my_e < e1) {
      my_j = __ldg(a.src + my_e);
      vx = __ldg(a.vec + 3 * (int64_t)my_e);
      vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
      vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
    }
    const int ne = min(32, e1 - base);
    if (sl == 0) {
      for (int k = 0; k < min(ne, kEdgeSlots); ++k) {
        const int j = __shfl_sync(kFull, my_j, k);
        if (lane == 0) fill(first + k, j);
      }
    }
    // the batch's path scalars (contiguous rows in receiver order), once for all warps
    for (int t = threadIdx.x; t < ne * S::P; t += blockDim.x) sbat[t] = __ldg(a.w + (int64_t)base * S::P + t);
    __syncthreads();
#pragma unroll 1
    for (int k = 0; k < ne; ++k) {
      const int f = first + k, s2 = f % kEdgeSlots;
      bool ok = !gather_failed;
      if (ok) ok = slot_wait(sm_addr(&full_bar[s2]), (uint32_t)((f / kEdgeSlots) & 1));
      ok = __all_sync(kFull, ok);
      if (!ok) gather_failed = 1;
      const float* xrow = reinterpret_cast<const float*>(esm + (size_t)s2 * row_bytes);
      float x[S::IN_PC];
      if (ok && act) S::load_in_shared(xrow, a.mul, c, x);
      // this warp is done with the slot; the last of the NSL warps refills it
      __syncwarp();
      int last = 0;
      if (lane == 0 && ok) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        uint32_t old;
        asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;" : "=r"(old) : "r"(sm_addr(&read_cnt[s2])) : "memory");
        last = old == NSL - 1;
      }
      last = __shfl_sync(kFull, last, 0);
      const int jnext = __shfl_sync(kFull, my_j, min(k + kEdgeSlots, 31));
      if (last && lane == 0) {
        read_cnt[s2] = 0;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (k + kEdgeSlots < ne) fill(f + kEdgeSlots, jnext);
      }
      if (!ok) continue;
      float sp[S::P];
#pragma unroll
      for (int p = 0; p < S::P; ++p) sp[p] = sbat[k * S::P + p] * (a.has_coeff ? a.coeff[p] : 1.f);
      const float ux = __shfl_sync(kFull, vx, k), uy = __shfl_sync(kFull, vy, k), uz = __shfl_sync(kFull, vz, k);
      float rx, ry, rz, ir;
      edge_geometry(ux, uy, uz, rx, ry, rz, ir);
      float Y[S::NSH];
      S::sh(rx, ry, rz, Y);
      if (act) S::uvw_edge(x, Y, sp, acc);
    }
    __syncthreads();   // every warp is done with this batch's slots
    first += ne;
  }
  if (gather_failed && threadIdx.x == 0) {   // let the issued copies land, then report
    for (int s2 = 0; s2 < kEdgeSlots; ++s2) {
      const int f = last_fill[s2];
      if (f < 0) continue;
      const uint32_t mb = sm_addr(&full_bar[s2]);
      const unsigned long long t0 = now_ns();
      while (!slot_ready(mb, (uint32_t)((f / kEdgeSlots) & 1)) && now_ns() - t0 < kGatherWaitNs) {
      }
    }
    report(a, kDevGatherTimeout);
  }
  if (act) S::store_uvw(a.A, a.N, a.mul, row, c, acc);
}

// Receiver pass with the per-edge coupling matrix K_e (S::km_build): one CTA per receiver,
// NW warps, every lane CH channels (c, and c + 32 when CH = 2, of its warp's 32 CH).  The
// row's edges are taken in batches of KB.  The K rows of a batch (the edge's harmonics, path
// scalars and CG entries folded once for all channels; 32 NW / KB threads per edge, each a
// part of the row) are written into one of two shared-memory buffers while the warps still
// walk the previous batch: its inputs (edge vectors and path scalars) are copied by
// cp.async at the start of that batch.  Every warp reads each sender's x row from a ring of
// copy-engine slots that runs ahead across batch boundaries, and accumulates
// A[(p, m3)] += x[a, m1] K_e two rows at a time.  Same sums as k_uvw_edge, in another
// association (per edge, C Y s first).  Needs no index checks and 16-byte aligned rows (the
// launcher checks).
template <class S, int NW, int KB, int CH, int MINB, int R = kEdgeSlots>
__global__ void __launch_bounds__(32 * NW, MINB) k_uvw_recv_km(const __grid_constant__ LaunchArgs a) {
  static_assert((32 * NW) % KB == 0, "threads per edge");
  constexpr int H = 32 * NW / KB;
  static_assert(H == 1 || H == 2 || H == 4 || H == 8, "parts of a K row");
  constexpr int NIN = S::P + 3;   // per edge: path scalars, edge vector
  extern __shared__ __align__(128) unsigned char esm[];
  __shared__ __align__(8) uint64_t full_bar[R];
  __shared__ uint32_t read_cnt[R];
  __shared__ int last_fill[R];
  __shared__ volatile int gather_failed;
  __shared__ float stage[2][KB * NIN];
  __shared__ int stage_src[2][KB + R];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int row = blockIdx.x;
  const int c0 = wid * 32 * CH + lane, c1 = c0 + 32;
  const bool act0 = c0 < a.mul, act1 = CH == 2 && c1 < a.mul;
  const int e0 = __ldg(a.rowptr + row), e1 = __ldg(a.rowptr + row + 1);
  const uint32_t row_bytes = (uint32_t)a.in_dim * 4u;
  float4* kbuf = reinterpret_cast<float4*>(esm + (size_t)R * row_bytes);   // [2][KB][KM_ROW]
  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < R; ++s2) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sm_addr(&full_bar[s2])) : "memory");
      read_cnt[s2] = 0;
      last_fill[s2] = -1;
    }
    gather_failed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // ring fill f carries the x row of edge e0 + f, sender j
  auto fill = [&](int f, int j) {
    const int s2 = f % R;
    const uint32_t mb = sm_addr(&full_bar[s2]);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mb), "r"(row_bytes) : "memory");
    bulk_g2s(sm_addr(esm + (size_t)s2 * row_bytes), a.x + (int64_t)j * a.in_dim, row_bytes, mb);
    last_fill[s2] = f;
  };
  // the inputs of the batch at edge b0 into stage buffer sb (cp.async, one group per thread):
  // path scalars and edge vectors of its edges, senders of its edges and the ring's lookahead
  auto stage_inputs = [&](int b0, int sb) {
    const int nb = min(KB, e1 - b0);
    for (int t = threadIdx.x; t < nb * NIN; t += 32 * NW) {
      const int k = t / NIN, v = t - k * NIN;
      const float* src = v < S::P ? a.w + (int64_t)(b0 + k) * S::P + v : a.vec + 3 * (int64_t)(b0 + k) + (v - S::P);
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sm_addr(&stage[sb][t])), "l"(src) : "memory");
    }
    const int ns = min(KB + R, e1 - b0);
    for (int t = threadIdx.x; t < ns; t += 32 * NW)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sm_addr(&stage_src[sb][t])), "l"(a.src + b0 + t) : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // K rows of the batch at edge b0 (stage buffer sb) into buffer kb
  auto build = [&](int b0, int sb, float4* kb) {
    const int k = threadIdx.x % KB, h = threadIdx.x / KB;
    if (b0 + k < e1) {
      const float* in = stage[sb] + k * NIN;
      float rx, ry, rz, ir;
      edge_geometry(in[S::P], in[S::P + 1], in[S::P + 2], rx, ry, rz, ir);
      float Y[S::NSH], cs[S::P];
      S::sh(rx, ry, rz, Y);
#pragma unroll
      for (int p = 0; p < S::P; ++p) cs[p] = in[p] * (a.has_coeff ? a.coeff[p] : 1.f);
      S::template km_build<H>(h, Y, cs, kb + (size_t)k * (S::KM_ROW / 4));
    }
  };
  float2 acc0[S::KM_PAIRS], acc1[CH == 2 ? S::KM_PAIRS : 1];
#pragma unroll
  for (int k = 0; k < S::KM_PAIRS; ++k) acc0[k] = make_float2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < (CH == 2 ? S::KM_PAIRS : 1); ++k) acc1[k] = make_float2(0.f, 0.f);
  const int ntot = e1 - e0;
  if (ntot > 0) {
    stage_inputs(e0, 0);
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0)
      for (int f = 0; f < min(ntot, R); ++f) fill(f, stage_src[0][f]);
    build(e0, 0, kbuf);
    __syncthreads();
  }
  int buf = 0;
  for (int base = e0; base < e1; base += KB) {
    const int ne = min(KB, e1 - base);
    const bool more = base + KB < e1;
    if (more) stage_inputs(base + KB, buf ^ 1);
    const float4* kcur = kbuf + (size_t)buf * KB * (S::KM_ROW / 4);
#pragma unroll 1
    for (int k = 0; k < ne; ++k) {
      const int f = base - e0 + k, s2 = f % R;
      bool ok = !gather_failed;
      if (ok) ok = slot_wait(sm_addr(&full_bar[s2]), (uint32_t)((f / R) & 1));
      ok = __all_sync(kFull, ok);
      if (!ok) gather_failed = 1;
      const float* xrow = reinterpret_cast<const float*>(esm + (size_t)s2 * row_bytes);
      float x0[S::IN_PC], x1[CH == 2 ? S::IN_PC : 1];
      if (ok) {
        if (act0) S::load_in_shared(xrow, a.mul, c0, x0);
        if constexpr (CH == 2) {
          if (act1) S::load_in_shared(xrow, a.mul, c1, x1);
        }
      }
      // this warp is done with the slot; the last of the NW warps refills it
      __syncwarp();
      int last = 0;
      if (lane == 0 && ok) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        uint32_t old;
        asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;" : "=r"(old) : "r"(sm_addr(&read_cnt[s2])) : "memory");
        last = old == NW - 1;
      }
      last = __shfl_sync(kFull, last, 0);
      if (last && lane == 0) {
        read_cnt[s2] = 0;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (f + R < ntot) fill(f + R, stage_src[buf][k + R]);
      }
      if (!ok) continue;
      const float4* kr = kcur + (size_t)k * (S::KM_ROW / 4);
      if constexpr (CH == 2) {
        if (act1) S::km_apply2(x0, x1, kr, acc0, acc1);
        else if (act0) S::km_apply1(x0, kr, acc0);
      } else if (act0) {
        S::km_apply1(x0, kr, acc0);
      }
    }
    if (more) {   // the next batch's K rows into the other buffer (last read two batches ago)
      asm volatile("cp.async.wait_all;" ::: "memory");
      __syncthreads();
      build(base + KB, buf ^ 1, kbuf + (size_t)(buf ^ 1) * KB * (S::KM_ROW / 4));
    }
    __syncthreads();
    buf ^= 1;
  }
  if (gather_failed && threadIdx.x == 0) {   // let the issued copies land, then report
    for (int s2 = 0; s2 < R; ++s2) {
      const int f = last_fill[s2];
      if (f < 0) continue;
      const uint32_t mb = sm_addr(&full_bar[s2]);
      const unsigned long long t0 = now_ns();
      while (!slot_ready(mb, (uint32_t)((f / R) & 1)) && now_ns() - t0 < kGatherWaitNs) {
      }
    }
    report(a, kDevGatherTimeout);
  }
  if (act0) S::km_store(a.A, a.N, a.mul, row, c0, acc0);
  if constexpr (CH == 2) {
    if (act1) S::km_store(a.A, a.N, a.mul, row, c1, acc1);
  }
}

// Wt[o][w][pl * mul + u] = W[path_of(o, pl)][u][w]: B operand of the forward mixing GEMM
// (hi at Wt, lo at Wt + P * mul * mul_out).
template <class S>
__global__ void k_uvw_prep_wt(const __grid_constant__ LaunchArgs a) {
  const int64_t per_path = (int64_t)a.mul * a.mul_out;
  const int64_t total = per_path * S::P;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    // t enumerates (o, w, pl, u) region by region
    int64_t rem = t, base = 0;
    int o = 0;
    for (; o < S::N_OUT; ++o) {
      const int64_t sz = (int64_t)S::out_cnt_at(o) * per_path;
      if (rem < sz) break;
      rem -= sz;
      base += sz;
    }
    const int K = S::out_cnt_at(o) * a.mul;
    const int w = (int)(rem / K), kk = (int)(rem % K);
    const int pl = kk / a.mul, u = kk % a.mul;
    const int p = S::path_of_at(o, pl);
    put_split(a.Wt + base + rem, total, a.W[(int64_t)p * per_path + (int64_t)u * a.mul_out + w]);
  }
}

// Backward B operands, per input irrep a (paths pl of that irrep), hi and lo each:
//   Wg[a][u][pl * mul_out + w]  = W[path_in(a, pl)][u][w]   (gx GEMM)       at Wt, Wt + n
//   Wx[a][pl * mul_out + w][u]  = W[path_in(a, pl)][u][w]   (x W GEMM)      at Wt + 2n, Wt + 3n
template <class S>
__global__ void k_uvw_prep_wg(const __grid_constant__ LaunchArgs a) {
  const int64_t per_path = (int64_t)a.mul * a.mul_out;
  const int64_t total = per_path * S::P;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    int64_t rem = t, base = 0;
    int ai = 0;
    for (; ai < S::N_IN; ++ai) {
      const int64_t sz = (int64_t)S::in_cnt_at(ai) * per_path;
      if (rem < sz) break;
      rem -= sz;
      base += sz;
    }
    const int K = S::in_cnt_at(ai) * a.mul_out;
    const int u = (int)(rem / K), kk = (int)(rem % K);
    const int pl = kk / a.mul_out, w = kk % a.mul_out;
    const int p = S::path_in_at(ai, pl);
    const float v = a.W[(int64_t)p * per_path + (int64_t)u * a.mul_out + w];
    put_split(a.Wt + base + rem, total, v);
    put_split(a.Wt + 2 * total + base + (int64_t)kk * a.mul + u, total, v);
  }
}

// xT[a][(j, m1)][u] = x[j, a, u, m1]: the input irreps as K-contiguous rows for the x W
// GEMM (and, read M-major, for the gW GEMM).  grid = N, one node row per CTA.
template <class S>
__global__ void k_uvw_xt(const __grid_constant__ LaunchArgs a) {
  const int j = blockIdx.x;
  const float* xr = a.x + (int64_t)j * a.in_dim;
  for (int ai = 0; ai < S::N_IN; ++ai) {
    const int d1 = S::in_d1_at(ai);
    const int n = d1 * a.mul;
    const int64_t xbase = (int64_t)a.mul * S::in_cum_at(ai);
    float* dst = a.xT + (int64_t)a.N * xbase + (int64_t)j * n;
    for (int t = threadIdx.x; t < n; t += blockDim.x) {
      const int m1 = t / a.mul, u = t - m1 * a.mul;
      dst[t] = __ldg(xr + xbase + (int64_t)u * d1 + m1);
    }
  }
}

// Warp-level epilogue stores.  T holds a rows x cols block (row stride ld) of the
// accumulator whose first element sits at global row r0, global column n0; the 32 lanes of
// one warp store it with one contiguous 128-byte run per instruction.

// Rows are (node, m) pairs, m < D; the output layout is [node][base + col * D + m], so the
// block of node i is one contiguous run of cols * D floats.
template <int D>
__device__ __forceinline__ void store_node_rows(float* out, int64_t row_stride, int64_t base, const float* T,
                                                int ld, int64_t r0, int rows, int64_t M, int n0, int cols,
                                                int lane) {
  const int64_t rlast = min(M, r0 + rows) - 1;
  if (rlast < r0) return;
  const int64_t i0 = r0 / D, i1 = rlast / D;
  for (int64_t i = i0; i <= i1; ++i) {
    float* dst = out + i * row_stride + base + (int64_t)n0 * D;
    for (int q = lane; q < cols * D; q += 32) {
      const int w = q / D, m = q - w * D;
      const int64_t row = i * D + m;
      if (row >= r0 && row <= rlast) dst[q] = T[(int)(row - r0) * ld + w];
    }
  }
}

// Row-major [M][Nn] output: lane = column, one row per instruction.
__device__ __forceinline__ void store_rows(float* out, int64_t Nn, const float* T, int ld, int64_t r0, int rows,
                                           int64_t M, int n0, int cols, int lane) {
  if (lane >= cols) return;
  const int nr = (int)min((int64_t)rows, M - r0);
  float* dst = out + r0 * Nn + n0 + lane;
  for (int r = 0; r < nr; ++r) dst[(int64_t)r * Nn] = T[r * ld + lane];
}

struct TcMaps {
  CUtensorMap tA, tA2, tB, tB2;
};

// y_o[(i, m3), w] = sum_k A_o[(i, m3), k] Wt_o[w, k],  k = (pl, u)
template <int D3>
struct MixFwdTc : TcMaps {
  int64_t M, Nn;
  int64_t ybase;
  int K;
  static constexpr int A_FMT = FMT_K, B_FMT = FMT_SPLIT, PROMOTE = 0;
  __device__ void k_range(const LaunchArgs&, int, int64_t& b, int64_t& e) const { b = 0; e = K; }
  __device__ void store_tile(const LaunchArgs& a, int, const float* T, int ld, int64_t r0, int rows, int n0,
                             int cols, int lane) const {
    store_node_rows<D3>(a.y, a.out_dim, ybase, T, ld, r0, rows, M, n0, cols, lane);
  }
};

// xt_a[(j, m1), (pl, w)] = sum_u xT_a[(j, m1), u] Wx_a[(pl, w), u]
template <int D1>
struct XtTc : TcMaps {
  int64_t M, Nn;
  int K;                 // mul
  float* out;            // region a of the xt buffer, row-major [M][Nn]
  static constexpr int A_FMT = FMT_K, B_FMT = FMT_SPLIT, PROMOTE = 0;
  __device__ void k_range(const LaunchArgs&, int, int64_t& b, int64_t& e) const { b = 0; e = K; }
  __device__ void store_tile(const LaunchArgs&, int, const float* T, int ld, int64_t r0, int rows, int n0,
                             int cols, int lane) const {
    store_rows(out, Nn, T, ld, r0, rows, M, n0, cols, lane);
  }
};

// gx[j, a, u, m1] = sum_k B_a[(j, m1), k] Wg_a[u, k],  k = (pl, w)
template <int D1>
struct GxTc : TcMaps {
  int64_t M, Nn;
  int64_t xbase;
  int K;
  static constexpr int A_FMT = FMT_K, B_FMT = FMT_SPLIT, PROMOTE = 0;
  __device__ void k_range(const LaunchArgs&, int, int64_t& b, int64_t& e) const { b = 0; e = K; }
  __device__ void store_tile(const LaunchArgs& a, int, const float* T, int ld, int64_t r0, int rows, int n0,
                             int cols, int lane) const {
    store_node_rows<D1>(a.gx, a.in_dim, xbase, T, ld, r0, rows, M, n0, cols, lane);
  }
};

// part[z][p][u][w] = sum_{(j, m1) in split z} xT_a[(j, m1), u] B_a[(j, m1), (pl, w)]
template <int D1>
struct GwTc : TcMaps {
  int64_t M, Nn;         // mul, cnt_a * mul_out
  int64_t rows;          // N * d1 (the reduction)
  int64_t wstride;
  int splits, mul_out, P;
  int paths[kMaxPaths];
  static constexpr int A_FMT = FMT_MN, B_FMT = FMT_MN, PROMOTE = 16;   // K = N * d1 / splits rows
  __device__ void k_range(const LaunchArgs&, int z, int64_t& b, int64_t& e) const {
    const int64_t chunk = ((rows + splits - 1) / splits + TC_BK - 1) / TC_BK * TC_BK;
    b = min(rows, (int64_t)z * chunk);
    e = min(rows, b + chunk);
  }
  __device__ void store_tile(const LaunchArgs& a, int z, const float* T, int ld, int64_t r0, int rows, int n0,
                             int cols, int lane) const {
    if (lane >= cols) return;
    const int n = n0 + lane;
    const int pl = n / mul_out, w = n - pl * mul_out;
    float* dst = a.part + ((int64_t)z * P + paths[pl]) * wstride + w;
    const int nr = (int)min((int64_t)rows, M - r0);
    for (int r = 0; r < nr; ++r) dst[(r0 + r) * mul_out] = T[r * ld + lane];
  }
};

// gW[idx] = sum_z part[z][idx] in split order (deterministic)
static __global__ void k_reduce_splits(const float* __restrict__ part, int splits, int64_t n, float* gW) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n; t += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int z = 0; z < splits; ++z) s += part[(int64_t)z * n + t];
    gW[t] = s;
  }
}

// ---------------------------------------------------------------------------------------
// Sender pass: B (per sender, per path), gs[e, p] and gvec[e]; lane = output channel w.
// gs and gvec are channel sums across all slices of the sender, which share one CTA.
// grid = N, block = 32 * NSL.
// ---------------------------------------------------------------------------------------
// Sums 16 values over the 32 lanes of a warp with 16 exchanges (against 80 for 16 separate
// butterflies): at each halving step a lane keeps half of its values and trades the other
// half with its partner.  Returns, in lanes 2v and 2v + 1, the warp sum of value v.
__device__ __forceinline__ float warp_reduce_scatter16(float* v, int lane) {
#pragma unroll
  for (int h = 8; h >= 1; h >>= 1) {
    const bool up = lane & (2 * h);
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = up ? v[i] : v[i + h];
      const float keep = up ? v[i + h] : v[i];
      v[i] = keep + __shfl_xor_sync(kFull, send, 2 * h);
    }
  }
  return v[0] + __shfl_xor_sync(kFull, v[0], 1);
}

// STAGED: the receivers' gy rows are fetched whole by cp.async.bulk into a ring of
// kSendSlots shared-memory slots that all NSL slice warps of the CTA read; the last warp to
// finish with a slot refills it with the row kSendSlots edges ahead.  Needs no index checks,
// a CTA that covers every output channel and 16-byte aligned rows (the launcher checks).
constexpr int kSendSlots = 3;

template <class S, bool GVEC, int NSL>
struct SendShape {
  static constexpr int NV = S::P + 4;
  static size_t smem_bytes(bool staged, int out_dim) {
    return (size_t)32 * NSL * NV * sizeof(float) + (staged ? (size_t)kSendSlots * out_dim * sizeof(float) : 0);
  }
};

template <class S, bool GVEC, int NSL, bool STAGED>
__global__ void __launch_bounds__(kMaxThreads) k_uvw_send(const __grid_constant__ LaunchArgs a) {
  extern __shared__ float smem[];
  constexpr int NV = S::P + 4;   // per edge and slice: P gs partials, 3 gvec partials, degree sum
  __shared__ __align__(8) uint64_t full_bar[kSendSlots];
  __shared__ uint32_t read_cnt[kSendSlots];
  __shared__ int last_fill[kSendSlots];
  __shared__ volatile int gather_failed;
  __shared__ int32_t rtab[kRowTab];
  __shared__ float sbat[STAGED ? 32 * S::P : 1];
  const int lane = threadIdx.x & 31;
  const int sl = threadIdx.x >> 5;
  const int node = blockIdx.x;
  const int c = sl * 32 + lane;
  const bool act = c < a.mul_out;
  int q0 = __ldg(a.colptr + node), q1 = __ldg(a.colptr + node + 1);
  if (a.check) {
    q0 = max(0, min(q0, a.E));
    q1 = max(q0, min(q1, a.E));
  }
  unsigned char* ring = reinterpret_cast<unsigned char*>(smem + 32 * NSL * NV);
  const uint32_t row_bytes = (uint32_t)a.out_dim * 4u;
  if constexpr (STAGED) {
    if (threadIdx.x == 0) {
      for (int s2 = 0; s2 < kSendSlots; ++s2) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sm_addr(&full_bar[s2])) : "memory");
        read_cnt[s2] = 0;
        last_fill[s2] = -1;
      }
      gather_failed = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  }
  const RowTab rt = load_row_tab(a.rowptr, a.N, rtab);
  __syncthreads();
  // fill f (a running index over this CTA's edges) -> slot f % kSendSlots
  auto fill = [&](int f, int i) {
    const int s2 = f % kSendSlots;
    const uint32_t mb = sm_addr(&full_bar[s2]);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mb), "r"(row_bytes) : "memory");
    bulk_g2s(sm_addr(ring + (size_t)s2 * row_bytes), a.gy + (int64_t)i * a.out_dim, row_bytes, mb);
    last_fill[s2] = f;
  };
  int first = 0;   // fill index of edge 0 of the current batch
  float xt[S::XT_PC], bt[S::XT_PC];
#pragma unroll
  for (int k = 0; k < S::XT_PC; ++k) {
    bt[k] = 0.f;
    xt[k] = 0.f;
  }
  if (act) S::load_xt(a.A, a.N, a.mul_out, node, c, xt);
  float* slot = smem;   // [32 edges][NSL][NV]

  for (int base = q0; base < q1; base += 32) {
    const int my_q = base + lane;
    int my_e = -1, my_i = 0;
    float vx = 0.f, vy = 0.f, vz = 0.f;
    if (my_q < q1) {
      my_e = __ldg(a.perm + my_q);
      if (a.check && (unsigned)my_e >= (unsigned)a.E) {
        report(a, kDevBadPerm);
        my_e = -1;
      } else {
        my_i = find_row_tab(a.rowptr, a.N, rtab, rt, my_e);
        vx = __ldg(a.vec + 3 * (int64_t)my_e);
        vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
        vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
      }
    }
    const int ne = min(32, q1 - base);
    if constexpr (STAGED) {
      if (sl == 0) {
        for (int k = 0; k < min(ne, kSendSlots); ++k) {
          const int i = __shfl_sync(kFull, my_i, k);
          if (lane == 0) fill(first + k, i);
        }
      }
      // the batch's path scalars, once for all slice warps
      for (int t = threadIdx.x; t < ne * S::P; t += blockDim.x) {
        const int kk = t / S::P;
        sbat[t] = __ldg(a.w + (int64_t)__ldg(a.perm + base + kk) * S::P + (t - kk * S::P));
      }
      __syncthreads();
    }
#pragma unroll 1
    for (int k = 0; k < ne; ++k) {
      const int e = __shfl_sync(kFull, my_e, k);
      const int i = __shfl_sync(kFull, my_i, k);
      const float* grow = nullptr;   // this edge's gy row (staged slot or global)
      if constexpr (STAGED) {
        const int f = first + k, s2 = f % kSendSlots;
        bool ok = !gather_failed;
        if (ok) ok = slot_wait(sm_addr(&full_bar[s2]), (uint32_t)((f / kSendSlots) & 1));
        ok = __all_sync(kFull, ok);
        if (!ok) gather_failed = 1;
        grow = ok ? reinterpret_cast<const float*>(ring + (size_t)s2 * row_bytes) : nullptr;
      } else {
        grow = a.gy + (int64_t)i * a.out_dim;
      }
      const float ux = __shfl_sync(kFull, vx, k);
      const float uy = __shfl_sync(kFull, vy, k);
      const float uz = __shfl_sync(kFull, vz, k);
      float rx, ry, rz, ir;
      edge_geometry(ux, uy, uz, rx, ry, rz, ir);
      float Y[S::NSH];
      S::sh(rx, ry, rz, Y);
      float gY[S::NSH], gs[S::P];
#pragma unroll
      for (int m = 0; m < S::NSH; ++m) gY[m] = 0.f;
#pragma unroll
      for (int p = 0; p < S::P; ++p) gs[p] = 0.f;
      if (e >= 0) {
        float s[S::P];
        if constexpr (STAGED) {
#pragma unroll
          for (int p = 0; p < S::P; ++p) s[p] = sbat[k * S::P + p] * (a.has_coeff ? a.coeff[p] : 1.f);
        } else {
          const float* srow = a.w + (int64_t)e * S::P;
#pragma unroll
          for (int p = 0; p < S::P; ++p) s[p] = __ldg(srow + p) * (a.has_coeff ? a.coeff[p] : 1.f);
        }
        if (act && grow) {
          float gyv[S::OUT_PC];
          if constexpr (STAGED) {
            S::load_out_shared(grow, a.mul_out, c, gyv);
          } else {
            S::load_out(grow, a.mul_out, c, gyv);
          }
          S::template uvw_send<GVEC>(xt, Y, s, gyv, bt, gs, gY);
        }
      }
      if constexpr (STAGED) {
        // this warp is done with the slot; the last of the NSL warps refills it
        __syncwarp();
        int last = 0;
        if (lane == 0 && grow) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          uint32_t old;
          asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;"
                       : "=r"(old)
                       : "r"(sm_addr(&read_cnt[(first + k) % kSendSlots]))
                       : "memory");
          last = old == NSL - 1;
        }
        last = __shfl_sync(kFull, last, 0);
        const int inext = __shfl_sync(kFull, my_i, min(k + kSendSlots, 31));
        if (last) {
          if (lane == 0) {
            read_cnt[(first + k) % kSendSlots] = 0;
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            if (k + kSendSlots < ne) fill(first + k + kSendSlots, inext);
          }
        }
      }
      float h0 = 0.f, h1 = 0.f, h2 = 0.f, sdeg = 0.f;
      if constexpr (GVEC) {
        float G[S::NSH][3];
        S::sh_grad(rx, ry, rz, G);
#pragma unroll
        for (int m = 0; m < S::NSH; ++m) {
          h0 = fmaf(gY[m], G[m][0], h0);
          h1 = fmaf(gY[m], G[m][1], h1);
          h2 = fmaf(gY[m], G[m][2], h2);
          sdeg = fmaf(S::sh_degree(m) * gY[m], Y[m], sdeg);
        }
      }
      // channel sums of the NR per-edge values: 16 at a time, each lane pair ends up
      // holding one of them (reduce-scatter), which one lane writes to the slice slot
      constexpr int NR = GVEC ? S::P + 4 : S::P;
      float r[(NR + 15) / 16 * 16];
#pragma unroll
      for (int v = 0; v < (NR + 15) / 16 * 16; ++v) r[v] = 0.f;
#pragma unroll
      for (int p = 0; p < S::P; ++p) r[p] = gs[p];
      if constexpr (GVEC) {
        r[S::P] = h0;
        r[S::P + 1] = h1;
        r[S::P + 2] = h2;
        r[S::P + 3] = sdeg;
      }
      float* sp = slot + ((size_t)k * NSL + sl) * NV;
#pragma unroll
      for (int g = 0; g < (NR + 15) / 16; ++g) {
        const float tot = warp_reduce_scatter16(&r[16 * g], lane);
        const int v = 16 * g + ((lane >> 1) & 15);
        if (!(lane & 1) && v < NR) sp[v] = tot;
      }
    }
    __syncthreads();
    if (sl == 0 && lane < ne && my_e >= 0) {
      float tot[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) tot[v] = 0.f;
      for (int s2 = 0; s2 < NSL; ++s2) {
        const float* sp = slot + ((size_t)lane * NSL + s2) * NV;
#pragma unroll
        for (int v = 0; v < NV; ++v) tot[v] += sp[v];
      }
      if (a.gw) {
        float* gsr = a.gw + (int64_t)my_e * S::P;
#pragma unroll
        for (int p = 0; p < S::P; ++p) gsr[p] = a.has_coeff ? tot[p] * a.coeff[p] : tot[p];
      }
      if constexpr (GVEC) {
        float rx, ry, rz, ir;
        edge_geometry(vx, vy, vz, rx, ry, rz, ir);
        const float sdeg = tot[S::P + 3];
        float* g = a.gvec + 3 * (int64_t)my_e;
        g[0] = ir * (tot[S::P] - rx * sdeg);
        g[1] = ir * (tot[S::P + 1] - ry * sdeg);
        g[2] = ir * (tot[S::P + 2] - rz * sdeg);
      }
    }
    __syncthreads();
    first += ne;
  }
  if constexpr (STAGED) {
    if (gather_failed && threadIdx.x == 0) {   // let the issued copies land, then report
      for (int s2 = 0; s2 < kSendSlots; ++s2) {
        const int f = last_fill[s2];
        if (f < 0) continue;
        const uint32_t mb = sm_addr(&full_bar[s2]);
        const unsigned long long t0 = now_ns();
        while (!slot_ready(mb, (uint32_t)((f / kSendSlots) & 1)) && now_ns() - t0 < kGatherWaitNs) {
        }
      }
      report(a, kDevGatherTimeout);
    }
  }
  if (act) S::store_xt(a.G, a.N, a.mul_out, node, c, bt);
}

// Sender pass with the transposed per-edge coupling matrix (S::kmt_build), without gvec: as
// the STAGED k_uvw_send (one CTA per sender, NSL slice warps, lane = output channel, the
// receivers' gy rows staged by the copy engine), but per batch of 32 out-edges the CTA first
// writes each edge's K row and path scalars into shared memory (warp h builds part h of every
// edge's row), so that per channel z = K gy, bt += s z and gs += xt . z are dense products
// evaluated two rows at a time.
template <class S, int NSL, int MINB, int KB>
__global__ void __launch_bounds__(32 * NSL, MINB) k_uvw_send_km(const __grid_constant__ LaunchArgs a) {
  static_assert(KB == 16 || KB == 32, "edges per batch");
  extern __shared__ float smem[];
  constexpr int NV = S::P;
  __shared__ __align__(8) uint64_t full_bar[kSendSlots];
  __shared__ uint32_t read_cnt[kSendSlots];
  __shared__ int last_fill[kSendSlots];
  __shared__ volatile int gather_failed;
  __shared__ int32_t rtab[kRowTab];
  const int lane = threadIdx.x & 31;
  const int sl = threadIdx.x >> 5;
  const int node = blockIdx.x;
  const int c = sl * 32 + lane;
  const bool act = c < a.mul_out;
  const int q0 = __ldg(a.colptr + node), q1 = __ldg(a.colptr + node + 1);
  // shared memory: [KB edges][NSL][NV] partials | K rows [KB][KMT_ROW] | gy ring
  float4* krows = reinterpret_cast<float4*>(smem + (KB * NSL * NV + 3) / 4 * 4);
  unsigned char* ring = reinterpret_cast<unsigned char*>(krows + KB * (S::KMT_ROW / 4));
  const uint32_t row_bytes = (uint32_t)a.out_dim * 4u;
  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < kSendSlots; ++s2) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sm_addr(&full_bar[s2])) : "memory");
      read_cnt[s2] = 0;
      last_fill[s2] = -1;
    }
    gather_failed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const RowTab rt = load_row_tab(a.rowptr, a.N, rtab);
  __syncthreads();
  auto fill = [&](int f, int i) {
    const int s2 = f % kSendSlots;
    const uint32_t mb = sm_addr(&full_bar[s2]);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mb), "r"(row_bytes) : "memory");
    bulk_g2s(sm_addr(ring + (size_t)s2 * row_bytes), a.gy + (int64_t)i * a.out_dim, row_bytes, mb);
    last_fill[s2] = f;
  };
  float2 xt[S::KMT_PAIRS], bt[S::KMT_PAIRS];
#pragma unroll
  for (int k = 0; k < S::KMT_PAIRS; ++k) xt[k] = bt[k] = make_float2(0.f, 0.f);
  if (act) S::kmt_load_xt(a.A, a.N, a.mul_out, node, c, xt);
  float* slot = smem;   // [KB edges][NSL][NV]
  int first = 0;
  for (int base = q0; base < q1; base += KB) {
    const int my_q = base + lane;
    int my_e = -1, my_i = 0;
    float vx = 0.f, vy = 0.f, vz = 0.f;
    if (lane < KB && my_q < q1) {
      my_e = __ldg(a.perm + my_q);
      my_i = find_row_tab(a.rowptr, a.N, rtab, rt, my_e);
      vx = __ldg(a.vec + 3 * (int64_t)my_e);
      vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
      vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
    }
    const int ne = min(KB, q1 - base);
    if (sl == 0) {
      for (int k = 0; k < min(ne, kSendSlots); ++k) {
        const int i = __shfl_sync(kFull, my_i, k);
        if (lane == 0) fill(first + k, i);
      }
    }
    if (my_e >= 0) {   // part sl of the K row of edge base + lane
      float rx, ry, rz, ir;
      edge_geometry(vx, vy, vz, rx, ry, rz, ir);
      float Y[S::NSH], cf[S::P], sv[S::P];
      S::sh(rx, ry, rz, Y);
#pragma unroll
      for (int p = 0; p < S::P; ++p) {
        cf[p] = a.has_coeff ? a.coeff[p] : 1.f;
        sv[p] = __ldg(a.w + (int64_t)my_e * S::P + p);
      }
      S::template kmt_build<NSL>(sl, Y, cf, sv, krows + (size_t)lane * (S::KMT_ROW / 4));
    }
    __syncthreads();
#pragma unroll 1
    for (int k = 0; k < ne; ++k) {
      const int f = first + k, s2 = f % kSendSlots;
      bool ok = !gather_failed;
      if (ok) ok = slot_wait(sm_addr(&full_bar[s2]), (uint32_t)((f / kSendSlots) & 1));
      ok = __all_sync(kFull, ok);
      if (!ok) gather_failed = 1;
      float gs[S::P];
#pragma unroll
      for (int p = 0; p < S::P; ++p) gs[p] = 0.f;
      if (ok && act) {
        float gyv[S::OUT_PC];
        S::load_out_shared(reinterpret_cast<const float*>(ring + (size_t)s2 * row_bytes), a.mul_out, c, gyv);
        S::kmt_apply(gyv, krows + (size_t)k * (S::KMT_ROW / 4), xt, bt, gs);
      }
      // this warp is done with the slot; the last of the NSL warps refills it
      __syncwarp();
      int last = 0;
      if (lane == 0 && ok) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        uint32_t old;
        asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;" : "=r"(old) : "r"(sm_addr(&read_cnt[s2])) : "memory");
        last = old == NSL - 1;
      }
      last = __shfl_sync(kFull, last, 0);
      const int inext = __shfl_sync(kFull, my_i, min(k + kSendSlots, KB - 1));
      if (last && lane == 0) {
        read_cnt[s2] = 0;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (k + kSendSlots < ne) fill(f + kSendSlots, inext);
      }
      float r[(NV + 15) / 16 * 16];
#pragma unroll
      for (int v = 0; v < (NV + 15) / 16 * 16; ++v) r[v] = v < NV ? gs[v < NV ? v : 0] : 0.f;
      float* sp = slot + ((size_t)k * NSL + sl) * NV;
#pragma unroll
      for (int g = 0; g < (NV + 15) / 16; ++g) {
        const float tot = warp_reduce_scatter16(&r[16 * g], lane);
        const int v = 16 * g + ((lane >> 1) & 15);
        if (!(lane & 1) && v < NV) sp[v] = tot;
      }
    }
    __syncthreads();
    if (sl == 0 && lane < ne && a.gw) {
      float* gsr = a.gw + (int64_t)my_e * S::P;
#pragma unroll
      for (int p = 0; p < S::P; ++p) {
        float t = 0.f;
        for (int s2 = 0; s2 < NSL; ++s2) t += slot[((size_t)lane * NSL + s2) * NV + p];
        gsr[p] = t;
      }
    }
    __syncthreads();
    first += ne;
  }
  if (gather_failed && threadIdx.x == 0) {   // let the issued copies land, then report
    for (int s2 = 0; s2 < kSendSlots; ++s2) {
      const int f = last_fill[s2];
      if (f < 0) continue;
      const uint32_t mb = sm_addr(&full_bar[s2]);
      const unsigned long long t0 = now_ns();
      while (!slot_ready(mb, (uint32_t)((f / kSendSlots) & 1)) && now_ns() - t0 < kGatherWaitNs) {
      }
    }
    report(a, kDevGatherTimeout);
  }
  if (act) S::kmt_store_bt(a.G, a.N, a.mul_out, node, c, bt);
}

// ---------------------------------------------------------------------------------------
// Host sequences
// ---------------------------------------------------------------------------------------
template <template <int> class Op, class F>
cudaError_t with_d(int d, F&& f) {
  switch (d) {
    case 1: return f(Op<1>{});
    case 3: return f(Op<3>{});
    case 5: return f(Op<5>{});
    default: return f(Op<7>{});
  }
}

template <class S>
cudaError_t launch_uvw_edge(const LaunchArgs& a, cudaStream_t s) {
  const int nsl = (a.mul + 31) / 32;
  if constexpr (S::KM_PAIRS <= 32) {
    if (!a.check && a.mul >= 64 && a.mul <= 128 && a.in_dim % 4 == 0 && (reinterpret_cast<uintptr_t>(a.x) & 15u) == 0) {
      // per-edge coupling matrices in shared memory, two channels per lane
      constexpr int KB = 16;
      auto go = [&](auto kern, int threads, int kb) -> cudaError_t {
        const size_t sm = (size_t)kEdgeSlots * a.in_dim * sizeof(float) + (size_t)2 * kb * S::KM_ROW * sizeof(float);
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)a.N, threads, sm, s>>>(a);
        count_launches(1);
        return cudaGetLastError();
      };
      // two warps, eight edges per K batch, six CTAs per SM (168 registers)
      if (a.mul > 64) return go(k_uvw_recv_km<S, 2, 8, 2, 6>, 64, 8);
      return go(k_uvw_recv_km<S, 1, KB, 2, 1>, 32, KB);
    }
  }
  if (!a.check && nsl == 4 && a.in_dim % 4 == 0 && (reinterpret_cast<uintptr_t>(a.x) & 15u) == 0) {
    // every slice of a receiver in one CTA, the x rows staged by the copy engine
    const size_t sm = (size_t)kEdgeSlots * a.in_dim * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(k_uvw_edge_staged<S, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k_uvw_edge_staged<S, 4><<<(unsigned)a.N, 128, sm, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
  }
  const size_t sm = (size_t)(a.split - 1) * S::A_PC * 32 * sizeof(float);
  k_uvw_edge<S><<<(unsigned)a.N * a.n_slices, 32 * a.split, sm, s>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

template <class S>
cudaError_t launch_uvw_fwd(const LaunchArgs& a, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  cudaError_t e = launch_uvw_edge<S>(a, s);
  if (e != cudaSuccess) return e;
  k_uvw_prep_wt<S><<<64, 256, 0, s>>>(a);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t n_shared = (int64_t)S::P * a.mul * a.mul_out;
  int64_t wt_off = 0;
  for (int o = 0; o < S::N_OUT; ++o) {
    const int d3 = S::out_d3_at(o), cnt = S::out_cnt_at(o);
    const int K = cnt * a.mul;
    e = with_d<MixFwdTc>(d3, [&](auto op) {
      op.M = (int64_t)a.N * d3;
      op.Nn = a.mul_out;
      op.K = K;
      op.ybase = (int64_t)a.mul_out * S::out_cumY_at(o);
      cudaError_t r = make_tmap(&op.tA, a.A + (int64_t)a.N * a.mul * S::out_cumA_at(o), K, op.M, K, FMT_K);
      if (r == cudaSuccess) r = make_tmap(&op.tB, a.Wt + wt_off, K, a.mul_out, K, FMT_SPLIT);
      if (r == cudaSuccess) r = make_tmap(&op.tB2, a.Wt + n_shared + wt_off, K, a.mul_out, K, FMT_SPLIT);
      if (r != cudaSuccess) return r;
      return launch_gemm_tc(a, op, 1, s);
    });
    if (e != cudaSuccess) return e;
    wt_off += (int64_t)K * a.mul_out;
  }
  return cudaSuccess;
}

template <class S>
cudaError_t launch_uvw_bwd(const LaunchArgs& a, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  cudaError_t e;
  k_uvw_prep_wg<S><<<64, 256, 0, s>>>(a);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_uvw_xt<S><<<(unsigned)a.N, 128, 0, s>>>(a);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t wstride = (int64_t)a.mul * a.mul_out;
  const int64_t n_shared = wstride * S::P;
  // xt = x W per input irrep
  int64_t wg_off = 0;
  for (int ai = 0; ai < S::N_IN; ++ai) {
    const int d1 = S::in_d1_at(ai), cnt = S::in_cnt_at(ai);
    if (cnt == 0) continue;
    e = with_d<XtTc>(d1, [&](auto op) {
      op.M = (int64_t)a.N * d1;
      op.Nn = (int64_t)cnt * a.mul_out;
      op.K = a.mul;
      op.out = a.A + (int64_t)a.N * a.mul_out * S::in_cumX_at(ai);
      const float* xT = a.xT + (int64_t)a.N * a.mul * S::in_cum_at(ai);
      cudaError_t r = make_tmap(&op.tA, xT, a.mul, op.M, a.mul, FMT_K);
      if (r == cudaSuccess) r = make_tmap(&op.tB, a.Wt + 2 * n_shared + wg_off, a.mul, op.Nn, a.mul, FMT_SPLIT);
      if (r == cudaSuccess) r = make_tmap(&op.tB2, a.Wt + 3 * n_shared + wg_off, a.mul, op.Nn, a.mul, FMT_SPLIT);
      if (r != cudaSuccess) return r;
      return launch_gemm_tc(a, op, 1, s);
    });
    if (e != cudaSuccess) return e;
    wg_off += (int64_t)cnt * wstride;
  }
  // sender pass: B, gs, gvec
  const int nsl = (a.mul_out + 31) / 32 <= 1 ? 1 : ((a.mul_out + 31) / 32 == 2 ? 2 : 4);
  const bool gv = a.gvec != nullptr;
  // stage the gy rows when the CTA covers every channel and the rows are 16-byte aligned
  const bool staged = !a.check && 32 * nsl >= a.mul_out && a.out_dim % 4 == 0 &&
                      (reinterpret_cast<uintptr_t>(a.gy) & 15u) == 0;
  auto send = [&](auto gvec_tag, auto nsl_tag) -> cudaError_t {
    constexpr bool G = decltype(gvec_tag)::value;
    constexpr int NS = decltype(nsl_tag)::value;
    const size_t sm = SendShape<S, G, NS>::smem_bytes(staged, a.out_dim);
    if (staged) {
      cudaError_t r = cudaFuncSetAttribute(k_uvw_send<S, G, NS, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      if (r != cudaSuccess) return r;
      k_uvw_send<S, G, NS, true><<<(unsigned)a.N, 32 * NS, sm, s>>>(a);
    } else {
      k_uvw_send<S, G, NS, false><<<(unsigned)a.N, 32 * NS, sm, s>>>(a);
    }
    return cudaSuccess;
  };
  using T1 = std::integral_constant<int, 1>;
  using T2 = std::integral_constant<int, 2>;
  using T4 = std::integral_constant<int, 4>;
  auto send_km = [&](auto nsl_tag) -> cudaError_t {
    constexpr int NS = decltype(nsl_tag)::value;
    constexpr int KB = 32;
    const size_t sm = sizeof(float) * ((size_t)(KB * NS * S::P + 3) / 4 * 4 + (size_t)KB * S::KMT_ROW) +
                      (size_t)kSendSlots * a.out_dim * sizeof(float);
    auto kern = k_uvw_send_km<S, NS, 12 / NS, KB>;   // three CTAs of four warps per SM
    cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (r != cudaSuccess) return r;
    kern<<<(unsigned)a.N, 32 * NS, sm, s>>>(a);
    return cudaSuccess;
  };
  if (staged && !gv && S::KMT_PAIRS <= 32) {
    // per-edge coupling matrices in shared memory (the direction gradient takes the CG form)
    if constexpr (S::KMT_PAIRS <= 32) {
      e = nsl == 1 ? send_km(T1{}) : nsl == 2 ? send_km(T2{}) : send_km(T4{});
    }
  } else if (nsl == 1) e = gv ? send(std::true_type{}, T1{}) : send(std::false_type{}, T1{});
  else if (nsl == 2) e = gv ? send(std::true_type{}, T2{}) : send(std::false_type{}, T2{});
  else e = gv ? send(std::true_type{}, T4{}) : send(std::false_type{}, T4{});
  if (e != cudaSuccess) return e;
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  wg_off = 0;
  for (int ai = 0; ai < S::N_IN; ++ai) {
    const int d1 = S::in_d1_at(ai), cnt = S::in_cnt_at(ai);
    if (cnt == 0) continue;
    const int K = cnt * a.mul_out;
    const int64_t rows = (int64_t)a.N * d1;
    const float* Bbuf = a.G + (int64_t)a.N * a.mul_out * S::in_cumX_at(ai);
    if (a.gx) {
      e = with_d<GxTc>(d1, [&](auto op) {
        op.M = rows;
        op.Nn = a.mul;
        op.K = K;
        op.xbase = (int64_t)a.mul * S::in_cum_at(ai);
        cudaError_t r = make_tmap(&op.tA, Bbuf, K, rows, K, FMT_K);
        if (r == cudaSuccess) r = make_tmap(&op.tB, a.Wt + wg_off, K, a.mul, K, FMT_SPLIT);
        if (r == cudaSuccess) r = make_tmap(&op.tB2, a.Wt + n_shared + wg_off, K, a.mul, K, FMT_SPLIT);
        if (r != cudaSuccess) return r;
        return launch_gemm_tc(a, op, 1, s);
      });
      if (e != cudaSuccess) return e;
    }
    if (a.gW) {
      e = with_d<GwTc>(d1, [&](auto op) {
        op.M = a.mul;
        op.Nn = K;
        op.rows = rows;
        op.splits = a.splits;
        op.mul_out = a.mul_out;
        op.P = S::P;
        op.wstride = wstride;
        for (int pl = 0; pl < cnt; ++pl) op.paths[pl] = S::path_in_at(ai, pl);
        const float* xT = a.xT + (int64_t)a.N * a.mul * S::in_cum_at(ai);
        cudaError_t r = make_tmap(&op.tA, xT, a.mul, rows, a.mul, FMT_MN);
        if (r == cudaSuccess) r = make_tmap(&op.tB, Bbuf, K, rows, K, FMT_MN);
        if (r != cudaSuccess) return r;
        return launch_gemm_tc(a, op, a.splits, s);
      });
      if (e != cudaSuccess) return e;
    }
    wg_off += (int64_t)cnt * wstride;
  }
  if (a.gW) {
    const int64_t n = (int64_t)S::P * wstride;
    k_reduce_splits<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, s>>>(a.part, a.splits, n, a.gW);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace tp
