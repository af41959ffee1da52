// Edge kernels of the tensor-product convolution, templated on a generated spec S.
//
// Operation ("Sobek: Streaming Equivariant Tensor Product Convolutions", abstract;
// "FlashTP", abstract): for each receiver i and each incoming edge e = (j -> i)
//   y[i, out(p), u, m3] += w[e, p, u] * sum_{m1,m2} C_p[m1, m2, m3] x[j, in(p), u, m1] Y_l2(r_e)[m2]
// with the real spherical harmonics Y of the edge direction evaluated in registers and
// only the non-zero C_p entries unrolled (S::fwd, generated).
//
// Schedule (B200): a CTA owns one node row and one 32-channel slice of it; lane = channel,
// so the per-channel work of an edge is identical on every lane and variable degree costs
// no divergence.  Up to four warps of a CTA ("phases") take interleaved edges of the same
// row and their register accumulators are summed in a fixed order through shared memory:
// the result is deterministic and no float atomics touch the output.  Rows are scheduled
// dynamically by the hardware block scheduler, which balances the degree spread.  Edge
// geometry (sender index, edge vector) is loaded 32 edges at a time, one per lane
// (coalesced), and broadcast with warp shuffles.  No edge-sized message, weight or adjoint
// is written anywhere: each edge's products are consumed straight into receiver (forward,
// double-backward receiver pass) or sender (backward, double-backward sender pass) state.
#pragma once
#include <algorithm>

#include "tp_common.h"

namespace tp {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ void edge_geometry(float vx, float vy, float vz, float& rx, float& ry,
                                              float& rz, float& inv_r) {
  const float r2 = fmaf(vx, vx, fmaf(vy, vy, vz * vz));
  inv_r = r2 > 0.f ? rsqrtf(r2) : 0.f;
  rx = vx * inv_r;
  ry = vy * inv_r;
  rz = vz * inv_r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Receiver of edge e: the last row i with rowptr[i] <= e (empty rows share their start).
__device__ __forceinline__ int find_row(const int32_t* __restrict__ rowptr, int N, int e) {
  int lo = 0, hi = N - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(rowptr + mid) <= e) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Receiver search with a coarse copy of rowptr in shared memory: tab[k] = rowptr[k * stride]
// for k < ntab (ntab <= kRowTab).  The coarse bracket is found in shared memory, the last
// log2(stride) steps read rowptr itself.
constexpr int kRowTab = 1024;

struct RowTab {
  int stride, ntab;
};

// Fills the table (all threads of the CTA take part; the caller synchronises afterwards).
__device__ __forceinline__ RowTab load_row_tab(const int32_t* __restrict__ rowptr, int N, int32_t* tab) {
  RowTab rt;
  rt.stride = max(1, (N + kRowTab - 2) / (kRowTab - 1));
  rt.ntab = N / rt.stride + 1;
  for (int k = threadIdx.x; k < rt.ntab; k += blockDim.x) tab[k] = __ldg(rowptr + (int64_t)k * rt.stride);
  return rt;
}

__device__ __forceinline__ int find_row_tab(const int32_t* __restrict__ rowptr, int N, const int32_t* tab,
                                            RowTab rt, int e) {
  int lo = 0, hi = rt.ntab - 1;   // last k with tab[k] <= e
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab[mid] <= e) lo = mid;
    else hi = mid - 1;
  }
  int rlo = lo * rt.stride, rhi = min(N - 1, rlo + rt.stride - 1);
  while (rlo < rhi) {
    const int mid = (rlo + rhi + 1) >> 1;
    if (__ldg(rowptr + mid) <= e) rlo = mid;
    else rhi = mid - 1;
  }
  return rlo;
}

__device__ __forceinline__ void report(const LaunchArgs& a, int code) {
  if (a.err) atomicCAS(a.err, 0, code);
}

template <int P>
__device__ __forceinline__ void load_path_weights(const LaunchArgs& a, const float* base, int nw, int mul,
                                                  bool has_coeff, int e, int c, float (&w)[P]) {
  if (base == nullptr) {
#pragma unroll
    for (int p = 0; p < P; ++p) w[p] = 0.f;
    return;
  }
  const float* row = base + (int64_t)e * nw + c;
#pragma unroll
  for (int p = 0; p < P; ++p) w[p] = __ldg(row + p * mul);
  if (has_coeff) {
#pragma unroll
    for (int p = 0; p < P; ++p) w[p] *= a.coeff[p];
  }
}

// Sums per-phase register arrays into phase 0 through shared memory, in phase order.
template <int N>
__device__ __forceinline__ void reduce_phases(float (&acc)[N], float* smem, int phase, int split,
                                              int lane, int group, int ngroups) {
  if (split <= 1) return;
  // layout: [(phase-1)][group][N][32]
  if (phase > 0) {
    float* dst = smem + (((size_t)(phase - 1) * ngroups + group) * N) * 32 + lane;
#pragma unroll
    for (int k = 0; k < N; ++k) dst[k * 32] = acc[k];
  }
  __syncthreads();
  if (phase == 0) {
    for (int ph = 1; ph < split; ++ph) {
      const float* s = smem + (((size_t)(ph - 1) * ngroups + group) * N) * 32 + lane;
#pragma unroll
      for (int k = 0; k < N; ++k) acc[k] += s[k * 32];
    }
  }
}

// ---------------------------------------------------------------------------------------
// Forward, uvu, receiver order.  grid = N * n_slices, block = 32 * split.
// ---------------------------------------------------------------------------------------
template <class S, bool PF, int MUL, bool FAST>
__global__ void __launch_bounds__(kMaxThreads, PF ? 4 : 1) k_fwd_uvu(const __grid_constant__ LaunchArgs a) {
  constexpr bool kFast = FAST;
  const int mul = MUL ? MUL : a.mul;
  const int nw = MUL ? S::P * MUL : a.nw;
  const int in_dim = MUL ? S::IN_PC * MUL : a.in_dim;
  const int out_dim = MUL ? S::OUT_PC * MUL : a.out_dim;
  const bool check = !kFast && a.check;
  const bool has_coeff = !kFast && a.has_coeff;
  (void)nw; (void)in_dim; (void)out_dim; (void)has_coeff;
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31;
  const int phase = threadIdx.x >> 5;
  const int row = blockIdx.x / a.n_slices;
  const int sl = blockIdx.x - row * a.n_slices;
  const int c = sl * 32 + lane;
  const bool act = c < mul;
  int e0 = __ldg(a.rowptr + row), e1 = __ldg(a.rowptr + row + 1);
  if (check) {  // never read outside [0, E) whatever rowptr holds
    e0 = max(0, min(e0, a.E));
    e1 = max(e0, min(e1, a.E));
  }
  const int st = a.split;
  float acc[S::OUT_PC];
  float2 acc2[PF ? S::OUT_PC : 1];
#pragma unroll
  for (int k = 0; k < S::OUT_PC; ++k) acc[k] = 0.f;
#pragma unroll
  for (int k = 0; k < (PF ? S::OUT_PC : 1); ++k) acc2[k] = make_float2(0.f, 0.f);

  for (int base = e0 + phase; base < e1; base += 32 * st) {
    const int my_e = base + lane * st;
    int my_j = 0;
    float vx = 0.f, vy = 0.f, vz = 0.f;
    if (my_e < e1) {
      my_j = __ldg(a.src + my_e);
      vx = __ldg(a.vec + 3 * (int64_t)my_e);
      vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
      vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
      if (check && (unsigned)my_j >= (unsigned)a.N) {
        report(a, kDevBadSrc);
        vx = vy = vz = 0.f;
        my_j = -1;
      }
    }
    const int ne = min(32, (e1 - base + st - 1) / st);
    float xa[S::IN_PC], wa[S::P];
    if constexpr (PF) {
      // edge pairs: both edges' gathers are in flight together and every CG FMA is a packed
      // __ffma2_rn over (edge k, edge k+1); an odd tail pairs with a zero-weight copy
      for (int k = 0; k < ne; k += 2) {
        const bool two = k + 1 < ne;
        const int kb = two ? k + 1 : k;
        int ja = __shfl_sync(kFull, my_j, k), jb = __shfl_sync(kFull, my_j, kb);
        const float ax = __shfl_sync(kFull, vx, k), ay = __shfl_sync(kFull, vy, k), az = __shfl_sync(kFull, vz, k);
        const float bx = __shfl_sync(kFull, vx, kb), by = __shfl_sync(kFull, vy, kb), bz = __shfl_sync(kFull, vz, kb);
        const bool oka = ja >= 0, okb = two && jb >= 0;
        if (!oka && !okb) continue;
        if (!oka) ja = jb;
        if (!okb) jb = ja;
        float2 x2[S::IN_PC], w2[S::P], Y2[S::NSH];
        if (act) {
          float xb[S::IN_PC], wb[S::P];
          S::load_in(a.x + (int64_t)ja * in_dim, mul, c, xa);
          S::load_in(a.x + (int64_t)jb * in_dim, mul, c, xb);
          load_path_weights(a, a.w, nw, mul, has_coeff, base + k * st, c, wa);
          load_path_weights(a, a.w, nw, mul, has_coeff, base + kb * st, c, wb);
#pragma unroll
          for (int q = 0; q < S::IN_PC; ++q) x2[q] = make_float2(xa[q], xb[q]);
#pragma unroll
          for (int q = 0; q < S::P; ++q) w2[q] = make_float2(oka ? wa[q] : 0.f, okb ? wb[q] : 0.f);
        }
        {
          float rx, ry, rz, ir, Ya[S::NSH], Yb[S::NSH];
          edge_geometry(ax, ay, az, rx, ry, rz, ir);
          S::sh(rx, ry, rz, Ya);
          edge_geometry(bx, by, bz, rx, ry, rz, ir);
          S::sh(rx, ry, rz, Yb);
#pragma unroll
          for (int q = 0; q < S::NSH; ++q) Y2[q] = make_float2(Ya[q], Yb[q]);
        }
        if (act) S::fwd2(x2, Y2, w2, acc2);
      }
    } else {
      // one edge at a time, gathers issued after the SH evaluation (fewer live registers)
      for (int k = 0; k < ne; ++k) {
        const int e = base + k * st;
        const int j = __shfl_sync(kFull, my_j, k);
        const float ux = __shfl_sync(kFull, vx, k);
        const float uy = __shfl_sync(kFull, vy, k);
        const float uz = __shfl_sync(kFull, vz, k);
        if (j < 0) continue;
        float rx, ry, rz, ir;
        edge_geometry(ux, uy, uz, rx, ry, rz, ir);
        float Y[S::NSH];
        S::sh(rx, ry, rz, Y);
        if (act) {
          S::load_in(a.x + (int64_t)j * in_dim, mul, c, xa);
          load_path_weights(a, a.w, nw, mul, has_coeff, e, c, wa);
          S::fwd(xa, Y, wa, acc);
        }
      }
    }
  }
  if constexpr (PF) {
#pragma unroll
    for (int k = 0; k < S::OUT_PC; ++k) acc[k] = acc2[k].x + acc2[k].y;
  }
  reduce_phases(acc, smem, phase, st, lane, 0, 1);
  if (phase == 0 && act) S::store_out(a.y + (int64_t)row * out_dim, mul, c, acc);
}


// ---------------------------------------------------------------------------------------
// Forward with the per-edge rows staged by the copy engine (lmax <= 2 specs, 32 channels,
// fast instance).  Same schedule and arithmetic as k_fwd_uvu's edge-pair path, but the two
// rows an edge needs -- the sender's x row (IN_PC * 32 floats, contiguous) and the edge's
// weight row (P * 32 floats, contiguous) -- are fetched by cp.async.bulk into a private ring
// of kGatherSlots shared-memory slots per warp, kGatherSlots - 2 edges ahead of the pair
// being computed, with an mbarrier per slot counting the bytes.  The gathers' latency then
// overlaps the CG arithmetic instead of stalling it.  Waits are bounded by the global
// timer; on a timeout the CTA records TP device error 6, lets the copies it issued land
// (again bounded) and stops.
// ---------------------------------------------------------------------------------------
constexpr int kGatherSlots = 4;
constexpr unsigned long long kGatherWaitNs = 4000000000ull;
constexpr int kDevGatherTimeout = 6;

__device__ __forceinline__ uint32_t sm_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(mbar)
               : "memory");
}

__device__ __forceinline__ bool slot_ready(uint32_t mbar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(mbar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Time-bounded wait on a slot; false on timeout.
__device__ __forceinline__ bool slot_wait(uint32_t mbar, uint32_t parity,
                                          unsigned long long limit_ns = kGatherWaitNs) {
  if (slot_ready(mbar, parity)) return true;
  const unsigned long long t0 = now_ns();
  while (!slot_ready(mbar, parity))
    if (now_ns() - t0 > limit_ns) return false;
  return true;
}

template <class S>
struct GatherFwd {
  static constexpr int XB = S::IN_PC * 32 * 4;   // bytes of one x row
  static constexpr int WB = S::P * 32 * 4;       // bytes of one weight row
  static constexpr int SLOT = XB + WB;
  static constexpr size_t smem_bytes(int split) {
    return (size_t)split * kGatherSlots * SLOT + (size_t)(split - 1) * S::OUT_PC * 32 * sizeof(float);
  }
};

template <class S>
__global__ void __launch_bounds__(kMaxThreads, S::IN_PC + S::P + S::OUT_PC <= 48 ? 4 : 2) k_fwd_uvu_gather(const __grid_constant__ LaunchArgs a) {
  using G = GatherFwd<S>;
  constexpr int MUL = 32;
  constexpr int in_dim = S::IN_PC * MUL, nw = S::P * MUL;
  extern __shared__ __align__(128) unsigned char gsm[];
  __shared__ __align__(8) uint64_t bars[kMaxThreads / 32][kGatherSlots];
  const int lane = threadIdx.x & 31;
  const int phase = threadIdx.x >> 5;
  const int st = a.split;
  const int row = blockIdx.x;
  const int e0 = __ldg(a.rowptr + row), e1 = __ldg(a.rowptr + row + 1);
  unsigned char* ring = gsm + (size_t)phase * kGatherSlots * G::SLOT;
  float* red = reinterpret_cast<float*>(gsm + (size_t)st * kGatherSlots * G::SLOT);
  if (lane == 0) {
    for (int s2 = 0; s2 < kGatherSlots; ++s2)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sm_addr(&bars[phase][s2])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  uint32_t parity = 0;   // bit s: phase of slot s's next completion
  int issued = 0;        // fills issued on this warp's ring (slot = fill % kGatherSlots)
  int consumed = 0;      // fills waited for, in fill order
  bool failed = false;

  float2 acc2[S::OUT_PC];
#pragma unroll
  for (int k = 0; k < S::OUT_PC; ++k) acc2[k] = make_float2(0.f, 0.f);

  for (int base = e0 + phase; base < e1 && !failed; base += 32 * st) {
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
    // copy edge k of this batch into the next ring slot (lane 0 issues; every lane learns j)
    auto fill = [&](int k) {
      const int j = __shfl_sync(kFull, my_j, k);
      if (lane == 0) {
        const int s2 = issued % kGatherSlots;
        unsigned char* slot = ring + (size_t)s2 * G::SLOT;
        const uint32_t mb = sm_addr(&bars[phase][s2]);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mb), "r"(G::SLOT) : "memory");
        bulk_g2s(sm_addr(slot), a.x + (int64_t)j * in_dim, G::XB, mb);
        bulk_g2s(sm_addr(slot + G::XB), a.w + (int64_t)(base + k * st) * nw, G::WB, mb);
      }
      ++issued;
    };
    const int first = issued;   // fill index of edge 0 of this batch
    for (int k = 0; k < min(ne, kGatherSlots); ++k) fill(k);
    for (int k = 0; k < ne; k += 2) {
      const bool two = k + 1 < ne;
      const int kb = two ? k + 1 : k;
      const int sa = (first + k) % kGatherSlots, sb = (first + kb) % kGatherSlots;
      bool ok = slot_wait(sm_addr(&bars[phase][sa]), (parity >> sa) & 1u);
      if (two) ok = ok && slot_wait(sm_addr(&bars[phase][sb]), (parity >> sb) & 1u);
      if (!__all_sync(kFull, ok)) {
        failed = true;
        break;
      }
      parity ^= 1u << sa;
      if (two) parity ^= 1u << sb;
      consumed += two ? 2 : 1;
      const float* xa = reinterpret_cast<const float*>(ring + (size_t)sa * G::SLOT);
      const float* xb = reinterpret_cast<const float*>(ring + (size_t)sb * G::SLOT);
      float2 x2[S::IN_PC], w2[S::P], Y2[S::NSH];
      {
        float ta[S::IN_PC], tb[S::IN_PC];
        S::load_in_shared(xa, MUL, lane, ta);
        S::load_in_shared(xb, MUL, lane, tb);
#pragma unroll
        for (int q = 0; q < S::IN_PC; ++q) x2[q] = make_float2(ta[q], two ? tb[q] : ta[q]);
        const float* wa = xa + G::XB / 4 + lane;
        const float* wb = xb + G::XB / 4 + lane;
#pragma unroll
        for (int p = 0; p < S::P; ++p) w2[p] = make_float2(wa[p * MUL], two ? wb[p * MUL] : 0.f);
      }
      // both slots are read: refill them with the edges kGatherSlots ahead
      __syncwarp();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      if (k + kGatherSlots < ne) fill(k + kGatherSlots);
      if (two && kb + kGatherSlots < ne) fill(kb + kGatherSlots);
      {
        const float ax = __shfl_sync(kFull, vx, k), ay = __shfl_sync(kFull, vy, k), az = __shfl_sync(kFull, vz, k);
        const float bx = __shfl_sync(kFull, vx, kb), by = __shfl_sync(kFull, vy, kb), bz = __shfl_sync(kFull, vz, kb);
        float rx, ry, rz, ir, Ya[S::NSH], Yb[S::NSH];
        edge_geometry(ax, ay, az, rx, ry, rz, ir);
        S::sh(rx, ry, rz, Ya);
        edge_geometry(bx, by, bz, rx, ry, rz, ir);
        S::sh(rx, ry, rz, Yb);
#pragma unroll
        for (int q = 0; q < S::NSH; ++q) Y2[q] = make_float2(Ya[q], Yb[q]);
      }
      S::fwd2(x2, Y2, w2, acc2);
    }
  }
  if (failed) {
    // let every copy this warp issued land before the CTA exits, then report
    if (lane == 0) {
      for (int f = consumed; f < issued; ++f) {
        const int s2 = f % kGatherSlots;
        const unsigned long long t0 = now_ns();
        while (!slot_ready(sm_addr(&bars[phase][s2]), (parity >> s2) & 1u) && now_ns() - t0 < kGatherWaitNs) {
        }
        parity ^= 1u << s2;
      }
      report(a, kDevGatherTimeout);
    }
  }
  float acc[S::OUT_PC];
#pragma unroll
  for (int k = 0; k < S::OUT_PC; ++k) acc[k] = acc2[k].x + acc2[k].y;
  reduce_phases(acc, red, phase, st, lane, 0, 1);
  if (phase == 0) S::store_out(a.y + (int64_t)row * (S::OUT_PC * MUL), MUL, lane, acc);
}

// ---------------------------------------------------------------------------------------
// Backward, uvu, sender order (through the stable transpose perm; each edge's receiver is
// found by a binary search of rowptr, one lane per edge).
//   gx[j]  = sum over edges leaving j (segmented, in registers)
//   gw[e]  = per edge, written at its own position
//   gvec[e]= per edge, channel sum: warp reduction, then across slice warps via smem.
// GVEC=false: grid = N * n_slices, block = 32*split (slices independent).
// GVEC=true : grid = N, block = 32*split*NSL (all slices of a row in one CTA).
// ---------------------------------------------------------------------------------------
template <class S, bool GVEC, int NSL, bool PF, int MUL, bool FAST>
__global__ void __launch_bounds__(kMaxThreads) k_bwd_uvu(const __grid_constant__ LaunchArgs a) {
  constexpr bool kFast = FAST;
  const int mul = MUL ? MUL : a.mul;
  const int nw = MUL ? S::P * MUL : a.nw;
  const int in_dim = MUL ? S::IN_PC * MUL : a.in_dim;
  const int out_dim = MUL ? S::OUT_PC * MUL : a.out_dim;
  const bool check = !kFast && a.check;
  const bool has_coeff = !kFast && a.has_coeff;
  (void)nw; (void)in_dim; (void)out_dim; (void)has_coeff;
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int st = a.split;
  const int phase = wid % st;
  int node, sl;
  if (GVEC) {
    node = blockIdx.x;
    sl = wid / st;
  } else {
    node = blockIdx.x / a.n_slices;
    sl = blockIdx.x - node * a.n_slices;
  }
  const int c = sl * 32 + lane;
  const bool act = c < mul;
  int q0 = __ldg(a.colptr + node), q1 = __ldg(a.colptr + node + 1);
  if (check) {
    q0 = max(0, min(q0, a.E));
    q1 = max(q0, min(q1, a.E));
  }

  float x[S::IN_PC];
  float gx[S::IN_PC];
#pragma unroll
  for (int k = 0; k < S::IN_PC; ++k) gx[k] = 0.f;
  if (act) S::load_in(a.x + (int64_t)node * in_dim, mul, c, x);
  else {
#pragma unroll
    for (int k = 0; k < S::IN_PC; ++k) x[k] = 0.f;
  }
  // gvec partial slots: [phase][edge-in-batch][slice][4]
  float* gslot = smem + (size_t)(st > 1 ? (st - 1) * NSL * S::IN_PC * 32 : 0);

  for (int base = q0 + phase; base < q1; base += 32 * st) {
    const int my_q = base + lane * st;
    int my_e = -1, my_i = 0;
    float vx = 0.f, vy = 0.f, vz = 0.f;
    if (my_q < q1) {
      my_e = __ldg(a.perm + my_q);
      if (check && (unsigned)my_e >= (unsigned)a.E) {
        report(a, kDevBadPerm);
        my_e = -1;
      } else {
        my_i = find_row(a.rowptr, a.N, my_e);
        vx = __ldg(a.vec + 3 * (int64_t)my_e);
        vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
        vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
      }
    }
    const int ne = min(32, (q1 - base + st - 1) / st);
    // gvec[e] = sum_m gY_m dY_m/dv with dY_m/dv = (grad P_m(r) - l_m Y_m r) / |v|; the
    // channel sum is a warp reduction, then (NSL > 1) a sum over the slice warps
    auto gvec_edge = [&](int k, int e, float rx, float ry, float rz, float ir, const float (&Y)[S::NSH],
                         const float (&gY)[S::NSH]) {
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
      if (NSL == 1) {
        if (lane == 0 && e >= 0) {
          float* g = a.gvec + 3 * (int64_t)e;
          g[0] = ir * (h0 - rx * sdeg);
          g[1] = ir * (h1 - ry * sdeg);
          g[2] = ir * (h2 - rz * sdeg);
        }
      } else if (lane == 0) {
        float* s = gslot + (((size_t)phase * 32 + k) * NSL + sl) * 4;
        s[0] = h0;
        s[1] = h1;
        s[2] = h2;
        s[3] = sdeg;
      }
    };
    // gathers of edge k: receiver slice gy[i] and the edge's weight row
    auto fetch = [&](int k, float (&gg)[S::OUT_PC], float (&ww)[S::P]) {
      const int e = __shfl_sync(kFull, my_e, k);
      const int i = __shfl_sync(kFull, my_i, k);
      if (act && e >= 0) {
        S::load_out(a.gy + (int64_t)i * out_dim, mul, c, gg);
        load_path_weights(a, a.w, nw, mul, has_coeff, e, c, ww);
      }
    };
    auto compute = [&](int k, const float (&gyv)[S::OUT_PC], const float (&w)[S::P]) {
      const int e = __shfl_sync(kFull, my_e, k);
      const float ux = __shfl_sync(kFull, vx, k);
      const float uy = __shfl_sync(kFull, vy, k);
      const float uz = __shfl_sync(kFull, vz, k);
      float rx, ry, rz, ir;
      edge_geometry(ux, uy, uz, rx, ry, rz, ir);
      float Y[S::NSH];
      S::sh(rx, ry, rz, Y);
      float gY[S::NSH];
#pragma unroll
      for (int m = 0; m < S::NSH; ++m) gY[m] = 0.f;
      if (act && e >= 0) {
        float gw[S::P];
        S::template bwd<GVEC>(x, Y, w, gyv, gx, gw, gY);
        if (a.gw) {
          float* row = a.gw + (int64_t)e * nw + c;
#pragma unroll
          for (int p = 0; p < S::P; ++p) row[(int64_t)p * mul] = has_coeff ? gw[p] * a.coeff[p] : gw[p];
        }
      }
      if constexpr (GVEC) gvec_edge(k, e, rx, ry, rz, ir, Y, gY);
    };
    float ga[S::OUT_PC], wa[S::P];
    if constexpr (PF) {
      float gb[S::OUT_PC], wb[S::P];
      fetch(0, ga, wa);
      for (int k = 0; k < ne; k += 2) {
        if (k + 1 < ne) fetch(k + 1, gb, wb);
        compute(k, ga, wa);
        if (k + 1 >= ne) break;
        if (k + 2 < ne) fetch(k + 2, ga, wa);
        compute(k + 1, gb, wb);
      }
    } else {
      // one edge at a time; the gathers are issued after the SH evaluation so that fewer
      // values are live at once (the lmax-3 bodies are register bound)
      for (int k = 0; k < ne; ++k) {
        const int e = __shfl_sync(kFull, my_e, k);
        const int i = __shfl_sync(kFull, my_i, k);
        const float ux = __shfl_sync(kFull, vx, k);
        const float uy = __shfl_sync(kFull, vy, k);
        const float uz = __shfl_sync(kFull, vz, k);
        float rx, ry, rz, ir;
        edge_geometry(ux, uy, uz, rx, ry, rz, ir);
        float Y[S::NSH];
        S::sh(rx, ry, rz, Y);
        float gY[S::NSH];
#pragma unroll
        for (int m = 0; m < S::NSH; ++m) gY[m] = 0.f;
        if (act && e >= 0) {
          S::load_out(a.gy + (int64_t)i * out_dim, mul, c, ga);
          load_path_weights(a, a.w, nw, mul, has_coeff, e, c, wa);
          float gw[S::P];
          S::template bwd<GVEC>(x, Y, wa, ga, gx, gw, gY);
          if (a.gw) {
            float* row = a.gw + (int64_t)e * nw + c;
#pragma unroll
            for (int p = 0; p < S::P; ++p) row[(int64_t)p * mul] = has_coeff ? gw[p] * a.coeff[p] : gw[p];
          }
        }
        if constexpr (GVEC) gvec_edge(k, e, rx, ry, rz, ir, Y, gY);
      }
    }
    if constexpr (GVEC && NSL > 1) {
      named_barrier(1 + phase, 32 * NSL);
      if (sl == 0 && lane < ne && my_e >= 0) {
        float h0 = 0.f, h1 = 0.f, h2 = 0.f, sdeg = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < NSL; ++s2) {
          const float* s = gslot + (((size_t)phase * 32 + lane) * NSL + s2) * 4;
          h0 += s[0];
          h1 += s[1];
          h2 += s[2];
          sdeg += s[3];
        }
        float rx, ry, rz, ir;
        edge_geometry(vx, vy, vz, rx, ry, rz, ir);
        float* g = a.gvec + 3 * (int64_t)my_e;
        g[0] = ir * (h0 - rx * sdeg);
        g[1] = ir * (h1 - ry * sdeg);
        g[2] = ir * (h2 - rz * sdeg);
      }
      named_barrier(1 + phase, 32 * NSL);
    }
  }
  reduce_phases(gx, smem, phase, st, lane, GVEC ? sl : 0, GVEC ? NSL : 1);
  if (phase == 0 && act && a.gx) S::store_in(a.gx + (int64_t)node * in_dim, mul, c, gx);
}

// ---------------------------------------------------------------------------------------
// Double backward, receiver pass: g_gy[i] = sum_e TP(ggx; Y, w) + TP(x; Y, ggw) + TP(x; dY[ggvec], w)
// ---------------------------------------------------------------------------------------
template <class S, int MUL, bool FAST>
__global__ void __launch_bounds__(kMaxThreads) k_dbwd_recv(const __grid_constant__ LaunchArgs a) {
  constexpr bool kFast = FAST;
  const int mul = MUL ? MUL : a.mul;
  const int nw = MUL ? S::P * MUL : a.nw;
  const int in_dim = MUL ? S::IN_PC * MUL : a.in_dim;
  const int out_dim = MUL ? S::OUT_PC * MUL : a.out_dim;
  const bool check = !kFast && a.check;
  const bool has_coeff = !kFast && a.has_coeff;
  (void)nw; (void)in_dim; (void)out_dim; (void)has_coeff;
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31;
  const int phase = threadIdx.x >> 5;
  const int row = blockIdx.x / a.n_slices;
  const int sl = blockIdx.x - row * a.n_slices;
  const int c = sl * 32 + lane;
  const bool act = c < mul;
  int e0 = __ldg(a.rowptr + row), e1 = __ldg(a.rowptr + row + 1);
  if (check) {  // never read outside [0, E) whatever rowptr holds
    e0 = max(0, min(e0, a.E));
    e1 = max(e0, min(e1, a.E));
  }
  const int st = a.split;
  float acc[S::OUT_PC];
#pragma unroll
  for (int k = 0; k < S::OUT_PC; ++k) acc[k] = 0.f;

  for (int base = e0 + phase; base < e1; base += 32 * st) {
    const int my_e = base + lane * st;
    int my_j = 0;
    float vx = 0.f, vy = 0.f, vz = 0.f, dx = 0.f, dy = 0.f, dz = 0.f;
    if (my_e < e1) {
      my_j = __ldg(a.src + my_e);
      vx = __ldg(a.vec + 3 * (int64_t)my_e);
      vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
      vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
      if (a.ggvec) {
        dx = __ldg(a.ggvec + 3 * (int64_t)my_e);
        dy = __ldg(a.ggvec + 3 * (int64_t)my_e + 1);
        dz = __ldg(a.ggvec + 3 * (int64_t)my_e + 2);
      }
      if (check && (unsigned)my_j >= (unsigned)a.N) {
        report(a, kDevBadSrc);
        my_j = -1;
      }
    }
    const int ne = min(32, (e1 - base + st - 1) / st);
    for (int k = 0; k < ne; ++k) {
      const int e = base + k * st;
      const int j = __shfl_sync(kFull, my_j, k);
      const float ux = __shfl_sync(kFull, vx, k);
      const float uy = __shfl_sync(kFull, vy, k);
      const float uz = __shfl_sync(kFull, vz, k);
      const float ddx = __shfl_sync(kFull, dx, k);
      const float ddy = __shfl_sync(kFull, dy, k);
      const float ddz = __shfl_sync(kFull, dz, k);
      if (j < 0) continue;
      float rx, ry, rz, ir;
      edge_geometry(ux, uy, uz, rx, ry, rz, ir);
      float Y[S::NSH], Yp[S::NSH];
      S::sh(rx, ry, rz, Y);
      {
        float G[S::NSH][3];
        S::sh_grad(rx, ry, rz, G);
        const float rd = fmaf(rx, ddx, fmaf(ry, ddy, rz * ddz));
#pragma unroll
        for (int m = 0; m < S::NSH; ++m) {
          const float gd = fmaf(G[m][0], ddx, fmaf(G[m][1], ddy, G[m][2] * ddz));
          Yp[m] = ir * (gd - S::sh_degree(m) * Y[m] * rd);
        }
      }
      if (act) {
        float x[S::IN_PC], ggx[S::IN_PC];
        S::load_in(a.x + (int64_t)j * in_dim, mul, c, x);
        if (a.ggx) S::load_in(a.ggx + (int64_t)j * in_dim, mul, c, ggx);
        else {
#pragma unroll
          for (int m = 0; m < S::IN_PC; ++m) ggx[m] = 0.f;
        }
        float w[S::P], ggw[S::P];
        load_path_weights(a, a.w, nw, mul, has_coeff, e, c, w);
        load_path_weights(a, a.ggw, nw, mul, has_coeff, e, c, ggw);
        S::dbwd_recv(x, ggx, Y, Yp, w, ggw, acc);
      }
    }
  }
  reduce_phases(acc, smem, phase, st, lane, 0, 1);
  if (phase == 0 && act) S::store_out(a.y + (int64_t)row * out_dim, mul, c, acc);
}

// ---------------------------------------------------------------------------------------
// Double backward, sender pass: g_x[j] (segmented), g_w[e], g_vec[e].
// PART 0 computes all three; large specs run PART 1 (g_x, g_w) and PART 2 (g_vec) as two
// launches, each with half of the generated straight-line body, so that the instruction
// working set of a kernel stays closer to what the instruction caches hold.
// ---------------------------------------------------------------------------------------
template <class S>
constexpr bool kSplitDbwd = S::P > 15;

template <class S, bool GVEC, int NSL, int MUL, bool FAST, int PART = 0>
__global__ void __launch_bounds__(kMaxThreads) k_dbwd_send(const __grid_constant__ LaunchArgs a) {
  constexpr bool kFast = FAST;
  const int mul = MUL ? MUL : a.mul;
  const int nw = MUL ? S::P * MUL : a.nw;
  const int in_dim = MUL ? S::IN_PC * MUL : a.in_dim;
  const int out_dim = MUL ? S::OUT_PC * MUL : a.out_dim;
  const bool check = !kFast && a.check;
  const bool has_coeff = !kFast && a.has_coeff;
  (void)nw; (void)in_dim; (void)out_dim; (void)has_coeff;
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int st = a.split;
  const int phase = wid % st;
  int node, sl;
  if (GVEC) {
    node = blockIdx.x;
    sl = wid / st;
  } else {
    node = blockIdx.x / a.n_slices;
    sl = blockIdx.x - node * a.n_slices;
  }
  const int c = sl * 32 + lane;
  const bool act = c < mul;
  int q0 = __ldg(a.colptr + node), q1 = __ldg(a.colptr + node + 1);
  if (check) {
    q0 = max(0, min(q0, a.E));
    q1 = max(q0, min(q1, a.E));
  }

  float x[S::IN_PC], ggx[S::IN_PC], gx[S::IN_PC];
#pragma unroll
  for (int k = 0; k < S::IN_PC; ++k) {
    gx[k] = 0.f;
    x[k] = 0.f;
    ggx[k] = 0.f;
  }
  if (act) {
    S::load_in(a.x + (int64_t)node * in_dim, mul, c, x);
    if (a.ggx) S::load_in(a.ggx + (int64_t)node * in_dim, mul, c, ggx);
  }
  float* gslot = smem + (size_t)(st > 1 ? (st - 1) * NSL * S::IN_PC * 32 : 0);

  for (int base = q0 + phase; base < q1; base += 32 * st) {
    const int my_q = base + lane * st;
    int my_e = -1, my_i = 0;
    float vx = 0.f, vy = 0.f, vz = 0.f, dx = 0.f, dy = 0.f, dz = 0.f;
    if (my_q < q1) {
      my_e = __ldg(a.perm + my_q);
      if (check && (unsigned)my_e >= (unsigned)a.E) {
        report(a, kDevBadPerm);
        my_e = -1;
      } else {
        my_i = find_row(a.rowptr, a.N, my_e);
        vx = __ldg(a.vec + 3 * (int64_t)my_e);
        vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
        vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
        if (a.ggvec) {
          dx = __ldg(a.ggvec + 3 * (int64_t)my_e);
          dy = __ldg(a.ggvec + 3 * (int64_t)my_e + 1);
          dz = __ldg(a.ggvec + 3 * (int64_t)my_e + 2);
        }
      }
    }
    const int ne = min(32, (q1 - base + st - 1) / st);
    for (int k = 0; k < ne; ++k) {
      const int e = __shfl_sync(kFull, my_e, k);
      const int i = __shfl_sync(kFull, my_i, k);
      const float ux = __shfl_sync(kFull, vx, k);
      const float uy = __shfl_sync(kFull, vy, k);
      const float uz = __shfl_sync(kFull, vz, k);
      const float ddx = __shfl_sync(kFull, dx, k);
      const float ddy = __shfl_sync(kFull, dy, k);
      const float ddz = __shfl_sync(kFull, dz, k);
      float rx, ry, rz, ir;
      edge_geometry(ux, uy, uz, rx, ry, rz, ir);
      const float rd = fmaf(rx, ddx, fmaf(ry, ddy, rz * ddz));
      float Y[S::NSH], Yp[S::NSH], G[S::NSH][3];
      S::sh(rx, ry, rz, Y);
      S::sh_grad(rx, ry, rz, G);
#pragma unroll
      for (int m = 0; m < S::NSH; ++m) {
        const float gd = fmaf(G[m][0], ddx, fmaf(G[m][1], ddy, G[m][2] * ddz));
        Yp[m] = ir * (gd - S::sh_degree(m) * Y[m] * rd);
      }
      float G1[S::NSH], G2[S::NSH];
#pragma unroll
      for (int m = 0; m < S::NSH; ++m) G1[m] = G2[m] = 0.f;
      if (act && e >= 0) {
        float gyv[S::OUT_PC];
        S::load_out(a.gy + (int64_t)i * out_dim, mul, c, gyv);
        float w[S::P], ggw[S::P];
        load_path_weights(a, a.w, nw, mul, has_coeff, e, c, w);
        load_path_weights(a, a.ggw, nw, mul, has_coeff, e, c, ggw);
        float gw[S::P];
        if constexpr (PART == 0) S::dbwd_send(x, ggx, Y, Yp, w, ggw, gyv, gx, gw, G1, G2);
        if constexpr (PART == 1) S::dbwd_send_gx(x, ggx, Y, Yp, w, ggw, gyv, gx, gw, G1, G2);
        if constexpr (PART == 2) S::dbwd_send_gv(x, ggx, Y, Yp, w, ggw, gyv, gx, gw, G1, G2);
        if (PART != 2 && a.gw) {
          float* row = a.gw + (int64_t)e * nw + c;
#pragma unroll
          for (int p = 0; p < S::P; ++p) row[(int64_t)p * mul] = has_coeff ? gw[p] * a.coeff[p] : gw[p];
        }
      }
      if constexpr (GVEC) {
        // g = sum_m G1_m dY_m/dv + G2_m (d^2 Y_m/dv^2) ggvec
        float HD[S::NSH][3];
        S::sh_hess_dot(rx, ry, rz, ddx, ddy, ddz, HD);
        float g0 = 0.f, g1 = 0.f, g2 = 0.f;
        const float ir2 = ir * ir;
#pragma unroll
        for (int m = 0; m < S::NSH; ++m) {
          const float l = S::sh_degree(m);
          const float gdm = fmaf(G[m][0], ddx, fmaf(G[m][1], ddy, G[m][2] * ddz));
          const float cJ = G1[m] * ir;                   // J_mk = ir (G_mk - l Y_m r_k)
          const float cK = G2[m] * ir2;                  // K_mk = ir^2 [ ... ]
          const float lY = l * Y[m];
          const float rcoef = -cJ * lY + cK * (-l * gdm + l * (l + 2.f) * Y[m] * rd);
          const float gcoef = cJ - cK * l * rd;
          const float dcoef = -cK * lY;
          g0 += gcoef * G[m][0] + cK * HD[m][0] + rcoef * rx + dcoef * ddx;
          g1 += gcoef * G[m][1] + cK * HD[m][1] + rcoef * ry + dcoef * ddy;
          g2 += gcoef * G[m][2] + cK * HD[m][2] + rcoef * rz + dcoef * ddz;
        }
        g0 = warp_sum(g0);
        g1 = warp_sum(g1);
        g2 = warp_sum(g2);
        if (NSL == 1) {
          if (lane == 0 && e >= 0) {
            float* g = a.gvec + 3 * (int64_t)e;
            g[0] = g0;
            g[1] = g1;
            g[2] = g2;
          }
        } else if (lane == 0) {
          float* s = gslot + (((size_t)phase * 32 + k) * NSL + sl) * 4;
          s[0] = g0;
          s[1] = g1;
          s[2] = g2;
        }
      }
    }
    if constexpr (GVEC && NSL > 1) {
      named_barrier(1 + phase, 32 * NSL);
      if (sl == 0 && lane < ne && my_e >= 0) {
        float g0 = 0.f, g1 = 0.f, g2 = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < NSL; ++s2) {
          const float* s = gslot + (((size_t)phase * 32 + lane) * NSL + s2) * 4;
          g0 += s[0];
          g1 += s[1];
          g2 += s[2];
        }
        float* g = a.gvec + 3 * (int64_t)my_e;
        g[0] = g0;
        g[1] = g1;
        g[2] = g2;
      }
      named_barrier(1 + phase, 32 * NSL);
    }
  }
  if constexpr (PART != 2) {
    reduce_phases(gx, smem, phase, st, lane, GVEC ? sl : 0, GVEC ? NSL : 1);
    if (phase == 0 && act && a.gx) S::store_in(a.gx + (int64_t)node * in_dim, mul, c, gx);
  }
}

// ---------------------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------------------
// Register double buffering of the per-edge gathers pays when the buffers are small (lmax
// <= 2); for lmax 3 the extra registers cost more occupancy than the overlap gains.
template <class S>
constexpr bool kPrefetch = S::IN_PC + S::P + S::OUT_PC <= 48;

// Calls f.template run<MUL, FAST>(): a specialisation with the channel count fixed at
// compile time (constant load offsets, no index checks, no path coefficients) when the spec
// ships one for a.mul and the call needs neither; otherwise the general kernel.
template <class S, class F>
cudaError_t dispatch_mul(const LaunchArgs& a, int mul, F&& f) {
  if (!a.check && !a.has_coeff) {
    if constexpr (S::FAST_MUL0 > 0)
      if (mul == S::FAST_MUL0) return f.template run<S::FAST_MUL0, true>();
    if constexpr (S::FAST_MUL1 > 0)
      if (mul == S::FAST_MUL1) return f.template run<S::FAST_MUL1, true>();
  }
  return f.template run<0, false>();
}

template <class S>
struct FwdLaunch {
  const LaunchArgs& a;
  cudaStream_t s;
  template <int MUL, bool FAST>
  cudaError_t run() const {
    if constexpr (MUL == 32 && FAST) {
      // rows start on 16-byte boundaries: stage them with the copy engine
      if (((reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.w)) & 15u) == 0) {
        const size_t sm = GatherFwd<S>::smem_bytes(a.split);
        cudaError_t e = cudaFuncSetAttribute(k_fwd_uvu_gather<S>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        k_fwd_uvu_gather<S><<<(unsigned)a.N, 32 * a.split, sm, s>>>(a);
        count_launches(1);
        return cudaGetLastError();
      }
    }
    const size_t sm = (size_t)(a.split - 1) * S::OUT_PC * 32 * sizeof(float);
    k_fwd_uvu<S, kPrefetch<S>, MUL, FAST><<<(unsigned)a.N * a.n_slices, 32 * a.split, sm, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
  }
};

template <class S>
cudaError_t launch_fwd_uvu(const LaunchArgs& a, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  return dispatch_mul<S>(a, a.mul, FwdLaunch<S>{a, s});
}

template <class S>
struct DbwdRecvLaunch {
  const LaunchArgs& a;
  cudaStream_t s;
  template <int MUL, bool FAST>
  cudaError_t run() const {
    const size_t sm = (size_t)(a.split - 1) * S::OUT_PC * 32 * sizeof(float);
    k_dbwd_recv<S, MUL, FAST><<<(unsigned)a.N * a.n_slices, 32 * a.split, sm, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
  }
};

template <class S>
cudaError_t launch_dbwd_recv(const LaunchArgs& a, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  return dispatch_mul<S>(a, a.mul, DbwdRecvLaunch<S>{a, s});
}

template <class S, bool GVEC, int NSL, bool DBWD>
struct SenderLaunch {
  const LaunchArgs& a;
  cudaStream_t s;
  template <int MUL, bool FAST>
  cudaError_t run() const {
    const int st = a.split;
    const int groups = GVEC ? NSL : 1;
    const size_t sm = (size_t)(st > 1 ? (st - 1) * groups * S::IN_PC * 32 : 0) * sizeof(float) +
                      (GVEC && NSL > 1 ? (size_t)st * 32 * NSL * 4 * sizeof(float) : 0);
    const unsigned grid = GVEC ? (unsigned)a.N : (unsigned)a.N * a.n_slices;
    if constexpr (DBWD && GVEC && kSplitDbwd<S>) {
      // g_x and g_w first (no g_vec work, slices independent), then g_vec
      const size_t sm1 = (size_t)(st > 1 ? (st - 1) * S::IN_PC * 32 : 0) * sizeof(float);
      k_dbwd_send<S, false, 1, MUL, FAST, 1><<<(unsigned)a.N * a.n_slices, 32 * st, sm1, s>>>(a);
      count_launches(1);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      k_dbwd_send<S, GVEC, NSL, MUL, FAST, 2><<<grid, 32 * st * groups, sm, s>>>(a);
    } else if constexpr (DBWD)
      k_dbwd_send<S, GVEC, NSL, MUL, FAST><<<grid, 32 * st * groups, sm, s>>>(a);
    else
      k_bwd_uvu<S, GVEC, NSL, kPrefetch<S>, MUL, FAST><<<grid, 32 * st * groups, sm, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
  }
};

// The host chooses split so that split * NSL <= 4 whenever gvec is requested.
template <class S, bool DBWD>
cudaError_t launch_sender(const LaunchArgs& a, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  if (a.gvec == nullptr) return dispatch_mul<S>(a, a.mul, SenderLaunch<S, false, 1, DBWD>{a, s});
  if (a.n_slices <= 1) return dispatch_mul<S>(a, a.mul, SenderLaunch<S, true, 1, DBWD>{a, s});
  if (a.n_slices == 2) return dispatch_mul<S>(a, a.mul, SenderLaunch<S, true, 2, DBWD>{a, s});
  return dispatch_mul<S>(a, a.mul, SenderLaunch<S, true, 4, DBWD>{a, s});
}

template <class S>
cudaError_t launch_bwd_uvu(const LaunchArgs& a, cudaStream_t s) { return launch_sender<S, false>(a, s); }

template <class S>
cudaError_t launch_dbwd_send(const LaunchArgs& a, cudaStream_t s) { return launch_sender<S, true>(a, s); }

}  // namespace tp
