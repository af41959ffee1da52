// uvw mode: fully connected multiplicity mixing per path, reassociated so that no edge-sized
// tensor exists ("Sobek: Streaming Equivariant Tensor Product Convolutions", abstract: the
// streaming formulation keeps fully connected multiplicity mixing; edge-sized intermediates
// are artifacts of the schedule).
//
//   y[i, o, w, m3] = sum_{p into o} sum_u W_p[u, w] A_p[i, u, m3]
//   A_p[i, u, m3]  = sum_{e into i} c_p s[e, p] sum_{m1,m2} C_p[m1,m2,m3] x[j, in(p), u, m1] Y(v_e)[m2]
//
// A is node-sized state (N x sum_p mul x (2 l3 + 1) floats), aggregated by the receiver-order
// edge pass below and consumed by the mixing GEMM.  Backward: gW_p = sum_i A_p[i]^T gy_o[i]
// (split-K GEMM with a fixed-order reduction), G_p[i] = W_p gy_o[i] (GEMM), then one
// sender-order pass that gives gx (segmented in registers), gs[e, p] and gvec[e].
#pragma once
#include <algorithm>

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

// Wt[o][w][pl * mul + u] = W[path_of[o][pl]][u][w]  (B operand of the forward mixing GEMM)
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
    a.Wt[base + rem] = a.W[(int64_t)p * per_path + (int64_t)u * a.mul_out + w];
  }
}

// ---------------------------------------------------------------------------------------
// SIMT fp32 GEMM  C[m, n] = sum_k A(m, k) B(n, k), tile 64 x 128 x 16, 256 threads, each
// thread 4 x 8 outputs.  The operand accessors define the three uvw contractions.
// ---------------------------------------------------------------------------------------
constexpr int GBM = 64, GBN = 128, GBK = 16;

template <class Op>
__global__ void __launch_bounds__(256) k_gemm_simt(const __grid_constant__ LaunchArgs a, const Op op) {
  __shared__ float As[GBK][GBM + 4];
  __shared__ float Bs[GBK][GBN + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = (int64_t)blockIdx.x * GBM;
  const int n0 = blockIdx.y * GBN;
  int64_t k_begin, k_end;
  op.k_range(a, blockIdx.z, k_begin, k_end);
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int64_t k0 = k_begin; k0 < k_end; k0 += GBK) {
#pragma unroll
    for (int r = 0; r < (GBM * GBK) / 256; ++r) {
      const int q = tid + 256 * r;
      const int mm = q / GBK, kk = q % GBK;
      const int64_t m = m0 + mm, k = k0 + kk;
      As[kk][mm] = (m < op.M(a) && k < k_end) ? op.A(a, m, k) : 0.f;
    }
#pragma unroll
    for (int r = 0; r < (GBN * GBK) / 256; ++r) {
      const int q = tid + 256 * r;
      const int nn = q / GBK, kk = q % GBK;
      const int n = n0 + nn;
      const int64_t k = k0 + kk;
      Bs[kk][nn] = (n < op.Nn(a) && k < k_end) ? op.B(a, n, k) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < GBK; ++kk) {
      float av[4], bv[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) bv[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t m = m0 + ty + 16 * i;
      const int n = n0 + tx + 16 * j;
      if (m < op.M(a) && n < op.Nn(a)) op.C(a, blockIdx.z, m, n, acc[i][j]);
    }
}

// y_o[(i, m3), w] = sum_{(pl, u)} A_o[(i, m3), (pl, u)] Wt_o[w, (pl, u)]
template <class S>
struct MixFwdOp {
  int o;
  __device__ int64_t M(const LaunchArgs& a) const { return (int64_t)a.N * S::out_d3_at(o); }
  __device__ int Nn(const LaunchArgs& a) const { return a.mul_out; }
  __device__ int K(const LaunchArgs& a) const { return S::out_cnt_at(o) * a.mul; }
  __device__ void k_range(const LaunchArgs& a, int, int64_t& b, int64_t& e) const { b = 0; e = K(a); }
  __device__ float A(const LaunchArgs& a, int64_t m, int64_t k) const {
    return a.A[(int64_t)a.N * a.mul * S::out_cumA_at(o) + m * K(a) + k];
  }
  __device__ float B(const LaunchArgs& a, int n, int64_t k) const {
    int64_t off = 0;
    for (int q = 0; q < o; ++q) off += (int64_t)S::out_cnt_at(q) * a.mul * a.mul_out;
    return a.Wt[off + (int64_t)n * K(a) + k];
  }
  __device__ void C(const LaunchArgs& a, int, int64_t m, int n, float v) const {
    const int d3 = S::out_d3_at(o);
    const int64_t i = m / d3;
    const int m3 = (int)(m - i * d3);
    a.y[i * a.out_dim + (int64_t)a.mul_out * S::out_cumY_at(o) + (int64_t)n * d3 + m3] = v;
  }
};

// G_o[(i, m3), (pl, u)] = sum_w gy_o[(i, m3), w] W_{p(pl)}[u, w]
template <class S>
struct GradStateOp {
  int o;
  __device__ int64_t M(const LaunchArgs& a) const { return (int64_t)a.N * S::out_d3_at(o); }
  __device__ int Nn(const LaunchArgs& a) const { return S::out_cnt_at(o) * a.mul; }
  __device__ void k_range(const LaunchArgs& a, int, int64_t& b, int64_t& e) const { b = 0; e = a.mul_out; }
  __device__ float A(const LaunchArgs& a, int64_t m, int64_t k) const {
    const int d3 = S::out_d3_at(o);
    const int64_t i = m / d3;
    const int m3 = (int)(m - i * d3);
    return a.gy[i * a.out_dim + (int64_t)a.mul_out * S::out_cumY_at(o) + k * d3 + m3];
  }
  __device__ float B(const LaunchArgs& a, int n, int64_t k) const {
    const int pl = n / a.mul, u = n - pl * a.mul;
    const int p = S::path_of_at(o, pl);
    return a.W[((int64_t)p * a.mul + u) * a.mul_out + k];
  }
  __device__ void C(const LaunchArgs& a, int, int64_t m, int n, float v) const {
    a.G[(int64_t)a.N * a.mul * S::out_cumA_at(o) + m * Nn(a) + n] = v;
  }
};

// part[z][p][u][w] = sum_{(i, m3) in split z} A_o[(i, m3), (pl, u)] gy_o[(i, m3), w]
template <class S>
struct GradWOp {
  int o;
  __device__ int64_t M(const LaunchArgs& a) const { return (int64_t)S::out_cnt_at(o) * a.mul; }
  __device__ int Nn(const LaunchArgs& a) const { return a.mul_out; }
  __device__ void k_range(const LaunchArgs& a, int z, int64_t& b, int64_t& e) const {
    const int64_t rows = (int64_t)a.N * S::out_d3_at(o);
    const int64_t chunk = ((rows + a.splits - 1) / a.splits + GBK - 1) / GBK * GBK;
    b = min(rows, (int64_t)z * chunk);
    e = min(rows, b + chunk);
  }
  __device__ float A(const LaunchArgs& a, int64_t m, int64_t k) const {
    return a.A[(int64_t)a.N * a.mul * S::out_cumA_at(o) + k * M(a) + m];
  }
  __device__ float B(const LaunchArgs& a, int n, int64_t k) const {
    const int d3 = S::out_d3_at(o);
    const int64_t i = k / d3;
    const int m3 = (int)(k - i * d3);
    return a.gy[i * a.out_dim + (int64_t)a.mul_out * S::out_cumY_at(o) + (int64_t)n * d3 + m3];
  }
  __device__ void C(const LaunchArgs& a, int z, int64_t m, int n, float v) const {
    const int pl = (int)(m / a.mul), u = (int)(m - (int64_t)pl * a.mul);
    const int p = S::path_of_at(o, pl);
    a.part[((int64_t)z * S::P + p) * a.mul * a.mul_out + (int64_t)u * a.mul_out + n] = v;
  }
};


// ---------------------------------------------------------------------------------------
// The same three contractions for the tcgen05 GEMM (tp_mma.cuh): element accessors, vector
// accessors for k-contiguous operands, and coalesced tile stores.
// ---------------------------------------------------------------------------------------
template <class S>
struct TcMixFwdOp {           // y_o[(i, m3), w] = sum_k A_o[(i, m3), k] Wt_o[w, k]
  int o;
  static constexpr bool A_KCONTIG = true, B_KCONTIG = true;
  __device__ int64_t M(const LaunchArgs& a) const { return (int64_t)a.N * S::out_d3_at(o); }
  __device__ int Nn(const LaunchArgs& a) const { return a.mul_out; }
  __device__ int K(const LaunchArgs& a) const { return S::out_cnt_at(o) * a.mul; }
  __device__ void k_range(const LaunchArgs& a, int, int64_t& b, int64_t& e) const { b = 0; e = K(a); }
  __device__ const float* Abase(const LaunchArgs& a) const { return a.A + (int64_t)a.N * a.mul * S::out_cumA_at(o); }
  __device__ const float* Bbase(const LaunchArgs& a) const {
    int64_t off = 0;
    for (int q = 0; q < o; ++q) off += (int64_t)S::out_cnt_at(q) * a.mul * a.mul_out;
    return a.Wt + off;
  }
  __device__ float A(const LaunchArgs& a, int64_t m, int64_t k) const { return Abase(a)[m * K(a) + k]; }
  __device__ float B(const LaunchArgs& a, int n, int64_t k) const { return Bbase(a)[(int64_t)n * K(a) + k]; }
  __device__ float4 A4(const LaunchArgs& a, int64_t m, int64_t k) const {
    return *reinterpret_cast<const float4*>(Abase(a) + m * K(a) + k);
  }
  __device__ float4 B4(const LaunchArgs& a, int n, int64_t k) const {
    return *reinterpret_cast<const float4*>(Bbase(a) + (int64_t)n * K(a) + k);
  }
  __device__ void store_tile(const LaunchArgs& a, int, const float* T, int ld, int64_t m0, int n0) const {
    const int d3 = S::out_d3_at(o);
    const int64_t Mx = M(a);
    const int64_t i0 = m0 / d3, i1 = (min(Mx, m0 + TC_BM) - 1) / d3;
    const int cols = min(TC_BN, a.mul_out - n0);
    const int per_i = cols * d3;
    const int64_t total = (i1 - i0 + 1) * per_i;
    for (int64_t t = threadIdx.x; t < total; t += blockDim.x) {
      const int64_t i = i0 + t / per_i;
      const int q = (int)(t % per_i);
      const int w = q / d3, m3 = q - (q / d3) * d3;
      const int64_t row = i * d3 + m3 - m0;
      if (row < 0 || row >= TC_BM || i * d3 + m3 >= Mx) continue;
      a.y[i * a.out_dim + (int64_t)a.mul_out * S::out_cumY_at(o) + (int64_t)(n0 + w) * d3 + m3] = T[row * ld + w];
    }
  }
};

template <class S>
struct TcGradStateOp {        // G_o[(i, m3), (pl, u)] = sum_w gy_o[(i, m3), w] W_p[u, w]
  int o;
  static constexpr bool A_KCONTIG = false, B_KCONTIG = true;
  __device__ int64_t M(const LaunchArgs& a) const { return (int64_t)a.N * S::out_d3_at(o); }
  __device__ int Nn(const LaunchArgs& a) const { return S::out_cnt_at(o) * a.mul; }
  __device__ void k_range(const LaunchArgs& a, int, int64_t& b, int64_t& e) const { b = 0; e = a.mul_out; }
  __device__ float A(const LaunchArgs& a, int64_t m, int64_t k) const {
    const int d3 = S::out_d3_at(o);
    const int64_t i = m / d3;
    const int m3 = (int)(m - i * d3);
    return a.gy[i * a.out_dim + (int64_t)a.mul_out * S::out_cumY_at(o) + k * d3 + m3];
  }
  __device__ float4 A4(const LaunchArgs& a, int64_t m, int64_t k) const {
    return make_float4(A(a, m, k), A(a, m, k + 1), A(a, m, k + 2), A(a, m, k + 3));
  }
  __device__ const float* Brow(const LaunchArgs& a, int n) const {
    const int pl = n / a.mul, u = n - pl * a.mul;
    return a.W + ((int64_t)S::path_of_at(o, pl) * a.mul + u) * a.mul_out;
  }
  __device__ float B(const LaunchArgs& a, int n, int64_t k) const { return Brow(a, n)[k]; }
  __device__ float4 B4(const LaunchArgs& a, int n, int64_t k) const {
    return *reinterpret_cast<const float4*>(Brow(a, n) + k);
  }
  __device__ void store_tile(const LaunchArgs& a, int, const float* T, int ld, int64_t m0, int n0) const {
    const int64_t Mx = M(a);
    const int Kn = Nn(a);
    const int cols = min(TC_BN, Kn - n0);
    float* G = a.G + (int64_t)a.N * a.mul * S::out_cumA_at(o);
    for (int t = threadIdx.x; t < TC_BM * cols; t += blockDim.x) {
      const int r = t / cols, c = t - r * cols;
      if (m0 + r < Mx) G[(m0 + r) * Kn + n0 + c] = T[r * ld + c];
    }
  }
};

template <class S>
struct TcGradWOp {            // part[z][p][u][w] = sum_{(i, m3) in split z} A_o[(i, m3), (pl, u)] gy_o[(i, m3), w]
  int o;
  static constexpr bool A_KCONTIG = false, B_KCONTIG = false;
  __device__ int64_t M(const LaunchArgs& a) const { return (int64_t)S::out_cnt_at(o) * a.mul; }
  __device__ int Nn(const LaunchArgs& a) const { return a.mul_out; }
  __device__ void k_range(const LaunchArgs& a, int z, int64_t& b, int64_t& e) const {
    const int64_t rows = (int64_t)a.N * S::out_d3_at(o);
    const int64_t chunk = ((rows + a.splits - 1) / a.splits + TC_BK - 1) / TC_BK * TC_BK;
    b = min(rows, (int64_t)z * chunk);
    e = min(rows, b + chunk);
  }
  __device__ float A(const LaunchArgs& a, int64_t m, int64_t k) const {
    return a.A[(int64_t)a.N * a.mul * S::out_cumA_at(o) + k * M(a) + m];
  }
  __device__ float4 A4(const LaunchArgs& a, int64_t m, int64_t k) const {
    return make_float4(A(a, m, k), A(a, m, k + 1), A(a, m, k + 2), A(a, m, k + 3));
  }
  __device__ float B(const LaunchArgs& a, int n, int64_t k) const {
    const int d3 = S::out_d3_at(o);
    const int64_t i = k / d3;
    const int m3 = (int)(k - i * d3);
    return a.gy[i * a.out_dim + (int64_t)a.mul_out * S::out_cumY_at(o) + (int64_t)n * d3 + m3];
  }
  __device__ float4 B4(const LaunchArgs& a, int n, int64_t k) const {
    return make_float4(B(a, n, k), B(a, n, k + 1), B(a, n, k + 2), B(a, n, k + 3));
  }
  __device__ void store_tile(const LaunchArgs& a, int z, const float* T, int ld, int64_t m0, int n0) const {
    const int64_t Mx = M(a);
    const int cols = min(TC_BN, a.mul_out - n0);
    for (int t = threadIdx.x; t < TC_BM * cols; t += blockDim.x) {
      const int r = t / cols, c = t - r * cols;
      const int64_t m = m0 + r;
      if (m >= Mx) continue;
      const int pl = (int)(m / a.mul), u = (int)(m - (int64_t)pl * a.mul);
      const int p = S::path_of_at(o, pl);
      a.part[((int64_t)z * S::P + p) * a.mul * a.mul_out + (int64_t)u * a.mul_out + n0 + c] = T[r * ld + c];
    }
  }
};

// The tensor-core path reads k-contiguous operand rows (A, G, Wt in the workspace and the
// caller's W) as float4: it needs multiplicities divisible by 4 and a 16-byte aligned W.
inline bool tc_usable(const LaunchArgs& a) {
  return a.use_tc && a.mul % 4 == 0 && a.mul_out % 4 == 0 && (reinterpret_cast<uintptr_t>(a.W) & 15u) == 0;
}

// gW[idx] = sum_z part[z][idx] in split order (deterministic)
static __global__ void k_reduce_splits(const float* __restrict__ part, int splits, int64_t n, float* gW) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n; t += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int z = 0; z < splits; ++z) s += part[(int64_t)z * n + t];
    gW[t] = s;
  }
}

// ---------------------------------------------------------------------------------------
// Sender pass: gx[j] (segmented), gs[e, p] and gvec[e] (channel sums across all slices of a
// row, which share one CTA).  grid = N, block = 32 * NSL (one edge phase).
// ---------------------------------------------------------------------------------------
template <class S, bool GVEC, int NSL>
__global__ void __launch_bounds__(kMaxThreads) k_uvw_send(const __grid_constant__ LaunchArgs a) {
  extern __shared__ float smem[];
  constexpr int NV = S::P + 4;   // per edge and slice: P gs partials, 3 gvec partials (+ degree sum)
  const int lane = threadIdx.x & 31;
  const int sl = threadIdx.x >> 5;
  const int node = blockIdx.x;
  const int c = sl * 32 + lane;
  const bool act = c < a.mul;
  int q0 = __ldg(a.colptr + node), q1 = __ldg(a.colptr + node + 1);
  if (a.check) {
    q0 = max(0, min(q0, a.E));
    q1 = max(q0, min(q1, a.E));
  }
  float x[S::IN_PC], gx[S::IN_PC];
#pragma unroll
  for (int k = 0; k < S::IN_PC; ++k) {
    gx[k] = 0.f;
    x[k] = 0.f;
  }
  if (act) S::load_in(a.x + (int64_t)node * a.in_dim, a.mul, c, x);
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
        my_i = find_row(a.rowptr, a.N, my_e);
        vx = __ldg(a.vec + 3 * (int64_t)my_e);
        vy = __ldg(a.vec + 3 * (int64_t)my_e + 1);
        vz = __ldg(a.vec + 3 * (int64_t)my_e + 2);
      }
    }
    const int ne = min(32, q1 - base);
#pragma unroll 1
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
      float gY[S::NSH], gs[S::P];
#pragma unroll
      for (int m = 0; m < S::NSH; ++m) gY[m] = 0.f;
#pragma unroll
      for (int p = 0; p < S::P; ++p) gs[p] = 0.f;
      if (e >= 0) {
        float s[S::P];
        const float* srow = a.w + (int64_t)e * S::P;
#pragma unroll
        for (int p = 0; p < S::P; ++p) s[p] = __ldg(srow + p) * (a.has_coeff ? a.coeff[p] : 1.f);
        if (act) {
          float g[S::A_PC];
          S::load_uvw(a.G, a.N, a.mul, i, c, g);
          S::template uvw_bwd<GVEC>(x, Y, s, g, gx, gs, gY);
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
        h0 = warp_sum(h0);
        h1 = warp_sum(h1);
        h2 = warp_sum(h2);
        sdeg = warp_sum(sdeg);
      }
#pragma unroll
      for (int p = 0; p < S::P; ++p) gs[p] = warp_sum(gs[p]);
      if (lane == 0) {
        float* sp = slot + ((size_t)k * NSL + sl) * NV;
#pragma unroll
        for (int p = 0; p < S::P; ++p) sp[p] = gs[p];
        sp[S::P] = h0;
        sp[S::P + 1] = h1;
        sp[S::P + 2] = h2;
        sp[S::P + 3] = sdeg;
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
  }
  if (act && a.gx) S::store_in(a.gx + (int64_t)node * a.in_dim, a.mul, c, gx);
}

// ---------------------------------------------------------------------------------------
// Host sequences
// ---------------------------------------------------------------------------------------
template <class Op>
static cudaError_t launch_gemm(const LaunchArgs& a, const Op& op, int64_t M, int Nn, int splits, cudaStream_t s) {
  if (M <= 0 || Nn <= 0) return cudaSuccess;
  dim3 grid((unsigned)((M + GBM - 1) / GBM), (unsigned)((Nn + GBN - 1) / GBN), (unsigned)splits);
  k_gemm_simt<Op><<<grid, 256, 0, s>>>(a, op);
  count_launches(1);
  return cudaGetLastError();
}

template <class S>
cudaError_t launch_uvw_edge(const LaunchArgs& a, cudaStream_t s) {
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
  const bool tc = tc_usable(a);
  for (int o = 0; o < S::N_OUT; ++o) {
    const int64_t M = (int64_t)a.N * S::out_d3_at(o);
    e = tc ? launch_gemm_tc(a, TcMixFwdOp<S>{o}, M, a.mul_out, 1, s) : launch_gemm(a, MixFwdOp<S>{o}, M, a.mul_out, 1, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <class S>
cudaError_t launch_uvw_bwd(const LaunchArgs& a, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  cudaError_t e = launch_uvw_edge<S>(a, s);
  if (e != cudaSuccess) return e;
  const bool tc = tc_usable(a);
  for (int o = 0; o < S::N_OUT; ++o) {
    const int64_t M = (int64_t)a.N * S::out_d3_at(o);
    const int K = S::out_cnt_at(o) * a.mul;
    e = tc ? launch_gemm_tc(a, TcGradStateOp<S>{o}, M, K, 1, s) : launch_gemm(a, GradStateOp<S>{o}, M, K, 1, s);
    if (e != cudaSuccess) return e;
    if (a.gW) {
      e = tc ? launch_gemm_tc(a, TcGradWOp<S>{o}, K, a.mul_out, a.splits, s)
             : launch_gemm(a, GradWOp<S>{o}, K, a.mul_out, a.splits, s);
      if (e != cudaSuccess) return e;
    }
  }
  if (a.gW) {
    const int64_t n = (int64_t)S::P * a.mul * a.mul_out;
    k_reduce_splits<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, s>>>(a.part, a.splits, n, a.gW);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (!a.gx && !a.gw && !a.gvec) return cudaSuccess;
  const int nsl = a.n_slices <= 1 ? 1 : (a.n_slices == 2 ? 2 : 4);
  const size_t sm = (size_t)32 * nsl * (S::P + 4) * sizeof(float);
  const bool gv = a.gvec != nullptr;
#define TP_UVW_SEND(G, NS) k_uvw_send<S, G, NS><<<(unsigned)a.N, 32 * NS, sm, s>>>(a)
  if (nsl == 1) { if (gv) TP_UVW_SEND(true, 1); else TP_UVW_SEND(false, 1); }
  else if (nsl == 2) { if (gv) TP_UVW_SEND(true, 2); else TP_UVW_SEND(false, 2); }
  else { if (gv) TP_UVW_SEND(true, 4); else TP_UVW_SEND(false, 4); }
#undef TP_UVW_SEND
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace tp
