// Node-side operators of the interaction layer (include/tp_block.h): the irreps-wise
// linear map, in two forms -- on the CUDA cores straight from the node rows (narrow maps or
// few nodes: k_lin_direct, k_lin_direct_gw) or on the tcgen05 tensor cores (3xTF32, the
// persistent GEMM of tp_mma.cuh with its own operand regrouping and epilogues) -- and the
// gate nonlinearity (elementwise, k_gate).
//
// Tensor-core linear, per irrep type t = (l, parity) that has instructions (every input
// block of type t is connected to every output block of type t):
//   XA_t[(n, m)][kc]  = x[n, b, u, m]          kc = (input block b of type t, channel u)
//   GA_t[(n, m)][oc]  = gy[n, o, w, m]         oc = (output block o of type t, channel w)
//   y_o   = XA_t . Wt_o^T     Wt_o[w][kc] = c_k W_k[u, w]      one GEMM per output block
//   gx_b  = GA_t . Wg_b^T     Wg_b[u][oc] = c_k W_k[u, w]      one GEMM per input block
//   G_t   = XA_t^T . GA_t     (split-K over the N (2l+1) rows) gW_k[u, w] = c_k G_t[kc, oc]
// The regrouped rows are node sized (they hold x or gy once more); the split weights are the
// size of W.  Every sum runs in a fixed order: the results are deterministic.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "../../include/tp_block.h"
#include "tp_common.h"
#include "tp_host.h"
#include "tp_kernels.cuh"   // warp helpers the GEMM header builds on
#include "tp_mma.cuh"

namespace tp {
namespace {

constexpr int kLinMaxInstr = 64;
constexpr int kLinMaxTypes = 8;     // (l <= 3) x (e, o)
constexpr int kLinMaxBlocks = 16;
constexpr int kLinSplits = 64;      // most split-K partials of a gW GEMM
constexpr int kLinPromote = 16;     // K blocks summed in TMEM before the fp32 promotion
constexpr int kLinGwChunks = 256;   // most node chunks (partials) of a CUDA-core gW

// ---------------------------------------------------------------------------------------
// Device side
// ---------------------------------------------------------------------------------------

// Regrouping of node rows into per-type [(n, m)][concatenated channel] rows, plus zeroing
// of the output blocks that no GEMM writes.
struct GatherArgs {
  const float* src;
  int64_t src_stride;
  float* dst;
  int64_t N;
  int n_groups;
  int d[kLinMaxTypes], K[kLinMaxTypes], nblk[kLinMaxTypes];
  int64_t cum[kLinMaxTypes];                       // group g starts at dst + N * cum[g]
  int boff[kLinMaxTypes][kLinMaxBlocks];           // block offset in the source row
  int bcat[kLinMaxTypes][kLinMaxBlocks];           // first concatenated channel of the block
  float* zdst;
  int64_t zstride;
  int nz;
  int zoff[kLinMaxBlocks], zlen[kLinMaxBlocks];
};

__global__ void k_lin_gather(const __grid_constant__ GatherArgs g) {
  for (int64_t n = blockIdx.x; n < g.N; n += gridDim.x) {
    const float* row = g.src + n * g.src_stride;
    for (int q = 0; q < g.n_groups; ++q) {
      const int d = g.d[q], K = g.K[q], total = d * K;
      float* dst = g.dst + g.N * g.cum[q] + n * (int64_t)total;
      for (int t = threadIdx.x; t < total; t += blockDim.x) {
        const int m = t / K, c = t - m * K;
        int b = 0;
        while (b + 1 < g.nblk[q] && c >= g.bcat[q][b + 1]) ++b;
        const int u = c - g.bcat[q][b];
        dst[t] = __ldg(row + g.boff[q][b] + u * d + m);
      }
    }
    for (int z = 0; z < g.nz; ++z) {
      float* zr = g.zdst + n * g.zstride + g.zoff[z];
      for (int t = threadIdx.x; t < g.zlen[z]; t += blockDim.x) zr[t] = 0.f;
    }
  }
}

// Per-instruction weight tables: the split operands (prep) and the split-K reduction.
struct InstrArgs {
  int n_instr;
  int64_t total;                       // n_weights
  int64_t woff[kLinMaxInstr];          // start of W_k in W
  int mul_in[kLinMaxInstr], mul_out[kLinMaxInstr];
  float coeff[kLinMaxInstr];
  int64_t base[kLinMaxInstr];          // prep: block base in Wt / Wg; reduce: (kc0, oc0) start in G_t
  int ld[kLinMaxInstr];                // prep: row length of the operand; reduce: row length of G_t
  int coff[kLinMaxInstr];              // prep: column offset of this instruction's channels
  int splits[kLinMaxInstr];            // reduce: partials of the instruction's type
  int transpose;                       // prep: 0 -> [w][kc] (forward), 1 -> [u][oc] (backward)
};

__device__ __forceinline__ int find_instr(const InstrArgs& a, int64_t t) {
  int k = 0;
  while (k + 1 < a.n_instr && t >= a.woff[k + 1]) ++k;
  return k;
}

// dst (hi) and dst + total (lo): c_k W_k[u, w] at row w, column coff + u (forward) or row
// u, column coff + w (backward).
__global__ void k_lin_prep(const __grid_constant__ InstrArgs a, const float* __restrict__ W, float* dst) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < a.total; t += (int64_t)gridDim.x * blockDim.x) {
    const int k = find_instr(a, t);
    const int64_t r = t - a.woff[k];
    const int u = (int)(r / a.mul_out[k]), w = (int)(r - (int64_t)u * a.mul_out[k]);
    const float v = a.coeff[k] * W[t];
    const int64_t idx = a.transpose ? a.base[k] + (int64_t)u * a.ld[k] + a.coff[k] + w
                                    : a.base[k] + (int64_t)w * a.ld[k] + a.coff[k] + u;
    const float h = tf32_hi(v);
    dst[idx] = h;
    dst[idx + a.total] = v - h;
  }
}

// gW[t] = c_k sum_z part[z][base_k + u * ld + w]: a CTA takes 32 consecutive weights (one
// per lane); warp i of 8 sums the partials z = i, i + 8, ... in order and the 8 warp sums
// are added in warp order, so the result is deterministic.
__global__ void __launch_bounds__(256) k_lin_reduce(const __grid_constant__ InstrArgs a, const float* __restrict__ part,
                                                    float* gW) {
  __shared__ float red[8][33];
  const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
  for (int64_t t0 = (int64_t)blockIdx.x * 32; t0 < a.total; t0 += (int64_t)gridDim.x * 32) {
    const int64_t t = t0 + lane;
    int k = 0, splits = 0;
    int64_t idx = 0;
    if (t < a.total) {
      k = find_instr(a, t);
      const int64_t r = t - a.woff[k];
      const int u = (int)(r / a.mul_out[k]), w = (int)(r - (int64_t)u * a.mul_out[k]);
      idx = a.base[k] + (int64_t)u * a.ld[k] + w;
      splits = a.splits[k];
    }
    float s = 0.f;
#pragma unroll 4
    for (int z = wp; z < splits; z += 8) s += __ldg(part + (int64_t)z * a.total + idx);
    red[wp][lane] = s;
    __syncthreads();
    if (wp == 0 && t < a.total) {
      float r = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) r += red[i][lane];
      gW[t] = a.coeff[k] * r;
    }
    __syncthreads();
  }
}

// Stores of a rows x cols accumulator block T (row stride ld; first element at global row
// r0 = (node, m) pair, global column n0) into node rows [node][base + col * D + m]: one
// contiguous run of cols * D floats per node, 32 lanes per instruction.
template <int D>
__device__ __forceinline__ void lin_store_rows(float* out, int64_t stride, int64_t base, const float* T, int ld,
                                               int64_t r0, int rows, int64_t M, int n0, int cols, int lane, int acc) {
  const int64_t rlast = min(M, r0 + rows) - 1;
  if (rlast < r0) return;
  for (int64_t i = r0 / D; i <= rlast / D; ++i) {
    float* dst = out + i * stride + base + (int64_t)n0 * D;
    for (int q = lane; q < cols * D; q += 32) {
      const int w = q / D, m = q - w * D;
      const int64_t row = i * D + m;
      if (row >= r0 && row <= rlast) {
        const float v = T[(int)(row - r0) * ld + w];
        dst[q] = acc ? dst[q] + v : v;
      }
    }
  }
}

// y_o[(n, m), w] (forward) or gx_b[(n, m), u] (backward): K-major regrouped rows times the
// split weights, stored into node rows.
template <int D>
struct LinRowsOp {
  CUtensorMap tA, tA2, tB, tB2;
  int64_t M, Nn;
  int K;
  float* out;
  int64_t stride, base;
  int acc;
  static constexpr int A_FMT = FMT_K, B_FMT = FMT_SPLIT, PROMOTE = 0;
  __device__ void k_range(const LaunchArgs&, int, int64_t& b, int64_t& e) const { b = 0; e = K; }
  __device__ void store_tile(const LaunchArgs&, int, const float* T, int ld, int64_t r0, int rows, int n0,
                             int cols, int lane) const {
    lin_store_rows<D>(out, stride, base, T, ld, r0, rows, M, n0, cols, lane, acc);
  }
};

// part[z][kc][oc] = sum over the rows of split z of XA_t[row][kc] GA_t[row][oc].
struct LinGwOp {
  CUtensorMap tA, tA2, tB, tB2;
  int64_t M, Nn;            // K_t, N_t
  int64_t rows;             // N (2l+1): the reduction
  int splits;
  float* part;              // this type's region of split 0
  int64_t split_stride;     // floats between the splits' regions
  static constexpr int A_FMT = FMT_MN, B_FMT = FMT_MN, PROMOTE = kLinPromote;
  __device__ void k_range(const LaunchArgs&, int z, int64_t& b, int64_t& e) const {
    const int64_t chunk = ((rows + splits - 1) / splits + TC_BK - 1) / TC_BK * TC_BK;
    b = min(rows, (int64_t)z * chunk);
    e = min(rows, b + chunk);
  }
  __device__ void store_tile(const LaunchArgs&, int z, const float* T, int ld, int64_t r0, int nrows, int n0,
                             int cols, int lane) const {
    if (lane >= cols) return;
    const int nr = (int)min((int64_t)nrows, M - r0);
    float* dst = part + (int64_t)z * split_stride + r0 * Nn + n0 + lane;
    for (int r = 0; r < nr; ++r) dst[(int64_t)r * Nn] = T[r * ld + lane];
  }
};

template <template <int> class Op, class F>
cudaError_t lin_with_d(int d, F&& f) {
  switch (d) {
    case 1: return f(Op<1>{});
    case 3: return f(Op<3>{});
    case 5: return f(Op<5>{});
    default: return f(Op<7>{});
  }
}

// ---------------------------------------------------------------------------------------
// Gate
// ---------------------------------------------------------------------------------------
struct GateArgs {
  int64_t N;
  int in_dim, out_dim;
  int n_scalar, n_gate;
  int n_sblk, smul_end[kLinMaxBlocks], spar[kLinMaxBlocks];   // scalar blocks: cumulative channel end, parity
  int n_gblk;
  int gcum[kLinMaxBlocks], gd[kLinMaxBlocks];                 // gated blocks: first gate channel, 2l+1
  int gin[kLinMaxBlocks], gout[kLinMaxBlocks];                // their offsets in the input / output row
  const float* x;
  const float* gy;
  const float* ggx;
  float* y;      // forward output / dbwd g_gy
  float* gx;     // bwd output / dbwd g_x
};

__device__ __forceinline__ float sigm(float v) { return 1.f / (1.f + __expf(-v)); }

// tanh from expm1 of -2|v| (no cancellation near 0): tanh|v| = -t / (2 + t)
__device__ __forceinline__ float tanh_of(float v) {
  const float t = expm1f(-2.f * fabsf(v));
  return copysignf(-t / (2.f + t), v);
}

// act, act', act'' of a scalar channel (SiLU for even, tanh for odd)
__device__ __forceinline__ void scalar_act(float v, int par, float& f, float& f1, float& f2) {
  if (par > 0) {
    const float s = sigm(v), s1 = s * (1.f - s);
    f = v * s;
    f1 = s + v * s1;
    f2 = s1 * (2.f + v * (1.f - 2.f * s));
  } else {
    const float t = tanh_of(v), t1 = 1.f - t * t;
    f = t;
    f1 = t1;
    f2 = -2.f * t * t1;
  }
}

// MODE 0 forward, 1 backward, 2 double backward.  One thread per (node, item): items are
// the scalar channels, then the gate channels (each with its gated channel's 2l+1 values).
template <int MODE>
__global__ void k_gate(const __grid_constant__ GateArgs a) {
  const int items = a.n_scalar + a.n_gate;
  const int64_t total = a.N * items;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = t / items;
    const int it = (int)(t - n * items);
    const float* xr = a.x + n * a.in_dim;
    if (it < a.n_scalar) {
      int b = 0;
      while (it >= a.smul_end[b]) ++b;
      float f, f1, f2;
      scalar_act(xr[it], a.spar[b], f, f1, f2);
      if (MODE == 0) {
        a.y[n * a.out_dim + it] = f;
      } else if (MODE == 1) {
        a.gx[n * a.in_dim + it] = f1 * a.gy[n * a.out_dim + it];
      } else {
        const float gg = a.ggx[n * a.in_dim + it];
        if (a.y) a.y[n * a.out_dim + it] = f1 * gg;
        if (a.gx) a.gx[n * a.in_dim + it] = f2 * a.gy[n * a.out_dim + it] * gg;
      }
      continue;
    }
    const int c = it - a.n_scalar;
    int b = 0;
    while (b + 1 < a.n_gblk && c >= a.gcum[b + 1]) ++b;
    const int d = a.gd[b], u = c - a.gcum[b];
    const float gv = xr[a.n_scalar + c];
    const float s = sigm(gv), s1 = s * (1.f - s);
    const float* v = xr + a.gin[b] + u * d;
    const int64_t oi = n * a.out_dim + a.gout[b] + (int64_t)u * d;
    const int64_t ii = n * a.in_dim + a.gin[b] + (int64_t)u * d;
    if (MODE == 0) {
      for (int m = 0; m < d; ++m) a.y[oi + m] = s * v[m];
    } else if (MODE == 1) {
      float dot = 0.f;
      for (int m = 0; m < d; ++m) {
        const float g = a.gy[oi + m];
        a.gx[ii + m] = s * g;
        dot += v[m] * g;
      }
      a.gx[n * a.in_dim + a.n_scalar + c] = s1 * dot;
    } else {
      const float ggg = a.ggx[n * a.in_dim + a.n_scalar + c];
      const float s2 = s1 * (1.f - 2.f * s);
      float vg = 0.f, gq = 0.f;
      for (int m = 0; m < d; ++m) {
        const float g = a.gy[oi + m], q = a.ggx[ii + m];
        if (a.y) a.y[oi + m] = s * q + s1 * v[m] * ggg;
        if (a.gx) a.gx[ii + m] = s1 * g * ggg;
        vg += v[m] * g;
        gq += g * q;
      }
      if (a.gx) a.gx[n * a.in_dim + a.n_scalar + c] = s1 * gq + s2 * ggg * vg;
    }
  }
}

// ---------------------------------------------------------------------------------------
// Linear on the CUDA cores, straight from the node rows: the form for small channel counts,
// where the map is bound by HBM or by launch latency and the regrouping of the tensor-core
// form would only add traffic and launches.  One CTA takes a tile of NB consecutive nodes,
// stages their rows in shared memory and produces every output block of them; each thread
// computes one (channel, m) output for all NB nodes, so a weight read from L1 serves NB FMAs.
//   out[n, off_j + c d + m] = sum_{terms t of j} c_t sum_v W[t](v, c) in[n, soff_t + v d + m]
// with W[t](v, c) = W[woff_t + v * sv + c * sc]: (sv, sc) = (mul_out, 1) in the forward
// (v = u, c = w) and (1, mul_out) for gx (v = w, c = u).
// ---------------------------------------------------------------------------------------
constexpr int kDirectThreads = 256;
constexpr int kDirectNB = 8;                    // nodes per tile
constexpr int kDirectSmemFloats = 56 * 1024;    // 224 KB: staged weights + rows

struct DirectArgs {
  int64_t N;
  const float* in;
  int64_t in_stride;
  float* out;
  int64_t out_stride;
  const float* W;
  int64_t n_weights, w_stage;                  // weights staged in shared memory (0: read from L2)
  int acc, n_groups, sc_is_ld, vec, vec_w, n_instr, out_cols;
  int o_off[kLinMaxBlocks], o_d[kLinMaxBlocks], t_begin[kLinMaxBlocks], t_count[kLinMaxBlocks];
  int s_off[kLinMaxInstr], s_mul[kLinMaxInstr], w_ld[kLinMaxInstr], g_ld[kLinMaxInstr];
  int i_mul_in[kLinMaxInstr], i_mul_out[kLinMaxInstr];
  int64_t w_off[kLinMaxInstr];
  float coeff[kLinMaxInstr];
  int64_t i_woff[kLinMaxInstr];                // per instruction, in W order (for the staging)
  float i_coeff[kLinMaxInstr];
};

// Copies count floats (a multiple of 4 when vec, with 16-byte aligned ends) into shared memory.
__device__ __forceinline__ void stage(float* dst, const float* src, int64_t count, int vec) {
  if (vec) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll 4
    for (int64_t t = threadIdx.x; t < (count >> 2); t += blockDim.x) d4[t] = __ldg(s4 + t);
  } else {
#pragma unroll 4
    for (int64_t t = threadIdx.x; t < count; t += blockDim.x) dst[t] = __ldg(src + t);
  }
}

template <bool WS>
__global__ void __launch_bounds__(kDirectThreads) k_lin_direct(const __grid_constant__ DirectArgs a) {
  extern __shared__ __align__(16) float dsm[];
  float* wsm = dsm;
  float* xs = dsm + a.w_stage;
  if constexpr (WS) {
    // c_k W_k once per CTA: in the global [u][w] layout for the map, as [w][u] for the
    // adjoint, so that a warp's consecutive output channels read consecutive words.  Every
    // W_k spans a multiple of 16 floats (channel counts are multiples of 4), so a float4
    // never straddles two of them.
    if (a.vec_w && !a.sc_is_ld) {
      const float4* w4 = reinterpret_cast<const float4*>(a.W);
#pragma unroll 4
      for (int64_t t = threadIdx.x; t < (a.n_weights >> 2); t += blockDim.x) {
        int k = 0;
        while (k + 1 < a.n_instr && 4 * t >= a.i_woff[k + 1]) ++k;
        float4 v = __ldg(w4 + t);
        const float ck = a.i_coeff[k];
        v.x *= ck;
        v.y *= ck;
        v.z *= ck;
        v.w *= ck;
        reinterpret_cast<float4*>(wsm)[t] = v;
      }
    } else {
      for (int64_t t = threadIdx.x; t < a.n_weights; t += blockDim.x) {
        int k = 0;
        while (k + 1 < a.n_instr && t >= a.i_woff[k + 1]) ++k;
        int64_t dst = t;
        if (a.sc_is_ld) {
          const int64_t r = t - a.i_woff[k];
          const int u = (int)(r / a.i_mul_out[k]), w = (int)(r - (int64_t)u * a.i_mul_out[k]);
          dst = a.i_woff[k] + (int64_t)w * a.i_mul_in[k] + u;
        }
        wsm[dst] = a.i_coeff[k] * __ldg(a.W + t);
      }
    }
  }
  for (int64_t n0 = (int64_t)blockIdx.x * kDirectNB; n0 < a.N; n0 += (int64_t)gridDim.x * kDirectNB) {
    const int nb_here = (int)min((int64_t)kDirectNB, a.N - n0);
    __syncthreads();
    stage(xs, a.in + n0 * a.in_stride, (int64_t)nb_here * a.in_stride, a.vec);
    __syncthreads();
    // all output blocks of the row in one pass: thread t takes row positions t, t + 256, ...
    for (int t = threadIdx.x; t < a.out_cols; t += blockDim.x) {
      int j = 0;
      while (j + 1 < a.n_groups && t >= a.o_off[j + 1]) ++j;
      const int d = a.o_d[j];
      const int r = t - a.o_off[j];
      const int c = r / d, m = r - c * d;
      if (a.acc && a.t_count[j] == 0) continue;      // accumulate leaves blocks without terms
      float acc[kDirectNB];
#pragma unroll
      for (int q = 0; q < kDirectNB; ++q) acc[q] = 0.f;
      for (int k = a.t_begin[j]; k < a.t_begin[j] + a.t_count[j]; ++k) {
        // staged: element (v, c) at w_off + v * ld + c for both the map and the adjoint
        const int ld = a.w_ld[k];
        const int64_t sv = (WS || !a.sc_is_ld) ? ld : 1, sc = (WS || !a.sc_is_ld) ? 1 : a.g_ld[k];
        const float ck = WS ? 1.f : a.coeff[k];
        const float* wp = (WS ? wsm : a.W) + a.w_off[k] + c * sc;
        const float* xp = xs + a.s_off[k] + m;
        for (int v = 0; v < a.s_mul[k]; v += 4) {      // channel counts are multiples of 4
          float wv[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) wv[i] = ck * (WS ? wp[(v + i) * sv] : __ldg(wp + (v + i) * sv));
#pragma unroll
          for (int q = 0; q < kDirectNB; ++q) {        // rows past nb_here hold stale data, never stored
            const float* xq = xp + q * a.in_stride + v * d;
            acc[q] = fmaf(wv[0], xq[0], acc[q]);
            acc[q] = fmaf(wv[1], xq[d], acc[q]);
            acc[q] = fmaf(wv[2], xq[2 * d], acc[q]);
            acc[q] = fmaf(wv[3], xq[3 * d], acc[q]);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < kDirectNB; ++q)
        if (q < nb_here) {
          float* o = a.out + (n0 + q) * a.out_stride + t;
          *o = a.acc ? *o + acc[q] : acc[q];
        }
    }
  }
}

// Per-CTA partial weight gradients on the CUDA cores: CTA (z, r) sums over the nodes of
// chunk z; each thread owns one 4 x 4 tile (u0..u0+3, w0..w0+3) of one W_k (channel counts
// are multiples of 4) and adds the outer products of x[n, in(k), u, m] and gy[n, out(k), w, m]
// over the chunk's (n, m): 8 shared-memory loads per 16 FMAs.
//   part[z][woff_k + u mul_out + w] = sum_{n in chunk z, m} x[n, in(k), u, m] gy[n, out(k), w, m]
// (coefficients are applied by the reduction, k_lin_reduce).
struct DirectGwArgs {
  int64_t N, chunk;
  const float* x;
  const float* gy;
  int64_t x_stride, gy_stride;
  float* part;
  int64_t n_weights;
  int n_instr, vec, n_tiles;
  int tile0[kLinMaxInstr + 1];      // first 4 x 4 tile of each instruction; tile0[n_instr] = n_tiles
  int64_t woff[kLinMaxInstr];
  int xoff[kLinMaxInstr], goff[kLinMaxInstr], mul_out[kLinMaxInstr], d[kLinMaxInstr];
};

__global__ void __launch_bounds__(kDirectThreads) k_lin_direct_gw(const __grid_constant__ DirectGwArgs a) {
  extern __shared__ __align__(16) float gsm[];
  float* xs = gsm;
  float* gs = gsm + kDirectNB * a.x_stride;
  const int64_t nb0 = (int64_t)blockIdx.x * a.chunk, nb1 = min(a.N, nb0 + a.chunk);
  const int T = blockIdx.y * kDirectThreads + threadIdx.x;
  const bool own = T < a.n_tiles;
  int k = 0, xo = 0, go = 0, d = 0, u0 = 0, w0 = 0;
  if (own) {
    while (k + 1 < a.n_instr && T >= a.tile0[k + 1]) ++k;
    const int tw_n = a.mul_out[k] / 4, r = T - a.tile0[k];
    u0 = 4 * (r / tw_n);
    w0 = 4 * (r - (r / tw_n) * tw_n);
    d = a.d[k];
    xo = a.xoff[k] + u0 * d;
    go = a.goff[k] + w0 * d;
  }
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int64_t n0 = nb0; n0 < nb1; n0 += kDirectNB) {
    const int nb_here = (int)min((int64_t)kDirectNB, nb1 - n0);
    __syncthreads();
    stage(xs, a.x + n0 * a.x_stride, (int64_t)nb_here * a.x_stride, a.vec);
    stage(gs, a.gy + n0 * a.gy_stride, (int64_t)nb_here * a.gy_stride, a.vec);
    __syncthreads();
    for (int q = 0; q < nb_here; ++q) {
      const float* xq = xs + q * a.x_stride + xo;
      const float* gq = gs + q * a.gy_stride + go;
      for (int m = 0; m < d; ++m) {
        float xv[4], gv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          xv[i] = xq[i * d + m];
          gv[i] = gq[i * d + m];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xv[i], gv[j], acc[i][j]);
      }
    }
  }
  if (own) {
    float* dst = a.part + (int64_t)blockIdx.x * a.n_weights + a.woff[k] + w0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4*>(dst + (int64_t)(u0 + i) * a.mul_out[k]) =
          make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
  }
}

size_t al256(size_t v) { return (v + 255) & ~size_t(255); }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

tp_status_t fail(tp_status_t st, const std::string& m) { return set_failure(st, m); }
tp_status_t cuda_failed(cudaError_t e, const char* where) {
  return set_failure(TP_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

int grid_for(int64_t work, int per_block) {
  const int64_t b = (work + per_block - 1) / per_block;
  return (int)std::max<int64_t>(1, std::min<int64_t>(b, (int64_t)sm_count() * 8));
}

}  // namespace
}  // namespace tp

using namespace tp;

// ---------------------------------------------------------------------------------------
// Host side: the linear handle
// ---------------------------------------------------------------------------------------
struct LinType {
  int l, parity, d;
  int nin, nout;
  int in_blk[kLinMaxBlocks], out_blk[kLinMaxBlocks];
  int in_cat[kLinMaxBlocks], out_cat[kLinMaxBlocks];
  int K, Nn;                       // concatenated input / output channels
  int64_t xa_cum, ga_cum, g_cum;   // per-node float offsets of XA_t and GA_t; offset of G_t
};

struct tp_linear_s {
  std::vector<IrrepTerm> in, out;
  std::vector<int64_t> in_off, out_off;
  int64_t in_dim = 0, out_dim = 0, n_weights = 0;
  int n_instr = 0;
  int ins_in[kLinMaxInstr], ins_out[kLinMaxInstr], ins_type[kLinMaxInstr];
  int64_t ins_woff[kLinMaxInstr];
  float coeff[kLinMaxInstr];
  int n_types = 0;
  LinType types[kLinMaxTypes];
  int64_t xa_per_node = 0, ga_per_node = 0;
  int64_t wt_base[kLinMaxBlocks];   // per output block: its rows of Wt
  int64_t wg_base[kLinMaxBlocks];   // per input block: its rows of Wg
  int type_of_in[kLinMaxBlocks], type_of_out[kLinMaxBlocks];
  uint32_t flags = 0;
};

namespace {

struct LinWs {
  size_t xa, ga, wsplit, part, total;
};

LinWs lin_ws(const tp_linear_s* L, int64_t N, bool bwd) {
  LinWs w{};
  size_t off = 0;
  w.xa = off;
  off += al256(sizeof(float) * (size_t)std::max<int64_t>(1, N * L->xa_per_node));
  w.ga = off;
  if (bwd) off += al256(sizeof(float) * (size_t)std::max<int64_t>(1, N * L->ga_per_node));
  w.wsplit = off;
  off += al256(sizeof(float) * 2 * (size_t)std::max<int64_t>(1, L->n_weights));
  w.part = off;
  if (bwd) off += al256(sizeof(float) * (size_t)std::max(kLinSplits, kLinGwChunks) * (size_t)std::max<int64_t>(1, L->n_weights));
  w.total = off;
  return w;
}

int lin_splits(int64_t rows) {
  const int64_t per = (int64_t)TC_BK * 4;   // short splits: many CTAs, little serial latency
  return (int)std::max<int64_t>(1, std::min<int64_t>(kLinSplits, (rows + per - 1) / per));
}

LaunchArgs gemm_args() {
  LaunchArgs a;
  std::memset(&a, 0, sizeof(a));
  a.err = device_error_ptr();
  return a;
}

// Regroups `src` rows by type: groups for the inputs (out_side = false) or the outputs.
GatherArgs gather_args(const tp_linear_s* L, int64_t N, const float* src, float* dst, bool out_side) {
  GatherArgs g;
  std::memset(&g, 0, sizeof(g));
  g.src = src;
  g.src_stride = out_side ? L->out_dim : L->in_dim;
  g.dst = dst;
  g.N = N;
  g.n_groups = L->n_types;
  for (int q = 0; q < L->n_types; ++q) {
    const LinType& T = L->types[q];
    g.d[q] = T.d;
    g.K[q] = out_side ? T.Nn : T.K;
    g.cum[q] = out_side ? T.ga_cum : T.xa_cum;
    g.nblk[q] = out_side ? T.nout : T.nin;
    for (int b = 0; b < g.nblk[q]; ++b) {
      const int blk = out_side ? T.out_blk[b] : T.in_blk[b];
      g.boff[q][b] = (int)(out_side ? L->out_off[blk] : L->in_off[blk]);
      g.bcat[q][b] = out_side ? T.out_cat[b] : T.in_cat[b];
    }
  }
  return g;
}

// Zero the blocks of `dst` rows (outputs, or input gradients) that no GEMM writes.
void add_zero_ranges(const tp_linear_s* L, GatherArgs& g, float* dst, bool out_side) {
  g.zdst = dst;
  g.zstride = out_side ? L->out_dim : L->in_dim;
  const auto& blocks = out_side ? L->out : L->in;
  const auto& offs = out_side ? L->out_off : L->in_off;
  const int* type_of = out_side ? L->type_of_out : L->type_of_in;
  for (size_t b = 0; b < blocks.size(); ++b)
    if (type_of[b] < 0) {
      g.zoff[g.nz] = (int)offs[b];
      g.zlen[g.nz] = blocks[b].mul * (2 * blocks[b].l + 1);
      ++g.nz;
    }
}

cudaError_t launch_gather(const GatherArgs& g, cudaStream_t s) {
  if (g.N == 0 || (g.n_groups == 0 && g.nz == 0)) return cudaSuccess;
  const unsigned grid = (unsigned)std::min<int64_t>(g.N, (int64_t)sm_count() * 16);
  k_lin_gather<<<grid, 128, 0, s>>>(g);
  count_launches(1);
  return cudaGetLastError();
}

InstrArgs instr_args(const tp_linear_s* L) {
  InstrArgs a;
  std::memset(&a, 0, sizeof(a));
  a.n_instr = L->n_instr;
  a.total = L->n_weights;
  for (int k = 0; k < L->n_instr; ++k) {
    a.woff[k] = L->ins_woff[k];
    a.mul_in[k] = L->in[L->ins_in[k]].mul;
    a.mul_out[k] = L->out[L->ins_out[k]].mul;
    a.coeff[k] = L->coeff[k];
  }
  return a;
}

int index_in(const int* arr, int n, int v) {
  for (int i = 0; i < n; ++i)
    if (arr[i] == v) return i;
  return -1;
}

// Split weights for the forward (transpose = 0: Wt_o[w][kc]) or the gx GEMMs (1: Wg_b[u][oc]).
cudaError_t launch_prep(const tp_linear_s* L, const float* W, float* dst, int transpose, cudaStream_t s) {
  if (L->n_weights == 0) return cudaSuccess;
  InstrArgs a = instr_args(L);
  a.transpose = transpose;
  for (int k = 0; k < L->n_instr; ++k) {
    const LinType& T = L->types[L->ins_type[k]];
    const int bi = index_in(T.in_blk, T.nin, L->ins_in[k]), oi = index_in(T.out_blk, T.nout, L->ins_out[k]);
    if (!transpose) {
      a.base[k] = L->wt_base[L->ins_out[k]];
      a.ld[k] = T.K;
      a.coff[k] = T.in_cat[bi];
    } else {
      a.base[k] = L->wg_base[L->ins_in[k]];
      a.ld[k] = T.Nn;
      a.coff[k] = T.out_cat[oi];
    }
  }
  k_lin_prep<<<grid_for(L->n_weights, 256), 256, 0, s>>>(a, W, dst);
  count_launches(1);
  return cudaGetLastError();
}

// The tensor-core form pays a regrouping pass and several launches; it wins when the
// channel counts make the map compute heavy and the node count fills the GPU.
bool use_tensor_cores(const tp_linear_s* L, int64_t N) {
  if (L->flags & TP_LINEAR_TENSOR_CORES) return true;
  if (L->flags & TP_LINEAR_CUDA_CORES) return false;
  if ((int64_t)kDirectNB * (L->in_dim + L->out_dim) > kDirectSmemFloats) return true;   // rows too wide to stage
  if (N < 4096 || L->n_types == 0) return false;
  for (int q = 0; q < L->n_types; ++q)
    if (std::min(L->types[q].K, L->types[q].Nn) < 64) return false;
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaError_t set_smem(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  if (bytes > 227 * 1024) return cudaErrorInvalidValue;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// out rows = the map (forward: in = x) or its adjoint (gx: in = gy) on the CUDA cores.
cudaError_t launch_direct(const tp_linear_s* L, int64_t N, const float* in, const float* W, float* out, int acc,
                          bool adjoint, cudaStream_t s) {
  DirectArgs a;
  std::memset(&a, 0, sizeof(a));
  a.N = N;
  a.in = in;
  a.in_stride = adjoint ? L->out_dim : L->in_dim;
  a.out = out;
  a.out_stride = adjoint ? L->in_dim : L->out_dim;
  a.W = W;
  a.acc = acc;
  a.sc_is_ld = adjoint ? 1 : 0;
  const auto& dst = adjoint ? L->in : L->out;
  const auto& dst_off = adjoint ? L->in_off : L->out_off;
  int nt = 0;
  for (int j = 0; j < (int)dst.size(); ++j) {
    a.o_off[j] = (int)dst_off[j];
    a.o_d[j] = 2 * dst[j].l + 1;
    a.t_begin[j] = nt;
    for (int k = 0; k < L->n_instr; ++k) {
      if ((adjoint ? L->ins_in[k] : L->ins_out[k]) != j) continue;
      const int src_blk = adjoint ? L->ins_out[k] : L->ins_in[k];
      a.s_off[nt] = (int)(adjoint ? L->out_off[src_blk] : L->in_off[src_blk]);
      a.s_mul[nt] = adjoint ? L->out[src_blk].mul : L->in[src_blk].mul;
      a.w_off[nt] = L->ins_woff[k];
      // row length of the staged layout ([u][w] for the map, [w][u] for the adjoint) and of
      // the global one ([u][w])
      a.w_ld[nt] = adjoint ? L->in[L->ins_in[k]].mul : L->out[L->ins_out[k]].mul;
      a.g_ld[nt] = L->out[L->ins_out[k]].mul;
      a.coeff[nt] = L->coeff[k];
      ++nt;
    }
    a.t_count[j] = nt - a.t_begin[j];
  }
  a.n_groups = (int)dst.size();
  a.out_cols = (int)a.out_stride;
  a.n_instr = L->n_instr;
  for (int k = 0; k < L->n_instr; ++k) {
    a.i_woff[k] = L->ins_woff[k];
    a.i_coeff[k] = L->coeff[k];
    a.i_mul_in[k] = L->in[L->ins_in[k]].mul;
    a.i_mul_out[k] = L->out[L->ins_out[k]].mul;
  }
  a.n_weights = L->n_weights;
  a.vec = aligned16(in) && a.in_stride % 4 == 0;
  a.vec_w = aligned16(W) && L->n_weights % 4 == 0;
  const int64_t rows = (int64_t)kDirectNB * a.in_stride;
  if (rows > kDirectSmemFloats) return cudaErrorInvalidValue;
  const bool ws = L->n_weights + rows + 4 <= kDirectSmemFloats;
  a.w_stage = ws ? (L->n_weights + 3) / 4 * 4 : 0;
  const size_t smem = sizeof(float) * (size_t)(a.w_stage + rows);
  const void* fn = ws ? reinterpret_cast<const void*>(k_lin_direct<true>) : reinterpret_cast<const void*>(k_lin_direct<false>);
  cudaError_t e = set_smem(fn, smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (N + kDirectNB - 1) / kDirectNB;
  const unsigned grid = (unsigned)std::min<int64_t>(tiles, (int64_t)sm_count() * 4);
  if (ws) k_lin_direct<true><<<grid, kDirectThreads, smem, s>>>(a);
  else k_lin_direct<false><<<grid, kDirectThreads, smem, s>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

// gW on the CUDA cores: per-CTA partials over node chunks, then the fixed-order reduction.
cudaError_t launch_direct_gw(const tp_linear_s* L, int64_t N, const float* x, const float* gy, float* part,
                             float* gW, cudaStream_t s) {
  DirectGwArgs a;
  std::memset(&a, 0, sizeof(a));
  const int64_t Z = std::max<int64_t>(1, std::min<int64_t>(kLinGwChunks, (N + kDirectNB - 1) / kDirectNB));
  a.N = N;
  a.chunk = (N + Z - 1) / Z;
  a.x = x;
  a.gy = gy;
  a.x_stride = L->in_dim;
  a.gy_stride = L->out_dim;
  a.part = part;
  a.n_weights = L->n_weights;
  a.n_instr = L->n_instr;
  a.vec = aligned16(x) && aligned16(gy) && L->in_dim % 4 == 0 && L->out_dim % 4 == 0;
  if ((int64_t)kDirectNB * (L->in_dim + L->out_dim) > kDirectSmemFloats) return cudaErrorInvalidValue;
  for (int k = 0; k < L->n_instr; ++k) {
    a.tile0[k] = a.n_tiles;
    a.n_tiles += (L->in[L->ins_in[k]].mul / 4) * (L->out[L->ins_out[k]].mul / 4);
    a.woff[k] = L->ins_woff[k];
    a.xoff[k] = (int)L->in_off[L->ins_in[k]];
    a.goff[k] = (int)L->out_off[L->ins_out[k]];
    a.mul_out[k] = L->out[L->ins_out[k]].mul;
    a.d[k] = 2 * L->in[L->ins_in[k]].l + 1;
  }
  const size_t smem = sizeof(float) * (size_t)kDirectNB * (size_t)(L->in_dim + L->out_dim);
  cudaError_t e = set_smem(reinterpret_cast<const void*>(k_lin_direct_gw), smem);
  if (e != cudaSuccess) return e;
  a.tile0[L->n_instr] = a.n_tiles;
  const int64_t tranges = (a.n_tiles + kDirectThreads - 1) / kDirectThreads;
  k_lin_direct_gw<<<dim3((unsigned)Z, (unsigned)tranges), kDirectThreads, smem, s>>>(a);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  InstrArgs r = instr_args(L);
  for (int k = 0; k < L->n_instr; ++k) {
    r.base[k] = L->ins_woff[k];
    r.ld[k] = L->out[L->ins_out[k]].mul;
    r.splits[k] = (int)Z;
  }
  k_lin_reduce<<<grid_for(L->n_weights, 32), 256, 0, s>>>(r, part, gW);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

extern "C" {

tp_status_t tp_linear_create(tp_linear_t* lin, const char* irreps_in, const char* irreps_out, const double* coeff,
                             uint32_t flags) {
  if (!lin) return fail(TP_ERR_INVALID_ARG, "lin is NULL");
  *lin = nullptr;
  if ((flags & ~3u) || flags == 3u) return fail(TP_ERR_INVALID_ARG, "flags: TP_LINEAR_TENSOR_CORES or TP_LINEAR_CUDA_CORES");
  std::vector<IrrepTerm> in, out;
  std::string why;
  if (!parse_irreps_terms(irreps_in, in, why)) return fail(TP_ERR_INVALID_ARG, "irreps_in: " + why);
  if (!parse_irreps_terms(irreps_out, out, why)) return fail(TP_ERR_INVALID_ARG, "irreps_out: " + why);
  if ((int)in.size() > kLinMaxBlocks || (int)out.size() > kLinMaxBlocks)
    return fail(TP_ERR_UNSUPPORTED, "at most 16 blocks per irreps string");
  for (const auto* v : {&in, &out})
    for (const IrrepTerm& t : *v) {
      if (t.l > 3) return fail(TP_ERR_UNSUPPORTED, "l > 3");
      if (t.mul % 4) return fail(TP_ERR_UNSUPPORTED, "multiplicities must be multiples of 4 (TMA row pitch)");
    }
  tp_linear_s* L = new (std::nothrow) tp_linear_s();
  if (!L) return fail(TP_ERR_INVALID_ARG, "out of host memory");
  L->in = in;
  L->out = out;
  L->flags = flags;
  for (const IrrepTerm& t : in) {
    L->in_off.push_back(L->in_dim);
    L->in_dim += (int64_t)t.mul * (2 * t.l + 1);
  }
  for (const IrrepTerm& t : out) {
    L->out_off.push_back(L->out_dim);
    L->out_dim += (int64_t)t.mul * (2 * t.l + 1);
  }
  for (int b = 0; b < kLinMaxBlocks; ++b) L->type_of_in[b] = L->type_of_out[b] = -1;
  // instructions in lexicographic (i_in, i_out) order; types in order of first appearance
  for (int i = 0; i < (int)in.size(); ++i)
    for (int o = 0; o < (int)out.size(); ++o) {
      if (in[i].l != out[o].l || in[i].parity != out[o].parity) continue;
      if (L->n_instr == kLinMaxInstr) {
        delete L;
        return fail(TP_ERR_UNSUPPORTED, "more than 64 instructions");
      }
      int q = 0;
      while (q < L->n_types && !(L->types[q].l == in[i].l && L->types[q].parity == in[i].parity)) ++q;
      if (q == L->n_types) {
        LinType& T = L->types[L->n_types++];
        std::memset(&T, 0, sizeof(T));
        T.l = in[i].l;
        T.parity = in[i].parity;
        T.d = 2 * T.l + 1;
        for (int b = 0; b < (int)in.size(); ++b)
          if (in[b].l == T.l && in[b].parity == T.parity) {
            T.in_blk[T.nin] = b;
            T.in_cat[T.nin++] = T.K;
            T.K += in[b].mul;
            L->type_of_in[b] = q;
          }
        for (int b = 0; b < (int)out.size(); ++b)
          if (out[b].l == T.l && out[b].parity == T.parity) {
            T.out_blk[T.nout] = b;
            T.out_cat[T.nout++] = T.Nn;
            T.Nn += out[b].mul;
            L->type_of_out[b] = q;
          }
      }
      const int k = L->n_instr++;
      L->ins_in[k] = i;
      L->ins_out[k] = o;
      L->ins_type[k] = q;
      L->ins_woff[k] = L->n_weights;
      L->coeff[k] = coeff ? (float)coeff[k] : 1.f;
      L->n_weights += (int64_t)in[i].mul * out[o].mul;
    }
  if (coeff)
    for (int k = 0; k < L->n_instr; ++k)
      if (!std::isfinite(coeff[k])) {
        delete L;
        return fail(TP_ERR_INVALID_ARG, "coefficients must be finite");
      }
  int64_t xa = 0, ga = 0, gc = 0, wt = 0, wg = 0;
  for (int q = 0; q < L->n_types; ++q) {
    LinType& T = L->types[q];
    T.xa_cum = xa;
    T.ga_cum = ga;
    T.g_cum = gc;
    xa += (int64_t)T.d * T.K;
    ga += (int64_t)T.d * T.Nn;
    gc += (int64_t)T.K * T.Nn;
  }
  L->xa_per_node = xa;
  L->ga_per_node = ga;
  for (int o = 0; o < (int)out.size(); ++o) {
    L->wt_base[o] = wt;
    if (L->type_of_out[o] >= 0) wt += (int64_t)out[o].mul * L->types[L->type_of_out[o]].K;
  }
  for (int b = 0; b < (int)in.size(); ++b) {
    L->wg_base[b] = wg;
    if (L->type_of_in[b] >= 0) wg += (int64_t)in[b].mul * L->types[L->type_of_in[b]].Nn;
  }
  *lin = L;
  return TP_OK;
}

tp_status_t tp_linear_destroy(tp_linear_t lin) {
  delete lin;
  return TP_OK;
}

tp_status_t tp_linear_query(tp_linear_t lin, int64_t* in_dim, int64_t* out_dim, int64_t* n_weights,
                            int32_t* n_instructions) {
  if (!lin) return fail(TP_ERR_INVALID_ARG, "lin is NULL");
  if (in_dim) *in_dim = lin->in_dim;
  if (out_dim) *out_dim = lin->out_dim;
  if (n_weights) *n_weights = lin->n_weights;
  if (n_instructions) *n_instructions = lin->n_instr;
  return TP_OK;
}

tp_status_t tp_linear_workspace_size(tp_linear_t lin, int64_t N, int32_t op, size_t* bytes) {
  if (!lin || !bytes) return fail(TP_ERR_INVALID_ARG, "lin and bytes must not be NULL");
  if (N < 0) return fail(TP_ERR_INVALID_ARG, "N must be non-negative");
  if (op != TP_OP_FWD && op != TP_OP_BWD) return fail(TP_ERR_INVALID_ARG, "op must be TP_OP_FWD or TP_OP_BWD");
  *bytes = lin_ws(lin, N, op == TP_OP_BWD).total;
  return TP_OK;
}

static tp_status_t lin_check(tp_linear_t lin, int64_t N, void* ws, size_t ws_bytes, bool bwd) {
  if (!lin) return fail(TP_ERR_INVALID_ARG, "lin is NULL");
  if (N < 0) return fail(TP_ERR_INVALID_ARG, "N must be non-negative");
  if (N * 7 >= ((int64_t)1 << 31)) return fail(TP_ERR_UNSUPPORTED, "N (2l+1) must be below 2^31");
  if (N == 0) return TP_OK;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return fail(TP_ERR_WORKSPACE, "workspace NULL or not 256-byte aligned");
  if (ws_bytes < lin_ws(lin, N, bwd).total) return fail(TP_ERR_WORKSPACE, "workspace too small");
  return TP_OK;
}

tp_status_t tp_linear_fwd(tp_linear_t lin, int64_t N, const float* x, const float* W, float* y, int32_t accumulate,
                          void* ws, size_t ws_bytes, tp_stream_t stream) {
  tp_status_t st = lin_check(lin, N, ws, ws_bytes, false);
  if (st != TP_OK || N == 0) return st;
  if (!x || !y || (lin->n_weights && !W)) return fail(TP_ERR_INVALID_ARG, "x, W and y must not be NULL");
  if (!aligned4(x) || !aligned4(y) || !aligned4(W)) return fail(TP_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!use_tensor_cores(lin, N)) {
    cudaError_t e = launch_direct(lin, N, x, W, y, accumulate ? 1 : 0, false, s);
    return e == cudaSuccess ? TP_OK : cuda_failed(e, "linear (CUDA cores)");
  }
  const LinWs L = lin_ws(lin, N, false);
  char* base = static_cast<char*>(ws);
  float* XA = reinterpret_cast<float*>(base + L.xa);
  float* Wt = reinterpret_cast<float*>(base + L.wsplit);
  cudaError_t e = launch_prep(lin, W, Wt, 0, s);
  if (e != cudaSuccess) return cuda_failed(e, "linear weight split");
  GatherArgs g = gather_args(lin, N, x, XA, false);
  if (!accumulate) add_zero_ranges(lin, g, y, true);
  if ((e = launch_gather(g, s)) != cudaSuccess) return cuda_failed(e, "linear regroup");
  const LaunchArgs a = gemm_args();
  for (int q = 0; q < lin->n_types; ++q) {
    const LinType& T = lin->types[q];
    const float* A = XA + N * T.xa_cum;
    for (int j = 0; j < T.nout; ++j) {
      const int o = T.out_blk[j];
      e = lin_with_d<LinRowsOp>(T.d, [&](auto op) {
        op.M = N * T.d;
        op.Nn = lin->out[o].mul;
        op.K = T.K;
        op.out = y;
        op.stride = lin->out_dim;
        op.base = lin->out_off[o];
        op.acc = accumulate ? 1 : 0;
        cudaError_t r = make_tmap(&op.tA, A, T.K, op.M, T.K, FMT_K);
        if (r == cudaSuccess) r = make_tmap(&op.tB, Wt + lin->wt_base[o], T.K, op.Nn, T.K, FMT_SPLIT);
        if (r == cudaSuccess) r = make_tmap(&op.tB2, Wt + lin->n_weights + lin->wt_base[o], T.K, op.Nn, T.K, FMT_SPLIT);
        if (r != cudaSuccess) return r;
        return launch_gemm_tc(a, op, 1, s);
      });
      if (e != cudaSuccess) return cuda_failed(e, "linear GEMM");
    }
  }
  return TP_OK;
}

tp_status_t tp_linear_bwd(tp_linear_t lin, int64_t N, const float* x, const float* W, const float* gy, float* gx,
                          float* gW, void* ws, size_t ws_bytes, tp_stream_t stream) {
  if (lin && N == 0 && gW && lin->n_weights) {
    // no rows: the weight gradient is zero
    cudaError_t e = cudaMemsetAsync(gW, 0, sizeof(float) * (size_t)lin->n_weights, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TP_OK : cuda_failed(e, "cudaMemsetAsync(gW)");
  }
  tp_status_t st = lin_check(lin, N, ws, ws_bytes, true);
  if (st != TP_OK || N == 0) return st;
  if (!gy) return fail(TP_ERR_INVALID_ARG, "gy must not be NULL");
  if (gx && lin->n_weights && !W) return fail(TP_ERR_INVALID_ARG, "gx needs W");
  if (gW && !x) return fail(TP_ERR_INVALID_ARG, "gW needs x");
  if (!aligned4(x) || !aligned4(W) || !aligned4(gy) || !aligned4(gx) || !aligned4(gW))
    return fail(TP_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  if (!gx && !gW) return TP_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const LinWs L = lin_ws(lin, N, true);
  if (!use_tensor_cores(lin, N)) {
    cudaError_t e = cudaSuccess;
    if (gx) e = launch_direct(lin, N, gy, W, gx, 0, true, s);
    if (e == cudaSuccess && gW && lin->n_weights)
      e = launch_direct_gw(lin, N, x, gy, reinterpret_cast<float*>(static_cast<char*>(ws) + L.part), gW, s);
    return e == cudaSuccess ? TP_OK : cuda_failed(e, "linear backward (CUDA cores)");
  }
  char* base = static_cast<char*>(ws);
  float* XA = reinterpret_cast<float*>(base + L.xa);
  float* GA = reinterpret_cast<float*>(base + L.ga);
  float* Wg = reinterpret_cast<float*>(base + L.wsplit);
  float* part = reinterpret_cast<float*>(base + L.part);
  cudaError_t e;
  GatherArgs g = gather_args(lin, N, gy, GA, true);
  if (gx) add_zero_ranges(lin, g, gx, false);
  if ((e = launch_gather(g, s)) != cudaSuccess) return cuda_failed(e, "linear regroup gy");
  const LaunchArgs a = gemm_args();
  if (gx) {
    if ((e = launch_prep(lin, W, Wg, 1, s)) != cudaSuccess) return cuda_failed(e, "linear weight split");
    for (int q = 0; q < lin->n_types; ++q) {
      const LinType& T = lin->types[q];
      const float* A = GA + N * T.ga_cum;
      for (int j = 0; j < T.nin; ++j) {
        const int b = T.in_blk[j];
        e = lin_with_d<LinRowsOp>(T.d, [&](auto op) {
          op.M = N * T.d;
          op.Nn = lin->in[b].mul;
          op.K = T.Nn;
          op.out = gx;
          op.stride = lin->in_dim;
          op.base = lin->in_off[b];
          op.acc = 0;
          cudaError_t r = make_tmap(&op.tA, A, T.Nn, op.M, T.Nn, FMT_K);
          if (r == cudaSuccess) r = make_tmap(&op.tB, Wg + lin->wg_base[b], T.Nn, op.Nn, T.Nn, FMT_SPLIT);
          if (r == cudaSuccess) r = make_tmap(&op.tB2, Wg + lin->n_weights + lin->wg_base[b], T.Nn, op.Nn, T.Nn, FMT_SPLIT);
          if (r != cudaSuccess) return r;
          return launch_gemm_tc(a, op, 1, s);
        });
        if (e != cudaSuccess) return cuda_failed(e, "linear gx GEMM");
      }
    }
  }
  if (gW && lin->n_weights) {
    GatherArgs gx_rows = gather_args(lin, N, x, XA, false);
    if ((e = launch_gather(gx_rows, s)) != cudaSuccess) return cuda_failed(e, "linear regroup x");
    InstrArgs r = instr_args(lin);
    for (int q = 0; q < lin->n_types; ++q) {
      const LinType& T = lin->types[q];
      const int64_t rows = N * T.d;
      LinGwOp op;
      std::memset(&op, 0, sizeof(op));
      op.M = T.K;
      op.Nn = T.Nn;
      op.rows = rows;
      op.splits = lin_splits(rows);
      op.part = part + T.g_cum;
      op.split_stride = lin->n_weights;
      e = make_tmap(&op.tA, XA + N * T.xa_cum, T.K, rows, T.K, FMT_MN);
      if (e == cudaSuccess) e = make_tmap(&op.tB, GA + N * T.ga_cum, T.Nn, rows, T.Nn, FMT_MN);
      if (e == cudaSuccess) e = launch_gemm_tc(a, op, op.splits, s);
      if (e != cudaSuccess) return cuda_failed(e, "linear gW GEMM");
      for (int k = 0; k < lin->n_instr; ++k)
        if (lin->ins_type[k] == q) {
          const int bi = index_in(T.in_blk, T.nin, lin->ins_in[k]), oi = index_in(T.out_blk, T.nout, lin->ins_out[k]);
          r.base[k] = T.g_cum + (int64_t)T.in_cat[bi] * T.Nn + T.out_cat[oi];
          r.ld[k] = T.Nn;
          r.splits[k] = op.splits;
        }
    }
    k_lin_reduce<<<grid_for(lin->n_weights, 32), 256, 0, s>>>(r, part, gW);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_failed(e, "linear gW reduction");
  }
  return TP_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Host side: the gate handle
// ---------------------------------------------------------------------------------------
struct tp_gate_s {
  GateArgs proto;   // layout fields filled, pointers and N zero
};

extern "C" {

tp_status_t tp_gate_create(tp_gate_t* gate, const char* irreps_scalars, const char* irreps_gates,
                           const char* irreps_gated) {
  if (!gate) return fail(TP_ERR_INVALID_ARG, "gate is NULL");
  *gate = nullptr;
  std::vector<IrrepTerm> sc, gt, gd;
  std::string why;
  auto parse = [&](const char* s, std::vector<IrrepTerm>& v, const char* name) -> bool {
    if (!s || !*s) return true;
    if (!parse_irreps_terms(s, v, why)) {
      why = std::string(name) + ": " + why;
      return false;
    }
    return true;
  };
  if (!parse(irreps_scalars, sc, "irreps_scalars") || !parse(irreps_gates, gt, "irreps_gates") ||
      !parse(irreps_gated, gd, "irreps_gated"))
    return fail(TP_ERR_INVALID_ARG, why);
  if ((int)sc.size() > kLinMaxBlocks || (int)gd.size() > kLinMaxBlocks)
    return fail(TP_ERR_UNSUPPORTED, "at most 16 scalar and 16 gated blocks");
  GateArgs a;
  std::memset(&a, 0, sizeof(a));
  for (const IrrepTerm& t : sc) {
    if (t.l != 0) return fail(TP_ERR_INVALID_ARG, "scalar blocks must have l = 0");
    a.n_scalar += t.mul;
    a.smul_end[a.n_sblk] = a.n_scalar;
    a.spar[a.n_sblk++] = t.parity;
  }
  for (const IrrepTerm& t : gt) {
    if (t.l != 0 || t.parity != 1) return fail(TP_ERR_INVALID_ARG, "gate blocks must be 0e");
    a.n_gate += t.mul;
  }
  int gated = 0, in_off = a.n_scalar + a.n_gate, out_off = a.n_scalar;
  for (const IrrepTerm& t : gd) {
    if (t.l > 3) return fail(TP_ERR_UNSUPPORTED, "l > 3");
    a.gcum[a.n_gblk] = gated;
    a.gd[a.n_gblk] = 2 * t.l + 1;
    a.gin[a.n_gblk] = in_off;
    a.gout[a.n_gblk++] = out_off;
    gated += t.mul;
    in_off += t.mul * (2 * t.l + 1);
    out_off += t.mul * (2 * t.l + 1);
  }
  if (gated != a.n_gate) return fail(TP_ERR_INVALID_ARG, "gate multiplicity must equal the gated multiplicity");
  a.in_dim = in_off;
  a.out_dim = out_off;
  tp_gate_s* G = new (std::nothrow) tp_gate_s();
  if (!G) return fail(TP_ERR_INVALID_ARG, "out of host memory");
  G->proto = a;
  *gate = G;
  return TP_OK;
}

tp_status_t tp_gate_destroy(tp_gate_t gate) {
  delete gate;
  return TP_OK;
}

tp_status_t tp_gate_query(tp_gate_t gate, int64_t* in_dim, int64_t* out_dim) {
  if (!gate) return fail(TP_ERR_INVALID_ARG, "gate is NULL");
  if (in_dim) *in_dim = gate->proto.in_dim;
  if (out_dim) *out_dim = gate->proto.out_dim;
  return TP_OK;
}

static tp_status_t gate_launch(tp_gate_t gate, int mode, int64_t N, const float* x, const float* gy,
                               const float* ggx, float* y, float* gx, tp_stream_t stream) {
  if (!gate) return fail(TP_ERR_INVALID_ARG, "gate is NULL");
  if (N < 0) return fail(TP_ERR_INVALID_ARG, "N must be non-negative");
  const GateArgs& p = gate->proto;
  const int items = p.n_scalar + p.n_gate;
  if (N == 0 || items == 0) return TP_OK;
  if (N * (int64_t)std::max(p.in_dim, 1) >= ((int64_t)1 << 40)) return fail(TP_ERR_UNSUPPORTED, "N too large");
  if (!x || (mode >= 1 && !gy) || (mode == 2 && !ggx)) return fail(TP_ERR_INVALID_ARG, "missing input");
  if (mode == 0 && !y) return fail(TP_ERR_INVALID_ARG, "y must not be NULL");
  if (mode == 1 && !gx) return fail(TP_ERR_INVALID_ARG, "gx must not be NULL");
  if (mode == 2 && !y && !gx) return TP_OK;
  if (!aligned4(x) || !aligned4(gy) || !aligned4(ggx) || !aligned4(y) || !aligned4(gx))
    return fail(TP_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  GateArgs a = p;
  a.N = N;
  a.x = x;
  a.gy = gy;
  a.ggx = ggx;
  a.y = y;
  a.gx = gx;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int grid = grid_for(N * items, 256);
  if (mode == 0) k_gate<0><<<grid, 256, 0, s>>>(a);
  else if (mode == 1) k_gate<1><<<grid, 256, 0, s>>>(a);
  else k_gate<2><<<grid, 256, 0, s>>>(a);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TP_OK : cuda_failed(e, "gate kernel");
}

tp_status_t tp_gate_fwd(tp_gate_t gate, int64_t N, const float* x, float* y, tp_stream_t stream) {
  return gate_launch(gate, 0, N, x, nullptr, nullptr, y, nullptr, stream);
}

tp_status_t tp_gate_bwd(tp_gate_t gate, int64_t N, const float* x, const float* gy, float* gx, tp_stream_t stream) {
  return gate_launch(gate, 1, N, x, gy, nullptr, nullptr, gx, stream);
}

tp_status_t tp_gate_dbwd(tp_gate_t gate, int64_t N, const float* x, const float* gy, const float* ggx, float* g_gy,
                         float* g_x, tp_stream_t stream) {
  return gate_launch(gate, 2, N, x, gy, ggx, g_gy, g_x, stream);
}

}  // extern "C"
