// CSR checks and the stable receiver->sender transpose used by the sender-order passes.
//
// The backward pass aggregates gradients by sender ("Sobek", abstract: the streaming
// formulation extends through backward and double backward, with no edge-sized adjoints),
// so it walks the edges grouped by sender.  colptr = exclusive scan of the sender
// histogram; perm = the stable sort of edge ids by sender (equal to a stable argsort of
// src), so every sender's edges are visited in increasing edge order and the segmented
// sums are reproducible bit for bit.
//
// Four kernels, no inter-CTA waits: an integer histogram (atomics on int counters are
// order independent), a single-CTA exclusive scan, an unordered scatter through atomic
// cursors, then a rank pass that places every edge at the position given by the number of
// smaller edge ids in its sender segment.  Workspace: counts[N] and tmp[E] int32.
#include "tp_common.h"

namespace tp {

__global__ void k_csr_validate(int N, int E, const int32_t* __restrict__ rowptr,
                               const int32_t* __restrict__ src, int* err) {
  const int64_t total = (int64_t)max(N + 1, E);
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    if (t < N) {
      if (rowptr[t + 1] < rowptr[t]) atomicCAS(err, 0, kDevBadRowptr);
    }
    if (t == 0) {
      if (rowptr[0] != 0 || rowptr[N] != E) atomicCAS(err, 0, kDevBadRowptr);
    }
    if (t < E) {
      const int s = src[t];
      if (s < 0 || s >= N) atomicCAS(err, 0, kDevBadSrc);
    }
  }
}

// Senders outside [0, N) are skipped by every transpose kernel (never an out-of-range write);
// with the index-check flag the validation kernel reports them.
__global__ void k_hist(int N, int E, const int32_t* __restrict__ src, int32_t* counts) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < E;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int32_t s = src[e];
    if ((unsigned)s < (unsigned)N) atomicAdd(counts + s, 1);
  }
}

// Exclusive scan of counts[0..N) into colptr[0..N]; counts becomes the scatter cursor.
__global__ void __launch_bounds__(1024) k_scan(int N, int32_t* counts, int32_t* colptr) {
  __shared__ int32_t warp_tot[32];
  const int t = threadIdx.x, nt = blockDim.x;
  const int chunk = (N + nt - 1) / nt;
  const int b = min(N, t * chunk), e = min(N, b + chunk);
  int32_t s = 0;
  for (int k = b; k < e; ++k) s += counts[k];
  // block-wide exclusive scan of s
  const int lane = t & 31, wid = t >> 5;
  int32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int32_t v = lane < (nt >> 5) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    warp_tot[lane] = v;   // inclusive over warps
  }
  __syncthreads();
  int32_t run = incl - s + (wid > 0 ? warp_tot[wid - 1] : 0);
  for (int k = b; k < e; ++k) {
    const int32_t c = counts[k];
    colptr[k] = run;
    counts[k] = run;
    run += c;
  }
  if (t == nt - 1) colptr[N] = warp_tot[(nt >> 5) - 1];
}

__global__ void k_scatter(int N, int E, const int32_t* __restrict__ src, int32_t* cursor, int32_t* tmp) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < E;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int32_t s = src[e];
    if ((unsigned)s >= (unsigned)N) continue;
    const int pos = atomicAdd(cursor + s, 1);
    tmp[pos] = (int32_t)e;
  }
}

__global__ void k_rank(int N, const int32_t* __restrict__ src, const int32_t* __restrict__ colptr,
                       const int32_t* __restrict__ tmp, int32_t* perm) {
  const int32_t nq = colptr[N];     // number of edges with a valid sender
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < nq;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int32_t e = tmp[q];
    const int32_t s = src[e];
    const int32_t lo = colptr[s], hi = colptr[s + 1];
    int32_t r = 0;
    for (int32_t t = lo; t < hi; ++t) r += (tmp[t] < e);
    perm[lo + r] = e;
  }
}

static unsigned grid_for(int64_t n, int block) {
  int64_t g = (n + block - 1) / block;
  const int64_t cap = 148 * 16;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return (unsigned)g;
}

cudaError_t launch_csr_validate(int N, int E, const int32_t* rowptr, const int32_t* src, int* err,
                                cudaStream_t s) {
  k_csr_validate<<<grid_for(max(N + 1, E), 256), 256, 0, s>>>(N, E, rowptr, src, err);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_csr_transpose(int N, int E, const int32_t* src, int32_t* colptr, int32_t* perm,
                                 int32_t* counts, int32_t* tmp, cudaStream_t s) {
  cudaError_t st = cudaMemsetAsync(counts, 0, sizeof(int32_t) * (size_t)max(N, 1), s);
  if (st != cudaSuccess) return st;
  if (E > 0) k_hist<<<grid_for(E, 256), 256, 0, s>>>(N, E, src, counts);
  k_scan<<<1, 1024, 0, s>>>(N, counts, colptr);
  if (E > 0) {
    k_scatter<<<grid_for(E, 256), 256, 0, s>>>(N, E, src, counts, tmp);
    k_rank<<<grid_for(E, 256), 256, 0, s>>>(N, src, colptr, tmp, perm);
  }
  count_launches(E > 0 ? 4 : 1);
  return cudaGetLastError();
}

}  // namespace tp
