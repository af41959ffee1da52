// CSR checks and the stable receiver->sender transpose used by the sender-order passes.
//
// The backward pass aggregates gradients by sender ("Sobek", abstract: the streaming
// formulation extends through backward and double backward, with no edge-sized adjoints),
// so it walks the edges grouped by sender.  colptr[s] = number of edges whose sender is
// below s; perm = the stable sort of edge ids by sender (equal to a stable argsort of src),
// so every sender's edges are visited in increasing edge order and the segmented sums are
// reproducible bit for bit.
//
// The sort is a least-significant-digit radix sort of the edge ids keyed by sender, O(E)
// work per pass whatever the degree distribution (a sender with a million edges costs what
// a million senders with one edge cost).  Keys are the sender ids clamped to [0, N]: an
// edge whose sender lies outside [0, N) gets key N and so lands after every valid edge, in
// edge order.  With b key bits the sort takes ceil(b / 11) passes of at most 11-bit digits
// (c2's 1,536 nodes: one pass; 100,000 nodes: two).  A pass is three kernels over tiles of
// 2,048 consecutive items, with no waits between CTAs:
//   k_radix_hist     per-tile digit histogram (warp-aggregated shared-memory counters);
//   k_radix_scan     per digit, the exclusive scan of its counts over the tiles, and the
//                    digit's total;
//   k_radix_scatter  each CTA scans the digit totals (digit bases), ranks its items within
//                    the tile in item order (warp match + per-warp counters, then a scan
//                    over the warps) and writes every item to base + tile offset + rank.
// Only edge ids move: the key of an item is re-read as src[id] (src is small enough to
// stay in L2).  colptr comes last from the sorted keys (k_colptr): position q is the
// start of every sender in (key[q - 1], key[q]].  Integer counts only, so every step is
// deterministic.
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

constexpr int kRadixThreads = 256;
constexpr int kRadixWarps = kRadixThreads / 32;
constexpr unsigned kAll = 0xffffffffu;

__device__ __forceinline__ uint32_t sender_key(const int32_t* __restrict__ src, int32_t e, int N) {
  const int32_t s = __ldg(src + e);
  return (unsigned)s < (unsigned)N ? (uint32_t)s : (uint32_t)N;
}

// Item order inside a tile: warp w, round r, lane l -> tile_base + w * 256 + r * 32 + l, so a
// round of a warp reads 32 consecutive items and the (warp, round, lane) order is the item
// order.
__device__ __forceinline__ int64_t tile_item(int tile, int warp, int r, int lane) {
  return (int64_t)tile * kRadixTile + warp * (32 * kRadixItems) + r * 32 + lane;
}

__global__ void __launch_bounds__(kRadixThreads) k_radix_hist(int E, int N, const int32_t* __restrict__ src,
                                                              const int32_t* __restrict__ vin, int shift, int R,
                                                              int tiles, int32_t* __restrict__ hist) {
  extern __shared__ int32_t cnt[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int d = tid; d < R; d += kRadixThreads) cnt[d] = 0;
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kRadixItems; ++r) {
    const int64_t q = tile_item(blockIdx.x, warp, r, lane);
    const bool valid = q < E;
    const unsigned vm = __ballot_sync(kAll, valid);
    if (valid) {
      const int32_t e = vin ? __ldg(vin + q) : (int32_t)q;
      const uint32_t d = (sender_key(src, e, N) >> shift) & (uint32_t)(R - 1);
      const unsigned peers = __match_any_sync(vm, d);
      if (lane == __ffs(peers) - 1) atomicAdd(cnt + d, __popc(peers));
    }
  }
  __syncthreads();
  for (int d = tid; d < R; d += kRadixThreads) hist[(int64_t)d * tiles + blockIdx.x] = cnt[d];
}

// One warp per digit: exclusive scan of the digit's per-tile counts (in place) and its total.
__global__ void __launch_bounds__(kRadixThreads) k_radix_scan(int R, int tiles, int32_t* __restrict__ hist,
                                                              int32_t* __restrict__ total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = blockIdx.x * kRadixWarps + warp;
  if (d >= R) return;
  int32_t* row = hist + (int64_t)d * tiles;
  int32_t carry = 0;
  for (int t0 = 0; t0 < tiles; t0 += 32) {
    const int t = t0 + lane;
    const int32_t v = t < tiles ? row[t] : 0;
    int32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u = __shfl_up_sync(kAll, incl, o);
      if (lane >= o) incl += u;
    }
    if (t < tiles) row[t] = carry + incl - v;
    carry += __shfl_sync(kAll, incl, 31);
  }
  if (lane == 0) total[d] = carry;
}

__global__ void __launch_bounds__(kRadixThreads) k_radix_scatter(int E, int N, const int32_t* __restrict__ src,
                                                                 const int32_t* __restrict__ vin,
                                                                 int32_t* __restrict__ vout, int shift, int R,
                                                                 int tiles, const int32_t* __restrict__ hist,
                                                                 const int32_t* __restrict__ total) {
  // 20 R bytes of shared memory (41 KB at R = 2,048), small enough to share an SM with the
  // CTAs of a convolution kernel running beside the transpose
  extern __shared__ int32_t sm[];
  int32_t* toff = sm;                                             // [R]: digit base + tile offset
  uint16_t* wcnt = reinterpret_cast<uint16_t*>(sm + R);           // [warp][R]: counts (<= 256), then
                                                                  // exclusive over the warps (<= 2,048)
  __shared__ int32_t wsum[kRadixWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  // digit bases: block-wide exclusive scan of the totals, each thread a run of `per` digits
  const int per = (R + kRadixThreads - 1) / kRadixThreads;   // 1..8
  int32_t loc[kRadixMaxDigits / kRadixThreads];
  int32_t s = 0;
#pragma unroll
  for (int k = 0; k < kRadixMaxDigits / kRadixThreads; ++k) {
    const int d = tid * per + k;
    loc[k] = (k < per && d < R) ? __ldg(total + d) : 0;
    s += loc[k];
  }
  int32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t u = __shfl_up_sync(kAll, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) wsum[warp] = incl;
  for (int i = tid; i < kRadixWarps * R; i += kRadixThreads) wcnt[i] = 0;
  __syncthreads();
  int32_t pre = incl - s;
  for (int w = 0; w < warp; ++w) pre += wsum[w];
#pragma unroll
  for (int k = 0; k < kRadixMaxDigits / kRadixThreads; ++k) {
    const int d = tid * per + k;
    if (k < per && d < R) toff[d] = pre + __ldg(hist + (int64_t)d * tiles + tile);
    pre += loc[k];
  }
  // ranks inside the warp, round by round in item order
  int32_t val[kRadixItems], rk[kRadixItems];
  uint32_t dig[kRadixItems];
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int r = 0; r < kRadixItems; ++r) {
    const int64_t q = tile_item(tile, warp, r, lane);
    const bool valid = q < E;
    const unsigned vm = __ballot_sync(kAll, valid);
    int32_t e = 0, before = 0;
    uint32_t d = 0;
    unsigned peers = 0;
    if (valid) {
      e = vin ? __ldg(vin + q) : (int32_t)q;
      d = (sender_key(src, e, N) >> shift) & (uint32_t)(R - 1);
      peers = __match_any_sync(vm, d);
      before = wcnt[warp * R + d];
    }
    __syncwarp();
    if (valid && lane == __ffs(peers) - 1) wcnt[warp * R + d] = (uint16_t)(before + __popc(peers));
    __syncwarp();
    val[r] = e;
    dig[r] = d;
    rk[r] = valid ? before + __popc(peers & lt) : -1;
  }
  __syncthreads();
  for (int d = tid; d < R; d += kRadixThreads) {
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < kRadixWarps; ++w) {
      const uint32_t c = wcnt[w * R + d];
      wcnt[w * R + d] = (uint16_t)run;
      run += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kRadixItems; ++r) {
    if (rk[r] >= 0) {
      const uint32_t d = dig[r];
      vout[toff[d] + wcnt[warp * R + d] + rk[r]] = val[r];
    }
  }
}

// colptr[s] = q for every s in (key[q - 1], key[q]], with key[-1] = -1 and key[E] = N + 1, so
// every entry of colptr[0..N] is written exactly once.  Long runs of senders without edges are
// written by the whole warp.
__global__ void __launch_bounds__(kRadixThreads) k_colptr(int E, int N, const int32_t* __restrict__ src,
                                                          const int32_t* __restrict__ perm,
                                                          int32_t* __restrict__ colptr) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * kRadixWarps;
  for (int64_t base = ((int64_t)blockIdx.x * kRadixWarps + (threadIdx.x >> 5)) * 32; base <= E;
       base += warps * 32) {
    const int64_t q = base + lane;
    const bool valid = q <= E;
    int64_t lo = 0, hi = -1;
    if (valid) {
      const int64_t kq = q < E ? (int64_t)sender_key(src, __ldg(perm + q), N) : (int64_t)N + 1;
      const int64_t kp = q > 0 ? (int64_t)sender_key(src, __ldg(perm + q - 1), N) : -1;
      lo = kp + 1;
      hi = min(kq, (int64_t)N);
    }
    const bool wide = hi - lo + 1 > 32;
    if (!wide)
      for (int64_t s = lo; s <= hi; ++s) colptr[s] = (int32_t)q;
    unsigned wm = __ballot_sync(kAll, wide);
    while (wm) {
      const int L = __ffs(wm) - 1;
      wm &= wm - 1;
      const int64_t l2 = __shfl_sync(kAll, lo, L), h2 = __shfl_sync(kAll, hi, L);
      const int32_t q2 = (int32_t)__shfl_sync(kAll, q, L);
      for (int64_t s = l2 + lane; s <= h2; s += 32) colptr[s] = q2;
    }
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
                                 int32_t* scratch, cudaStream_t s) {
  const RadixPlan rp = radix_plan(N, E);
  int launches = 0;
  if (E > 0) {
    int32_t* vtmp = scratch;
    int32_t* hist = scratch + (rp.passes > 1 ? (int64_t)E : 0);
    int32_t* total = hist + (int64_t)rp.radix * rp.tiles;
    const size_t sm_hist = sizeof(int32_t) * (size_t)rp.radix;
    const size_t sm_scat = (sizeof(int32_t) + sizeof(uint16_t) * kRadixWarps) * (size_t)rp.radix;
    if (sm_scat > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(k_radix_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_scat);
      if (e != cudaSuccess) return e;
    }
    const int32_t* vin = nullptr;
    for (int p = 0; p < rp.passes; ++p) {
      // the last pass writes perm; earlier passes alternate so that no pass reads what it writes
      int32_t* vout = ((rp.passes - 1 - p) % 2 == 0) ? perm : vtmp;
      const int shift = p * rp.bits;
      k_radix_hist<<<(unsigned)rp.tiles, kRadixThreads, sm_hist, s>>>(E, N, src, vin, shift, rp.radix, (int)rp.tiles,
                                                                     hist);
      k_radix_scan<<<(unsigned)((rp.radix + kRadixWarps - 1) / kRadixWarps), kRadixThreads, 0, s>>>(
          rp.radix, (int)rp.tiles, hist, total);
      k_radix_scatter<<<(unsigned)rp.tiles, kRadixThreads, sm_scat, s>>>(E, N, src, vin, vout, shift, rp.radix,
                                                                        (int)rp.tiles, hist, total);
      launches += 3;
      vin = vout;
    }
  }
  k_colptr<<<grid_for((int64_t)E + 1, kRadixThreads), kRadixThreads, 0, s>>>(E, N, src, perm, colptr);
  count_launches(launches + 1);
  return cudaGetLastError();
}

}  // namespace tp
