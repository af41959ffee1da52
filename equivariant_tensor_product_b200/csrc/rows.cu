// Row movement for receiver-range sharding over several GPUs: the halo exchange of sender
// rows (gather before the send) and the return of halo gradients (add after the receive).
//
// A rank that owns a contiguous range of receiver rows needs, for its forward, the x rows of
// the senders of its edges that other ranks own (the halo), and after its backward sends
// the gradient partials of those halo senders back to their owners, who add them to their
// own rows ("Sobek", abstract: graphs a hundred times larger than fit before, by keeping
// the state bounded per device).  Both steps are plain row copies; the exchange between
// the steps is a collective of the caller (NCCL all-to-all over NVLink).
#include "../../include/tp.h"
#include "tp_common.h"

namespace tp {
namespace {

// dst[k, :] = src[idx[k], :], one warp per row, float4 when the row allows it
__global__ void k_gather_rows(const float* __restrict__ src, int64_t row_len, const int32_t* __restrict__ idx,
                              int64_t n, float* __restrict__ dst, int vec4) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t k = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); k < n; k += warps) {
    const int64_t r = __ldg(idx + k);
    if (vec4) {
      const float4* s = reinterpret_cast<const float4*>(src + r * row_len);
      float4* d = reinterpret_cast<float4*>(dst + k * row_len);
      for (int64_t c = lane; c < row_len / 4; c += 32) d[c] = __ldg(s + c);
    } else {
      for (int64_t c = lane; c < row_len; c += 32) dst[k * row_len + c] = __ldg(src + r * row_len + c);
    }
  }
}

// dst[idx[k], :] += src[k, :]; the indices of one call must be distinct (no two warps add to
// the same row), so the result does not depend on the schedule
__global__ void k_add_rows(float* __restrict__ dst, int64_t row_len, const int32_t* __restrict__ idx, int64_t n,
                           const float* __restrict__ src) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t k = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); k < n; k += warps) {
    const int64_t r = __ldg(idx + k);
    for (int64_t c = lane; c < row_len; c += 32) dst[r * row_len + c] += __ldg(src + k * row_len + c);
  }
}

unsigned rows_grid(int64_t n) {
  int64_t g = (n + 7) / 8;
  if (g > 148 * 16) g = 148 * 16;
  return (unsigned)(g < 1 ? 1 : g);
}

bool bad(int64_t n, int64_t row_len, const void* a, const void* b, const void* c) {
  if (n < 0 || row_len <= 0) return true;
  if (n > 0 && (!a || !b || !c)) return true;
  return ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b) | reinterpret_cast<uintptr_t>(c)) & 3u) != 0;
}

}  // namespace
}  // namespace tp

extern "C" {

tp_status_t tp_gather_rows(const float* src, int64_t row_len, const int32_t* idx, int64_t n, float* dst,
                           tp_stream_t stream) {
  if (tp::bad(n, row_len, src, idx, dst)) return TP_ERR_INVALID_ARG;
  if (n == 0) return TP_OK;
  const int vec4 = (row_len % 4 == 0) &&
                   ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u) == 0;
  tp::k_gather_rows<<<tp::rows_grid(n), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(src, row_len, idx, n, dst,
                                                                                          vec4);
  tp::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

tp_status_t tp_add_rows(float* dst, int64_t row_len, const int32_t* idx, int64_t n, const float* src,
                        tp_stream_t stream) {
  if (tp::bad(n, row_len, src, idx, dst)) return TP_ERR_INVALID_ARG;
  if (n == 0) return TP_OK;
  tp::k_add_rows<<<tp::rows_grid(n), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(dst, row_len, idx, n, src);
  tp::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

}  // extern "C"
