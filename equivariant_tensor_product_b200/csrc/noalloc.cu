// tp_csr_transpose_noalloc: the stable receiver->sender transpose with its scratch memory
// held by the library itself, for callers that cannot allocate device memory.
//
// Some hosts of this library cannot hand it a workspace: an MD engine or plugin whose device
// memory belongs to a pool it does not control, a framework that has reserved (almost) all
// of the GPU up front so a fresh cudaMalloc would fail, or a loop that must not call
// cudaMalloc/cudaFree because those calls synchronise the device.  This entry point needs
// nothing from them beyond the inputs and outputs: the scratch that tp_csr_transpose takes
// from the caller's workspace (the radix sort's second id buffer and its per-tile digit
// counts) lives in one file-scope __device__ array instead.
//
// Costs and rules of that choice:
//   * every GPU that loads the library holds the array (kScratchInts int32, about 5.3 MB)
//     until the process exits;
//   * N <= kNoAllocMaxN and E <= kNoAllocMaxE, larger graphs are rejected
//     (TP_ERR_UNSUPPORTED) before any work is enqueued;
//   * all calls share the array: two calls whose work overlaps on the GPU (different
//     streams, or different host threads, without ordering between them) race and produce
//     wrong results; order them on one stream or synchronise between them;
//   * the array keeps whatever the last call left in it; every kernel of a call writes the
//     part it later reads (digit counts, scans, ids) before reading it, so nothing needs
//     clearing;
//   * the first call on each device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current; make that first call before any
//     stream capture.  The address is kept until exit: a cudaDeviceReset between calls is
//     not supported.
#include <mutex>

#include "../../include/tp.h"
#include "tp_common.h"

namespace {

constexpr int64_t kNoAllocMaxN = 1 << 17;   // 131,072 nodes
constexpr int64_t kNoAllocMaxE = 1 << 20;   // 1,048,576 edges

// The largest transpose scratch over every N <= kNoAllocMaxN at E = kNoAllocMaxE (the digit
// width, and so the count table, depends on the number of key bits of N).
constexpr int64_t max_scratch_ints() {
  int64_t best = tp::transpose_scratch_ints(kNoAllocMaxN, kNoAllocMaxE);
  for (int64_t n = 1; n < kNoAllocMaxN; n = 2 * n + 1) {
    const int64_t v = tp::transpose_scratch_ints(n, kNoAllocMaxE);
    if (v > best) best = v;
  }
  return best;
}
constexpr int64_t kScratchInts = max_scratch_ints();
constexpr int kMaxDevices = 64;

// The radix sort's scratch (see csr.cu): an id buffer and per-tile digit counts.
static __device__ __align__(256) int32_t g_transpose_scratch[kScratchInts];

std::mutex g_mu;
int32_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device (host code must not use the symbol
// itself: on the host it names a stand-in, not device memory).
cudaError_t scratch_for_current_device(int32_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_transpose_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" tp_status_t tp_csr_transpose_noalloc(int64_t N, int64_t E, const int32_t* rowptr,
                                                const int32_t* src, int32_t* colptr, int32_t* perm,
                                                tp_stream_t stream) {
  (void)rowptr;
  if (N < 0 || E < 0) return TP_ERR_INVALID_ARG;
  // graphs larger than the fixed array: use tp_csr_transpose with a caller workspace
  if (N > kNoAllocMaxN || E > kNoAllocMaxE) return TP_ERR_UNSUPPORTED;
  if (!colptr || (E > 0 && (!src || !perm))) return TP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(colptr) |
       reinterpret_cast<uintptr_t>(perm)) & 3u)
    return TP_ERR_INVALID_ARG;
  int32_t* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return TP_ERR_CUDA;
  if (tp::transpose_scratch_ints(N, E) > kScratchInts) return TP_ERR_UNSUPPORTED;
  if (tp::launch_csr_transpose((int)N, (int)E, src, colptr, perm, scratch, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return TP_ERR_CUDA;
  return TP_OK;
}
