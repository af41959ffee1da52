// tp_check_bounded_waits: runs the two wait primitives every pipelined kernel of the
// library is built on -- the copy-engine slot wait of the staged edge passes and the
// mbarrier wait with abort flag of the tensor-core GEMM -- against an mbarrier that nothing
// ever signals, with a caller-given limit, and reports which of them gave up.  Both must:
// a kernel whose producer never delivers ends with an error status instead of hanging.
#include "../../include/tp.h"
#include "tp_kernels.cuh"
#include "tp_mma.cuh"

namespace {

__device__ int g_selftest_result;

__global__ void k_check_bounded_waits(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tp::sm_addr(&bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_flag = 0;
  }
  __syncthreads();
  // nothing arrives on `bar`: phase 0 never completes
  const bool slot_ok = tp::slot_wait(tp::sm_addr(&bar), 0u, limit_ns);
  const bool mbar_ok = tp::mbar_wait(tp::sm_addr(&bar), 0u, &abort_flag, limit_ns);
  __syncthreads();
  if (threadIdx.x == 0) g_selftest_result = (slot_ok ? 0 : 1) | (mbar_ok ? 0 : 2) | (abort_flag ? 4 : 0);
}

}  // namespace

extern "C" tp_status_t tp_check_bounded_waits(int64_t limit_ns, tp_stream_t stream, int32_t* gave_up) {
  if (!gave_up || limit_ns <= 0 || limit_ns > 1000000000ll) return TP_ERR_INVALID_ARG;
  *gave_up = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  k_check_bounded_waits<<<1, 32, 0, s>>>((unsigned long long)limit_ns);
  tp::count_launches(1);
  int v = 0;
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbolAsync(&v, g_selftest_result, sizeof(int), 0, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return TP_ERR_CUDA;
  *gave_up = v;
  return TP_OK;
}
