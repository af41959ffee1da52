// Dense fp32 contraction on the 5th-generation tensor cores (tcgen05, accumulator in TMEM),
// used only for the uvw multiplicity mixing.  fp32 accuracy comes from 3xTF32 operand
// splitting: a = a_hi + a_lo with a_hi = a truncated to TF32 (exact) and a_lo = a - a_hi
// (exact in fp32), and D = A_hi B_hi + A_hi B_lo + A_lo B_hi accumulated in fp32 (the
// dropped A_lo B_lo term is ~2^-20 relative).  Published as "3xTF32" split-precision GEMM
// (e.g. Ootomo & Yokota, 2022).
//
// CTA tile: M = 128 rows, N = 128 columns, K in blocks of 32 fp32 (one 128-byte swizzle
// row).  All 128 threads stage operand blocks (global -> registers -> hi/lo split -> shared
// memory in the canonical K-major 128B-swizzled layout); one elected thread issues the
// tcgen05.mma instructions (kind::tf32, M128 N128 K8) and commits them to an mbarrier; two
// stages let the staging of block k+1 overlap the MMAs of block k.  The epilogue moves the
// accumulator TMEM -> registers (tcgen05.ld 32x32b) -> shared memory, and the operation
// functor writes it out with coalesced stores.  Every wait is bounded: on timeout the CTA
// records TP device error 6, stops issuing work and releases its TMEM.
#pragma once
#include <cstdint>

#include "tp_common.h"

namespace tp {

constexpr int TC_BM = 128, TC_BN = 128, TC_BK = 32;
constexpr int TC_TILE_BYTES = TC_BM * TC_BK * 4;           // 16 KB: one 128 x 32 fp32 operand block
constexpr int TC_STAGE_BYTES = 4 * TC_TILE_BYTES;          // A_hi, A_lo, B_hi, B_lo
constexpr int TC_STAGES = 2;
constexpr int TC_EPI_LD = TC_BN + 1;                       // padded row of the staged accumulator
constexpr int TC_SMEM_BYTES = TC_STAGES * TC_STAGE_BYTES + 1024;   // + alignment slack
constexpr int kDevTimeout = 6;
constexpr long long kWaitPolls = 1ll << 26;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Canonical K-major, 128B-swizzled operand descriptor (sm_100 smem matrix descriptor):
// start address >> 4 in bits [0,14), leading byte offset (unused for swizzled K-major, 1)
// in [16,30), stride byte offset 1024 B >> 4 between 8-row groups in [32,46), version 1 in
// [46,48), layout type SWIZZLE_128B (2) in [61,64).
__device__ __forceinline__ uint64_t kmajor_sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFF) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: D f32 (bits 4-5 = 1), A and B tf32 (bits 7-9, 10-12 = 2), both
// K-major, N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t kIdescTf32 = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(TC_BN >> 3) << 17) |
                                ((uint32_t)(TC_BM >> 4) << 24);

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kIdescTf32), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
               : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t mbar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(mbar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait; false after kWaitPolls unsuccessful polls.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
  for (long long it = 0; it < kWaitPolls; ++it)
    if (mbar_try_wait(mbar, parity)) return true;
  return false;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ float tf32_hi(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u); }

// Byte offset of element (row, k) inside a 128 x 32 fp32 K-major SW128 block: row r is 128
// bytes, its 16-byte chunk c is stored at chunk c ^ (r & 7).
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Stages four consecutive k of one row (hi and lo parts) into a block pair.
__device__ __forceinline__ void stage4(char* hi_blk, char* lo_blk, int row, int chunk, float4 v) {
  float4 h = make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
  float4 l = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
  const uint32_t off = sw128_off(row, chunk);
  *reinterpret_cast<float4*>(hi_blk + off) = h;
  *reinterpret_cast<float4*>(lo_blk + off) = l;
}

// Operand addressing.  Element (r, k) of an operand lives at
//   base[row(r) + kpart(k)],  kpart(k) = (k / kd) * ks1 + (k % kd) * ks2   (kd = 0: k * ks1)
// row(r) is any per-row offset (computed once per row and K block); the k part is affine or
// splits k into (outer, inner) with a small inner extent, which covers every uvw layout.
struct TcOperand {
  const float* base;
  int kd;              // 0: plain stride ks1; else k = (k / kd, k % kd)
  int64_t ks1, ks2;
  bool vec4;           // rows are k-contiguous and 16-byte aligned: load 4 k at once
  __device__ __forceinline__ int64_t kpart(int64_t k) const {
    if (kd == 0) return k * ks1;
    const int64_t q = k / kd;
    return q * ks1 + (k - q * kd) * ks2;
  }
};

// Op interface:
//   int64_t M, Nn; void k_range(a, z, &k0, &k1)
//   TcOperand A, B (set on the host);  static constexpr bool A_KCONTIG, B_KCONTIG (thread mapping)
//   __device__ int64_t a_row(a, m), b_row(a, n)   (offset of row m of A / row n of B)
//   __device__ void store_tile(a, z, const float* T, int ld, int64_t m0, int n0)
// A thread of the CTA stages a fixed (row, chunk) set of a 128 x 32 block: with k-contiguous
// operands consecutive threads walk along k, otherwise along rows (coalesced either way).
template <class Op, bool IS_A>
struct TcStager {
  static constexpr bool KC = IS_A ? Op::A_KCONTIG : Op::B_KCONTIG;
  static constexpr int NIT = (TC_BM * TC_BK / 4) / 128;   // 8 chunks of 4 per thread
  float4 v[NIT];
  __device__ __forceinline__ static void slot(int it, int& row, int& chunk) {
    const int q = threadIdx.x + 128 * it;
    if (KC) {
      row = q >> 3;
      chunk = q & 7;
    } else {
      row = q & 127;
      chunk = q >> 7;
    }
  }
  __device__ __forceinline__ void load(const LaunchArgs& a, const Op& op, int64_t r0, int64_t rows, int64_t k0,
                                       int64_t k1) {
    const TcOperand& od = IS_A ? op.A : op.B;
#pragma unroll
    for (int it = 0; it < NIT; ++it) {
      int row, chunk;
      slot(it, row, chunk);
      const int64_t r = r0 + row, k = k0 + 4 * chunk;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < rows && k < k1) {
        const float* p = od.base + (IS_A ? op.a_row(a, r) : op.b_row(a, r));
        if (od.vec4 && k + 3 < k1) {
          x = *reinterpret_cast<const float4*>(p + k);
        } else {
          float e[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) e[j] = (k + j < k1) ? __ldg(p + od.kpart(k + j)) : 0.f;
          x = make_float4(e[0], e[1], e[2], e[3]);
        }
      }
      v[it] = x;
    }
  }
  __device__ __forceinline__ void store(char* hi, char* lo) const {
#pragma unroll
    for (int it = 0; it < NIT; ++it) {
      int row, chunk;
      slot(it, row, chunk);
      stage4(hi, lo, row, chunk, v[it]);
    }
  }
};

template <class Op>
__global__ void __launch_bounds__(128, 1) k_gemm_tc(const __grid_constant__ LaunchArgs a, const __grid_constant__ Op op) {
  extern __shared__ __align__(1024) char tc_smem_raw[];
  __shared__ uint64_t mbar[TC_STAGES];
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = (int64_t)blockIdx.x * TC_BM;
  const int n0 = blockIdx.y * TC_BN;
  int64_t k_begin, k_end;
  op.k_range(a, blockIdx.z, k_begin, k_end);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_holder)),
                 "r"(TC_BN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    for (int s = 0; s < TC_STAGES; ++s) mbar_init(smem_u32(&mbar[s]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_flag = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;

  const int nkb = (int)((k_end - k_begin + TC_BK - 1) / TC_BK);
  TcStager<Op, true> sa;
  TcStager<Op, false> sb;
  if (nkb > 0) {
    sa.load(a, op, m0, op.M, k_begin, k_end);
    sb.load(a, op, n0, op.Nn, k_begin, k_end);
  }
  for (int kb = 0; kb < nkb; ++kb) {
    const int s = kb % TC_STAGES;
    char* st = smem + s * TC_STAGE_BYTES;
    if (kb >= TC_STAGES) {   // the MMAs that read this stage (block kb - TC_STAGES) must be done
      const uint32_t parity = (uint32_t)((kb / TC_STAGES - 1) & 1);
      if (!mbar_wait(smem_u32(&mbar[s]), parity)) atomicExch(&abort_flag, 1);
    }
    __syncthreads();
    if (abort_flag) break;
    sa.store(st, st + TC_TILE_BYTES);
    sb.store(st + 2 * TC_TILE_BYTES, st + 3 * TC_TILE_BYTES);
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ah = smem_u32(st), al = ah + TC_TILE_BYTES;
      const uint32_t bh = ah + 2 * TC_TILE_BYTES, bl = ah + 3 * TC_TILE_BYTES;
#pragma unroll
      for (int ks = 0; ks < TC_BK / 8; ++ks) {      // K = 8 tf32 (32 bytes) per MMA
        const uint32_t kofs = ks * 32;
        const uint32_t acc0 = (kb > 0 || ks > 0) ? 1u : 0u;
        mma_tf32(tmem, kmajor_sw128_desc(ah + kofs), kmajor_sw128_desc(bh + kofs), acc0);
        mma_tf32(tmem, kmajor_sw128_desc(ah + kofs), kmajor_sw128_desc(bl + kofs), 1u);
        mma_tf32(tmem, kmajor_sw128_desc(al + kofs), kmajor_sw128_desc(bh + kofs), 1u);
      }
      mma_commit(smem_u32(&mbar[s]));
    }
    // global loads of the next block are in flight while the tensor cores work on this one
    if (kb + 1 < nkb) {
      const int64_t k0 = k_begin + (int64_t)(kb + 1) * TC_BK;
      sa.load(a, op, m0, op.M, k0, k_end);
      sb.load(a, op, n0, op.Nn, k0, k_end);
    }
  }
  // wait for the last committed group of each stage
  if (!abort_flag && nkb > 0) {
    const int last = nkb - 1;
    if (!mbar_wait(smem_u32(&mbar[last % TC_STAGES]), (uint32_t)((last / TC_STAGES) & 1))) atomicExch(&abort_flag, 1);
    if (nkb > 1) {
      const int prev = nkb - 2;
      if (!mbar_wait(smem_u32(&mbar[prev % TC_STAGES]), (uint32_t)((prev / TC_STAGES) & 1)))
        atomicExch(&abort_flag, 1);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (abort_flag) {
    if (tid == 0 && a.err) atomicCAS(a.err, 0, kDevTimeout);
  } else {
    // TMEM -> registers -> shared staging tile (fp32, padded rows), then the op's stores
    float* T = reinterpret_cast<float*>(smem);
    const int row = warp * 32 + lane;
#pragma unroll 1
    for (int c0 = 0; c0 < TC_BN; c0 += 32) {
      float v[32];
      if (nkb > 0) {
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) T[row * TC_EPI_LD + c0 + i] = v[i];
    }
    tc_fence_before();
    __syncthreads();
    op.store_tile(a, blockIdx.z, T, TC_EPI_LD, m0, n0);
  }
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TC_BN));
}

template <class Op>
cudaError_t launch_gemm_tc(const LaunchArgs& a, const Op& op, int splits, cudaStream_t s) {
  const int64_t M = op.M;
  const int Nn = (int)op.Nn;
  if (M <= 0 || Nn <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<Op>, cudaFuncAttributeMaxDynamicSharedMemorySize, TC_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((M + TC_BM - 1) / TC_BM), (unsigned)((Nn + TC_BN - 1) / TC_BN), (unsigned)splits);
  k_gemm_tc<Op><<<grid, 128, TC_SMEM_BYTES, s>>>(a, op);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace tp
