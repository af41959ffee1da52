// Dense fp32 contraction on the 5th-generation tensor cores (tcgen05, accumulator in TMEM),
// used only for the uvw multiplicity mixing.  fp32 accuracy comes from 3xTF32 operand
// splitting: a = a_hi + a_lo with a_hi = a truncated to TF32 (exact) and a_lo = a - a_hi
// (exact in fp32), and D = A_hi B_hi + A_hi B_lo + A_lo B_hi accumulated in fp32 (the
// dropped A_lo B_lo term is ~2^-20 relative).  Published as "3xTF32" split-precision GEMM
// (e.g. Ootomo & Yokota, 2022).
//
// CTA tile: M = 128 rows, N = 128 columns, K in blocks of 32 fp32 (one 128-byte swizzle
// row).  Persistent and warp-specialised: one CTA per SM walks a static list of tiles with
// 320 threads:
//   warp 0     one lane issues the TMA loads of every K block of every tile into a ring of
//              stages;
//   warp 1     owns two TMEM accumulators (256 columns); one lane issues tcgen05.mma
//              (kind::tf32, M128 N128 K8, three per K step for the split) into them in turn
//              and commits each stage back to the producer and each finished accumulator
//              to the epilogue;
//   warps 2-5  split the raw fp32 operand tiles into TF32 hi/lo tiles in the canonical
//              K-major 128B-swizzled layout (transposing tiles that arrive M/N-major);
//   warps 6-9  epilogue: tcgen05.ld 32x32b -> registers -> a 128 x 32 shared tile -> the
//              op's stores, while the MMAs of the next tile run on the other accumulator.
// Operands come in one of three forms (per op, at compile time):
//   FMT_K      [rows][K] fp32, K contiguous: TMA with the 128B swizzle lands the tile in the
//              MMA layout; the split rewrites it in place (hi) and writes lo beside it;
//   FMT_MN     [K][rows] fp32, rows contiguous: TMA lands a plain 32 x 128 tile, the split
//              transposes it;
//   FMT_SPLIT  two K-major arrays already split into hi and lo (the shared weights, split
//              once per call): TMA straight into the MMA tiles, no conversion.
// The tensor-core accumulator does not round to nearest, so its error grows with the number
// of MMAs summed into it.  Ops with a deep K (the split-K gW GEMM) set PROMOTE = R: every R K
// blocks the epilogue warps add the TMEM accumulator into fp32 registers (round to nearest)
// and the MMAs restart from zero, which bounds that growth at R blocks.
// Every wait is bounded: on timeout the CTA records TP device error 6, the other roles see
// the abort flag and stop, loads and MMAs already issued are waited for (again bounded) and
// the TMEM is released.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "tp_common.h"

namespace tp {

constexpr int TC_BM = 128, TC_BN = 128, TC_BK = 32;
constexpr int TC_TILE_BYTES = TC_BM * TC_BK * 4;           // 16 KB: one 128 x 32 fp32 operand block
constexpr int TC_SMEM_BUDGET = 196608;                     // ring of stages (192 KB)
constexpr int TC_EPI_COLS = 32;                            // epilogue sub-tile: 128 rows x 32 columns
constexpr int TC_EPI_LD = TC_EPI_COLS + 1;                 // padded row of the staged sub-tile
constexpr int TC_EPI_BYTES = (TC_BM * TC_EPI_LD * 4 + 1023) / 1024 * 1024;
constexpr int TC_THREADS = 320;
constexpr int kDevTimeout = 6;
constexpr unsigned long long kWaitNs = 4000000000ull;   // a wait gives up after 4 s

enum TcFmt { FMT_K = 0, FMT_MN = 1, FMT_SPLIT = 2 };

__host__ __device__ constexpr int tc_operand_bytes(int fmt) {
  return fmt == FMT_MN ? 3 * TC_TILE_BYTES : 2 * TC_TILE_BYTES;   // (raw +) hi + lo
}
__host__ __device__ constexpr int tc_load_bytes(int fmt) {
  return fmt == FMT_SPLIT ? 2 * TC_TILE_BYTES : TC_TILE_BYTES;
}
template <class Op>
struct TcShape {
  static constexpr int A_BYTES = tc_operand_bytes(Op::A_FMT);
  static constexpr int STAGE_BYTES = A_BYTES + tc_operand_bytes(Op::B_FMT);
  static constexpr int STAGES = TC_SMEM_BUDGET / STAGE_BYTES > 4 ? 4 : TC_SMEM_BUDGET / STAGE_BYTES;
  static constexpr uint32_t TX_BYTES = tc_load_bytes(Op::A_FMT) + tc_load_bytes(Op::B_FMT);
  static constexpr int SMEM = STAGES * STAGE_BYTES + TC_EPI_BYTES + 1024;   // + alignment slack
  static_assert(STAGES >= 2, "ring needs two stages");
};

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

__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
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

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait bounded in time (a try_wait may suspend the thread for a while, so the bound is on
// the clock, not on the number of polls) that also gives up when another role has aborted.
// On its own timeout it raises the abort flag.  Returns false when the caller must stop.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit_ns = kWaitNs) {
  if (mbar_try_wait(mbar, parity)) return true;   // the common case reads no clock
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(mbar, parity)) return true;
    if (*abort_flag) return false;
    if (global_ns() - t0 > limit_ns) break;
  }
  *abort_flag = 1;
  return false;
}

// Time-bounded wait that ignores the abort flag: used to drain work already issued.
__device__ __forceinline__ void mbar_drain(uint32_t mbar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(mbar, parity))
    if (global_ns() - t0 > kWaitNs) return;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t mbar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(mbar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Tile t of the static schedule -> (m block, n block, split); n runs fastest so that the
// CTAs working at the same time share their A tile through L2.
struct TcTile {
  int64_t m0;
  int n0, z;
};
__device__ __forceinline__ TcTile tc_tile(int64_t t, int64_t mtiles, int ntiles) {
  const int64_t per_z = mtiles * ntiles;
  TcTile r;
  r.z = (int)(t / per_z);
  const int64_t rem = t - (int64_t)r.z * per_z;
  r.m0 = (rem / ntiles) * TC_BM;
  r.n0 = (int)(rem % ntiles) * TC_BN;
  return r;
}

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

// Split of one operand tile of a stage by converter thread ct (of 128).
template <int FMT>
__device__ __forceinline__ void tc_split(char* op_base, int ct) {
  if constexpr (FMT == FMT_K) {
    // the raw tile is already in the swizzled layout at op_base (it becomes hi); lo follows
    char* lo = op_base + TC_TILE_BYTES;
#pragma unroll
    for (int i = 0; i < TC_TILE_BYTES / 16 / 128; ++i) {
      const uint32_t off = (uint32_t)(ct + 128 * i) * 16u;
      const float4 v = *reinterpret_cast<const float4*>(op_base + off);
      const float4 h = make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
      *reinterpret_cast<float4*>(op_base + off) = h;
      *reinterpret_cast<float4*>(lo + off) = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
    }
  } else if constexpr (FMT == FMT_MN) {
    // raw [32 k][128 rows] at op_base; the hi and lo K-major swizzled tiles follow it
    const float* raw = reinterpret_cast<const float*>(op_base);
    char* hi = op_base + TC_TILE_BYTES;
    char* lo = op_base + 2 * TC_TILE_BYTES;
    const int r = ct;
#pragma unroll
    for (int c = 0; c < TC_BK / 4; ++c) {
      const float4 v = make_float4(raw[(4 * c + 0) * TC_BM + r], raw[(4 * c + 1) * TC_BM + r],
                                   raw[(4 * c + 2) * TC_BM + r], raw[(4 * c + 3) * TC_BM + r]);
      const float4 h = make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
      const uint32_t off = sw128_off(r, c);
      *reinterpret_cast<float4*>(hi + off) = h;
      *reinterpret_cast<float4*>(lo + off) = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
    }
  }
}

// Shared-memory address of the hi MMA tile of an operand in a stage (lo follows it).
template <int FMT>
__device__ __forceinline__ uint32_t tc_hi(uint32_t op_base) {
  return FMT == FMT_MN ? op_base + TC_TILE_BYTES : op_base;
}

// Issues the TMA load(s) of one K block of an operand.  FMT_K / FMT_SPLIT maps are
// (K inner, rows) with box (32, 128); FMT_MN maps are (rows inner, K) with box (128, 32).
template <int FMT>
__device__ __forceinline__ void tc_load(uint32_t op_base, const CUtensorMap* m0, const CUtensorMap* m1,
                                        uint32_t mbar, int k0, int r0) {
  if constexpr (FMT == FMT_K) {
    tma_load_2d(op_base, m0, mbar, k0, r0);
  } else if constexpr (FMT == FMT_MN) {
    tma_load_2d(op_base, m0, mbar, r0, k0);
  } else {
    tma_load_2d(op_base, m0, mbar, k0, r0);
    tma_load_2d(op_base + TC_TILE_BYTES, m1, mbar, k0, r0);
  }
}

// Op interface:
//   int64_t M, Nn;  static constexpr int A_FMT, B_FMT, PROMOTE (0: off, else chunk of K blocks);
//   CUtensorMap tA, tA2, tB, tB2   (tA2 / tB2 used only by FMT_SPLIT: the lo array)
//   __device__ void k_range(a, z, &k0, &k1)   (k0 a multiple of 32)
//   __device__ void store_tile(a, z, const float* T, int ld, int64_t r0, int rows, int n0, int cols, int lane)
//     stores, with the 32 lanes of one warp, the rows x cols block T (row stride ld) whose
//     first element is at global row r0 and global column n0.
template <class Op>
__global__ void __launch_bounds__(TC_THREADS, 1) k_gemm_tc(const __grid_constant__ LaunchArgs a,
                                                           const __grid_constant__ Op op, int splits) {
  using SH = TcShape<Op>;
  constexpr int ST = SH::STAGES;
  constexpr int R = Op::PROMOTE;
  extern __shared__ __align__(1024) char tc_smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[ST];
  __shared__ __align__(8) uint64_t conv_bar[ST];
  __shared__ __align__(8) uint64_t empty_bar[ST];
  __shared__ __align__(8) uint64_t accf_bar[2];
  __shared__ __align__(8) uint64_t acce_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_holder;
  __shared__ volatile int abort_flag;
  // aligned by an offset from the shared array itself, so that the compiler keeps the accesses
  // in the shared window (a round trip through an integer would make them generic)
  char* smem = tc_smem_raw + ((1024u - (smem_u32(tc_smem_raw) & 1023u)) & 1023u);
  float* T = reinterpret_cast<float*>(smem + ST * SH::STAGE_BYTES);
  const uint32_t smem_s = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t mtiles = (op.M + TC_BM - 1) / TC_BM;
  const int ntiles = (int)((op.Nn + TC_BN - 1) / TC_BN);
  const int64_t tiles = mtiles * ntiles * splits;
  // K blocks of the tile and its accumulation segments (R K blocks each when promoting)
  auto tile_kb = [&](const TcTile& tt, int64_t& kb0) {
    int64_t k0, k1;
    op.k_range(a, tt.z, k0, k1);
    kb0 = k0;
    return k1 > k0 ? (int)((k1 - k0 + TC_BK - 1) / TC_BK) : 0;
  };

  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_holder)),
                 "r"(2 * TC_BN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&conv_bar[s]), 128);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&accf_bar[b]), 1);
      mbar_init(smem_u32(&acce_bar[b]), 128);
    }
    mbar_init(smem_u32(&drain_bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_flag = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int64_t q = 0;   // position in the ring over all tiles
      for (int64_t t = blockIdx.x; t < tiles && !abort_flag; t += gridDim.x) {
        const TcTile tt = tc_tile(t, mtiles, ntiles);
        int64_t kb0;
        const int nkb = tile_kb(tt, kb0);
        for (int kb = 0; kb < nkb; ++kb, ++q) {
          const int s = (int)(q % ST);
          if (q >= ST && !mbar_wait(smem_u32(&empty_bar[s]), (uint32_t)((q / ST - 1) & 1), &abort_flag)) break;
          const uint32_t st = smem_s + (uint32_t)(s * SH::STAGE_BYTES);
          const uint32_t fb = smem_u32(&full_bar[s]);
          mbar_expect_tx(fb, SH::TX_BYTES);
          const int k0 = (int)(kb0 + (int64_t)kb * TC_BK);
          tc_load<Op::A_FMT>(st, &op.tA, &op.tA2, fb, k0, (int)tt.m0);
          tc_load<Op::B_FMT>(st + SH::A_BYTES, &op.tB, &op.tB2, fb, k0, tt.n0);
        }
      }
      if (abort_flag) {   // let the loads already issued land before the CTA exits
        for (int64_t u = q > ST ? q - ST : 0; u < q; ++u)
          mbar_drain(smem_u32(&full_bar[u % ST]), (uint32_t)((u / ST) & 1));
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int64_t q = 0, g = 0;   // ring position, accumulation segment
      bool issued = false;
      for (int64_t t = blockIdx.x; t < tiles && !abort_flag; t += gridDim.x) {
        const TcTile tt = tc_tile(t, mtiles, ntiles);
        int64_t kb0;
        const int nkb = tile_kb(tt, kb0);
        for (int kb = 0; kb < nkb; ++kb, ++q) {
          const int kc = R > 0 ? kb % R : kb;   // position inside the segment
          const int b = (int)(g & 1);
          if (kc == 0 && g >= 2 &&
              !mbar_wait(smem_u32(&acce_bar[b]), (uint32_t)(((g >> 1) - 1) & 1), &abort_flag))
            break;
          const int s = (int)(q % ST);
          if (!mbar_wait(smem_u32(&conv_bar[s]), (uint32_t)((q / ST) & 1), &abort_flag)) break;
          tc_fence_after();
          const uint32_t st = smem_s + (uint32_t)(s * SH::STAGE_BYTES);
          const uint32_t ah = tc_hi<Op::A_FMT>(st), al = ah + TC_TILE_BYTES;
          const uint32_t bh = tc_hi<Op::B_FMT>(st + SH::A_BYTES), bl = bh + TC_TILE_BYTES;
          const uint32_t acc = tmem + (uint32_t)(b * TC_BN);
          for (int ks = 0; ks < TC_BK / 8; ++ks) {   // K = 8 tf32 (32 bytes) per MMA
            const uint32_t kofs = ks * 32;
            const uint32_t acc0 = (kc > 0 || ks > 0) ? 1u : 0u;
            mma_tf32(acc, kmajor_sw128_desc(ah + kofs), kmajor_sw128_desc(bh + kofs), acc0);
            mma_tf32(acc, kmajor_sw128_desc(ah + kofs), kmajor_sw128_desc(bl + kofs), 1u);
            mma_tf32(acc, kmajor_sw128_desc(al + kofs), kmajor_sw128_desc(bh + kofs), 1u);
          }
          issued = true;
          mma_commit(smem_u32(&empty_bar[s]));
          if ((R > 0 && kc == R - 1) || kb == nkb - 1) {   // end of a segment
            mma_commit(smem_u32(&accf_bar[b]));
            ++g;
          }
        }
      }
      if (abort_flag && issued) {   // every MMA issued above must finish before TMEM is freed
        mma_commit(smem_u32(&drain_bar));
        mbar_drain(smem_u32(&drain_bar), 0u);
      }
    }
  } else if (warp < 6) {
    // ---------------- split (warps 2-5) ----------------
    const int ct = tid - 64;
    int64_t q = 0;
    for (int64_t t = blockIdx.x; t < tiles && !abort_flag; t += gridDim.x) {
      const TcTile tt = tc_tile(t, mtiles, ntiles);
      int64_t kb0;
      const int nkb = tile_kb(tt, kb0);
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb, ++q) {
        const int s = (int)(q % ST);
        if (!mbar_wait(smem_u32(&full_bar[s]), (uint32_t)((q / ST) & 1), &abort_flag)) {
          ok = false;
          break;
        }
        char* st = smem + s * SH::STAGE_BYTES;
        tc_split<Op::A_FMT>(st, ct);
        tc_split<Op::B_FMT>(st + SH::A_BYTES, ct);
        fence_async_smem();
        mbar_arrive(smem_u32(&conv_bar[s]));
      }
      if (!ok) break;
    }
  } else {
    // ---------------- epilogue (warps 6-9) ----------------
    // Each warp owns the 32 accumulator rows of its TMEM lane quarter (warp id % 4) and
    // stages and stores them on its own: no barrier spans warps, and every wait result is
    // made warp-uniform before the warp-collective TMEM loads.
    const int qd = warp & 3;
    float* Tw = T + qd * 32 * TC_EPI_LD;
    int64_t g = 0;
    for (int64_t t = blockIdx.x; t < tiles && !abort_flag; t += gridDim.x) {
      const TcTile tt = tc_tile(t, mtiles, ntiles);
      int64_t kb0;
      const int nkb = tile_kb(tt, kb0);
      const int nseg = nkb == 0 ? 0 : (R > 0 ? (nkb + R - 1) / R : 1);
      const int cols_all = (int)min((int64_t)TC_BN, op.Nn - tt.n0);
      const int64_t r0 = tt.m0 + qd * 32;
      bool ok = true;
      if constexpr (R > 0) {
        // segments add into fp32 registers (round to nearest)
        float acc[TC_BN];
#pragma unroll
        for (int i = 0; i < TC_BN; ++i) acc[i] = 0.f;
        for (int sg = 0; sg < nseg; ++sg, ++g) {
          const int b = (int)(g & 1);
          ok = __all_sync(kFull, mbar_wait(smem_u32(&accf_bar[b]), (uint32_t)((g >> 1) & 1), &abort_flag));
          if (!ok) break;
          tc_fence_after();
          const uint32_t tq = tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)(b * TC_BN);
#pragma unroll
          for (int c0 = 0; c0 < TC_BN; c0 += 32) {
            float v[32];
            tmem_ld32(tq + (uint32_t)c0, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[c0 + i] += v[i];
          }
          tc_fence_before();
          mbar_arrive(smem_u32(&acce_bar[b]));
        }
        if (!ok) break;
#pragma unroll
        for (int c0 = 0; c0 < TC_BN; c0 += TC_EPI_COLS) {
          if (c0 < cols_all) {
#pragma unroll
            for (int i = 0; i < TC_EPI_COLS; ++i) Tw[lane * TC_EPI_LD + i] = acc[c0 + i];
            __syncwarp();
            op.store_tile(a, tt.z, Tw, TC_EPI_LD, r0, 32, tt.n0 + c0, min(TC_EPI_COLS, cols_all - c0), lane);
            __syncwarp();
          }
        }
      } else {
        const int b = (int)(g & 1);
        if (nseg > 0) {
          ok = __all_sync(kFull, mbar_wait(smem_u32(&accf_bar[b]), (uint32_t)((g >> 1) & 1), &abort_flag));
          if (!ok) break;
        }
        tc_fence_after();
        const uint32_t tq = tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)(b * TC_BN);
#pragma unroll 1
        for (int c0 = 0; c0 < TC_BN; c0 += TC_EPI_COLS) {
          float v[32];
          if (nseg > 0) {
            tmem_ld32(tq + (uint32_t)c0, v);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
          }
          if (nseg > 0 && c0 + TC_EPI_COLS == TC_BN) {   // accumulator fully read: hand it back
            tc_fence_before();
            mbar_arrive(smem_u32(&acce_bar[b]));
          }
          if (c0 < cols_all) {
#pragma unroll
            for (int i = 0; i < TC_EPI_COLS; ++i) Tw[lane * TC_EPI_LD + i] = v[i];
            __syncwarp();
            op.store_tile(a, tt.z, Tw, TC_EPI_LD, r0, 32, tt.n0 + c0, min(TC_EPI_COLS, cols_all - c0), lane);
            __syncwarp();
          }
        }
        g += nseg;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && abort_flag && a.err) atomicCAS(a.err, 0, kDevTimeout);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * TC_BN));
  }
}

// ---------------------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------------------
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D fp32 tensor map over `rows` rows of `inner` elements (row pitch `pitch` floats).
// FMT_K / FMT_SPLIT: box 32 (inner) x 128 rows with the 128-byte swizzle;
// FMT_MN:            box 128 (inner) x 32 rows, no swizzle.
// Box elements outside the tensor read as zero.  Needs a 16-byte aligned base and pitch.
inline cudaError_t make_tmap(CUtensorMap* m, const float* base, int64_t inner, int64_t rows, int64_t pitch,
                             int fmt) {
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  if ((reinterpret_cast<uintptr_t>(base) & 15u) || (pitch * 4) % 16 != 0 || inner <= 0 || rows <= 0 ||
      pitch < inner)
    return cudaErrorInvalidValue;
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)pitch * 4};
  const cuuint32_t box_k[2] = {TC_BK, TC_BM};
  const cuuint32_t box_mn[2] = {TC_BM, TC_BK};
  const cuuint32_t estr[2] = {1, 1};
  const bool mn = fmt == FMT_MN;
  const CUresult r =
      enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, mn ? box_mn : box_k, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, mn ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

inline int sm_count() {
  static int n = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  });
  return n;
}

template <class Op>
cudaError_t launch_gemm_tc(const LaunchArgs& a, const Op& op, int splits, cudaStream_t s) {
  const int64_t M = op.M;
  const int64_t Nn = op.Nn;
  if (M <= 0 || Nn <= 0 || splits <= 0) return cudaSuccess;
  constexpr int smem = TcShape<Op>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<Op>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((M + TC_BM - 1) / TC_BM) * ((Nn + TC_BN - 1) / TC_BN) * splits;
  const unsigned grid = (unsigned)std::min<int64_t>(tiles, sm_count());   // persistent: one CTA per SM
  k_gemm_tc<Op><<<grid, TC_THREADS, smem, s>>>(a, op, splits);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace tp
