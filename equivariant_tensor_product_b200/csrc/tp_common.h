// Shared host/device declarations of the tensor-product convolution library (internal).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace tp {

constexpr int kMaxPaths = 64;
constexpr int kMaxBlocks = 16;
constexpr int kMaxThreads = 128;   // launch bound of every edge kernel

// Device error codes written to the workspace error word (debug index checks).
enum DeviceError : int {
  kDevOk = 0,
  kDevBadRowptr = 1,
  kDevBadSrc = 2,
  kDevBadPerm = 3,
};

// Everything an edge kernel needs, passed by value as a kernel parameter.
struct LaunchArgs {
  int N;               // nodes
  int E;               // edges
  int mul;             // channels per irrep block (uniform), uvu: in == out
  int mul_out;         // uvw: output channels
  int in_dim, out_dim, nw, a_dim;
  int split;           // warps per node row that split its edges (1..4)
  int n_slices;        // 32-channel slices per row = ceil(mul / 32)
  int has_coeff;       // path coefficients differ from 1
  int check;           // bounds-check indices and report through *err
  const int32_t* rowptr;
  const int32_t* src;
  const int32_t* colptr;
  const int32_t* perm;
  const float* x;
  const float* vec;
  const float* w;       // uvu w[E, P, mul]; uvw s[E, P]
  const float* gy;
  const float* ggx;
  const float* ggw;
  const float* ggvec;
  const float* W;       // uvw: shared mixing matrices [P][mul][mul_out]
  float* A;             // uvw forward: per-path receiver state (workspace), S::store_uvw layout;
                        // uvw backward: x W per path and sender, S::load_xt layout
  float* G;             // uvw backward: sender state B (workspace), S::store_xt layout
  float* Wt;            // uvw: W regrouped for the GEMM B operands, TF32 hi and lo (workspace)
  float* xT;            // uvw backward: x per input irrep as [node][m1][u] rows (workspace)
  float* gW;            // uvw: gradient of W (output)
  float* part;          // uvw: split-K partials of gW (workspace)
  int splits;           // uvw: number of split-K partials
  float* y;             // fwd output / dbwd g_gy
  float* gx;
  float* gw;
  float* gvec;
  int* err;
  float coeff[kMaxPaths];
};

// Runtime path table: plans whose path list has no compiled specialisation run kernels that
// take this table by value and dispatch every path to the unrolled contractions of its
// (l1, l2, l3) triple (generic.cu).
constexpr int kGenMaxTasks = 256;

struct GenPath {
  int16_t l1, l2, l3, tid;   // degrees and the triple id of the generated contractions
  int32_t in_off;            // offset of the path's input block in a row of x (uvw: of x W)
  int32_t out_off;           // offset of its output block in a row of y
  int32_t mul;               // channels (uvu: of the path; uvw: output channels)
  int32_t w_off;             // uvu: first weight of the path in an edge's w row; uvw: path index
  int32_t in_block, out_block;
  float coeff;
};

struct GenTable {
  int n_paths, n_in, n_out, lmax_sh;
  int uvw;                   // uvw: path p reads the rows of x W_p (offset path[p].in_off in a row of
  int xt_dim;                // xt_dim floats), mul_in / mul_out uniform; W is [P][mul_in][mul_out]
  int mul_in, mul_out;
  int in_off[kMaxBlocks], in_mul[kMaxBlocks], in_l[kMaxBlocks];
  int out_off[kMaxBlocks], out_mul[kMaxBlocks], out_l[kMaxBlocks];
  int out_first[kMaxBlocks + 1], out_paths[kMaxPaths];   // paths into each output block, path order
  int in_first[kMaxBlocks + 1], in_paths[kMaxPaths];     // paths reading each input block
  int n_rtask, n_stask;                                  // receiver / sender tasks: (block, 32-channel slice)
  uint8_t rtask_block[kGenMaxTasks], rtask_slice[kGenMaxTasks];
  uint8_t stask_block[kGenMaxTasks], stask_slice[kGenMaxTasks];
  GenPath path[kMaxPaths];
};

// Id of the (l1, l2, l3) triple in the generated contractions, or -1.
int gen_triple_id(int l1, int l2, int l3);
cudaError_t launch_gen_fwd(const LaunchArgs& a, const GenTable& T, cudaStream_t s);
cudaError_t launch_gen_bwd(const LaunchArgs& a, const GenTable& T, cudaStream_t s);
cudaError_t launch_gen_dbwd(const LaunchArgs& a, const GenTable& T, bool recv, bool send, cudaStream_t s);
// uvw through the path table.  fwd: a.A = x W per path [N, xt_dim] (workspace).  bwd: a.A as
// in fwd, a.G = its gradient B [N, xt_dim], a.part = a.splits node-chunk partials of gW.
cudaError_t launch_gen_uvw_fwd(const LaunchArgs& a, const GenTable& T, cudaStream_t s);
cudaError_t launch_gen_uvw_bwd(const LaunchArgs& a, const GenTable& T, cudaStream_t s);

// Convolution with the radial projection fused in (radial.cu): the uvu weights are formed on
// chip as w[e, c] = sum_k h[e, k] W_r[k, c] from the radial network's last hidden layer h[E, H]
// and its output layer W_r[H, nw]; the table is the plan's path table (built for every uvu plan).
struct RadArgs {
  int N, E, H;               // H: hidden width, a multiple of 4, at most kRadMaxHidden
  int nw, nwp;               // weights per edge; row pitch of the shared-memory weight tiles
  int in_dim, out_dim;
  int check, splits;         // index checks; edge chunks of the gW_r partials
  int spec;                  // compiled whole path list of the plan: 2 = all paths of lmax 2, 3 = of lmax 3, 0 = none
  int mul;                   // its (uniform) multiplicity
  const int32_t* rowptr;
  const int32_t* src;
  const int32_t* colptr;
  const int32_t* perm;
  const float* x;
  const float* vec;
  const float* h;            // [E, H]
  const float* Wr;           // [H, nw]
  const float* gy;
  float* y;
  float* gx;
  float* gh;                 // [E, H]
  float* gvec;
  float* gWr;                // [H, nw]
  float* WrT;                // workspace: W_r transposed, [nw, H]
  float* part;               // workspace: gW_r partials, [splits, H, nw]
  int* err;
};
constexpr int kRadMaxHidden = 64;
// Edges per shared-memory chunk (4, 8, 16 or 32) and the bytes of dynamic shared memory of
// the forward (bwd = false) or sender pass (bwd = true); 0 edges when even 4 do not fit.
int rad_chunk(const RadArgs& a, bool bwd, size_t* smem_bytes);
int rad_splits(const GenTable& T, int64_t E);
cudaError_t launch_rad_fwd(const RadArgs& a, const GenTable& T, cudaStream_t s);
cudaError_t launch_rad_bwd(const RadArgs& a, const GenTable& T, cudaStream_t s);

// Number of kernels the library has launched in this process (diagnostics).
void count_launches(int n);

// Host-side launchers of one compiled specialisation.
typedef cudaError_t (*LaunchFn)(const LaunchArgs&, cudaStream_t);

struct SpecOps {
  const char* name;
  int n_in, in_ls[kMaxBlocks];
  int n_sh, sh_ls[kMaxBlocks];
  int n_out, out_ls[kMaxBlocks];
  int n_paths, paths[kMaxPaths][3];
  int IN_PC, OUT_PC, NSH, P, A_PC, XT_PC;
  LaunchFn fwd_uvu;         // y = conv(x)
  LaunchFn bwd_uvu;         // gx, gw (gvec when args.gvec != nullptr), sender order
  LaunchFn dbwd_recv;       // g_gy, receiver order
  LaunchFn dbwd_send;       // g_x, g_w, g_vec, sender order
  LaunchFn uvw_fwd;         // edge pass into A, then y = mix(A, W)
  LaunchFn uvw_bwd;         // x W, the sender pass for B, gs, gvec, then gx = B W^T, gW = x^T B
};

extern const SpecOps* const kRegistry[];
extern const int kRegistrySize;

// CSR helpers (csr.cu)
cudaError_t launch_csr_validate(int N, int E, const int32_t* rowptr, const int32_t* src, int* err,
                                cudaStream_t s);

// The transpose is a radix sort of edge ids keyed by sender (keys 0..N, N = invalid sender):
// tiles of kRadixTile edges, passes of at most kRadixMaxBits-bit digits.
constexpr int kRadixItems = 8;                         // items per thread of a tile
constexpr int kRadixTile = 256 * kRadixItems;          // 2,048 edges per CTA
constexpr int kRadixMaxBits = 11;
constexpr int kRadixMaxDigits = 1 << kRadixMaxBits;

struct RadixPlan {
  int passes, bits, radix;   // passes of `bits`-bit digits, radix = 2^bits buckets
  int64_t tiles;
};

constexpr RadixPlan radix_plan(int64_t N, int64_t E) {
  int key_bits = 1;                                    // keys lie in [0, N]
  while (key_bits < 32 && ((int64_t)1 << key_bits) <= N) ++key_bits;
  const int passes = (key_bits + kRadixMaxBits - 1) / kRadixMaxBits;
  const int bits = (key_bits + passes - 1) / passes;
  return RadixPlan{passes, bits, 1 << bits, (E + kRadixTile - 1) / kRadixTile};
}

// int32 scratch of one transpose: a second id buffer when there is more than one pass, and
// the per-digit, per-tile counts followed by the digit totals.
constexpr int64_t transpose_scratch_ints(int64_t N, int64_t E) {
  const RadixPlan p = radix_plan(N, E);
  return (p.passes > 1 ? E : 0) + (int64_t)p.radix * (p.tiles + 1);
}

// colptr[N+1] and perm[E] of the stable receiver->sender transpose; scratch holds
// transpose_scratch_ints(N, E) int32.
cudaError_t launch_csr_transpose(int N, int E, const int32_t* src, int32_t* colptr, int32_t* perm,
                                 int32_t* scratch, cudaStream_t s);

}  // namespace tp
