/*
 * tp.h -- C ABI of the B200 edge-conditioned E(3)-equivariant tensor-product convolution.
 *
 * The operation ("Sobek: Streaming Equivariant Tensor Product Convolutions", abstract;
 * "FlashTP: Fused, Sparsity-Aware Tensor Product for Machine Learning Interatomic
 * Potentials", abstract; "The GPU Workload That Rewrites Molecular Physics", section
 * "Equivariant feature transforms"): for every directed edge e = (j -> i) of a graph,
 * couple the sender features x[j] with the real spherical harmonics Y(v_e / |v_e|) of the
 * edge vector through the real Clebsch-Gordan tensor C_p of each path p = (in, sh, out),
 * scale by the edge's radial weights and sum into the receiver:
 *
 *   y[i, out(p), w, m3] = sum_{e into i} sum_p sum_{m1,m2} C_p[m1,m2,m3] Y_sh(p)(v_e)[m2] X_pe[w,m1]
 *     uvu mode: X_pe[u, m1] = c_p * w[e, p, u] * x[j, in(p), u, m1]
 *     uvw mode: X_pe[w, m1] = c_p * s[e, p] * sum_u W[p, u, w] * x[j, in(p), u, m1]
 *
 * tp_conv_bwd returns the vector-Jacobian product against gy; tp_conv_dbwd the VJP of the
 * backward map (x, vec, w, gy) -> (gx, gw, gvec) against (ggx, ggw, ggvec) ("Sobek",
 * abstract: forward, backward and double backward).
 *
 * Conventions.  Real spherical harmonics, m = -l..l, component normalisation
 * (sum_m Y_lm^2 = 2l+1, Y_0 = 1), no Condon-Shortley phase; l = 1 is sqrt(3)(y, z, x).  A
 * zero edge vector has Y_0 = 1, Y_{l>0} = 0 and zero derivatives.  Real CG tensors have
 * ||C||_F^2 = 2 l3 + 1 and a positive first non-zero entry in row-major (m1, m2, m3)
 * order.  l <= 3 everywhere.
 *
 * Layouts (all row-major, fp32 unless noted, device memory):
 *   x     [N, in_dim]   blocks in irreps order, inside a block [u][m] (m fastest)
 *   y     [N, out_dim]  same rule on the output irreps
 *   vec   [E, 3]        edge vector of edge e (any convention; the bench uses sender - receiver)
 *   w     [E, P, mul]   uvu radial weights, paths outer, channel inner
 *   s     [E, P]        uvw per-edge path scalars (passed as `w`)
 *   W     [P, mul_in, mul_out]  uvw shared mixing matrices (NULL in uvu)
 *   rowptr[N+1], src[E] int32: receiver-sorted CSR, edges of receiver i are
 *                       rowptr[i] .. rowptr[i+1]-1 and src[e] is their sender
 *   colptr[N+1], perm[E] int32: sender-sorted transpose, perm = stable argsort(src)
 *
 * Ownership.  The caller owns every buffer, including the workspace (size it with
 * tp_workspace_size).  The library owns only the plan (host memory).  Inputs are read
 * only; outputs are fully overwritten, never accumulated.
 *
 * Streams.  Every call only enqueues work on `stream` and returns; nothing synchronises
 * except tp_get_device_error.
 *
 * Errors.  Host-side checks (null pointers, sizes, 4-byte alignment, irreps and path
 * rules) return a status before any work is enqueued.  No C++ exception crosses the ABI.
 * CUDA launch failures return TP_ERR_CUDA.  Kernels never trap: with TP_FLAG_CHECK_INDICES
 * they bounds-check rowptr/src/perm, skip bad entries and record the first problem in the
 * workspace error word, readable with tp_get_device_error; outputs are then unspecified.
 * Every device-side wait (the copy-engine rings of the staged edge passes, the tensor-core
 * pipeline of the uvw GEMMs) is bounded by the GPU clock (4 s); a wait that gives up records
 * code 6 (= TP_ERR_TIMEOUT) -- in the workspace word in check mode, otherwise in a per-device
 * word -- and the kernel drains its copies and returns; tp_get_device_error reports it.
 *
 * Alignment.  4 bytes is required.  Rows that start on 16-byte boundaries (any torch
 * allocation) let the 32-channel lmax-2 forward and the uvw edge passes stage them with the
 * copy engine; otherwise the same results come from the unstaged kernels.
 * tp_last_error_message returns this thread's detail text of the last failing call.
 */
#ifndef TP_H_
#define TP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* tp_stream_t; /* identical to cudaStream_t; NULL = legacy default stream */
typedef struct tp_plan_s* tp_plan_t;

typedef enum {
  TP_OK = 0,
  TP_ERR_INVALID_ARG = 1,  /* null pointer, negative size, misalignment, bad irreps string */
  TP_ERR_UNSUPPORTED = 2,  /* valid request this build has no kernel for (l > 3, ...) */
  TP_ERR_BAD_GRAPH = 3,    /* inconsistent CSR found on the host (sizes) */
  TP_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than tp_workspace_size */
  TP_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed */
  TP_ERR_TIMEOUT = 6       /* a bounded device wait gave up (device error code 6) */
} tp_status_t;

enum { TP_MODE_UVU = 0, TP_MODE_UVW = 1 };
enum { TP_FLAG_CHECK_INDICES = 1 };
enum { TP_OP_FWD = 0, TP_OP_BWD = 1, TP_OP_DBWD = 2 };

/* Builds a plan from irreps strings and a path list ("FlashTP: Fused, Sparsity-Aware Tensor
 * Product for Machine Learning Interatomic Potentials", abstract: the tensor product over the
 * model's paths; "Sobek: Streaming Equivariant Tensor Product Convolutions", abstract: uvu and
 * uvw operator families).
 *   irreps_in/out: "32x0e+32x1o+32x2e" (mul x l parity); irreps_sh: "1x0e+1x1o+1x2e"
 *   (multiplicity 1, parity (-1)^l).  paths: [n_paths][3] = (i_in, i_sh, i_out) block
 *   indices, any subset, order or repetition of allowed triples (at most 64 paths); their
 *   order fixes the weight layout: uvu w[e] holds the paths in list order, each path's
 *   mul_in(path) channels contiguous; uvw s[e, p] and W[p][mul_in][mul_out].  Rules:
 *   triangle |l1-l2| <= l3 <= l1+l2, parity p3 = p1 * p2, uvu needs mul_in == mul_out per
 *   path (blocks may differ from each other), uvw needs one multiplicity for all input
 *   blocks and one for all output blocks.  Output blocks no path reaches are zero.
 *   path_coeff: NULL = all 1.0.
 * The lists the build compiles whole (all paths of lmax 1, 2 and 3, and the 4-path lmax-1
 * list, with uniform multiplicities; uvw with multiplicities that are multiples of 4, the
 * TMA row-pitch rule of its tensor-core GEMMs) run their specialised kernels; every other
 * valid list runs the runtime path table (per-triple unrolled contractions chosen at run
 * time).
 * Errors: TP_ERR_INVALID_ARG (syntax, rule violations), TP_ERR_UNSUPPORTED (l > 3, more than
 * 64 paths or 16 blocks, more than 256 32-channel slices, uvw with blocks of different
 * multiplicities). */
tp_status_t tp_plan_create(tp_plan_t* plan, const char* irreps_in, const char* irreps_sh,
                           const char* irreps_out, const int32_t* paths, int32_t n_paths,
                           int32_t mode, const double* path_coeff, uint32_t flags);
tp_status_t tp_plan_destroy(tp_plan_t plan);

/* Sizes of the plan: feature widths, per-edge weights per edge, shared uvw weights. */
tp_status_t tp_plan_query(tp_plan_t plan, int64_t* in_dim, int64_t* out_dim,
                          int64_t* n_edge_weights, int64_t* n_shared_weights);

/* Bytes of device workspace a call of kind op (TP_OP_*) needs for N nodes and E edges:
 * forward 0 (256 with TP_FLAG_CHECK_INDICES, for the error word); backward and double
 * backward 256 + int32 colptr[N+1] + perm[E] + the transpose's scratch
 * (tp_csr_transpose_workspace_size), room to build the transpose in place; only the
 * 256-byte header is used when colptr/perm are given.  uvw adds node- and weight-sized
 * float regions.  The workspace never holds an edge x feature float tensor. */
tp_status_t tp_workspace_size(tp_plan_t plan, int64_t N, int64_t E, int32_t op, size_t* bytes);

/* Bytes of scratch tp_csr_transpose needs for N nodes and E edges. */
tp_status_t tp_csr_transpose_workspace_size(int64_t N, int64_t E, size_t* bytes);

/* Stable receiver->sender transpose (the sender order of the backward passes):
 * colptr[N+1] = exclusive scan of bincount(src), perm[E] = stable argsort of src (bit
 * exact), computed as a radix sort of the edge ids keyed by sender: O(E) work per pass and
 * ceil(log2(N+1) / 11) passes, whatever the degree distribution.  rowptr may be NULL.
 * Senders should lie in [0, N); an edge whose sender does not is placed after all valid
 * edges (perm[colptr[N]..E) lists those edges in increasing order) and colptr[N] counts the
 * valid edges.  Workspace: ws 4-byte aligned, ws_bytes >= tp_csr_transpose_workspace_size
 * (int32 scratch: an id buffer of E when more than one pass is needed, plus per-tile digit
 * counts, about 4 bytes per edge at most).  TP_ERR_INVALID_ARG for null or misaligned
 * pointers or sizes outside [0, 2^31), TP_ERR_WORKSPACE for a short workspace. */
tp_status_t tp_csr_transpose(int64_t N, int64_t E, const int32_t* rowptr, const int32_t* src,
                             int32_t* colptr, int32_t* perm, void* ws, size_t ws_bytes,
                             tp_stream_t stream);

/* Same result as tp_csr_transpose (bit for bit), for callers that cannot allocate device
 * memory -- e.g. an MD engine whose device memory is owned by a pool it does not control,
 * a framework that has reserved nearly all of the GPU up front, or a loop that must avoid
 * cudaMalloc/cudaFree because they synchronise the device.  It takes no workspace: its
 * scratch (the radix sort's second id buffer and digit counts) is a fixed int32 array
 * inside the library (about 5.3 MB, held on every GPU that loads the library until exit).
 * The source pages have no counterpart; this is an interface convenience.
 *   Limits: N <= 131072 and E <= 1048576, else TP_ERR_UNSUPPORTED with nothing enqueued.
 *   Senders outside [0, N) are handled as by tp_csr_transpose (placed last, not counted).
 *   Calls share the array: calls whose work overlaps on the GPU race; order them on one
 *   stream.  Every call writes the parts of the array it reads before reading them.  The
 *   first call on a device looks up the array's device address with that device current:
 *   make it before any stream capture.  The address is kept for the life of the process, so
 *   a cudaDeviceReset between calls is not supported.  Other errors: TP_ERR_INVALID_ARG
 *   (null, misaligned, negative sizes), TP_ERR_CUDA.  No message is set for
 *   tp_last_error_message. */
tp_status_t tp_csr_transpose_noalloc(int64_t N, int64_t E, const int32_t* rowptr,
                                     const int32_t* src, int32_t* colptr, int32_t* perm,
                                     tp_stream_t stream);

/* Forward: y[N, out_dim].  W is NULL in uvu mode. */
tp_status_t tp_conv_fwd(tp_plan_t plan, int64_t N, int64_t E, const int32_t* rowptr,
                        const int32_t* src, const float* x, const float* vec, const float* w,
                        const float* W, float* y, void* ws, size_t ws_bytes, tp_stream_t stream);

/* Backward against gy[N, out_dim].  colptr/perm: a transpose from tp_csr_transpose, or both
 * NULL to have it built in the workspace.  Outputs gx[N, in_dim], gw[E, nw] (uvu w or uvw
 * s), gvec[E, 3], gW[P, mul_in, mul_out] (uvw); each NULL output is skipped. */
tp_status_t tp_conv_bwd(tp_plan_t plan, int64_t N, int64_t E, const int32_t* rowptr,
                        const int32_t* src, const int32_t* colptr, const int32_t* perm,
                        const float* x, const float* vec, const float* w, const float* W,
                        const float* gy, float* gx, float* gw, float* gvec, float* gW, void* ws,
                        size_t ws_bytes, tp_stream_t stream);

/* Double backward (uvu): inputs ggx[N, in_dim], ggw[E, nw], ggvec[E, 3], each NULL = zero;
 * outputs g_gy[N, out_dim], g_x[N, in_dim], g_w[E, nw], g_vec[E, 3], each NULL = skipped. */
tp_status_t tp_conv_dbwd(tp_plan_t plan, int64_t N, int64_t E, const int32_t* rowptr,
                         const int32_t* src, const int32_t* colptr, const int32_t* perm,
                         const float* x, const float* vec, const float* w, const float* W,
                         const float* gy, const float* ggx, const float* ggw, const float* ggvec,
                         float* g_gy, float* g_x, float* g_w, float* g_vec, void* ws,
                         size_t ws_bytes, tp_stream_t stream);

/* The uvu convolution with the radial projection fused in ("Sobek: Streaming Equivariant
 * Tensor Product Convolutions", abstract: the radial projection reordered so that
 * edge-specific weights are never materialised).  Instead of w[E, nw] the caller passes the
 * radial network's last hidden layer and its bias-free output layer,
 *   h   [E, H]   fp32, row e belongs to edge e (receiver-sorted order, like vec); 16-byte aligned
 *   Wr  [H, nw]  fp32, nw = n_edge_weights of the plan, columns in the w layout above
 * and the library forms w[e, c] = sum_k h[e, k] Wr[k, c] in on-chip memory, chunk by chunk,
 * and uses it there (fp32, k ascending): y equals tp_conv_fwd with that w, and no edge x nw
 * tensor exists at any point.  H is a multiple of 4 in [4, 64]; any uvu plan (the path table
 * runs the coupling); uvw plans give TP_ERR_UNSUPPORTED, as do plans whose weight rows do not
 * fit four edges' on-chip tiles (nw above about 6,000).  Errors and ownership as tp_conv_fwd.
 *
 * tp_radial_workspace_size: bytes for op TP_OP_FWD (0, or 256 with TP_FLAG_CHECK_INDICES) or
 * TP_OP_BWD (the transpose region of tp_workspace_size, Wr transposed and per-split partials
 * of gWr: H x nw floats per split, at most 256 splits; nothing edge-sized).
 *
 * tp_conv_bwd_radial: the VJP against gy[N, out_dim] with respect to x, vec, h and Wr:
 * gx[N, in_dim], gh[E, H], gWr[H, nw], gvec[E, 3]; each NULL output is skipped; colptr/perm
 * as in tp_conv_bwd (NULL: built in the workspace).  gW_r is a deterministic sum of fixed
 * edge-range partials. */
tp_status_t tp_radial_workspace_size(tp_plan_t plan, int64_t N, int64_t E, int32_t H, int32_t op,
                                     size_t* bytes);
tp_status_t tp_conv_fwd_radial(tp_plan_t plan, int64_t N, int64_t E, int32_t H, const int32_t* rowptr,
                               const int32_t* src, const float* x, const float* vec, const float* h,
                               const float* Wr, float* y, void* ws, size_t ws_bytes, tp_stream_t stream);
tp_status_t tp_conv_bwd_radial(tp_plan_t plan, int64_t N, int64_t E, int32_t H, const int32_t* rowptr,
                               const int32_t* src, const int32_t* colptr, const int32_t* perm,
                               const float* x, const float* vec, const float* h, const float* Wr,
                               const float* gy, float* gx, float* gh, float* gWr, float* gvec,
                               void* ws, size_t ws_bytes, tp_stream_t stream);

/* Row movement of receiver-range sharding over several GPUs (one process per GPU): a rank
 * owning a contiguous range of receivers gathers the x rows its peers need before the halo
 * exchange, and adds the gradient partials its peers send back for the senders it owns
 * ("Sobek: Streaming Equivariant Tensor Product Convolutions", abstract: graphs far beyond
 * one device's memory; the exchange itself is the caller's collective).
 *   tp_gather_rows: dst[k, :] = src[idx[k], :] for k < n (rows of row_len floats).
 *   tp_add_rows:    dst[idx[k], :] += src[k, :] for k < n; the n indices of one call must be
 *                   distinct, which makes the result independent of the schedule.
 * idx holds valid row indices of the respective arrays (not checked on the device).
 * TP_ERR_INVALID_ARG for n < 0, row_len <= 0, NULL or non-4-byte-aligned pointers with n > 0. */
tp_status_t tp_gather_rows(const float* src, int64_t row_len, const int32_t* idx, int64_t n, float* dst,
                           tp_stream_t stream);
tp_status_t tp_add_rows(float* dst, int64_t row_len, const int32_t* idx, int64_t n, const float* src,
                        tp_stream_t stream);

/* Reads (and clears) the device error word after the work on `stream` finished;
 * synchronises the stream.  Check-mode plans read the word of workspace `ws`; other plans,
 * and plan == NULL, read the per-device word (ws unused) -- the word the linear maps of
 * tp_block.h report their bounded-wait timeouts to as well.  *code: 0 = none, 1 = bad rowptr, 2 = bad src,
 * 3 = bad perm / transpose entry, 6 = a bounded device wait gave up. */
tp_status_t tp_get_device_error(tp_plan_t plan, void* ws, tp_stream_t stream, int32_t* code);

/* Self-check of the bounded waits (no counterpart on the pages; failure detection).  Runs the
 * two wait primitives the pipelined kernels use -- the copy-engine slot wait and the
 * tensor-core pipeline wait with its abort flag -- on a barrier that is never signalled,
 * with limit_ns (1 ns .. 1 s), and synchronises `stream`.  *gave_up: bit 0 = slot wait gave
 * up, bit 1 = pipeline wait gave up, bit 2 = it raised the abort flag; 7 is the designed
 * outcome.  TP_ERR_INVALID_ARG for a NULL result or a limit outside (0, 1 s]. */
tp_status_t tp_check_bounded_waits(int64_t limit_ns, tp_stream_t stream, int32_t* gave_up);

/* Number of kernels this library has launched in the calling process (diagnostics: lets a
 * benchmark count its own launches in a timed region). */
int64_t tp_launch_count(void);

const char* tp_status_string(tp_status_t status);
const char* tp_last_error_message(void);
const char* tp_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TP_H_ */
