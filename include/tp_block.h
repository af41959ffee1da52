/*
 * tp_block.h -- C ABI of the node-side operators of an equivariant interaction layer, which
 * sit around the tensor-product convolution of tp.h: the irreps-wise linear map
 * (self-interaction before the convolution, mixing of its path-concatenated outputs after
 * it) and the gate nonlinearity.  The 1/(average degree) scale of the aggregated messages
 * is either the convolution plan's path coefficient (tp_plan_create, path_coeff) or, since
 * it commutes with the linear map, that map's instruction coefficients -- the cheaper form:
 * the convolution's compiled fast instances take unit path coefficients.
 *
 * The pages name these layers without defining them ("Accelerating Tensor Products in
 * E(3)-Equivariant Graph Neural Networks", abstract: NequIP's equivariant interaction layers,
 * dominated by the tensor-product convolution; "The GPU Workload That Rewrites Molecular
 * Physics", section "What Makes MLFF Workloads Structurally Different": every atom
 * aggregates its neighbours and transforms the result through a neural network).  The
 * definitions below are the plainest equivariant readings.
 *
 * Linear.  Instructions are every block pair (i_in, i_out) of irreps_in and irreps_out with
 * equal (l, parity), in lexicographic (i_in, i_out) order.  Instruction k owns the matrix
 * W_k[mul_in(k)][mul_out(k)] (row-major; the matrices are concatenated in instruction order
 * into W[n_weights]) and a coefficient c_k (default 1):
 *
 *   y[n, o, w, m] = sum_{k: out(k) = o} c_k sum_u W_k[u, w] x[n, in(k), u, m]
 *
 * Output blocks that no instruction reaches are zero.  Wide maps on many nodes run on the
 * tcgen05 tensor cores in 3xTF32 (fp32-accurate, see tp.h) as one GEMM per output block over
 * the concatenated input channels of its irrep, after the inputs are regrouped into
 * [(node, m)][channel] rows in the workspace; narrow maps run on the CUDA cores straight from
 * the node rows (see tp_linear_create).  Backward: gx = the adjoint map applied to gy,
 * gW_k[u, w] = c_k sum_{n, m} x[n, in(k), u, m] gy[n, out(k), w, m] (split-K GEMM, fixed
 * split order: deterministic).  Second order needs no entry point of its own: with
 * cotangents (ggx, ggW) of (gx, gW),
 *   g_gy = fwd(ggx; W) + fwd(x; ggW)      (the second call with accumulate = 1)
 *   g_x  = bwd(gy; ggW).gx,   g_W = bwd(x := ggx, gy).gW.
 *
 * Gate.  The input row is [scalars | gates | gated] (the three irreps strings concatenated),
 * the output row [act(scalars) | gated * sigmoid(gates)]: 0e scalars take SiLU
 * (x sigmoid(x)), 0o scalars tanh (odd, so parity is kept), and gated channel c (the
 * channels of the gated blocks counted in order) is multiplied by sigmoid(gate channel c).
 * Gates must be 0e and their total multiplicity must equal that of the gated blocks.
 *
 * Layouts as in tp.h: [N, dim] row-major fp32 device arrays, blocks in irreps order, [u][m]
 * inside a block.  Ownership: the caller owns every buffer (workspace included); the
 * library owns the linear and gate handles (host memory).  Streams: every call enqueues on
 * `stream` and returns.  Errors: host checks return a status before anything is enqueued
 * (NULL arguments, sizes, 4-byte alignment, irreps rules); TP_ERR_CUDA for a failed launch.
 * The GEMMs' device waits are bounded (4 s) and a wait that gives up records code 6 in the
 * per-device error word, which tp_get_device_error(NULL, NULL, stream, &code) reads.
 */
#ifndef TP_BLOCK_H_
#define TP_BLOCK_H_

#include "tp.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tp_linear_s* tp_linear_t;
typedef struct tp_gate_s* tp_gate_t;

enum { TP_LINEAR_TENSOR_CORES = 1, TP_LINEAR_CUDA_CORES = 2 };

/* Builds a linear map.  irreps strings as in tp.h ("32x0e+32x1o"); l <= 3; every
 * multiplicity a multiple of 4 (TMA row pitch), else TP_ERR_UNSUPPORTED.  coeff: one double
 * per instruction, or NULL for 1.0.  At most 64 instructions and 16 blocks per string.
 * flags: 0 picks the form per call -- the tcgen05 GEMMs when N >= 4096 and every irrep has
 * at least 64 input and 64 output channels, otherwise the CUDA-core form, which reads the
 * node rows in place (one launch for y or gx, two for gW); TP_LINEAR_TENSOR_CORES or
 * TP_LINEAR_CUDA_CORES forces one.  Both give the same sums to fp32 rounding. */
tp_status_t tp_linear_create(tp_linear_t* lin, const char* irreps_in, const char* irreps_out, const double* coeff,
                             uint32_t flags);
tp_status_t tp_linear_destroy(tp_linear_t lin);

/* Feature widths, weight count (sum of mul_in * mul_out over instructions), instructions. */
tp_status_t tp_linear_query(tp_linear_t lin, int64_t* in_dim, int64_t* out_dim, int64_t* n_weights,
                            int32_t* n_instructions);

/* Device workspace bytes for N nodes: op TP_OP_FWD (regrouped inputs + split weights) or
 * TP_OP_BWD (regrouped inputs and output gradients, split weights, split-K partials), enough
 * for either form; 256-byte aligned (any torch allocation is). */
tp_status_t tp_linear_workspace_size(tp_linear_t lin, int64_t N, int32_t op, size_t* bytes);

/* y[N, out_dim] = linear(x[N, in_dim]; W[n_weights]); accumulate = 1 adds into y instead of
 * overwriting it (blocks no instruction reaches are then left as they are). */
tp_status_t tp_linear_fwd(tp_linear_t lin, int64_t N, const float* x, const float* W, float* y,
                          int32_t accumulate, void* ws, size_t ws_bytes, tp_stream_t stream);

/* Against gy[N, out_dim]: gx[N, in_dim] and gW[n_weights]; each NULL output is skipped (x
 * may then be NULL when gW is). */
tp_status_t tp_linear_bwd(tp_linear_t lin, int64_t N, const float* x, const float* W, const float* gy,
                          float* gx, float* gW, void* ws, size_t ws_bytes, tp_stream_t stream);

/* Builds a gate.  Any of the three strings may be empty ("" or NULL) as long as the
 * multiplicities match; scalars l = 0, gates 0e, gated l <= 3. */
tp_status_t tp_gate_create(tp_gate_t* gate, const char* irreps_scalars, const char* irreps_gates,
                           const char* irreps_gated);
tp_status_t tp_gate_destroy(tp_gate_t gate);
tp_status_t tp_gate_query(tp_gate_t gate, int64_t* in_dim, int64_t* out_dim);

/* y[N, out_dim] = gate(x[N, in_dim]).  No workspace. */
tp_status_t tp_gate_fwd(tp_gate_t gate, int64_t N, const float* x, float* y, tp_stream_t stream);

/* gx[N, in_dim] = J(x)^T gy. */
tp_status_t tp_gate_bwd(tp_gate_t gate, int64_t N, const float* x, const float* gy, float* gx,
                        tp_stream_t stream);

/* VJP of (x, gy) -> gx against ggx[N, in_dim]: g_gy[N, out_dim] = J(x) ggx and
 * g_x[N, in_dim] = the second-derivative terms; each NULL output is skipped. */
tp_status_t tp_gate_dbwd(tp_gate_t gate, int64_t N, const float* x, const float* gy, const float* ggx,
                         float* g_gy, float* g_x, tp_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* TP_BLOCK_H_ */
