// C ABI of the tensor-product convolution: plans, argument checks, workspace layout and
// dispatch to the compiled specialisations.  See include/tp.h for the contract.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "../../include/tp.h"
#include "tp_common.h"
#include "tp_host.h"

using namespace tp;

struct IrrepBlock {
  int mul, l, parity;
};

struct tp_plan_s {
  const SpecOps* ops;   // compiled specialisation, or NULL: runtime path table `gen`
  GenTable* gen;
  GenTable* rad;        // uvu: the path table of the fused radial projection (== gen when set)
  int mode;
  int mul_in, mul_out;
  int64_t in_dim, out_dim, nw, n_shared;
  int n_paths;
  int has_coeff;
  float coeff[kMaxPaths];
  uint32_t flags;
};

#include <atomic>
#include <mutex>
namespace tp {
static std::atomic<long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
}  // namespace tp

namespace {

thread_local std::string g_msg;

tp_status_t fail(tp_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_msg = buf;
  return st;
}

tp_status_t cuda_fail(cudaError_t e, const char* where) {
  return fail(TP_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool parse_irreps(const char* s, std::vector<IrrepBlock>& out, std::string& why) {
  out.clear();
  if (!s) {
    why = "null irreps string";
    return false;
  }
  std::string str;
  for (const char* p = s; *p; ++p)
    if (*p != ' ') str.push_back(*p);
  if (str.empty()) {
    why = "empty irreps string";
    return false;
  }
  size_t pos = 0;
  while (pos <= str.size()) {
    size_t end = str.find('+', pos);
    if (end == std::string::npos) end = str.size();
    std::string term = str.substr(pos, end - pos);
    size_t x = term.find('x');
    if (x == std::string::npos || x == 0 || x + 2 > term.size()) {
      why = "bad irreps term '" + term + "'";
      return false;
    }
    const std::string mul_s = term.substr(0, x), l_s = term.substr(x + 1, term.size() - x - 2);
    const char par = term.back();
    if (l_s.empty() || (par != 'e' && par != 'o') || mul_s.size() > 7 || l_s.size() > 3) {
      why = "bad irreps term '" + term + "'";
      return false;
    }
    for (char ch : mul_s + l_s)
      if (ch < '0' || ch > '9') {
        why = "bad irreps term '" + term + "'";
        return false;
      }
    IrrepBlock b{std::atoi(mul_s.c_str()), std::atoi(l_s.c_str()), par == 'e' ? 1 : -1};
    if (b.mul <= 0) {
      why = "multiplicity must be positive";
      return false;
    }
    out.push_back(b);
    if (end == str.size()) break;
    pos = end + 1;
    if (pos == str.size()) {
      why = "trailing '+'";
      return false;
    }
  }
  return true;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct WsLayout {
  size_t header, colptr, perm, scratch, total;
};

// header (error word) | colptr[N+1] | perm[E] | transpose scratch (int32, see csr.cu)
WsLayout ws_layout(int64_t N, int64_t E) {
  WsLayout L{};
  size_t off = 0;
  L.header = off;
  off += 256;
  L.colptr = off;
  off += align256(sizeof(int32_t) * (size_t)(N + 1));
  L.perm = off;
  off += align256(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
  L.scratch = off;
  off += align256(sizeof(int32_t) * (size_t)transpose_scratch_ints(N, E));
  L.total = off;
  return L;
}

// uvw regions (floats, 256-byte aligned).  Forward: A | Wt (hi, lo).  Backward, after the
// transpose region: A (x W) | G (B) | xT | Wt (Wg hi, lo, Wx hi, lo) | part.
// Split-K partials of the gW GEMM: one per 1,536 nodes, at most 64.  Every split then
// reduces at least ~768 * d1 rows (24 or more K blocks), so the fp32 promotion of the
// accumulator (every 16 K blocks) runs at every size beyond a few hundred nodes, and a large
// graph keeps 64 splits of parallel work.
int uvw_splits(int64_t N) { return (int)std::min<int64_t>(64, std::max<int64_t>(1, (N + 1535) / 1536)); }
struct UvwLayout {
  size_t A, G, xT, Wt, part, total;
};
UvwLayout uvw_layout(tp_plan_t plan, int64_t N, int64_t E, bool bwd) {
  UvwLayout U{};
  size_t off = bwd ? ws_layout(N, E).total : 256;
  // forward: receiver state A (A_PC x mul per node); backward: x W and B (XT_PC x mul_out)
  const size_t a_bytes = bwd ? sizeof(float) * (size_t)N * plan->ops->XT_PC * plan->mul_out
                             : sizeof(float) * (size_t)N * plan->ops->A_PC * plan->mul_in;
  const size_t w_bytes = sizeof(float) * (size_t)plan->n_shared;
  U.A = off;
  off += align256(a_bytes > 0 ? a_bytes : 1);
  U.G = off;
  if (bwd) off += align256(a_bytes > 0 ? a_bytes : 1);
  U.xT = off;
  if (bwd) off += align256(sizeof(float) * (size_t)(N > 0 ? N : 1) * plan->in_dim);
  U.Wt = off;
  off += align256(w_bytes * (bwd ? 4 : 2));
  U.part = off;
  if (bwd) off += align256(w_bytes * uvw_splits(N));
  U.total = off;
  return U;
}

// uvw through the path table: x W per path (fwd and bwd), its gradient B and the gW node-chunk
// partials (bwd), after the transpose region in the backward.
UvwLayout gen_uvw_layout(tp_plan_t plan, int64_t N, int64_t E, bool bwd) {
  UvwLayout U{};
  size_t off = bwd ? ws_layout(N, E).total : 256;
  const size_t xt_bytes = sizeof(float) * (size_t)(N > 0 ? N : 1) * plan->gen->xt_dim;
  U.A = off;
  off += align256(xt_bytes);
  U.G = off;
  if (bwd) off += align256(xt_bytes);
  U.xT = U.Wt = U.part = off;
  if (bwd) off += align256(sizeof(float) * (size_t)plan->n_shared * uvw_splits(N));
  U.total = off;
  return U;
}

int pick_split(int64_t N, int64_t E) {
  if (N <= 0) return 1;
  const double avg = (double)E / (double)N;
  if (avg >= 24.0) return 4;
  if (avg >= 8.0) return 2;
  return 1;
}

tp_status_t check_sizes(tp_plan_t plan, int64_t N, int64_t E) {
  if (!plan) return fail(TP_ERR_INVALID_ARG, "plan is NULL");
  if (N < 0 || E < 0) return fail(TP_ERR_INVALID_ARG, "N and E must be non-negative");
  if (N >= (int64_t)1 << 31 || E >= (int64_t)1 << 31)
    return fail(TP_ERR_UNSUPPORTED, "N and E must be below 2^31 (int32 indices)");
  const int64_t slices = (plan->mul_in + 31) / 32;
  if (N * slices >= (int64_t)1 << 31) return fail(TP_ERR_UNSUPPORTED, "N * channel slices must be below 2^31");
  return TP_OK;
}

LaunchArgs base_args(tp_plan_t plan, int64_t N, int64_t E) {
  LaunchArgs a;
  std::memset(&a, 0, sizeof(a));
  a.N = (int)N;
  a.E = (int)E;
  a.mul = plan->mul_in;
  a.mul_out = plan->mul_out;
  a.in_dim = (int)plan->in_dim;
  a.out_dim = (int)plan->out_dim;
  a.nw = (int)plan->nw;
  a.split = pick_split(N, E);
  a.n_slices = (plan->mul_in + 31) / 32;
  a.has_coeff = plan->has_coeff;
  a.check = (plan->flags & TP_FLAG_CHECK_INDICES) ? 1 : 0;


  std::memcpy(a.coeff, plan->coeff, sizeof(a.coeff));
  return a;
}

// Validates the CSR on the device (debug flag only) and resets the error word.
// Sticky per-device error word for plans without TP_FLAG_CHECK_INDICES: the pipelined
// kernels record a wait that gave up (code 6) here; tp_get_device_error reads and clears it.
__device__ int g_device_error;

int* device_error_word() {
  static std::mutex mu;
  static int* ptr[64] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    ptr[dev] = static_cast<int*>(p);
  }
  return ptr[dev];
}

tp_status_t debug_prologue(tp_plan_t plan, int64_t N, int64_t E, const int32_t* rowptr,
                           const int32_t* src, void* ws, cudaStream_t s, int** err) {
  *err = nullptr;
  if (!(plan->flags & TP_FLAG_CHECK_INDICES)) {
    *err = device_error_word();
    return TP_OK;
  }
  if (!ws) return fail(TP_ERR_WORKSPACE, "TP_FLAG_CHECK_INDICES needs a workspace for the error word");
  int* e = reinterpret_cast<int*>(ws);
  cudaError_t st = cudaMemsetAsync(e, 0, sizeof(int), s);
  if (st != cudaSuccess) return cuda_fail(st, "cudaMemsetAsync(error word)");
  st = launch_csr_validate((int)N, (int)E, rowptr, src, e, s);
  if (st != cudaSuccess) return cuda_fail(st, "csr_validate");
  *err = e;
  return TP_OK;
}

// The runtime path table of a plan without a compiled specialisation: block offsets, paths
// per block and the (block, 32-channel slice) tasks of the receiver and sender passes.
bool build_gen_table(const std::vector<IrrepBlock>& bi, const std::vector<IrrepBlock>& bs,
                     const std::vector<IrrepBlock>& bo, const int32_t* paths, int n_paths, const double* coeff,
                     bool uvw, GenTable& T, std::string& why) {
  std::memset(&T, 0, sizeof(T));
  T.uvw = uvw ? 1 : 0;
  T.mul_in = bi[0].mul;
  T.mul_out = bo[0].mul;
  T.n_paths = n_paths;
  T.n_in = (int)bi.size();
  T.n_out = (int)bo.size();
  int off = 0;
  for (int k = 0; k < T.n_in; ++k) {
    T.in_off[k] = off;
    T.in_mul[k] = bi[k].mul;
    T.in_l[k] = bi[k].l;
    off += bi[k].mul * (2 * bi[k].l + 1);
  }
  off = 0;
  for (int k = 0; k < T.n_out; ++k) {
    T.out_off[k] = off;
    T.out_mul[k] = bo[k].mul;
    T.out_l[k] = bo[k].l;
    off += bo[k].mul * (2 * bo[k].l + 1);
  }
  int w_off = 0;
  for (int p = 0; p < n_paths; ++p) {
    const int a = paths[3 * p], b = paths[3 * p + 1], o = paths[3 * p + 2];
    GenPath& P = T.path[p];
    P.l1 = (int16_t)bi[a].l;
    P.l2 = (int16_t)bs[b].l;
    P.l3 = (int16_t)bo[o].l;
    P.tid = (int16_t)gen_triple_id(bi[a].l, bs[b].l, bo[o].l);
    if (P.tid < 0) {
      why = "path outside the generated triples";
      return false;
    }
    P.in_off = uvw ? T.xt_dim : T.in_off[a];     // uvw: the path's block in a row of x W
    P.out_off = T.out_off[o];
    P.mul = uvw ? bo[o].mul : bi[a].mul;
    P.w_off = uvw ? p : w_off;
    if (uvw) T.xt_dim += bo[o].mul * (2 * bi[a].l + 1);
    P.in_block = a;
    P.out_block = o;
    P.coeff = coeff ? (float)coeff[p] : 1.0f;
    w_off += bi[a].mul;
    T.lmax_sh = std::max(T.lmax_sh, bs[b].l);
  }
  int q = 0;
  for (int o = 0; o < T.n_out; ++o) {
    T.out_first[o] = q;
    for (int p = 0; p < n_paths; ++p)
      if (paths[3 * p + 2] == o) T.out_paths[q++] = p;
  }
  T.out_first[T.n_out] = q;
  q = 0;
  for (int a = 0; a < T.n_in; ++a) {
    T.in_first[a] = q;
    for (int p = 0; p < n_paths; ++p)
      if (paths[3 * p] == a) T.in_paths[q++] = p;
  }
  T.in_first[T.n_in] = q;
  for (int pass = 0; pass < 2; ++pass) {
    const auto& blocks = pass == 0 ? bo : bi;
    int n = 0;
    for (int k = 0; k < (int)blocks.size(); ++k)
      for (int sl = 0; sl < (blocks[k].mul + 31) / 32; ++sl) {
        if (n >= kGenMaxTasks || sl > 255) {
          why = "too many 32-channel slices for the runtime path table (at most 256 over all blocks)";
          return false;
        }
        (pass == 0 ? T.rtask_block : T.stask_block)[n] = (uint8_t)k;
        (pass == 0 ? T.rtask_slice : T.stask_slice)[n] = (uint8_t)sl;
        ++n;
      }
    (pass == 0 ? T.n_rtask : T.n_stask) = n;
  }
  return true;
}

}  // namespace

namespace tp {

bool parse_irreps_terms(const char* s, std::vector<IrrepTerm>& out, std::string& why) {
  std::vector<IrrepBlock> blocks;
  out.clear();
  if (!parse_irreps(s, blocks, why)) return false;
  for (const IrrepBlock& b : blocks) out.push_back(IrrepTerm{b.mul, b.l, b.parity});
  return true;
}

tp_status_t set_failure(tp_status_t st, const std::string& msg) {
  g_msg = msg;
  return st;
}

int* device_error_ptr() { return device_error_word(); }

}  // namespace tp

namespace {

// Host checks shared by the radial entry points; fills the sizes of `a`.
tp_status_t radial_args(tp_plan_t plan, int64_t N, int64_t E, int32_t H, RadArgs& a) {
  tp_status_t st = check_sizes(plan, N, E);
  if (st != TP_OK) return st;
  if (plan->mode != TP_MODE_UVU || !plan->rad)
    return fail(TP_ERR_UNSUPPORTED, "the fused radial projection is implemented for uvu plans");
  if (H < 4 || H > kRadMaxHidden || H % 4 != 0)
    return fail(TP_ERR_UNSUPPORTED, "hidden width must be a multiple of 4 in [4, %d]", kRadMaxHidden);
  std::memset(&a, 0, sizeof(a));
  a.N = (int)N;
  a.E = (int)E;
  a.H = H;
  a.nw = (int)plan->nw;
  a.nwp = (a.nw + 3) & ~3;
  a.in_dim = (int)plan->in_dim;
  a.out_dim = (int)plan->out_dim;
  a.check = (plan->flags & TP_FLAG_CHECK_INDICES) ? 1 : 0;
  a.splits = rad_splits(*plan->rad, E);
  a.mul = plan->mul_in;
  a.spec = 0;
  if (plan->ops && std::strcmp(plan->ops->name, "full_l2") == 0) a.spec = 2;
  if (plan->ops && std::strcmp(plan->ops->name, "full_l3") == 0) a.spec = 3;
  if (rad_chunk(a, false, nullptr) == 0 || rad_chunk(a, true, nullptr) == 0)
    return fail(TP_ERR_UNSUPPORTED, "%d weights per edge do not fit the shared-memory chunk of four edges", a.nw);
  return TP_OK;
}

struct RadLayout {
  size_t WrT, part, total;
};
// backward: the transpose region, then W_r^T [nw, H] and the gW_r partials [splits, H, nw]
RadLayout rad_layout(const RadArgs& a) {
  RadLayout L{};
  size_t off = ws_layout(a.N, a.E).total;
  L.WrT = off;
  off += align256(sizeof(float) * (size_t)a.H * a.nw);
  L.part = off;
  off += align256(sizeof(float) * (size_t)a.H * a.nw * a.splits);
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

const char* tp_version(void) { return "tp-b200 0.1 (sm_100a)"; }

int64_t tp_launch_count(void) { return tp::g_launches.load(std::memory_order_relaxed); }

const char* tp_status_string(tp_status_t s) {
  switch (s) {
    case TP_OK: return "ok";
    case TP_ERR_INVALID_ARG: return "invalid argument";
    case TP_ERR_UNSUPPORTED: return "unsupported";
    case TP_ERR_BAD_GRAPH: return "bad graph";
    case TP_ERR_WORKSPACE: return "workspace too small";
    case TP_ERR_CUDA: return "CUDA error";
    case TP_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* tp_last_error_message(void) { return g_msg.c_str(); }

tp_status_t tp_plan_create(tp_plan_t* plan, const char* irreps_in, const char* irreps_sh,
                           const char* irreps_out, const int32_t* paths, int32_t n_paths, int32_t mode,
                           const double* path_coeff, uint32_t flags) {
  if (!plan) return fail(TP_ERR_INVALID_ARG, "plan out-pointer is NULL");
  *plan = nullptr;
  std::vector<IrrepBlock> bi, bs, bo;
  std::string why;
  if (!parse_irreps(irreps_in, bi, why)) return fail(TP_ERR_INVALID_ARG, "irreps_in: %s", why.c_str());
  if (!parse_irreps(irreps_sh, bs, why)) return fail(TP_ERR_INVALID_ARG, "irreps_sh: %s", why.c_str());
  if (!parse_irreps(irreps_out, bo, why)) return fail(TP_ERR_INVALID_ARG, "irreps_out: %s", why.c_str());
  if (mode != TP_MODE_UVU && mode != TP_MODE_UVW) return fail(TP_ERR_INVALID_ARG, "mode must be TP_MODE_UVU or TP_MODE_UVW");
  if (!paths || n_paths <= 0) return fail(TP_ERR_INVALID_ARG, "empty path list");
  if (n_paths > kMaxPaths) return fail(TP_ERR_UNSUPPORTED, "at most %d paths", kMaxPaths);
  if ((int)bi.size() > kMaxBlocks || (int)bs.size() > kMaxBlocks || (int)bo.size() > kMaxBlocks)
    return fail(TP_ERR_UNSUPPORTED, "at most %d irreps blocks", kMaxBlocks);
  for (auto* v : {&bi, &bs, &bo})
    for (auto& b : *v)
      if (b.l > 3) return fail(TP_ERR_UNSUPPORTED, "l = %d > 3", b.l);
  for (auto& b : bs)
    if (b.mul != 1 || b.parity != ((b.l & 1) ? -1 : 1))
      return fail(TP_ERR_INVALID_ARG, "spherical-harmonic irreps must be 1x<l> with parity (-1)^l");
  for (int p = 0; p < n_paths; ++p) {
    const int a = paths[3 * p], b = paths[3 * p + 1], o = paths[3 * p + 2];
    if (a < 0 || a >= (int)bi.size() || b < 0 || b >= (int)bs.size() || o < 0 || o >= (int)bo.size())
      return fail(TP_ERR_INVALID_ARG, "path %d: block index out of range", p);
    const int l1 = bi[a].l, l2 = bs[b].l, l3 = bo[o].l;
    if (l3 < std::abs(l1 - l2) || l3 > l1 + l2)
      return fail(TP_ERR_INVALID_ARG, "path %d (%d,%d,%d): triangle rule violated", p, l1, l2, l3);
    if (bo[o].parity != bi[a].parity * bs[b].parity)
      return fail(TP_ERR_INVALID_ARG, "path %d: parity rule violated", p);
    if (mode == TP_MODE_UVU && bi[a].mul != bo[o].mul)
      return fail(TP_ERR_INVALID_ARG, "path %d: uvu needs equal input and output multiplicity", p);
  }
  int mul_in = 0, mul_out = 0;
  bool uniform = true;
  for (auto& b : bi) {
    uniform = uniform && b.mul == bi[0].mul;
    mul_in = std::max(mul_in, b.mul);
  }
  for (auto& b : bo) {
    uniform = uniform && b.mul == bo[0].mul;
    mul_out = std::max(mul_out, b.mul);
  }
  // the compiled specialisation of this irreps / path list, if the build ships one
  const SpecOps* found = nullptr;
  for (int r = 0; r < kRegistrySize && !found && uniform; ++r) {
    const SpecOps* s = kRegistry[r];
    if (s->n_in != (int)bi.size() || s->n_sh != (int)bs.size() || s->n_out != (int)bo.size() ||
        s->n_paths != n_paths)
      continue;
    bool ok = true;
    for (int k = 0; k < s->n_in && ok; ++k) ok = s->in_ls[k] == bi[k].l;
    for (int k = 0; k < s->n_sh && ok; ++k) ok = s->sh_ls[k] == bs[k].l;
    for (int k = 0; k < s->n_out && ok; ++k) ok = s->out_ls[k] == bo[k].l;
    for (int p = 0; p < n_paths && ok; ++p)
      ok = s->paths[p][0] == paths[3 * p] && s->paths[p][1] == paths[3 * p + 1] &&
           s->paths[p][2] == paths[3 * p + 2];
    if (ok) found = s;
  }
  // uvw shares one W_p [mul_in, mul_out] per path: one multiplicity per side
  if (mode == TP_MODE_UVW && !uniform)
    return fail(TP_ERR_UNSUPPORTED, "uvw needs one multiplicity for all input blocks and one for all output blocks");
  if (found && mode == TP_MODE_UVW && (!found->uvw_fwd || !found->uvw_bwd)) found = nullptr;
  // the compiled uvw GEMMs load their operands by TMA, whose row pitches are multiples of 16
  // bytes; other multiplicities take the path table
  if (found && mode == TP_MODE_UVW && (mul_in % 4 != 0 || mul_out % 4 != 0)) found = nullptr;
  GenTable* gen = nullptr;
  if (!found) {
    gen = new (std::nothrow) GenTable;
    if (!gen) return fail(TP_ERR_INVALID_ARG, "out of host memory");
    std::string why2;
    if (!build_gen_table(bi, bs, bo, paths, n_paths, path_coeff, mode == TP_MODE_UVW, *gen, why2)) {
      delete gen;
      return fail(TP_ERR_UNSUPPORTED, "%s", why2.c_str());
    }
  }
  // the fused radial projection runs through the path table for every uvu plan
  GenTable* rad = gen;
  if (mode == TP_MODE_UVU && !rad) {
    rad = new (std::nothrow) GenTable;
    std::string why3;
    if (rad && !build_gen_table(bi, bs, bo, paths, n_paths, path_coeff, false, *rad, why3)) {
      delete rad;
      rad = nullptr;
    }
  }
  tp_plan_s* pl = new (std::nothrow) tp_plan_s;
  if (!pl) {
    if (rad != gen) delete rad;
    delete gen;
    return fail(TP_ERR_INVALID_ARG, "out of host memory");
  }
  std::memset(pl, 0, sizeof(*pl));
  pl->ops = found;
  pl->gen = gen;
  pl->rad = mode == TP_MODE_UVU ? rad : nullptr;
  pl->mode = mode;
  pl->mul_in = mul_in;
  pl->mul_out = mul_out;
  int64_t in_dim = 0, out_dim = 0;
  for (auto& b : bi) in_dim += (int64_t)b.mul * (2 * b.l + 1);
  for (auto& b : bo) out_dim += (int64_t)b.mul * (2 * b.l + 1);
  pl->in_dim = in_dim;
  pl->out_dim = out_dim;
  pl->n_paths = n_paths;
  int64_t nw = 0;
  for (int p = 0; p < n_paths; ++p) nw += bi[paths[3 * p]].mul;
  pl->nw = mode == TP_MODE_UVU ? nw : n_paths;
  pl->n_shared = mode == TP_MODE_UVW ? (int64_t)n_paths * mul_in * mul_out : 0;
  pl->has_coeff = 0;
  for (int p = 0; p < kMaxPaths; ++p) pl->coeff[p] = 1.0f;
  if (path_coeff) {
    for (int p = 0; p < n_paths; ++p) {
      if (!std::isfinite(path_coeff[p])) {
        if (pl->rad != pl->gen) delete pl->rad;
        delete pl->gen;
        delete pl;
        return fail(TP_ERR_INVALID_ARG, "path_coeff[%d] is not finite", p);
      }
      pl->coeff[p] = (float)path_coeff[p];
      if (path_coeff[p] != 1.0) pl->has_coeff = 1;
    }
  }
  pl->flags = flags;
  *plan = pl;
  return TP_OK;
}

tp_status_t tp_plan_destroy(tp_plan_t plan) {
  if (plan && plan->rad != plan->gen) delete plan->rad;
  if (plan) delete plan->gen;
  delete plan;
  return TP_OK;
}

tp_status_t tp_plan_query(tp_plan_t plan, int64_t* in_dim, int64_t* out_dim, int64_t* n_edge_weights,
                          int64_t* n_shared_weights) {
  if (!plan) return fail(TP_ERR_INVALID_ARG, "plan is NULL");
  if (in_dim) *in_dim = plan->in_dim;
  if (out_dim) *out_dim = plan->out_dim;
  if (n_edge_weights) *n_edge_weights = plan->nw;
  if (n_shared_weights) *n_shared_weights = plan->n_shared;
  return TP_OK;
}

tp_status_t tp_workspace_size(tp_plan_t plan, int64_t N, int64_t E, int32_t op, size_t* bytes) {
  tp_status_t st = check_sizes(plan, N, E);
  if (st != TP_OK) return st;
  if (!bytes) return fail(TP_ERR_INVALID_ARG, "bytes is NULL");
  if (op != TP_OP_FWD && op != TP_OP_BWD && op != TP_OP_DBWD) return fail(TP_ERR_INVALID_ARG, "bad op");
  size_t need = 0;
  if (plan->mode == TP_MODE_UVW) {
    if (op == TP_OP_DBWD) return fail(TP_ERR_UNSUPPORTED, "double backward is implemented for uvu");
    need = plan->gen ? gen_uvw_layout(plan, N, E, op == TP_OP_BWD).total : uvw_layout(plan, N, E, op == TP_OP_BWD).total;
  } else if (op == TP_OP_FWD) {
    need = (plan->flags & TP_FLAG_CHECK_INDICES) ? 256 : 0;
  } else {
    need = ws_layout(N, E).total;   // enough to build the transpose in place
  }
  *bytes = need;
  return TP_OK;
}

tp_status_t tp_csr_transpose_workspace_size(int64_t N, int64_t E, size_t* bytes) {
  if (!bytes) return fail(TP_ERR_INVALID_ARG, "bytes is NULL");
  if (N < 0 || E < 0 || N >= (int64_t)1 << 31 || E >= (int64_t)1 << 31)
    return fail(TP_ERR_INVALID_ARG, "N and E must be in [0, 2^31)");
  *bytes = sizeof(int32_t) * (size_t)transpose_scratch_ints(N, E);
  return TP_OK;
}

tp_status_t tp_csr_transpose(int64_t N, int64_t E, const int32_t* rowptr, const int32_t* src,
                             int32_t* colptr, int32_t* perm, void* ws, size_t ws_bytes,
                             tp_stream_t stream) {
  (void)rowptr;
  if (N < 0 || E < 0 || N >= (int64_t)1 << 31 || E >= (int64_t)1 << 31)
    return fail(TP_ERR_INVALID_ARG, "N and E must be in [0, 2^31)");
  if (!colptr || (E > 0 && (!src || !perm))) return fail(TP_ERR_INVALID_ARG, "null pointer");
  if (!aligned4(src) || !aligned4(colptr) || !aligned4(perm)) return fail(TP_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  const size_t need = sizeof(int32_t) * (size_t)transpose_scratch_ints(N, E);
  if (!ws || ws_bytes < need) return fail(TP_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  if (reinterpret_cast<uintptr_t>(ws) & 3u) return fail(TP_ERR_INVALID_ARG, "workspace must be 4-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_csr_transpose((int)N, (int)E, src, colptr, perm, static_cast<int32_t*>(ws), s);
  if (e != cudaSuccess) return cuda_fail(e, "csr_transpose");
  return TP_OK;
}

tp_status_t tp_conv_fwd(tp_plan_t plan, int64_t N, int64_t E, const int32_t* rowptr, const int32_t* src,
                        const float* x, const float* vec, const float* w, const float* W, float* y,
                        void* ws, size_t ws_bytes, tp_stream_t stream) {
  tp_status_t st = check_sizes(plan, N, E);
  if (st != TP_OK) return st;
  if (N == 0) return TP_OK;
  if (!rowptr || !y) return fail(TP_ERR_INVALID_ARG, "rowptr and y must not be NULL");
  if (E > 0 && (!src || !x || !vec || !w)) return fail(TP_ERR_INVALID_ARG, "src, x, vec and w must not be NULL");
  if (plan->mode == TP_MODE_UVW && !W) return fail(TP_ERR_INVALID_ARG, "uvw mode needs W");
  for (const void* p : {(const void*)rowptr, (const void*)src, (const void*)x, (const void*)vec,
                        (const void*)w, (const void*)W, (const void*)y})
    if (!aligned4(p)) return fail(TP_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  size_t need = 0;
  tp_workspace_size(plan, N, E, TP_OP_FWD, &need);
  if (need > 0 && (!ws || ws_bytes < need)) return fail(TP_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  LaunchArgs a = base_args(plan, N, E);
  st = debug_prologue(plan, N, E, rowptr, src, ws, s, &a.err);
  if (st != TP_OK) return st;
  a.rowptr = rowptr;
  a.src = src;
  a.x = x;
  a.vec = vec;
  a.w = w;
  a.y = y;
  cudaError_t e;
  if (plan->mode == TP_MODE_UVW && plan->gen) {
    const UvwLayout U = gen_uvw_layout(plan, N, E, false);
    a.W = W;
    a.A = reinterpret_cast<float*>(static_cast<char*>(ws) + U.A);
    a.nw = plan->n_paths;
    e = launch_gen_uvw_fwd(a, *plan->gen, s);
  } else if (plan->mode == TP_MODE_UVW) {
    const UvwLayout U = uvw_layout(plan, N, E, false);
    char* wsb = static_cast<char*>(ws);
    a.W = W;
    a.A = reinterpret_cast<float*>(wsb + U.A);
    a.Wt = reinterpret_cast<float*>(wsb + U.Wt);
    a.nw = plan->n_paths;
    e = plan->ops->uvw_fwd(a, s);
  } else if (plan->gen) {
    e = launch_gen_fwd(a, *plan->gen, s);
  } else {
    e = plan->ops->fwd_uvu(a, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "tp_conv_fwd launch");
  return TP_OK;
}

namespace {

// Puts colptr / perm in place, building the transpose in the workspace when not supplied.
tp_status_t sender_order(int64_t N, int64_t E, const int32_t* src, const int32_t*& colptr,
                         const int32_t*& perm, void* ws, size_t ws_bytes, cudaStream_t s) {
  if ((colptr == nullptr) != (perm == nullptr))
    return fail(TP_ERR_INVALID_ARG, "colptr and perm must both be given or both be NULL");
  if (colptr) return TP_OK;
  const WsLayout L = ws_layout(N, E);
  if (!ws || ws_bytes < L.total) return fail(TP_ERR_WORKSPACE, "workspace needs %zu bytes", L.total);
  char* w = static_cast<char*>(ws);
  int32_t* cp = reinterpret_cast<int32_t*>(w + L.colptr);
  int32_t* pm = reinterpret_cast<int32_t*>(w + L.perm);
  cudaError_t e = launch_csr_transpose((int)N, (int)E, src, cp, pm, reinterpret_cast<int32_t*>(w + L.scratch), s);
  if (e != cudaSuccess) return cuda_fail(e, "csr_transpose");
  colptr = cp;
  perm = pm;
  return TP_OK;
}

}  // namespace

tp_status_t tp_conv_bwd(tp_plan_t plan, int64_t N, int64_t E, const int32_t* rowptr, const int32_t* src,
                        const int32_t* colptr, const int32_t* perm, const float* x, const float* vec,
                        const float* w, const float* W, const float* gy, float* gx, float* gw, float* gvec,
                        float* gW, void* ws, size_t ws_bytes, tp_stream_t stream) {
  tp_status_t st = check_sizes(plan, N, E);
  if (st != TP_OK) return st;
  if (N == 0) return TP_OK;
  if (!rowptr || !gy || !x) return fail(TP_ERR_INVALID_ARG, "rowptr, x and gy must not be NULL");
  if (E > 0 && (!src || !vec || !w)) return fail(TP_ERR_INVALID_ARG, "src, vec and w must not be NULL");
  if (plan->mode == TP_MODE_UVW && !W) return fail(TP_ERR_INVALID_ARG, "uvw mode needs W");
  for (const void* p : {(const void*)rowptr, (const void*)src, (const void*)colptr, (const void*)perm,
                        (const void*)x, (const void*)vec, (const void*)w, (const void*)W, (const void*)gy,
                        (const void*)gx, (const void*)gw, (const void*)gvec, (const void*)gW})
    if (!aligned4(p)) return fail(TP_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  LaunchArgs a = base_args(plan, N, E);
  st = debug_prologue(plan, N, E, rowptr, src, ws, s, &a.err);
  if (st != TP_OK) return st;
  if (!gx && !gw && !gvec && !gW) return TP_OK;
  if (plan->mode == TP_MODE_UVW) {
    size_t need = 0;
    tp_workspace_size(plan, N, E, TP_OP_BWD, &need);
    if (!ws || ws_bytes < need) return fail(TP_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  }
  st = sender_order(N, E, src, colptr, perm, ws, ws_bytes, s);
  if (st != TP_OK) return st;
  a.rowptr = rowptr;
  a.src = src;
  a.colptr = colptr;
  a.perm = perm;
  a.x = x;
  a.vec = vec;
  a.w = w;
  a.gy = gy;
  a.gx = gx;
  a.gw = gw;
  a.gvec = gvec;
  if (plan->mode == TP_MODE_UVW && plan->gen) {
    const UvwLayout U = gen_uvw_layout(plan, N, E, true);
    char* wsb = static_cast<char*>(ws);
    a.W = W;
    a.A = reinterpret_cast<float*>(wsb + U.A);
    a.G = reinterpret_cast<float*>(wsb + U.G);
    a.part = reinterpret_cast<float*>(wsb + U.part);
    a.splits = uvw_splits(N);
    a.gW = gW;
    a.nw = plan->n_paths;
    cudaError_t e = launch_gen_uvw_bwd(a, *plan->gen, s);
    if (e != cudaSuccess) return cuda_fail(e, "tp_conv_bwd (uvw) launch");
    return TP_OK;
  }
  if (plan->mode == TP_MODE_UVW) {
    const UvwLayout U = uvw_layout(plan, N, E, true);
    char* wsb = static_cast<char*>(ws);
    a.W = W;
    a.A = reinterpret_cast<float*>(wsb + U.A);
    a.G = reinterpret_cast<float*>(wsb + U.G);
    a.Wt = reinterpret_cast<float*>(wsb + U.Wt);
    a.xT = reinterpret_cast<float*>(wsb + U.xT);
    a.part = reinterpret_cast<float*>(wsb + U.part);
    a.splits = uvw_splits(N);
    a.gW = gW;
    a.nw = plan->n_paths;
    cudaError_t e = plan->ops->uvw_bwd(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "tp_conv_bwd (uvw) launch");
    return TP_OK;
  }
  if (plan->gen) {
    cudaError_t e = launch_gen_bwd(a, *plan->gen, s);
    if (e != cudaSuccess) return cuda_fail(e, "tp_conv_bwd launch");
    return TP_OK;
  }
  if (gvec) {
    const int nsl = a.n_slices <= 1 ? 1 : (a.n_slices == 2 ? 2 : 4);
    while (a.split * nsl > 4) a.split >>= 1;
  }
  cudaError_t e = plan->ops->bwd_uvu(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "tp_conv_bwd launch");
  return TP_OK;
}

tp_status_t tp_conv_dbwd(tp_plan_t plan, int64_t N, int64_t E, const int32_t* rowptr, const int32_t* src,
                         const int32_t* colptr, const int32_t* perm, const float* x, const float* vec,
                         const float* w, const float* W, const float* gy, const float* ggx, const float* ggw,
                         const float* ggvec, float* g_gy, float* g_x, float* g_w, float* g_vec, void* ws,
                         size_t ws_bytes, tp_stream_t stream) {
  tp_status_t st = check_sizes(plan, N, E);
  if (st != TP_OK) return st;
  if (N == 0) return TP_OK;
  (void)W;
  if (plan->mode != TP_MODE_UVU) return fail(TP_ERR_UNSUPPORTED, "double backward is implemented for uvu");
  if (!rowptr || !gy || !x) return fail(TP_ERR_INVALID_ARG, "rowptr, x and gy must not be NULL");
  if (E > 0 && (!src || !vec || !w)) return fail(TP_ERR_INVALID_ARG, "src, vec and w must not be NULL");
  for (const void* p : {(const void*)rowptr, (const void*)src, (const void*)colptr, (const void*)perm,
                        (const void*)x, (const void*)vec, (const void*)w, (const void*)gy, (const void*)ggx,
                        (const void*)ggw, (const void*)ggvec, (const void*)g_gy, (const void*)g_x,
                        (const void*)g_w, (const void*)g_vec})
    if (!aligned4(p)) return fail(TP_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  LaunchArgs a = base_args(plan, N, E);
  st = debug_prologue(plan, N, E, rowptr, src, ws, s, &a.err);
  if (st != TP_OK) return st;
  a.rowptr = rowptr;
  a.src = src;
  a.x = x;
  a.vec = vec;
  a.w = w;
  a.gy = gy;
  a.ggx = ggx;
  a.ggw = ggw;
  a.ggvec = ggvec;
  if (g_gy) {
    a.y = g_gy;
    cudaError_t e = plan->gen ? launch_gen_dbwd(a, *plan->gen, true, false, s) : plan->ops->dbwd_recv(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "tp_conv_dbwd receiver pass");
  }
  if (!g_x && !g_w && !g_vec) return TP_OK;
  st = sender_order(N, E, src, colptr, perm, ws, ws_bytes, s);
  if (st != TP_OK) return st;
  a.colptr = colptr;
  a.perm = perm;
  a.gx = g_x;
  a.gw = g_w;
  a.gvec = g_vec;
  if (plan->gen) {
    cudaError_t e = launch_gen_dbwd(a, *plan->gen, false, true, s);
    if (e != cudaSuccess) return cuda_fail(e, "tp_conv_dbwd sender pass");
    return TP_OK;
  }
  if (g_vec) {
    const int nsl = a.n_slices <= 1 ? 1 : (a.n_slices == 2 ? 2 : 4);
    while (a.split * nsl > 4) a.split >>= 1;
  }
  cudaError_t e = plan->ops->dbwd_send(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "tp_conv_dbwd sender pass");
  return TP_OK;
}

tp_status_t tp_radial_workspace_size(tp_plan_t plan, int64_t N, int64_t E, int32_t H, int32_t op, size_t* bytes) {
  RadArgs a;
  tp_status_t st = radial_args(plan, N, E, H, a);
  if (st != TP_OK) return st;
  if (!bytes) return fail(TP_ERR_INVALID_ARG, "bytes is NULL");
  if (op == TP_OP_FWD) *bytes = (plan->flags & TP_FLAG_CHECK_INDICES) ? 256 : 0;
  else if (op == TP_OP_BWD) *bytes = rad_layout(a).total;
  else return fail(TP_ERR_UNSUPPORTED, "the fused radial projection has a forward and a backward");
  return TP_OK;
}

tp_status_t tp_conv_fwd_radial(tp_plan_t plan, int64_t N, int64_t E, int32_t H, const int32_t* rowptr,
                               const int32_t* src, const float* x, const float* vec, const float* h,
                               const float* Wr, float* y, void* ws, size_t ws_bytes, tp_stream_t stream) {
  RadArgs a;
  tp_status_t st = radial_args(plan, N, E, H, a);
  if (st != TP_OK) return st;
  if (N == 0) return TP_OK;
  if (!rowptr || !x || !y || !Wr) return fail(TP_ERR_INVALID_ARG, "rowptr, x, Wr and y must not be NULL");
  if (E > 0 && (!src || !vec || !h)) return fail(TP_ERR_INVALID_ARG, "src, vec and h must not be NULL");
  for (const void* p : {(const void*)rowptr, (const void*)src, (const void*)x, (const void*)vec, (const void*)h,
                        (const void*)Wr, (const void*)y})
    if (!aligned4(p)) return fail(TP_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  if ((reinterpret_cast<uintptr_t>(h) & 15u) != 0) return fail(TP_ERR_INVALID_ARG, "h must be 16-byte aligned");
  if ((plan->flags & TP_FLAG_CHECK_INDICES) && (!ws || ws_bytes < 256))
    return fail(TP_ERR_WORKSPACE, "TP_FLAG_CHECK_INDICES needs a 256-byte workspace");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = debug_prologue(plan, N, E, rowptr, src, ws, s, &a.err);
  if (st != TP_OK) return st;
  a.rowptr = rowptr;
  a.src = src;
  a.x = x;
  a.vec = vec;
  a.h = h;
  a.Wr = Wr;
  a.y = y;
  cudaError_t e = launch_rad_fwd(a, *plan->rad, s);
  if (e != cudaSuccess) return cuda_fail(e, "tp_conv_fwd_radial launch");
  return TP_OK;
}

tp_status_t tp_conv_bwd_radial(tp_plan_t plan, int64_t N, int64_t E, int32_t H, const int32_t* rowptr,
                               const int32_t* src, const int32_t* colptr, const int32_t* perm, const float* x,
                               const float* vec, const float* h, const float* Wr, const float* gy, float* gx,
                               float* gh, float* gWr, float* gvec, void* ws, size_t ws_bytes, tp_stream_t stream) {
  RadArgs a;
  tp_status_t st = radial_args(plan, N, E, H, a);
  if (st != TP_OK) return st;
  if (N == 0) {
    if (gWr && H > 0) {
      cudaError_t e = cudaMemsetAsync(gWr, 0, sizeof(float) * (size_t)H * plan->nw, reinterpret_cast<cudaStream_t>(stream));
      if (e != cudaSuccess) return cuda_fail(e, "tp_conv_bwd_radial");
    }
    return TP_OK;
  }
  if (!rowptr || !x || !gy || !Wr) return fail(TP_ERR_INVALID_ARG, "rowptr, x, Wr and gy must not be NULL");
  if (E > 0 && (!src || !vec || !h)) return fail(TP_ERR_INVALID_ARG, "src, vec and h must not be NULL");
  for (const void* p : {(const void*)rowptr, (const void*)src, (const void*)colptr, (const void*)perm,
                        (const void*)x, (const void*)vec, (const void*)h, (const void*)Wr, (const void*)gy,
                        (const void*)gx, (const void*)gh, (const void*)gWr, (const void*)gvec})
    if (!aligned4(p)) return fail(TP_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  if ((reinterpret_cast<uintptr_t>(h) & 15u) != 0) return fail(TP_ERR_INVALID_ARG, "h must be 16-byte aligned");
  if (!gx && !gh && !gWr && !gvec) return TP_OK;
  const RadLayout L = rad_layout(a);
  if (!ws || ws_bytes < L.total) return fail(TP_ERR_WORKSPACE, "workspace needs %zu bytes", L.total);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = debug_prologue(plan, N, E, rowptr, src, ws, s, &a.err);
  if (st != TP_OK) return st;
  st = sender_order(N, E, src, colptr, perm, ws, ws_bytes, s);
  if (st != TP_OK) return st;
  char* wsb = static_cast<char*>(ws);
  a.rowptr = rowptr;
  a.src = src;
  a.colptr = colptr;
  a.perm = perm;
  a.x = x;
  a.vec = vec;
  a.h = h;
  a.Wr = Wr;
  a.gy = gy;
  a.gx = gx;
  a.gh = gh;
  a.gvec = gvec;
  a.gWr = gWr;
  a.WrT = reinterpret_cast<float*>(wsb + L.WrT);
  a.part = reinterpret_cast<float*>(wsb + L.part);
  cudaError_t e = launch_rad_bwd(a, *plan->rad, s);
  if (e != cudaSuccess) return cuda_fail(e, "tp_conv_bwd_radial launch");
  return TP_OK;
}

tp_status_t tp_get_device_error(tp_plan_t plan, void* ws, tp_stream_t stream, int32_t* code) {
  if (!code) return fail(TP_ERR_INVALID_ARG, "code must not be NULL");
  *code = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!plan || !(plan->flags & TP_FLAG_CHECK_INDICES)) {
    int* word = device_error_word();
    if (!word) return fail(TP_ERR_CUDA, "device error word unavailable");
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, word, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemsetAsync(word, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return cuda_fail(e, "tp_get_device_error");
    *code = v;
    return TP_OK;
  }
  if (!ws) return fail(TP_ERR_WORKSPACE, "workspace is NULL");
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(int32_t), s);
  if (e != cudaSuccess) return cuda_fail(e, "tp_get_device_error");
  *code = v;
  return TP_OK;
}

}  // extern "C"
