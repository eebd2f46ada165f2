// C ABI of the blocked Shampoo step (include/shampoo.h): argument checking,
// caller-owned state / scratch layout, and the order of work in one step.
//
// Step order ("Shampoo optimizer" notes, matrix-case listing: preconditioners
// first, then the parameters; podcast "Preconditioned optimization without the
// full matrix cost", cue 28: roots recomputed only every so many steps):
//   1. stack     gradient blocks -> Gs (B x B) and Gt (transposed), zero-padded
//   2. stats     L <- beta L + Gs Gs^T, R <- beta R + Gt Gt^T     (one GEMM launch)
//   3. roots     if step % refresh_every == 0: XL, XR of the damped, scaled stats
//   4. apply     T = XL G (GEMM; on other steps it joins the launch of 2), then
//                W -= lr T XR fused into the second GEMM's epilogue, masked to
//                each block's real extent.
#include <algorithm>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/shampoo.h"
#include "internal.h"

using namespace shampoo;

namespace {

constexpr size_t kAlignBytes = 256;
constexpr size_t kRootBudget = size_t(16) << 30;  // solver scratch per step (chunks beyond)

size_t al(size_t x) { return (x + kAlignBytes - 1) / kAlignBytes * kAlignBytes; }

struct Shapes {
  int nb = 0;
  std::vector<int> table;  // nb x {param, row0, col0, r, c}
};

int validate_config(const shampoo_config* c) {
  if (!c) return set_error(SHAMPOO_ERR_INVALID_ARG, "config is NULL");
  if (c->block < 32 || c->block > 1024 || c->block % 32)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "block %d: need a multiple of 32 in [32, 1024]", c->block);
  if (!(c->beta >= 0.f) || !(c->beta <= 1.f)) return set_error(SHAMPOO_ERR_INVALID_ARG, "beta must be in [0, 1]");
  if (!(c->eps >= 0.f)) return set_error(SHAMPOO_ERR_INVALID_ARG, "eps must be >= 0");
  if (!(c->lr == c->lr)) return set_error(SHAMPOO_ERR_INVALID_ARG, "lr is NaN");
  if (c->root_p != 2 && c->root_p != 4) return set_error(SHAMPOO_ERR_INVALID_ARG, "root_p must be 2 or 4");
  if (c->solver < 0 || c->solver > kMaxSolver) return set_error(SHAMPOO_ERR_INVALID_ARG, "unknown solver %d", c->solver);
  if (c->solver != SHAMPOO_SOLVER_CHEBYSHEV && (c->iters < 1 || c->iters > 1000))
    return set_error(SHAMPOO_ERR_INVALID_ARG, "iters must be in [1, 1000]");
  if (!(c->tol >= 0.f)) return set_error(SHAMPOO_ERR_INVALID_ARG, "tol must be >= 0");
  if (c->refresh_every < 1) return set_error(SHAMPOO_ERR_INVALID_ARG, "refresh_every must be >= 1");
  if (c->solver == SHAMPOO_SOLVER_CHEBYSHEV) {
    if (c->cheb_degree < 2 || c->cheb_degree > kMaxChebDegree)
      return set_error(SHAMPOO_ERR_INVALID_ARG, "cheb_degree must be in [2, %d]", kMaxChebDegree);
    if (!(c->cheb_lo > 0.f) && !(c->eps > 0.f))
      return set_error(SHAMPOO_ERR_INVALID_ARG, "Chebyshev needs cheb_lo > 0 or eps > 0");
  }
  if (c->grad_dtype != SHAMPOO_F32 && c->grad_dtype != SHAMPOO_BF16)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "grad_dtype must be SHAMPOO_F32 or SHAMPOO_BF16");
  if (!(c->momentum >= 0.f) || !(c->momentum < 1.f))
    return set_error(SHAMPOO_ERR_INVALID_ARG, "momentum must be in [0, 1)");
  return SHAMPOO_OK;
}

int build_table(int B, int32_t nparams, const int64_t* rows, const int64_t* cols, Shapes& out) {
  if (nparams < 1 || nparams > kMaxParams)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "nparams %d: need 1..%d", nparams, kMaxParams);
  if (!rows || !cols) return set_error(SHAMPOO_ERR_INVALID_ARG, "rows/cols is NULL");
  out.table.clear();
  for (int i = 0; i < nparams; ++i) {
    if (rows[i] < 1 || cols[i] < 1 || rows[i] > (1 << 20) || cols[i] > (1 << 20))
      return set_error(SHAMPOO_ERR_INVALID_ARG, "param %d has shape %lld x %lld", i, (long long)rows[i],
                       (long long)cols[i]);
    for (int64_t r0 = 0; r0 < rows[i]; r0 += B)
      for (int64_t c0 = 0; c0 < cols[i]; c0 += B) {
        out.table.push_back(i);
        out.table.push_back(static_cast<int>(r0));
        out.table.push_back(static_cast<int>(c0));
        out.table.push_back(static_cast<int>(std::min<int64_t>(B, rows[i] - r0)));
        out.table.push_back(static_cast<int>(std::min<int64_t>(B, cols[i] - c0)));
      }
  }
  out.nb = static_cast<int>(out.table.size() / 5);
  if (out.nb > 65535) return set_error(SHAMPOO_ERR_UNSUPPORTED, "%d blocks exceed 65535", out.nb);
  return SHAMPOO_OK;
}

// State layout (bytes, each part 256-aligned):
//   status word | block table (nb x 5 int32) | valid extents (2nb int32: r of L_b, c of R_b)
//   | wrows (nb) | wcols (nb) | statistics (2nb, B, B; fp64 with the fp64-iterate solver) | roots (2nb, B, B)
//   | momentum (nb, B, B; only with momentum > 0) | power flag | power iterates (2nb, B)
// Bytes per statistics element: the fp64-iterate solver keeps L and R in
// fp64 in the blocked step (fp32 statistics would set the update's error
// floor whatever the iterates' precision).
size_t stats_elem_bytes(int solver) { return solver == SHAMPOO_SOLVER_NEWTON_CUBIC_F64 ? 8 : 4; }

struct StateLayout {
  size_t status, table, valid, wrows, wcols, stats, roots, mom, pflag, pvec, total;
};
StateLayout state_layout(int nb, int B, bool momentum, size_t stats_elem) {
  StateLayout s;
  size_t o = 0;
  s.status = o, o += al(4);
  s.table = o, o += al(size_t(nb) * 5 * 4);
  s.valid = o, o += al(size_t(2) * nb * 4);
  s.wrows = o, o += al(size_t(nb) * 4);
  s.wcols = o, o += al(size_t(nb) * 4);
  s.stats = o, o += al(plain_floats(2 * nb, B) * stats_elem);
  s.roots = o, o += al(plain_floats(2 * nb, B) * 4);
  s.mom = o;
  if (momentum) o += al(plain_floats(nb, B) * 4);
  s.pflag = o, o += al(4);
  s.pvec = o, o += al(size_t(2) * nb * B * 4);
  s.total = o;
  return s;
}
// bf16 gradients with fp32 statistics and no momentum: the first apply
// product reads the roots XL as three bf16 planes (split once per refresh) and
// G^T from the bf16 stack, all on the bf16 MMA; no fp32 G^T stack is kept.
bool apply_planes(const shampoo_config* c) {
  return c->grad_dtype == SHAMPOO_BF16 && c->solver != SHAMPOO_SOLVER_NEWTON_CUBIC_F64 && !(c->momentum > 0.f);
}
// Roots kept for several steps: the second apply product reads XR split into
// its tf32 hi and lo parts (once per refresh) instead of splitting it on chip
// every step.  With a refresh every step the split pass would cost more than
// it saves.
bool presplit_xr(const shampoo_config* c) { return c->refresh_every > 1; }

// Scratch layout: Gs | Gt (none with XL planes) | Tapply | XL planes (3 nb bf16 matrices, with XL planes only)
//   | XR split (nb tf32 hi, then nb lo matrices; with refresh_every > 1 only) | blk_wptr (nb ptrs) | blk_ld (nb)
//   | solver scratch
struct ScratchLayout {
  size_t gs, gt, tap, xlp, xrs, wptr, ld, root, root_bytes, total;
};
ScratchLayout scratch_layout(int nb, int B, int solver, int p, bool planes, bool xr_split) {
  ScratchLayout s;
  size_t o = 0;
  s.gs = o, o += al(plain_floats(nb, B) * 4);
  s.gt = o;
  if (!planes) o += al(plain_floats(nb, B) * 4);
  s.tap = o, o += al(plain_floats(nb, B) * 4);
  s.xlp = o;
  if (planes) o += al(plain_floats(nb, B) * 3 * 2);
  s.xrs = o;
  if (xr_split) o += al(plain_floats(2 * nb, B) * 4);
  s.wptr = o, o += al(size_t(nb) * 8);
  s.ld = o, o += al(size_t(nb) * 4);
  s.root = o;
  const size_t per = root_scratch_per_matrix(B, solver, p);
  const size_t want = root_scratch_header() + per * size_t(2 * nb);
  s.root_bytes = std::min(want, std::max(kRootBudget, root_scratch_header() + per));
  o += al(s.root_bytes);
  s.total = o;
  return s;
}

bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }

}  // namespace

int shampoo::build_block_table(int B, int32_t nparams, const int64_t* rows, const int64_t* cols,
                               std::vector<int>& table) {
  Shapes sh;
  int rc = build_table(B, nparams, rows, cols, sh);
  if (rc) return rc;
  table = sh.table;
  return SHAMPOO_OK;
}

struct shampoo_ctx {
  shampoo_config cfg;
  int nparams = 0;
  std::vector<int64_t> rows, cols;
  Shapes shapes;
  StateLayout sl;
  ScratchLayout xl;
  char* state = nullptr;
  char* scratch = nullptr;
  int* d_status = nullptr;
  int* d_table = nullptr;
  int* d_valid = nullptr;
  int* d_wrows = nullptr;
  int* d_wcols = nullptr;
  float* stats = nullptr;
  float* roots = nullptr;
  float* mom = nullptr;  // momentum stack (momentum > 0 only)
  float* Gs = nullptr;
  float* Gt = nullptr;
  float* Tap = nullptr;
  float** blk_wptr = nullptr;
  int* blk_ld = nullptr;
  StackMaps mGs, mGt, mRoots, mTap, mMom;
  // bf16 gradients with fp32 statistics: G and G^T also as bf16 stacks (in the
  // Gs region), the statistics' operands on the kind::f16 MMA
  uint16_t* Gs16 = nullptr;
  uint16_t* Gt16 = nullptr;
  StackMaps mGs16, mGt16;
  // XL as three bf16 planes (apply_planes): rebuilt after every refresh, and
  // before the next apply whenever the roots may have changed otherwise
  // (a new handle, shampoo_set_step after restoring a state)
  uint16_t* xlp = nullptr;
  StackMaps mXlp;
  // XR split into its tf32 hi and lo parts (the second apply's right operand),
  // rebuilt on the same schedule as the XL planes
  float* xrs = nullptr;
  StackMaps mXrs;
  bool planes_stale = true;
  double stats_flops_L = 0, stats_flops_R = 0, stack_bytes = 0;
  int64_t step = 0;
  int power_refreshed = 0;  // a refresh has stored power iterates (profiler byte count only)
  bool stats_f64 = false;   // L, R kept in fp64 (fp64-iterate solver)
  cudaStream_t last_stream = nullptr;
};

extern "C" {

const char* shampoo_status_string(int code) {
  switch (code) {
    case SHAMPOO_OK: return "SHAMPOO_OK";
    case SHAMPOO_ERR_INVALID_ARG: return "SHAMPOO_ERR_INVALID_ARG";
    case SHAMPOO_ERR_UNSUPPORTED: return "SHAMPOO_ERR_UNSUPPORTED";
    case SHAMPOO_ERR_WORKSPACE: return "SHAMPOO_ERR_WORKSPACE";
    case SHAMPOO_ERR_CUDA: return "SHAMPOO_ERR_CUDA";
    case SHAMPOO_ERR_DEVICE: return "SHAMPOO_ERR_DEVICE";
    default: return "SHAMPOO_UNKNOWN_STATUS";
  }
}

int shampoo_query_sizes(const shampoo_config* cfg, int32_t nparams, const int64_t* rows, const int64_t* cols,
                        size_t* state_bytes, size_t* scratch_bytes) {
  int rc = validate_config(cfg);
  if (rc) return rc;
  Shapes sh;
  if ((rc = build_table(cfg->block, nparams, rows, cols, sh))) return rc;
  if (!state_bytes || !scratch_bytes) return set_error(SHAMPOO_ERR_INVALID_ARG, "output pointer is NULL");
  *state_bytes = state_layout(sh.nb, cfg->block, cfg->momentum > 0.f, stats_elem_bytes(cfg->solver)).total;
  *scratch_bytes =
      scratch_layout(sh.nb, cfg->block, cfg->solver, cfg->root_p, apply_planes(cfg), presplit_xr(cfg)).total;
  return SHAMPOO_OK;
}

int shampoo_init(const shampoo_config* cfg, int32_t nparams, const int64_t* rows, const int64_t* cols, void* d_state,
                 size_t state_bytes, void* d_scratch, size_t scratch_bytes, void* stream, shampoo_handle* out) {
  int rc = validate_config(cfg);
  if (rc) return rc;
  if (!out) return set_error(SHAMPOO_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  Shapes sh;
  if ((rc = build_table(cfg->block, nparams, rows, cols, sh))) return rc;
  if (!d_state || !d_scratch) return set_error(SHAMPOO_ERR_INVALID_ARG, "state/scratch is NULL");
  if (!aligned256(d_state) || !aligned256(d_scratch))
    return set_error(SHAMPOO_ERR_UNSUPPORTED, "state/scratch must be 256-byte aligned");
  const int B = cfg->block, nb = sh.nb;
  StateLayout sl = state_layout(nb, B, cfg->momentum > 0.f, stats_elem_bytes(cfg->solver));
  ScratchLayout xl = scratch_layout(nb, B, cfg->solver, cfg->root_p, apply_planes(cfg), presplit_xr(cfg));
  if (state_bytes < sl.total) return set_error(SHAMPOO_ERR_WORKSPACE, "state %zu < %zu bytes", state_bytes, sl.total);
  if (scratch_bytes < xl.total)
    return set_error(SHAMPOO_ERR_WORKSPACE, "scratch %zu < %zu bytes", scratch_bytes, xl.total);

  shampoo_ctx* h = new (std::nothrow) shampoo_ctx;
  if (!h) return set_error(SHAMPOO_ERR_INVALID_ARG, "out of host memory");
  h->cfg = *cfg;
  h->nparams = nparams;
  h->rows.assign(rows, rows + nparams);
  h->cols.assign(cols, cols + nparams);
  h->shapes = sh;
  h->sl = sl;
  h->xl = xl;
  h->state = static_cast<char*>(d_state);
  h->scratch = static_cast<char*>(d_scratch);
  h->d_status = reinterpret_cast<int*>(h->state + sl.status);
  h->d_table = reinterpret_cast<int*>(h->state + sl.table);
  h->d_valid = reinterpret_cast<int*>(h->state + sl.valid);
  h->d_wrows = reinterpret_cast<int*>(h->state + sl.wrows);
  h->d_wcols = reinterpret_cast<int*>(h->state + sl.wcols);
  h->stats = reinterpret_cast<float*>(h->state + sl.stats);
  h->stats_f64 = cfg->solver == SHAMPOO_SOLVER_NEWTON_CUBIC_F64;
  h->roots = reinterpret_cast<float*>(h->state + sl.roots);
  h->mom = cfg->momentum > 0.f ? reinterpret_cast<float*>(h->state + sl.mom) : nullptr;
  h->Gs = reinterpret_cast<float*>(h->scratch + xl.gs);
  h->Gt = apply_planes(cfg) ? nullptr : reinterpret_cast<float*>(h->scratch + xl.gt);
  h->xlp = apply_planes(cfg) ? reinterpret_cast<uint16_t*>(h->scratch + xl.xlp) : nullptr;
  h->xrs = presplit_xr(cfg) ? reinterpret_cast<float*>(h->scratch + xl.xrs) : nullptr;
  h->Tap = reinterpret_cast<float*>(h->scratch + xl.tap);
  h->blk_wptr = reinterpret_cast<float**>(h->scratch + xl.wptr);
  if (cfg->grad_dtype == SHAMPOO_BF16 && !h->stats_f64) {
    h->Gs16 = reinterpret_cast<uint16_t*>(h->scratch + xl.gs);
    h->Gt16 = h->Gs16 + plain_floats(nb, B);
  }
  h->blk_ld = reinterpret_cast<int*>(h->scratch + xl.ld);

  std::vector<int> valid(2 * nb), wr(nb), wc(nb);
  double fl = 0, fr = 0, sb = 0;
  for (int b = 0; b < nb; ++b) {
    const double r = sh.table[5 * b + 3], c = sh.table[5 * b + 4];
    valid[b] = sh.table[5 * b + 3];
    valid[nb + b] = sh.table[5 * b + 4];
    wr[b] = sh.table[5 * b + 3];
    wc[b] = sh.table[5 * b + 4];
    fl += 2 * r * r * c;
    fr += 2 * r * c * c;
    // G read; G and G^T written: fp32 (or bf16 both plus fp32 G^T), bf16 both with XL planes
    sb += r * c * (cfg->grad_dtype == SHAMPOO_BF16 ? 2 : 4) + (apply_planes(cfg) ? 4.0 : 8.0) * B * B;
    if (cfg->momentum > 0.f) sb += 8.0 * B * B;                                 // M read and written
  }
  h->stats_flops_L = fl / nb;
  h->stats_flops_R = fr / nb;
  h->stack_bytes = sb;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  auto up = [&](void* dst, const void* src, size_t bytes) {
    return check_cuda(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, st), "upload block table");
  };
  if ((rc = up(h->d_table, sh.table.data(), sh.table.size() * 4)) || (rc = up(h->d_valid, valid.data(), valid.size() * 4)) ||
      (rc = up(h->d_wrows, wr.data(), wr.size() * 4)) || (rc = up(h->d_wcols, wc.data(), wc.size() * 4)) ||
      (rc = check_cuda(cudaMemsetAsync(h->d_status, 0, 4, st), "zero status")) ||
      (rc = check_cuda(cudaMemsetAsync(h->stats, 0, plain_floats(2 * nb, B) * stats_elem_bytes(cfg->solver), st),
                       "zero statistics")) ||
      (rc = check_cuda(cudaMemsetAsync(h->roots, 0, plain_floats(2 * nb, B) * 4, st), "zero roots")) ||
      (h->mom && (rc = check_cuda(cudaMemsetAsync(h->mom, 0, plain_floats(nb, B) * 4, st), "zero momentum"))) ||
      (rc = check_cuda(cudaMemsetAsync(h->state + sl.pflag, 0, sl.total - sl.pflag, st), "zero power store")) ||
      (rc = check_cuda(cudaStreamSynchronize(st), "init sync"))) {
    delete h;
    return rc;
  }
  if ((rc = make_stack_maps(h->mGs, h->Gs, nb, B)) || (h->Gt && (rc = make_stack_maps(h->mGt, h->Gt, nb, B))) ||
      (h->xlp && (rc = make_stack_maps_bf16(h->mXlp, h->xlp, 3 * int64_t(nb), B))) ||
      (h->xrs && (rc = make_stack_maps(h->mXrs, h->xrs, 2 * int64_t(nb), B))) ||
      (rc = make_stack_maps(h->mRoots, h->roots, 2 * nb, B)) || (rc = make_stack_maps(h->mTap, h->Tap, nb, B)) ||
      (h->mom && (rc = make_stack_maps(h->mMom, h->mom, nb, B))) ||
      (h->Gs16 && ((rc = make_stack_maps_bf16(h->mGs16, h->Gs16, nb, B)) ||
                   (rc = make_stack_maps_bf16(h->mGt16, h->Gt16, nb, B))))) {
    delete h;
    return rc;
  }
  *out = h;
  return SHAMPOO_OK;
}

int shampoo_step(shampoo_handle h, float* const* d_weights, const void* const* d_grads, void* stream) {
  return shampoo_step_strided(h, d_weights, d_grads, nullptr, stream);
}

int shampoo_step_strided(shampoo_handle h, float* const* d_weights, const void* const* d_grads, const int64_t* ld,
                         void* stream) {
  if (!h) return set_error(SHAMPOO_ERR_INVALID_ARG, "handle is NULL");
  if (!d_weights || !d_grads) return set_error(SHAMPOO_ERR_INVALID_ARG, "weights/grads array is NULL");
  const shampoo_config& c = h->cfg;
  const int B = c.block, nb = h->shapes.nb;
  StackArgs args;
  for (int i = 0; i < h->nparams; ++i) {
    if (!d_weights[i] || !d_grads[i]) return set_error(SHAMPOO_ERR_INVALID_ARG, "param %d has a NULL pointer", i);
    const int64_t ldi = ld ? ld[i] : h->cols[i];
    if (ldi < h->cols[i] || ldi > 0x7fffffff)
      return set_error(SHAMPOO_ERR_INVALID_ARG, "param %d: row stride %lld outside [cols, 2^31)", i,
                       static_cast<long long>(ldi));
    args.g[i] = d_grads[i];
    args.w[i] = d_weights[i];
    args.ld[i] = static_cast<int>(ldi);
    // 16-byte (fp32) / 8-byte (bf16) gradient loads need every row aligned.
    const size_t esize = c.grad_dtype == SHAMPOO_BF16 ? 2 : 4;
    args.vec[i] = (ldi % 4 == 0 && reinterpret_cast<uintptr_t>(d_grads[i]) % (4 * esize) == 0) ? 1 : 0;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  int rc;
  // 1. partition / stack (and, with momentum, M <- alpha M + G per block)
  if ((rc = launch_stack(args, h->d_table, nb, B, c.grad_dtype, h->Gs, h->Gt, h->mom, c.momentum, 1.f,
                         h->blk_wptr, h->blk_ld, st, h->stack_bytes, h->Gs16, h->Gt16)))
    return rc;
  // Widened bf16 gradients are exact in tf32: their lo parts are zero, so
  // the products that take G as an operand skip the MMAs with those parts.
  const int g_exact = c.grad_dtype == SHAMPOO_BF16 ? 1 : 0;
  // 2. statistics: L <- beta L + G G^T (first nb matrices), R <- beta R + G^T G (next nb).
  // On steps that keep the previous roots, the first apply product T = XL G
  // (T = XL M with momentum, M read as a true product) depends on neither, so
  // it joins the same launch.
  const bool refresh = h->step % c.refresh_every == 0;
  // The apply products' split forms of the roots: XL as bf16 planes (bf16
  // gradients), XR as tf32 hi and lo parts.
  auto split_roots = [&]() -> int {
    int r;
    const int64_t cnt = plain_floats(nb, B);
    if (h->xlp && (r = launch_split_planes(h->roots, cnt, h->xlp, st))) return r;
    if (h->xrs && (r = launch_split_tf32(h->roots + cnt, cnt, h->xrs, h->xrs + cnt, st))) return r;
    h->planes_stale = false;
    return SHAMPOO_OK;
  };
  if (h->planes_stale && !refresh && (rc = split_roots())) return rc;  // roots not split since they were set
  auto add_apply1 = [&](Builder& b) {
    if (h->xlp) {  // T = (XL0 + XL1 + XL2) G: three bf16 planes of XL against G^T in bf16
      Epilogue& e = b.add(nb, B, h->mXlp, 0, h->mGt16, 0, h->stats_flops_L);
      b.L.g[b.L.ngroups - 1].a_planes = 3;
      b.L.g[b.L.ngroups - 1].a_plane_stride = nb;
      e.D = h->Tap;
      e.flags = h->d_status;
    } else if (h->mom) {
      Epilogue& e = b.add(nb, B, h->mRoots, 0, h->mMom, 0, h->stats_flops_L, B_MN_MAJOR);
      e.D = h->Tap;
      e.flags = h->d_status;
    } else {
      Epilogue& e = b.add(nb, B, h->mRoots, 0, h->mGt, 0, h->stats_flops_L);
      b.L.g[b.L.ngroups - 1].b_exact = g_exact;
      e.D = h->Tap;
      e.flags = h->d_status;
    }
  };
  if (h->stats_f64) {
    // fp64 statistics: L <- beta L + Gs Gt and R <- beta R + Gt Gs (Gt = Gs^T,
    // true products) on the fp64 MMA, the fp32 stacks widened exactly
    double* L64 = reinterpret_cast<double*>(h->stats);
    DGemmGroup g[2];
    g[0].A = h->Gs;
    g[0].B = h->Gt;
    g[0].C = L64;
    g[0].D = L64;
    g[0].beta = c.beta;
    g[1].A = h->Gt;
    g[1].B = h->Gs;
    g[1].C = L64 + plain_floats(nb, B);
    g[1].D = L64 + plain_floats(nb, B);
    g[1].beta = c.beta;
    // symmetric: the tiles below the diagonal are filled in on refresh steps
    if ((rc = launch_dgemm(g, 2, nb, B, nullptr, nullptr, h->d_status, st, true, true))) return rc;
    if (refresh && (rc = launch_mirror_lower_f64(L64, 2 * int64_t(nb), B, st))) return rc;
    if (!refresh) {
      Builder b;
      add_apply1(b);
      if ((rc = b.launch(st))) return rc;
    }
  } else {
    Builder b;
    // bf16 gradients: both statistics products on the kind::f16 MMA (G exact in bf16)
    Epilogue& eL = b.add(nb, B, h->Gs16 ? h->mGs16 : h->mGs, 0, h->Gs16 ? h->mGs16 : h->mGs, 0, h->stats_flops_L);
    b.L.g[0].a_exact = b.L.g[0].b_exact = g_exact;
    b.L.g[0].sym = 1;  // symmetric: the tiles below the diagonal come from the mirror pass
    eL.beta = c.beta;
    eL.C = h->stats;
    eL.D = h->stats;
    eL.flags = h->d_status;
    Epilogue& eR = b.add(nb, B, h->Gs16 ? h->mGt16 : h->mGt, 0, h->Gs16 ? h->mGt16 : h->mGt, 0, h->stats_flops_R);
    b.L.g[1].a_exact = b.L.g[1].b_exact = g_exact;
    b.L.g[1].sym = 1;
    eR.beta = c.beta;
    eR.C = h->stats + plain_floats(nb, B);
    eR.D = h->stats + plain_floats(nb, B);
    eR.flags = h->d_status;
    if (!refresh) add_apply1(b);
    if ((rc = b.launch(st))) return rc;
    // Only the roots read the tiles below the diagonal, so they are filled in
    // on refresh steps alone (shampoo_sync_statistics fills them for readers).
    if (refresh && (rc = launch_mirror_lower(h->stats, 2 * nb, B, st))) return rc;
  }
  // 3. roots of all 2 nb damped statistics, every refresh_every steps
  if (refresh) {
    RootJob job;
    job.batch = 2 * nb;
    job.n = B;
    job.p = c.root_p;
    job.solver = c.solver;
    job.iters = c.iters;
    job.cheb_degree = c.cheb_degree;
    job.eps = c.eps;
    job.tol = c.tol;
    job.cheb_lo = c.cheb_lo;
    job.A = h->stats_f64 ? nullptr : h->stats;
    job.A64 = h->stats_f64 ? reinterpret_cast<const double*>(h->stats) : nullptr;
    job.valid = h->d_valid;
    job.X = h->roots;
    job.iters_used = nullptr;
    job.flags = h->d_status;
    if (!h->stats_f64) {  // fp64 statistics are scaled by their Frobenius norm
      job.power_vec = reinterpret_cast<float*>(h->state + h->sl.pvec);
      job.power_warm = reinterpret_cast<int*>(h->state + h->sl.pflag);
    }
    job.power_warm_hint = h->power_refreshed;
    if ((rc = run_inverse_roots(job, h->scratch + h->xl.root, h->xl.root_bytes, st))) return rc;
    h->power_refreshed = 1;
    if ((rc = split_roots())) return rc;
    // 4a. apply, first product: T = XL G (with the fresh roots)
    Builder b;
    add_apply1(b);
    if ((rc = b.launch(st))) return rc;
  }
  // 4b. apply, second product: W -= lr T XR (masked scatter into the weights)
  {
    Builder b;
    Epilogue& e = h->xrs ? b.add(nb, B, h->mTap, 0, h->mXrs, 0, h->stats_flops_R)  // XR as its hi and lo parts
                         : b.add(nb, B, h->mTap, 0, h->mRoots, nb, h->stats_flops_R);
    if (h->xrs) {
      b.L.g[0].b_presplit = 1;
      b.L.g[0].b_plane_stride = nb;
    }
    e.wptr = h->blk_wptr;
    e.wld = h->blk_ld;
    e.wrows = h->d_wrows;
    e.wcols = h->d_wcols;
    e.lr = c.lr;
    e.flags = h->d_status;
    if ((rc = b.launch(st))) return rc;
  }
  h->step += 1;
  return SHAMPOO_OK;
}

int shampoo_get_status(shampoo_handle h, int32_t* status, int32_t reset) {
  if (!h || !status) return set_error(SHAMPOO_ERR_INVALID_ARG, "handle/status is NULL");
  int rc = check_cuda(cudaStreamSynchronize(h->last_stream), "status sync");
  if (rc) return rc;
  int v = 0;
  if ((rc = check_cuda(cudaMemcpy(&v, h->d_status, 4, cudaMemcpyDeviceToHost), "read status"))) return rc;
  *status = v;
  if (reset && (rc = check_cuda(cudaMemset(h->d_status, 0, 4), "reset status"))) return rc;
  return SHAMPOO_OK;
}

int shampoo_block_table(shampoo_handle h, int32_t* nb, int64_t* table) {
  if (!h || !nb) return set_error(SHAMPOO_ERR_INVALID_ARG, "handle/nb is NULL");
  *nb = h->shapes.nb;
  if (table)
    for (size_t i = 0; i < h->shapes.table.size(); ++i) table[i] = h->shapes.table[i];
  return SHAMPOO_OK;
}

int shampoo_state_views(shampoo_handle h, float** L, float** R, float** rootL, float** rootR, int64_t* step) {
  if (!h) return set_error(SHAMPOO_ERR_INVALID_ARG, "handle is NULL");
  const int nb = h->shapes.nb, B = h->cfg.block;
  if (L) *L = h->stats;
  if (R)  // R follows the nb L matrices, whose elements are fp64 with the fp64-iterate solver
    *R = h->stats_f64 ? reinterpret_cast<float*>(reinterpret_cast<double*>(h->stats) + plain_floats(nb, B))
                      : h->stats + plain_floats(nb, B);
  if (rootL) *rootL = h->roots;
  if (rootR) *rootR = h->roots + plain_floats(nb, B);
  if (step) *step = h->step;
  return SHAMPOO_OK;
}

int shampoo_sync_statistics(shampoo_handle h, void* stream) {
  if (!h) return set_error(SHAMPOO_ERR_INVALID_ARG, "handle is NULL");
  const int64_t batch = 2 * int64_t(h->shapes.nb);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (h->stats_f64) return launch_mirror_lower_f64(reinterpret_cast<double*>(h->stats), batch, h->cfg.block, st);
  return launch_mirror_lower(h->stats, batch, h->cfg.block, st);
}

int shampoo_momentum_view(shampoo_handle h, float** M) {
  if (!h || !M) return set_error(SHAMPOO_ERR_INVALID_ARG, "handle/M is NULL");
  *M = h->mom;
  return SHAMPOO_OK;
}

int shampoo_set_step(shampoo_handle h, int64_t step) {
  if (!h || step < 0) return set_error(SHAMPOO_ERR_INVALID_ARG, "bad handle or step");
  h->step = step;
  h->planes_stale = true;  // the roots may have been restored
  return SHAMPOO_OK;
}

void shampoo_destroy(shampoo_handle h) { delete h; }

int inv_root_scratch_bytes(int64_t batch, int32_t n, int32_t solver, size_t* bytes) {
  return inv_root_scratch_bytes_p(batch, n, solver, 4, bytes);
}

int inv_root_scratch_bytes_p(int64_t batch, int32_t n, int32_t solver, int32_t p, size_t* bytes) {
  if (!bytes) return set_error(SHAMPOO_ERR_INVALID_ARG, "bytes is NULL");
  if (batch < 0 || n < 32 || n > 1024 || n % 32 || solver < 0 || solver > kMaxSolver)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "bad batch / n / solver");
  if (p != 2 && p != 4 && p != 6 && p != 8) return set_error(SHAMPOO_ERR_INVALID_ARG, "p must be 2, 4, 6 or 8");
  *bytes = root_scratch_header() +
           root_scratch_per_matrix(n, solver, p) * static_cast<size_t>(std::max<int64_t>(batch, 1));
  return SHAMPOO_OK;
}

}  // extern "C"

int shampoo::inv_root_batched_impl(const float* d_A, float* d_X, int64_t batch, int n, int p, float eps, int solver,
                                   int iters, float tol, int cheb_degree, float cheb_lo, void* d_scratch,
                                   size_t scratch_bytes, int* d_iters_used, int* d_status, cudaStream_t st,
                                   bool plain_launches) {
  if (batch < 0) return set_error(SHAMPOO_ERR_INVALID_ARG, "batch < 0");
  if (batch == 0) return SHAMPOO_OK;
  if (!d_A || !d_X || !d_scratch) return set_error(SHAMPOO_ERR_INVALID_ARG, "NULL device pointer");
  if (n < 32 || n > 1024 || n % 32) return set_error(SHAMPOO_ERR_INVALID_ARG, "n %d: need a multiple of 32 in [32, 1024]", n);
  if (p != 2 && p != 4 && p != 6 && p != 8) return set_error(SHAMPOO_ERR_INVALID_ARG, "p must be 2, 4, 6 or 8");
  if (solver == SHAMPOO_SOLVER_NEWTON_DB && p > 4)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "Newton-DB computes p = 2 and p = 4 only");
  if (!(eps >= 0.f)) return set_error(SHAMPOO_ERR_INVALID_ARG, "eps must be >= 0");
  if (solver < 0 || solver > kMaxSolver) return set_error(SHAMPOO_ERR_INVALID_ARG, "unknown solver %d", solver);
  if (solver != SHAMPOO_SOLVER_CHEBYSHEV && (iters < 1 || iters > 1000))
    return set_error(SHAMPOO_ERR_INVALID_ARG, "iters must be in [1, 1000]");
  if (!(tol >= 0.f)) return set_error(SHAMPOO_ERR_INVALID_ARG, "tol must be >= 0");
  if (solver == SHAMPOO_SOLVER_CHEBYSHEV) {
    if (cheb_degree < 2 || cheb_degree > kMaxChebDegree)
      return set_error(SHAMPOO_ERR_INVALID_ARG, "cheb_degree must be in [2, %d]", kMaxChebDegree);
    if (!(cheb_lo > 0.f) && !(eps > 0.f))
      return set_error(SHAMPOO_ERR_INVALID_ARG, "Chebyshev needs cheb_lo > 0 or eps > 0");
  }
  if (!aligned256(d_scratch) || (reinterpret_cast<uintptr_t>(d_A) & 15) || (reinterpret_cast<uintptr_t>(d_X) & 15))
    return set_error(SHAMPOO_ERR_UNSUPPORTED, "scratch must be 256-byte and A, X 16-byte aligned");
  RootJob job;
  job.batch = batch;
  job.n = n;
  job.p = p;
  job.solver = solver;
  job.iters = iters;
  job.cheb_degree = cheb_degree;
  job.eps = eps;
  job.tol = tol;
  job.cheb_lo = cheb_lo;
  job.A = d_A;
  job.valid = nullptr;
  job.X = d_X;
  job.iters_used = d_iters_used;
  job.flags = d_status;
  job.plain_launches = plain_launches ? 1 : 0;
  return run_inverse_roots(job, d_scratch, scratch_bytes, st);
}

extern "C" {

int inv_root_batched(const float* d_A, float* d_X, int64_t batch, int32_t n, int32_t p, float eps, int32_t solver,
                     int32_t iters, float tol, int32_t cheb_degree, float cheb_lo, void* d_scratch,
                     size_t scratch_bytes, int32_t* d_iters_used, int32_t* d_status, void* stream) {
  return inv_root_batched_impl(d_A, d_X, batch, n, p, eps, solver, iters, tol, cheb_degree, cheb_lo, d_scratch,
                               scratch_bytes, d_iters_used, d_status, static_cast<cudaStream_t>(stream), false);
}


int shampoo_gemm_scratch_bytes(int64_t batch, int32_t n, size_t* bytes) {
  if (!bytes || batch < 0 || n < 32 || n > 4096 || n % 32)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "bad arguments");
  *bytes = 0;  // the operands are read in place
  return SHAMPOO_OK;
}

int shampoo_gemm_batched(const float* d_A, const float* d_B, const float* d_C, float* d_D, int64_t batch, int32_t n,
                         int32_t op_b, float alpha, float beta, float gamma, void* d_scratch, size_t scratch_bytes,
                         int32_t* d_status, void* stream) {
  (void)d_scratch;
  (void)scratch_bytes;
  if (batch < 0 || n < 32 || n > 4096 || n % 32) return set_error(SHAMPOO_ERR_INVALID_ARG, "bad batch / n");
  if (op_b != 0 && op_b != 1) return set_error(SHAMPOO_ERR_INVALID_ARG, "op_b must be 0 (B^T) or 1 (B)");
  if (batch == 0) return SHAMPOO_OK;
  if (batch > 0x7fffffff / 32) return set_error(SHAMPOO_ERR_UNSUPPORTED, "batch too large");
  if (!d_A || !d_B || !d_D) return set_error(SHAMPOO_ERR_INVALID_ARG, "NULL device pointer");
  if ((reinterpret_cast<uintptr_t>(d_A) & 15) || (reinterpret_cast<uintptr_t>(d_B) & 15) ||
      (reinterpret_cast<uintptr_t>(d_D) & 15) || (reinterpret_cast<uintptr_t>(d_C) & 15))
    return set_error(SHAMPOO_ERR_UNSUPPORTED, "A, B, C, D must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc;
  StackMaps ma, mb;
  if ((rc = make_stack_maps(ma, d_A, batch, n)) || (rc = make_stack_maps(mb, d_B, batch, n))) return rc;
  Builder b;
  Epilogue& e = b.add(static_cast<int>(batch), n, ma, 0, mb, 0, 2.0 * n * double(n) * n,
                      op_b ? B_MN_MAJOR : B_TRANSPOSED);
  e.alpha = alpha;
  e.beta = d_C ? beta : 0.f;
  e.gamma = gamma;
  e.C = d_C;
  e.D = d_D;
  e.flags = d_status;
  return b.launch(st);
}

}  // extern "C"
