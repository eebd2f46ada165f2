// Batched inverse p-th roots X_i ~ (A_i + eps I)^{-1/p} of stacked symmetric
// matrices: host-side driver of the tensor-core GEMM and the prologue /
// check / output kernels.
//
// The pages name the solvers (DASH abstract: Newton-DB iteration and Chebyshev
// polynomial approximation for inverse matrix roots; matrix scaling) without
// defining them.  The iterations implemented here are published methods:
//   coupled Newton  (Guo & Higham 2006): X0 = I, M0 = A'; T = ((p+1) I - M)/p;
//                   X <- X T; M <- T^p M   (4 GEMMs per iteration for p = 4,
//                   3 for p = 2);
//   coupled Newton, second-degree correction: the same coupled form with T
//                   the degree-2 truncation of the binomial series of
//                   M^{-1/p} = (I - (I - M))^{-1/p}; the degree-1 truncation is
//                   the Newton T above.  One more GEMM per iteration (T is
//                   formed from D = I - M, which the M update writes, as
//                   c2 D D + c1 D + I), cubic local convergence, and an
//                   eigenvalue mu << 1 of M grows by (1 + c1 + c2)^p instead
//                   of ((p+1)/p)^p per iteration (3.91 against 2.44 at p = 4);
//                   the first iteration is a plain Newton step;
//   Newton-DB       coupled Denman-Beavers-family square-root iteration in its
//                   multiplication-only form: Y0 = A', Z0 = I;
//                   T = (3 I - Z Y)/2; Y <- Y T; Z <- T Z (3 GEMMs); p = 4 runs
//                   a second stage on Y ~ A'^{1/2};
//   Chebyshev       Clenshaw evaluation of the degree-d interpolant of x^{-1/p}
//                   on [a, 1] (d - 1 GEMMs).
// Operand orientation.  The iterates are symmetric in exact arithmetic, so
// A B^T (both operands K-major) equals the wanted product A B up to rounding,
// but the rounding's antisymmetric part K then never dies out: in coupled
// Newton it flips sign every iteration, is amplified with the small
// eigenvalues during the linear phase (to ||K||_F ~ 0.08 at n = 256), and its
// second-order term 2 (2 c2 + c1^2) K^T K shifts the fixed point of M above I
// (by 2e-5 for the Newton T, 1e-4 with the second-degree correction; the
// signed trace residual settles at -3e-6, resp. -2e-5, and the latter never
// reaches a 1e-5 tolerance).  With true products A B (B read MN-major) K
// decays quadratically with the rest of the error, the residual settles near
// +3e-8 and M's eigenvalues within 3e-7 of 1, so both Newton forms use true
// products.  The Newton-DB fixed point is outright unstable along K under
// A B^T (the error grows about 1.5x per iteration): true products as well.
// The Clenshaw recurrence is a fixed number of steps with no fixed point to
// shift and keeps A B^T.
// Convergence is measured by |tr(I - M)|/n (Newton) or |tr(I - Z Y)|/n
// (Newton-DB): the iterations keep every eigenvalue of M (or Z Y) at or below
// 1 in exact arithmetic, so the trace bounds the largest eigenvalue error and
// ignores any antisymmetric rounding component.
// A' = (A + eps I)/s, unscaled by s^{-1/p} at the end.  Newton-DB and
// Chebyshev take s = ||A + eps I||_F (Frobenius pre-scaling); coupled Newton
// takes s = min(||A + eps I||_F, 1.25 x a power-iteration estimate of the
// largest eigenvalue).  With tol > 0 the residual is checked after every
// iteration and converged matrices drop out of later launches (their tiles
// exit at once); iters is then the cap.
#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "internal.h"

namespace shampoo {
namespace {

constexpr int NEWTON_B = B_MN_MAJOR;

// Scratch stacks per solver (plain fp32, n x n per matrix):
//   Newton    : M0 M1 X0 X1 T T2 T4 (both correction degrees), and T^p for p = 6, 8
//   Newton-DB : Y0 Y1 Z0 Z1 T
//   Chebyshev : Xt b0 b1 b2
int stacks_for(int solver, int p) {
  if (solver == 0 || solver == 3 || solver == 4) return p >= 6 ? 8 : 7;
  return solver == 1 ? 5 : 4;
}
// Bytes per stack element: fp64 iterates for solver 4, fp32 otherwise.
size_t stack_elem_bytes(int solver) { return solver == 4 ? 8 : 4; }

constexpr size_t kAlign = 256;
constexpr size_t kHeader = 64 * 1024;  // covers the alignment padding of the arrays
constexpr int kVecInts = 8;            // s sc sf res prev done iters iters1
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// First iteration at which a stalled residual counts as stagnation: an
// eigenvalue mu of M (scaled input 2^-24 <= mu << 1) grows by ((p+1)/p)^p per
// coupled-Newton iteration (2.44 at p = 4, 2.25 at p = 2) and by 9/4 per
// square-root iteration, reaching 1/2 within 18 (resp. 20) iterations; a few
// quadratic steps and a margin give the values below.  With the
// second-degree correction the growth is (1 + c1 + c2)^p (3.91 at p = 4,
// 3.52 at p = 2), reaching 1/2 within 13 (resp. 14) iterations counting the
// plain first step, followed by cubic steps.
int kmin_newton(int p, bool order2) {
  // p = 6, 8 grow small eigenvalues at least as fast as p = 4 ((7/6)^6 = 2.52,
  // (9/8)^8 = 2.57; second degree 4.08, 4.17) and take its thresholds.
  if (order2) return p >= 4 ? 17 : 18;
  return p >= 4 ? 24 : 26;
}
constexpr int kPowerIters = 12;     // power-iteration steps of the coupled-Newton scale
constexpr int kPowerItersWarm = 4;  // ... from the previous refresh's iterate
constexpr int kKminSqrt = 26;

struct Layout {
  int* counter;  // [0] iterations done, [1] matrices still active (written by the check kernel)
  float* s;
  float* sc;
  float* sf;  // Frobenius norm of A + eps I (the damping floor's reference)
  float* res;
  float* prev;
  int* done;
  int* iters;
  int* iters1;
  float* coef;
  float* stack[8];
};

Layout carve(void* base, int64_t cb, int n, int solver, int root_p) {
  Layout L;
  std::memset(&L, 0, sizeof(L));
  char* p = static_cast<char*>(base);
  auto take = [&](size_t bytes) {
    char* r = p;
    p += align_up(bytes);
    return r;
  };
  L.counter = reinterpret_cast<int*>(take(8));
  L.s = reinterpret_cast<float*>(take(cb * 4));
  L.sc = reinterpret_cast<float*>(take(cb * 4));
  L.sf = reinterpret_cast<float*>(take(cb * 4));
  L.res = reinterpret_cast<float*>(take(cb * 4));
  L.prev = reinterpret_cast<float*>(take(cb * 4));
  L.done = reinterpret_cast<int*>(take(cb * 4));
  L.iters = reinterpret_cast<int*>(take(cb * 4));
  L.iters1 = reinterpret_cast<int*>(take(cb * 4));
  L.coef = reinterpret_cast<float*>(take(cb * 4 * (kMaxChebDegree + 2)));
  for (int k = 0; k < stacks_for(solver, root_p); ++k)
    L.stack[k] = reinterpret_cast<float*>(take(plain_floats(cb, n) * stack_elem_bytes(solver)));
  return L;
}

// ---------------------------------------------------------------------------
// Residual-checked loops as CUDA graphs.  After iteration 0, the remaining
// iterations run as one graph with a WHILE node; its body holds two
// iterations (so the ping-pong buffers line up again after every pass) and
// each body's check kernel sets the loop condition to "some matrix still
// active".  The device ends the loop as soon as every matrix has converged,
// stagnated or reached the cap, instead of the host launching the cap's worth
// of iterations.  Executable graphs are cached by everything their kernels'
// arguments depend on.
// ---------------------------------------------------------------------------
struct LoopKey {
  int dev, solver, p, n, cap;
  int64_t cb;
  float tol;
  const void* scratch;
  const int* valid;
  const int* flags;
  bool operator<(const LoopKey& o) const {
    return std::tie(dev, solver, p, n, cap, cb, tol, scratch, valid, flags) <
           std::tie(o.dev, o.solver, o.p, o.n, o.cap, o.cb, o.tol, o.scratch, o.valid, o.flags);
  }
};

struct LoopGraph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  uint64_t used = 0;
};

std::mutex g_loop_mu;
std::map<LoopKey, LoopGraph> g_loops;
uint64_t g_loop_clock = 0;
bool g_loops_unavailable = false;  // a graph call failed once: plain launches from then on
constexpr size_t kMaxLoopGraphs = 64;

void destroy_loop(LoopGraph& g) {
  if (g.exec) cudaGraphExecDestroy(g.exec);
  if (g.graph) cudaGraphDestroy(g.graph);
  g.exec = nullptr;
  g.graph = nullptr;
}

// Graph loops are used unless profiling is on (per-launch events need plain
// launches), the caller's stream is being captured, or graphs failed before.
bool use_graph_loop(cudaStream_t st) {
  if (profiling_enabled()) return false;
  {
    std::lock_guard<std::mutex> lk(g_loop_mu);
    if (g_loops_unavailable) return false;
  }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return cs == cudaStreamCaptureStatusNone;
}

// Builds the graph: one WHILE node whose body `body(capture_stream, loop)`
// issues by stream capture.  Returns 0 or a CUDA error (nothing enqueued).
template <class Body>
int build_loop(LoopGraph& out, int kernels_per_iter, Body&& body) {
  cudaGraph_t g = nullptr;
  cudaStream_t cs = nullptr;
  auto fail = [&](cudaError_t e, const char* what) {
    if (cs) {
      cudaGraph_t tmp = nullptr;
      cudaStreamEndCapture(cs, &tmp);
      cudaStreamDestroy(cs);
    }
    if (g) cudaGraphDestroy(g);
    cudaGetLastError();
    return set_error(-4, "graph loop: %s failed (%s)", what, cudaGetErrorString(e));
  };
  cudaError_t e = cudaGraphCreate(&g, 0);
  if (e != cudaSuccess) return fail(e, "cudaGraphCreate");
  cudaGraphConditionalHandle h;
  e = cudaGraphConditionalHandleCreate(&h, g, 1, cudaGraphCondAssignDefault);
  if (e != cudaSuccess) return fail(e, "cudaGraphConditionalHandleCreate");
  cudaGraphNodeParams np = {cudaGraphNodeTypeConditional};
  np.conditional.handle = h;
  np.conditional.type = cudaGraphCondTypeWhile;
  np.conditional.size = 1;
  cudaGraphNode_t node;
  e = cudaGraphAddNode(&node, g, nullptr, 0, &np);
  if (e != cudaSuccess) return fail(e, "cudaGraphAddNode(while)");
  cudaGraph_t bodyg = np.conditional.phGraph_out[0];
  e = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking);
  if (e != cudaSuccess) return fail(e, "cudaStreamCreate");
  e = cudaStreamBeginCaptureToGraph(cs, bodyg, nullptr, nullptr, 0, cudaStreamCaptureModeThreadLocal);
  if (e != cudaSuccess) return fail(e, "cudaStreamBeginCaptureToGraph");
  GraphLoop loop{h, kernels_per_iter};
  int rc;
  {
    CaptureScope capture;  // launches recorded here are not executed launches
    rc = body(cs, &loop);
  }
  cudaGraph_t ended = nullptr;
  e = cudaStreamEndCapture(cs, &ended);
  cudaStreamDestroy(cs);
  cs = nullptr;
  if (rc) {
    cudaGraphDestroy(g);
    return rc;
  }
  if (e != cudaSuccess) return fail(e, "cudaStreamEndCapture");
  cudaGraphExec_t exec = nullptr;
  e = cudaGraphInstantiate(&exec, g, 0);
  if (e != cudaSuccess) return fail(e, "cudaGraphInstantiate");
  out.graph = g;
  out.exec = exec;
  return 0;
}

// Runs the loop for `key` on st (building and caching its graph on first
// use).  *done = false when graphs are unavailable (the caller then issues
// the iterations itself; nothing was enqueued).
template <class Body>
int run_loop(const LoopKey& key, int kernels_per_iter, Body&& body, cudaStream_t st, bool* done) {
  *done = false;
  std::lock_guard<std::mutex> lk(g_loop_mu);
  auto it = g_loops.find(key);
  if (it == g_loops.end()) {
    if (g_loops.size() >= kMaxLoopGraphs) {  // evict the least recently used
      auto old = g_loops.begin();
      for (auto i = g_loops.begin(); i != g_loops.end(); ++i)
        if (i->second.used < old->second.used) old = i;
      destroy_loop(old->second);
      g_loops.erase(old);
    }
    LoopGraph lg;
    if (build_loop(lg, kernels_per_iter, body)) {
      g_loops_unavailable = true;
      return 0;
    }
    it = g_loops.emplace(key, lg).first;
  }
  it->second.used = ++g_loop_clock;
  int rc = check_cuda(cudaGraphLaunch(it->second.exec, st), "cudaGraphLaunch(solver loop)");
  if (rc) return rc;
  note_graph_loop_launch();
  *done = true;
  return 0;
}

}  // namespace

size_t root_scratch_header() { return kHeader; }

size_t root_scratch_per_matrix(int n, int solver, int p) {
  return static_cast<size_t>(stacks_for(solver, p)) * n * n * stack_elem_bytes(solver) +
         4 * (kVecInts + kMaxChebDegree + 2);
}

int run_inverse_roots(const RootJob& job, void* scratch, size_t scratch_bytes, cudaStream_t st) {
  const int n = job.n;
  const int p = job.p;
  if (job.A64 && job.solver != 4) return set_error(-1, "fp64 input needs the fp64-iterate solver");
  const bool residual = job.tol > 0.f && job.solver != 2;
  const size_t per = root_scratch_per_matrix(n, job.solver, p);
  if (scratch_bytes < kHeader + per)
    return set_error(-3, "inverse-root scratch too small: %zu < %zu bytes", scratch_bytes, kHeader + per);
  const int64_t cb_max = std::min<int64_t>(job.batch, static_cast<int64_t>((scratch_bytes - kHeader) / per));
  // grid.z limit of the prologues (and of the fp64 GEMM's two groups); the
  // chunks are then balanced, so that no last chunk runs a few matrices alone
  const int64_t cb_lim = std::min<int64_t>(cb_max, job.solver == 4 ? 32767 : 65535);
  const int64_t nchunks = (job.batch + cb_lim - 1) / cb_lim;
  const int64_t cb_cap = (job.batch + nchunks - 1) / nchunks;
  const double f1 = 2.0 * n * static_cast<double>(n) * n;  // one GEMM(n), algorithmic
  int rc = 0;
  for (int64_t off = 0; off < job.batch; off += cb_cap) {
    const int64_t cb = std::min<int64_t>(cb_cap, job.batch - off);
    const int cbi = static_cast<int>(cb);
    Layout S = carve(scratch, cb, n, job.solver, p);
    const float* A = job.A ? job.A + off * static_cast<int64_t>(n) * n : nullptr;
    const double* A64 = job.A64 ? job.A64 + off * static_cast<int64_t>(n) * n : nullptr;
    const int* valid = job.valid ? job.valid + off : nullptr;
    float* out = job.X + off * static_cast<int64_t>(n) * n;
    int* iters_out = job.iters_used ? job.iters_used + off : nullptr;
    StackMaps sm[8];
    if (job.solver != 4)  // the fp64 GEMM reads its operands without tensor maps
      for (int k = 0; k < stacks_for(job.solver, p); ++k)
        if ((rc = make_stack_maps(sm[k], S.stack[k], cb, n))) return rc;
    // Coupled Newton scales by the power-iteration estimate (bounded by the
    // Frobenius norm); Newton-DB (convergent only on (0, 2)) and Chebyshev
    // (an exact upper bound is needed) by the Frobenius norm.
    if (A64) {
      if ((rc = launch_frob_f64(A64, cb, n, valid, job.eps, S.s, S.sf, st))) return rc;
    } else if (job.solver == 0 || job.solver == 3 || job.solver == 4) {
      float* pv = job.power_vec ? job.power_vec + off * n : nullptr;
      // one flag for all chunks: read by every chunk's scale kernel, set by the
      // last chunk's root prologue
      if ((rc = launch_spectral_scale(A, cb, n, valid, job.eps, p, kPowerIters, S.s, S.sc, S.sf, pv,
                                      job.power_vec ? job.power_warm : nullptr, kPowerItersWarm,
                                      job.power_vec && job.power_warm_hint, st)))
        return rc;
    } else {
      if ((rc = launch_frob_norm(A, cb, n, valid, job.eps, p, S.s, S.sc, st))) return rc;
    }
    if (residual) {
      if ((rc = check_cuda(cudaMemsetAsync(S.done, 0, cb * 4, st), "memset done"))) return rc;
      if ((rc = check_cuda(cudaMemsetAsync(S.res, 0, cb * 4, st), "memset res"))) return rc;
      if ((rc = check_cuda(cudaMemsetAsync(S.prev, 0, cb * 4, st), "memset prev"))) return rc;
      if ((rc = check_cuda(cudaMemsetAsync(S.counter, 0, 8, st), "memset counter"))) return rc;
    }
    const int* skip = residual ? S.done : nullptr;
    int dev = 0;
    if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;
    const LoopKey key{dev, job.solver, p, n, job.iters, cb, job.tol, scratch, valid, job.flags};
    // Iterations 1.. of a residual-checked loop: one graph with a WHILE node
    // when available, else plain launches up to the cap.
    auto run_rest = [&](auto&& iterate, int kernels_per_iter) -> int {
      if (job.iters <= 1) return 0;
      if (!job.plain_launches && use_graph_loop(st)) {
        bool ran = false;
        int r = run_loop(key, kernels_per_iter,
                         [&](cudaStream_t cs, const GraphLoop* lp) {
                           int q = iterate(1, cs, lp);
                           return q ? q : iterate(2, cs, lp);
                         },
                         st, &ran);
        if (r || ran) return r;
      }
      // Plain launches.  With profiling on (per-launch events) the host reads
      // the active count after each iteration and stops where the device loop
      // would, so that the profile covers the same kernels as a graph run.
      const bool follow = profiling_enabled();
      for (int j = 1; j < job.iters; ++j) {
        int r = iterate(j, st, nullptr);
        if (r) return r;
        if (follow) {
          int active = 0;
          if ((r = check_cuda(cudaMemcpyAsync(&active, S.counter + 1, 4, cudaMemcpyDeviceToHost, st),
                              "read active count")) ||
              (r = check_cuda(cudaStreamSynchronize(st), "profiling sync")))
            return r;
          if (active == 0) break;
        }
      }
      return 0;
    };
    auto common = [&](Epilogue& e) {
      e.skip = skip;
      e.flags = job.flags;
    };

    if (job.solver == 4) {
      // ------------------------------------------------ coupled Newton, fp64 iterates
      // The second-degree iteration of solver 3 below, step for step, with the
      // same stack rotation, on fp64 stacks through the fp64 GEMM.
      double* Mb[2] = {reinterpret_cast<double*>(S.stack[0]), reinterpret_cast<double*>(S.stack[1])};
      double* Xb[2] = {reinterpret_cast<double*>(S.stack[2]), reinterpret_cast<double*>(S.stack[3])};
      double* Q[3] = {reinterpret_cast<double*>(S.stack[4]), reinterpret_cast<double*>(S.stack[5]),
                      reinterpret_cast<double*>(S.stack[6])};
      double* Tp = reinterpret_cast<double*>(S.stack[7]);
      const double c1 = 1.0 / p, c2 = (p + 1.0) / (2.0 * p * p);
      int* set_flag = (job.power_vec && job.power_warm && off + cb == job.batch) ? job.power_warm : nullptr;
      // The damping floor is the input's own rounding, below which it may be
      // indefinite: 2^-24 ||A + eps I||_F for fp32 input (as for the fp32
      // solvers); for fp64 statistics n 2^-53 ||A + eps I||_F, the size of
      // their accumulated rounding
      const float floor_rel = A64 ? static_cast<float>(n * 1.1102230246251565e-16) : 5.9604645e-8f;
      if ((rc = launch_prologue_f64(A64 ? static_cast<const void*>(A64) : static_cast<const void*>(A), A64 ? 1 : 0,
                                    cb, n, valid, job.eps, floor_rel, p, S.s, S.sf, Mb[0], Q[0], Xb[1], set_flag,
                                    st)))
        return rc;
      auto dg = [](const double* a, const double* b, double* d) {
        DGemmGroup g;
        g.A = a;
        g.B = b;
        g.D = d;
        return g;
      };
      auto iterate = [&](int j, cudaStream_t cs, const GraphLoop* lp) -> int {
        int r;
        double* Tb = Q[0];
        double* T2b = Q[1];
        double* T4b = Q[2];
        if (j >= 1) {
          double* Db = p >= 4 ? Q[j & 1] : Q[0];
          Tb = p >= 4 ? Q[(j + 1) & 1] : Q[1];
          T2b = Q[2];
          T4b = Db;
          DGemmGroup g = dg(Db, Db, Tb);  // T = c2 D D + c1 D + I
          g.C = Db;
          g.alpha = c2;
          g.beta = c1;
          g.gamma = 1.0;
          if ((r = launch_dgemm(&g, 1, cb, n, valid, skip, job.flags, cs))) return r;
        }
        double* Dnext = p >= 4 ? Q[(j + 1) & 1] : Q[0];
        const bool last = !residual && j == job.iters - 1;
        {
          DGemmGroup g[2];
          int ng = 0;
          if (!last) g[ng++] = dg(Tb, Tb, T2b);                      // T2 = T T
          if (j >= 1) g[ng++] = dg(Xb[j & 1], Tb, Xb[(j + 1) & 1]);  // X <- X T
          if (ng && (r = launch_dgemm(g, ng, cb, n, valid, skip, job.flags, cs))) return r;
        }
        if (last) return 0;
        double* P = T2b;
        if (p >= 4) {
          DGemmGroup g = dg(T2b, T2b, T4b);  // T4 = T2 T2
          if ((r = launch_dgemm(&g, 1, cb, n, valid, skip, job.flags, cs))) return r;
          P = T4b;
        }
        if (p >= 6) {
          DGemmGroup g = dg(T4b, p == 6 ? T2b : T4b, Tp);
          if ((r = launch_dgemm(&g, 1, cb, n, valid, skip, job.flags, cs))) return r;
          P = Tp;
        }
        {
          DGemmGroup g = dg(P, Mb[j & 1], Mb[(j + 1) & 1]);  // M <- T^p M, next D = I - M
          g.E = Dnext;
          g.e_mul = -1.0;
          g.e_add = 1.0;
          g.res = residual ? S.res : nullptr;
          if ((r = launch_dgemm(&g, 1, cb, n, valid, skip, job.flags, cs))) return r;
        }
        if (residual)
          return launch_check(S.res, S.prev, S.done, S.iters, valid, cb, n, job.tol, S.counter, job.iters,
                              kmin_newton(p, true), job.flags, lp, cs);
        return 0;
      };
      if (residual) {
        const int per_iter = (p == 2 ? 3 : (p == 4 ? 4 : 5)) + 1;
        if ((rc = iterate(0, st, nullptr)) || (rc = run_rest(iterate, per_iter))) return rc;
      } else {
        for (int j = 0; j < job.iters; ++j)
          if ((rc = iterate(j, st, nullptr))) return rc;
      }
      if ((rc = launch_finalize_f64(Xb[0], Xb[1], residual ? S.iters : nullptr, job.iters, S.s, p, cb, n, out,
                                    job.flags, st)))
        return rc;
      if ((iters_out || residual) &&
          (rc = launch_report(residual ? S.iters : nullptr, nullptr, residual ? S.done : nullptr, cb, job.iters,
                              iters_out, job.flags, residual, st)))
        return rc;
    } else if (job.solver == 0 || job.solver == 3) {
      // ------------------------------------------------------------ coupled Newton
      StackMaps* M = &sm[0];  // M[0], M[1]
      StackMaps* X = &sm[2];  // X[0], X[1]
      StackMaps& T = sm[4];
      StackMaps& T2 = sm[5];
      StackMaps& T4 = sm[6];
      StackMaps& Tp = sm[7];  // T^6 or T^8 (p = 6, 8 only)
      // Second-degree correction (solver 3): from iteration 1 on,
      // T = I + c1 (I - M) + c2 (I - M)^2 with c1 = 1/p, c2 = (p+1)/(2p^2),
      // the first three terms of the binomial series of M^{-1/p} about I,
      // which is one GEMM: T = c2 M M + (-c1 - 2 c2) M + (1 + c1 + c2) I.
      // Iteration 0 is a plain Newton step; it maps every eigenvalue in
      // (0, p+1) into (0, 1], where the second-degree steps keep eigenvalues
      // increasing to 1.
      const bool order2 = job.solver == 3;
      const float c1 = 1.f / p, c2 = (p + 1.f) / (2.f * p * p);
      int* set_flag = (job.power_vec && job.power_warm && off + cb == job.batch) ? job.power_warm : nullptr;
      if ((rc = launch_root_prologue(0, A, cb, n, valid, job.eps, p, S.s, S.sf, M[0].base, T.base, X[1].base,
                                     set_flag, st)))
        return rc;
      // With the second-degree correction the M update also writes
      // D = I - M (exact in fp32 from the accumulator value), and T is formed
      // from D: T = c2 D D + c1 D + I.  The product of D carries rounding
      // relative to |D|^2 only, so T is as accurate as the Newton T = I + D/p
      // (a product of M itself would add rounding of order |M|^2 = 1, above
      // the residual tolerance).  The three stacks T, T2, T4 then rotate
      // (p = 4, period 2; p = 2, period 1), so that no launch writes a stack
      // that another of its tiles reads:
      //   p = 4, j >= 1: D in Q[j&1], T -> Q[(j+1)&1], T2 -> Q2, T4 -> Q[j&1],
      //                  next D -> Q[(j+1)&1];
      //   p = 2, j >= 1: D in Q0, T -> Q1, T2 -> Q2, next D -> Q0;
      //   j = 0 (plain step): T in Q0, T2 -> Q1, T4 -> Q2, next D -> Q1
      //                  (p = 4) or Q0 (p = 2).
      StackMaps* Q[3] = {&T, &T2, &T4};
      // One iteration j on stream cs (inside a graph loop when lp != NULL).
      auto iterate = [&](int j, cudaStream_t cs, const GraphLoop* lp) -> int {
        int r;
        StackMaps* Tb = Q[0];
        StackMaps* T2b = Q[1];
        StackMaps* T4b = Q[2];
        StackMaps* Dnext = nullptr;
        if (order2) {
          if (j >= 1) {
            StackMaps* Db = p >= 4 ? Q[j & 1] : Q[0];
            Tb = p >= 4 ? Q[(j + 1) & 1] : Q[1];
            T2b = Q[2];
            T4b = Db;
            Builder b;
            Epilogue& e = b.add(cbi, n, *Db, 0, *Db, 0, f1, NEWTON_B);  // T = c2 D D + c1 D + I
            e.alpha = c2;
            e.C = Db->base;
            e.beta = c1;
            e.gamma = 1.f;
            e.D = Tb->base;
            common(e);
            if ((r = b.launch(cs))) return r;
          }
          Dnext = p >= 4 ? Q[(j + 1) & 1] : Q[0];
        }
        // The last iteration of a fixed count only needs X <- X T.
        const bool last = !residual && j == job.iters - 1;
        if (j >= 1 || !last) {
          Builder b;
          if (!last) {
            Epilogue& e = b.add(cbi, n, *Tb, 0, *Tb, 0, f1, NEWTON_B);  // T2 = T T
            e.D = T2b->base;
            common(e);
          }
          if (j >= 1) {
            Epilogue& ex = b.add(cbi, n, X[j & 1], 0, *Tb, 0, f1, NEWTON_B);  // X <- X T
            ex.D = X[(j + 1) & 1].base;
            common(ex);
          }
          if ((r = b.launch(cs))) return r;
        }
        if (last) return 0;
        StackMaps* P = T2b;
        if (p >= 4) {
          Builder b;
          Epilogue& e = b.add(cbi, n, *T2b, 0, *T2b, 0, f1, NEWTON_B);  // T4 = T2 T2
          e.D = T4b->base;
          common(e);
          if ((r = b.launch(cs))) return r;
          P = T4b;
        }
        if (p >= 6) {  // T6 = T4 T2, or T8 = T4 T4, into a stack no later launch of this iteration writes
          Builder b;
          Epilogue& e = b.add(cbi, n, *T4b, 0, p == 6 ? *T2b : *T4b, 0, f1, NEWTON_B);
          e.D = Tp.base;
          common(e);
          if ((r = b.launch(cs))) return r;
          P = &Tp;
        }
        {
          Builder b;
          Epilogue& e = b.add(cbi, n, *P, 0, M[j & 1], 0, f1, NEWTON_B);  // M <- T^p M
          e.D = M[(j + 1) & 1].base;
          if (order2) {
            e.E = Dnext->base;  // next D = I - M
            e.e_mul = -1.f;
            e.e_add = 1.f;
          } else {
            e.E = T.base;  // next T = ((p+1) I - M) / p
            e.e_mul = -1.f / p;
            e.e_add = static_cast<float>(p + 1) / p;
          }
          e.res = residual ? S.res : nullptr;
          e.valid = valid;
          common(e);
          if ((r = b.launch(cs))) return r;
        }
        if (residual)
          return launch_check(S.res, S.prev, S.done, S.iters, valid, cb, n, job.tol, S.counter, job.iters,
                              kmin_newton(p, order2), job.flags, lp, cs);
        return 0;
      };
      if (residual) {
        const int per_iter = (p == 2 ? 3 : (p == 4 ? 4 : 5)) + (order2 ? 1 : 0);
        if ((rc = iterate(0, st, nullptr)) || (rc = run_rest(iterate, per_iter))) return rc;
      } else {
        for (int j = 0; j < job.iters; ++j)
          if ((rc = iterate(j, st, nullptr))) return rc;
      }
      if ((rc = launch_finalize(X[0].base, X[1].base, residual ? S.iters : nullptr, job.iters, S.sc, cb, n, out,
                                job.flags, st)))
        return rc;
      if ((iters_out || residual) &&
          (rc = launch_report(residual ? S.iters : nullptr, nullptr, residual ? S.done : nullptr, cb, job.iters,
                              iters_out, job.flags, residual, st)))
        return rc;
    } else if (job.solver == 1) {
      // ------------------------------------------------------------ Newton-DB
      StackMaps* Y = &sm[0];
      StackMaps* Z = &sm[2];
      StackMaps& T = sm[4];
      if ((rc = launch_root_prologue(1, A, cb, n, valid, job.eps, p, S.s, nullptr, Y[0].base, T.base, Z[1].base,
                                     nullptr, st)))
        return rc;
      const int stages = (p == 4) ? 2 : 1;
      for (int stage = 0; stage < stages; ++stage) {
        if (stage == 1) {
          // Stage-1 results: Y_final at parity iters1; its square root seeds stage 2.
          if (residual) {
            // Flags stage-1 matrices that reached the cap (per-matrix signs report stage 2).
            if ((rc = launch_report(S.iters, nullptr, S.done, cb, job.iters, nullptr, job.flags, true, st))) return rc;
            if ((rc = check_cuda(cudaMemcpyAsync(S.iters1, S.iters, cb * 4, cudaMemcpyDeviceToDevice, st),
                                 "copy iters")))
              return rc;
            if ((rc = check_cuda(cudaMemsetAsync(S.done, 0, cb * 4, st), "memset done"))) return rc;
            if ((rc = check_cuda(cudaMemsetAsync(S.res, 0, cb * 4, st), "memset res"))) return rc;
            if ((rc = check_cuda(cudaMemsetAsync(S.prev, 0, cb * 4, st), "memset prev"))) return rc;
            if ((rc = check_cuda(cudaMemsetAsync(S.counter, 0, 8, st), "memset counter"))) return rc;
          } else {
            if ((rc = launch_fill_iters(S.iters1, cb, job.iters, st))) return rc;
          }
          if ((rc = launch_db_stage2_prologue(Y[0].base, Y[1].base, S.iters1, cb, n, Y[0].base, T.base, Z[1].base,
                                              st)))
            return rc;
        }
        auto iterate = [&](int j, cudaStream_t cs, const GraphLoop* lp) -> int {
          int r;
          {
            Builder b;
            Epilogue& ey = b.add(cbi, n, Y[j & 1], 0, T, 0, f1, B_MN_MAJOR);  // Y <- Y T
            ey.D = Y[(j + 1) & 1].base;
            common(ey);
            if (j >= 1) {
              Epilogue& ez = b.add(cbi, n, T, 0, Z[j & 1], 0, f1, B_MN_MAJOR);  // Z <- T Z
              ez.D = Z[(j + 1) & 1].base;
              common(ez);
            }
            if ((r = b.launch(cs))) return r;
          }
          if (!residual && j == job.iters - 1) return 0;
          {
            Builder b;
            Epilogue& e = b.add(cbi, n, Z[(j + 1) & 1], 0, Y[(j + 1) & 1], 0, f1, B_MN_MAJOR);  // T = (3I - Z Y)/2
            e.alpha = -0.5f;
            e.gamma = 1.5f;
            e.D = T.base;
            e.res = residual ? S.res : nullptr;
            e.valid = valid;
            common(e);
            if ((r = b.launch(cs))) return r;
          }
          if (residual)
            return launch_check(S.res, S.prev, S.done, S.iters, valid, cb, n, job.tol, S.counter, job.iters,
                                kKminSqrt, job.flags, lp, cs);
          return 0;
        };
        if (residual) {
          if ((rc = iterate(0, st, nullptr)) || (rc = run_rest(iterate, 3))) return rc;
        } else {
          for (int j = 0; j < job.iters; ++j)
            if ((rc = iterate(j, st, nullptr))) return rc;
        }
      }
      if ((rc = launch_finalize(Z[0].base, Z[1].base, residual ? S.iters : nullptr, job.iters, S.sc, cb, n, out,
                                job.flags, st)))
        return rc;
      const int* add = (p == 4 && residual) ? S.iters1 : nullptr;
      const int default_total = (p == 4) ? 2 * job.iters : job.iters;
      if ((iters_out || residual) &&
          (rc = launch_report(residual ? S.iters : nullptr, add, residual ? S.done : nullptr, cb, default_total,
                              iters_out, job.flags, residual, st)))
        return rc;
    } else {
      // ------------------------------------------------------------ Chebyshev
      const int d = job.cheb_degree;
      StackMaps& Xt = sm[0];
      StackMaps* b = &sm[1];  // b[k % 3]
      if ((rc = launch_cheb_setup(A, cb, n, valid, job.eps, p, d, job.cheb_lo, S.s, S.coef, S.sc, Xt.base,
                                  b[d % 3].base, b[(d - 1) % 3].base, st)))
        return rc;
      for (int k = d - 2; k >= 1; --k) {  // b_k = 2 Xt b_{k+1} - b_{k+2} + c_k I
        Builder bl;
        Epilogue& e = bl.add(cbi, n, Xt, 0, b[(k + 1) % 3], 0, f1, B_TRANSPOSED);
        e.alpha = 2.f;
        e.beta = -1.f;
        e.C = b[(k + 2) % 3].base;
        e.gamma_vec = S.coef + k;
        e.gamma_stride = d + 2;
        e.D = b[k % 3].base;
        e.flags = job.flags;
        if ((rc = bl.launch(st))) return rc;
      }
      {  // X = s^{-1/p} (Xt b_1 - b_2 + c_0 I)
        Builder bl;
        Epilogue& e = bl.add(cbi, n, Xt, 0, b[1], 0, f1, B_TRANSPOSED);
        e.alpha = 1.f;
        e.beta = -1.f;
        e.C = b[2].base;
        e.gamma_vec = S.coef;
        e.gamma_stride = d + 2;
        e.scale_vec = S.sc;
        e.D = out;
        e.flags = job.flags;
        if ((rc = bl.launch(st))) return rc;
      }
      if (iters_out && (rc = launch_fill_iters(iters_out, cb, d, st))) return rc;
    }
  }
  return 0;
}

}  // namespace shampoo
