// Batched symmetric eigendecomposition A_i = Q_i diag(lam_i) Q_i^T for the
// eigenbasis SOAP runs Adam in (pith.science SOAP record: Adam in the
// eigenbasis of Shampoo's preconditioner; Substack SOAP survey: the
// eigendecompositions are Shampoo's bottleneck).  The pages name no method;
// two published ones are used:
//   eigenvectors  cyclic Jacobi with the round-robin parallel ordering
//                 (Golub & Van Loan, "Matrix Computations", sec. 8.5): each
//                 round rotates n/2 disjoint index pairs (p, q), zeroing a_pq,
//                 as the two-sided update A <- J^T A J and V <- V J; one CTA per
//                 matrix, the working copy in global memory (L2 resident).  A
//                 warm start from an approximate basis X runs Jacobi on the
//                 nearly diagonal X^T A X (a few sweeps) and takes X V;
//   orthogonality Newton-Schulz steps toward the nearest orthogonal matrix
//                 (Bjorck & Bowie 1971): X <- X + X (I - X^T X) / 2 =
//                 1.5 X - 0.5 X (X^T X), GEMM only.  The products of a warm start
//                 carry 3xTF32 rounding into X's orthogonality; each step
//                 squares that error.  (An eigenvector-correcting refinement
//                 such as Ogita & Aishima's divides rounding in X^T A X by
//                 eigenvalue gaps and, evaluated in fp32, degrades an
//                 fp32-accurate basis; it is not used.)
// Matrices of a ragged block use their leading `valid` x `valid` part; the
// rest of Q is the identity.
#include <algorithm>
#include <cmath>

#include "../../include/shampoo.h"
#include "common.cuh"
#include "internal.h"

namespace shampoo {
namespace {

constexpr int kJacobiThreads = 1024;
// Sweeps stop once ||offdiag(W)||_F <= kJacobiTol ||W||_F (fp32 rounding of
// the rotations leaves off-diagonal mass of a few u ||A||_F per sweep).
constexpr float kJacobiTol = 1e-5f;

// Index at position j of round r of the round-robin schedule over m (even)
// indices: position 0 is fixed, the others rotate by one per round.  Round r
// pairs position k with position m - 1 - k.
__device__ __forceinline__ int rr_index(int j, int r, int m) { return j == 0 ? 0 : 1 + (j - 1 + r) % (m - 1); }

// One CTA per matrix.  W: working copy (n x n), V: eigenvectors (columns),
// lam (nullable): eigenvalues (the diagonal of the converged W).
__global__ void __launch_bounds__(kJacobiThreads) jacobi_eig_kernel(const float* __restrict__ A, int n,
                                                                    const int* __restrict__ valid, float* W, float* V,
                                                                    float* lam, int max_sweeps, float tol,
                                                                    int* flags) {
  __shared__ float cs[512][2];
  __shared__ int pq[512][2];
  __shared__ double red[32];
  __shared__ double total;
  const int i = blockIdx.x;
  const int tid = threadIdx.x;
  const size_t nn = static_cast<size_t>(n) * n;
  const float* a = A + i * nn;
  float* w = W + i * nn;
  float* v = V + i * nn;
  const int m = valid ? valid[i] : n;
  // working copy: sym(A) on the valid part, zero elsewhere; V = I
  for (size_t e = tid; e < nn; e += blockDim.x) {
    const int r = static_cast<int>(e / n), c = static_cast<int>(e % n);
    w[e] = (r < m && c < m) ? 0.5f * (a[e] + a[static_cast<size_t>(c) * n + r]) : 0.f;
    v[e] = (r == c) ? 1.f : 0.f;
  }
  __syncthreads();
  auto block_sum = [&](double x) -> double {
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if ((tid & 31) == 0) red[tid >> 5] = x;
    __syncthreads();
    if (tid < 32) {
      double y = (tid < static_cast<int>(blockDim.x >> 5)) ? red[tid] : 0.0;
      for (int o = 16; o > 0; o >>= 1) y += __shfl_xor_sync(0xffffffffu, y, o);
      if (tid == 0) total = y;
    }
    __syncthreads();
    const double r = total;
    __syncthreads();
    return r;
  };
  const int me = m + (m & 1);  // even count; index m (if added) is a dummy that never rotates
  const int pairs = me / 2;
  bool converged = m < 2;
  for (int sweep = 0; sweep < max_sweeps && !converged; ++sweep) {
    double off = 0.0, fro = 0.0;
    for (size_t e = tid; e < static_cast<size_t>(m) * m; e += blockDim.x) {
      const int r = static_cast<int>(e / m), c = static_cast<int>(e % m);
      const double x = w[static_cast<size_t>(r) * n + c];
      fro += x * x;
      if (r != c) off += x * x;
    }
    off = block_sum(off);
    fro = block_sum(fro);
    if (off <= static_cast<double>(tol) * tol * fro) {
      converged = true;
      break;
    }
    for (int rnd = 0; rnd < me - 1; ++rnd) {
      for (int k = tid; k < pairs; k += blockDim.x) {
        int p = rr_index(k, rnd, me), q = rr_index(me - 1 - k, rnd, me);
        if (p > q) {
          const int t = p;
          p = q;
          q = t;
        }
        float c = 1.f, s = 0.f;
        if (q < m) {
          const float apq = w[static_cast<size_t>(p) * n + q];
          if (apq != 0.f) {
            const float app = w[static_cast<size_t>(p) * n + p], aqq = w[static_cast<size_t>(q) * n + q];
            const float tau = (aqq - app) / (2.f * apq);
            const float t = (tau >= 0.f ? 1.f : -1.f) / (fabsf(tau) + sqrtf(1.f + tau * tau));
            c = rsqrtf(1.f + t * t);
            s = t * c;
          }
        }
        pq[k][0] = p;
        pq[k][1] = q;
        cs[k][0] = c;
        cs[k][1] = s;
      }
      __syncthreads();
      // rows: A <- J^T A (rows p and q of every pair)
      for (int e = tid; e < pairs * m; e += blockDim.x) {
        const int k = e / m, col = e % m;
        const int p = pq[k][0], q = pq[k][1];
        if (q >= m || cs[k][1] == 0.f) continue;
        const float c = cs[k][0], s = cs[k][1];
        float* rp = w + static_cast<size_t>(p) * n + col;
        float* rq = w + static_cast<size_t>(q) * n + col;
        const float x = *rp, y = *rq;
        *rp = c * x - s * y;
        *rq = s * x + c * y;
      }
      __syncthreads();
      // columns: A <- A J and V <- V J (columns p and q of every pair); the
      // pair index runs fastest, so a warp's accesses fall in one or two rows
      for (int e = tid; e < pairs * m; e += blockDim.x) {
        const int k = e % pairs, row = e / pairs;
        const int p = pq[k][0], q = pq[k][1];
        if (q >= m || cs[k][1] == 0.f) continue;
        const float c = cs[k][0], s = cs[k][1];
        float* ap = w + static_cast<size_t>(row) * n;
        const float x = ap[p], y = ap[q];
        ap[p] = c * x - s * y;
        ap[q] = s * x + c * y;
        float* vp = v + static_cast<size_t>(row) * n;
        const float vx = vp[p], vy = vp[q];
        vp[p] = c * vx - s * vy;
        vp[q] = s * vx + c * vy;
      }
      __syncthreads();
    }
  }
  if (tid == 0 && !converged && m >= 2) raise_flag(flags, DEV_FLAG_NOT_CONVERGED);
  if (lam)
    for (int j = tid; j < n; j += blockDim.x) lam[static_cast<size_t>(i) * n + j] = j < m ? w[static_cast<size_t>(j) * n + j] : 0.f;
}

// Batched transpose, Xt_i = X_i^T.  grid (n/32, n/32, batch), block (32, 8).
__global__ void transpose_kernel(const float* __restrict__ X, int n, float* __restrict__ Xt) {
  pdl_launch_dependents();
  __shared__ float t[32][33];
  const int i = blockIdx.z, bi = blockIdx.y, bj = blockIdx.x;
  const size_t nn = static_cast<size_t>(n) * n;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    t[threadIdx.y + 8 * k][threadIdx.x] = X[i * nn + static_cast<size_t>(bi * 32 + threadIdx.y + 8 * k) * n + bj * 32 + threadIdx.x];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k)
    Xt[i * nn + static_cast<size_t>(bj * 32 + threadIdx.y + 8 * k) * n + bi * 32 + threadIdx.x] =
        t[threadIdx.x][threadIdx.y + 8 * k];
}

// Eigenvalues as Rayleigh quotients of the final basis: lam_j = q_j^T A q_j =
// sum_i Q[i][j] (A Q)[i][j] (more accurate than the diagonal Jacobi's
// rotations leave, which carries their accumulated rounding).  One thread per
// column, rows in order (coalesced across the threads of a row).
__global__ void rayleigh_kernel(const float* __restrict__ Q, const float* __restrict__ AQ, int n,
                                const int* __restrict__ valid, float* __restrict__ lam) {
  const int i = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int m = valid ? valid[i] : n;
  const size_t nn = static_cast<size_t>(n) * n;
  double acc = 0.0;
  if (j < m)
    for (int r = 0; r < m; ++r)
      acc += static_cast<double>(Q[i * nn + static_cast<size_t>(r) * n + j]) * AQ[i * nn + static_cast<size_t>(r) * n + j];
  lam[static_cast<size_t>(i) * n + j] = static_cast<float>(acc);
}

}  // namespace

size_t eig_scratch_per_matrix(int n) { return static_cast<size_t>(5) * n * n * 4; }

int run_eigh(const float* A, float* Q, float* lam, int64_t batch, int n, const int* valid, int warm_start,
             int jacobi_sweeps, int refine_iters, void* scratch, size_t scratch_bytes, int* flags, cudaStream_t st) {
  if (batch == 0) return 0;
  const size_t per = eig_scratch_per_matrix(n);
  const size_t nn = static_cast<size_t>(n) * n;
  // at most 65535 matrices per chunk (grid.y / grid.z of the per-matrix kernels)
  const int64_t cb_max = std::min<int64_t>(static_cast<int64_t>(scratch_bytes / per), 65535);
  if (cb_max < 1) return set_error(-3, "eigensolver scratch too small: %zu < %zu bytes", scratch_bytes, per);
  int rc;
  for (int64_t off = 0; off < batch; off += cb_max) {
    const int64_t cb = std::min<int64_t>(cb_max, batch - off);
    const float* Ai = A + off * nn;
    float* Qi = Q + off * nn;
    float* li = lam ? lam + off * n : nullptr;
    const int* vi = valid ? valid + off : nullptr;
    float* base = static_cast<float*>(scratch);
    float* Xt = base;            // X^T
    float* Rm = Xt + cb * nn;    // the Jacobi working copy
    float* T = Rm + cb * nn;     // A X, then the new basis
    float* S = T + cb * nn;      // X^T A X, then X^T X
    float* E = S + cb * nn;      // Jacobi's rotation of X^T A X
    const double f1 = 2.0 * n * static_cast<double>(n) * n;
    const int cbi = static_cast<int>(cb);
    StackMaps mA, mX, mXt, mT, mE;
    if ((rc = make_stack_maps(mA, Ai, cb, n)) || (rc = make_stack_maps(mX, Qi, cb, n)) ||
        (rc = make_stack_maps(mXt, Xt, cb, n)) || (rc = make_stack_maps(mT, T, cb, n)) ||
        (rc = make_stack_maps(mE, E, cb, n)))
      return rc;
    dim3 tgrid(n / 32, n / 32, static_cast<unsigned>(cb)), tblock(32, 8);
    auto jacobi = [&](const float* in, float* vout) -> int {
      ProfScope ps(K_EIGEN, st, 0.0, 8.0 * cb * nn);
      // the Jacobi working copy lives in Rm
      jacobi_eig_kernel<<<static_cast<unsigned>(cb), kJacobiThreads, 0, st>>>(in, n, vi, Rm, vout, nullptr,
                                                                          jacobi_sweeps, kJacobiTol, flags);
      count_launch();
      return check_cuda(cudaGetLastError(), "jacobi_eig_kernel");
    };
    if (!warm_start) {
      if ((rc = jacobi(Ai, Qi))) return rc;
    } else {
      {  // Xt = X^T
        ProfScope ps(K_EIGEN, st, 0.0, 8.0 * cb * nn);
        transpose_kernel<<<tgrid, tblock, 0, st>>>(Qi, n, Xt);
        count_launch();
        if ((rc = check_cuda(cudaGetLastError(), "transpose_kernel"))) return rc;
      }
      {  // T = A X
        Builder b;
        Epilogue& e = b.add(cbi, n, mA, 0, mX, 0, f1, B_MN_MAJOR);
        e.D = T;
        e.flags = flags;
        if ((rc = b.launch(st))) return rc;
      }
      {  // S = X^T A X (nearly diagonal for a good basis)
        Builder b;
        Epilogue& e = b.add(cbi, n, mXt, 0, mT, 0, f1, B_MN_MAJOR);
        e.D = S;
        e.flags = flags;
        if ((rc = b.launch(st))) return rc;
      }
      if ((rc = jacobi(S, E))) return rc;  // S = V diag V^T
      {  // X <- X V
        Builder b;
        Epilogue& e = b.add(cbi, n, mX, 0, mE, 0, f1, B_MN_MAJOR);
        e.D = T;
        e.flags = flags;
        if ((rc = b.launch(st))) return rc;
      }
      if ((rc = check_cuda(cudaMemcpyAsync(Qi, T, cb * nn * 4, cudaMemcpyDeviceToDevice, st), "rotated basis")))
        return rc;
    }
    for (int it = 0; it < refine_iters; ++it) {
      {
        ProfScope ps(K_EIGEN, st, 0.0, 8.0 * cb * nn);
        transpose_kernel<<<tgrid, tblock, 0, st>>>(Qi, n, Xt);
        count_launch();
        if ((rc = check_cuda(cudaGetLastError(), "transpose_kernel"))) return rc;
      }
      {  // S = X^T X (= Xt Xt^T)
        Builder b;
        Epilogue& e = b.add(cbi, n, mXt, 0, mXt, 0, f1, B_TRANSPOSED);
        e.D = S;
        e.flags = flags;
        if ((rc = b.launch(st))) return rc;
      }
      StackMaps mS;
      if ((rc = make_stack_maps(mS, S, cb, n))) return rc;
      {  // X <- 1.5 X - 0.5 X (X^T X), into T, then back to Q
        Builder b;
        Epilogue& e = b.add(cbi, n, mX, 0, mS, 0, f1, B_MN_MAJOR);
        e.alpha = -0.5f;
        e.C = Qi;
        e.beta = 1.5f;
        e.D = T;
        e.flags = flags;
        if ((rc = b.launch(st))) return rc;
      }
      if ((rc = check_cuda(cudaMemcpyAsync(Qi, T, cb * nn * 4, cudaMemcpyDeviceToDevice, st), "orthogonalised basis")))
        return rc;
    }
    if (li) {  // eigenvalues: Rayleigh quotients of the final basis
      {
        Builder b;
        Epilogue& e = b.add(cbi, n, mA, 0, mX, 0, f1, B_MN_MAJOR);  // T = A Q
        e.D = T;
        e.flags = flags;
        if ((rc = b.launch(st))) return rc;
      }
      ProfScope ps(K_EIGEN, st, 0.0, 8.0 * cb * nn);
      rayleigh_kernel<<<dim3((n + 127) / 128, static_cast<unsigned>(cb)), 128, 0, st>>>(Qi, T, n, vi, li);
      count_launch();
      if ((rc = check_cuda(cudaGetLastError(), "rayleigh_kernel"))) return rc;
    }
  }
  return 0;
}

}  // namespace shampoo

extern "C" {

int eigh_scratch_bytes(int64_t batch, int32_t n, size_t* bytes) {
  if (!bytes) return shampoo::set_error(SHAMPOO_ERR_INVALID_ARG, "bytes is NULL");
  if (batch < 0 || n < 32 || n > 1024 || n % 32) return shampoo::set_error(SHAMPOO_ERR_INVALID_ARG, "bad batch / n");
  *bytes = shampoo::eig_scratch_per_matrix(n) * static_cast<size_t>(batch < 1 ? 1 : batch);
  return SHAMPOO_OK;
}

int eigh_batched(const float* d_A, float* d_Q, float* d_lam, int64_t batch, int32_t n, int32_t warm_start,
                 int32_t jacobi_sweeps, int32_t refine_iters, void* d_scratch, size_t scratch_bytes,
                 int32_t* d_status, void* stream) {
  using namespace shampoo;
  if (batch < 0) return set_error(SHAMPOO_ERR_INVALID_ARG, "batch < 0");
  if (batch == 0) return SHAMPOO_OK;
  if (!d_A || !d_Q || !d_scratch) return set_error(SHAMPOO_ERR_INVALID_ARG, "NULL device pointer");
  if (n < 32 || n > 1024 || n % 32) return set_error(SHAMPOO_ERR_INVALID_ARG, "n %d: need a multiple of 32 in [32, 1024]", n);
  if (warm_start != 0 && warm_start != 1) return set_error(SHAMPOO_ERR_INVALID_ARG, "warm_start must be 0 or 1");
  if (jacobi_sweeps < 1 || jacobi_sweeps > 100 || refine_iters < 0 || refine_iters > 100)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "jacobi_sweeps in [1, 100], refine_iters in [0, 100]");
  if ((reinterpret_cast<uintptr_t>(d_scratch) & 255) || (reinterpret_cast<uintptr_t>(d_A) & 15) ||
      (reinterpret_cast<uintptr_t>(d_Q) & 15))
    return set_error(SHAMPOO_ERR_UNSUPPORTED, "scratch must be 256-byte and A, Q 16-byte aligned");
  return run_eigh(d_A, d_Q, d_lam, batch, n, nullptr, warm_start, jacobi_sweeps, refine_iters, d_scratch,
                  scratch_bytes, d_status, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
