// Order-k tensor Shampoo (podcast transcript "Preconditioned optimization
// without the full matrix cost", cue 26: one preconditioner per dimension of
// the gradient tensor, built from the gradient contracted with itself over
// every other dimension, applied by a contraction along its own dimension with
// the power -1/(2k); the order of the modes does not matter).
//
// For a parameter of order k with dimensions d_0 .. d_{k-1}, every step:
//   1. unfold   U_i = mode-i unfolding of G (d_i x prod_{l != i} d_l, the other
//               indices in row-major order), zero-padded to npad_i x Kpad_i
//               (multiples of 32);
//   2. stats    H_i <- beta H_i + U_i U_i^T        (one GEMM launch, k groups);
//   3. roots    every refresh_every steps, X_i = (H_i + eps I)^{-1/(2k)} for all
//               modes of all parameters, batched by (npad, k);
//   4. apply    V = X_0 U_0; then for i = 1 .. k-1: V <- X_i unfold_i(fold_{i-1}(V))
//               (a permutation pass between the products), and the last
//               fold writes W <- W - lr P into the weight.
// Short modes (d_i <= 32, e.g. the 3 x 3 spatial modes of a convolution
// kernel) skip the unfolding, whose 32-row padding would be most of its
// bytes: their statistic is summed over the tensor's fibres along the mode
// in its natural layout, and their product is applied to those fibres in
// place of a layout change (one pass, read and write once).  They go first;
// the longer modes follow as above.  The modes commute, so the order does
// not change the result.
// Diagonal variant (cue 28): a dimension longer than the threshold keeps only
// h_i = diag(H_i) (the row sums of squares of U_i), is refreshed to
// d_i = (h_i + eps)^{-1/(2k)} elementwise, and its "product" scales the rows
// of the mode-i unfolding by d_i.
#include <algorithm>
#include <cstring>
#include <map>
#include <new>
#include <vector>

#include "../../include/shampoo.h"
#include "common.cuh"
#include "internal.h"

using namespace shampoo;

namespace {

constexpr int kMaxOrder = 4;
constexpr int kMaxTensorParams = 256;
constexpr size_t kAlignT = 256;
constexpr size_t kTensorRootBudget = size_t(8) << 30;

size_t alt(size_t x) { return (x + kAlignT - 1) / kAlignT * kAlignT; }
int up32(int64_t x) { return static_cast<int>((x + 31) / 32 * 32); }

// Layout of one side of a permutation: the natural row-major tensor
// (mode = -1) or the mode-`mode` unfolding with row stride `ld`.
struct PermSide {
  int mode;
  int64_t ld;
};

struct PermArgs {
  int k;
  int dims[kMaxOrder];
  const void* src;
  int src_bf16;
  PermSide s;
  float* dst;
  PermSide d;
  int rows, cols;  // destination extent written (unfolding: padded rows x padded cols)
  float lr;        // fold into the weight: dst[idx] -= lr * value
  int update;
};

// Multi-index of column c of the mode-m unfolding (other indices row-major).
__device__ __forceinline__ void unfold_col_index(const PermArgs& a, int m, int64_t c, int* idx) {
#pragma unroll
  for (int l = kMaxOrder - 1; l >= 0; --l) {
    if (l >= a.k || l == m) continue;
    idx[l] = static_cast<int>(c % a.dims[l]);
    c /= a.dims[l];
  }
}

__device__ __forceinline__ int64_t natural_offset(const PermArgs& a, const int* idx) {
  int64_t o = 0;
#pragma unroll
  for (int l = 0; l < kMaxOrder; ++l)
    if (l < a.k) o = o * a.dims[l] + idx[l];
  return o;
}

__device__ __forceinline__ int64_t unfold_offset(const PermArgs& a, const PermSide& sd, const int* idx) {
  int64_t c = 0;
#pragma unroll
  for (int l = 0; l < kMaxOrder; ++l)
    if (l < a.k && l != sd.mode) c = c * a.dims[l] + idx[l];
  return static_cast<int64_t>(idx[sd.mode]) * sd.ld + c;
}

// One thread per destination element.  Unfolding destinations are written
// whole, zeros in the padding; a natural destination (the weight) is updated
// in place, W[idx] -= lr * P[idx].
__global__ void tensor_permute_kernel(const __grid_constant__ PermArgs a, int64_t total) {
  pdl_launch_dependents();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= total) return;
  int idx[kMaxOrder] = {0, 0, 0, 0};
  bool inside = true;
  int64_t dst_off;
  if (a.d.mode < 0) {
    int64_t r = t;
#pragma unroll
    for (int l = kMaxOrder - 1; l >= 0; --l) {
      if (l >= a.k) continue;
      idx[l] = static_cast<int>(r % a.dims[l]);
      r /= a.dims[l];
    }
    dst_off = t;
  } else {
    const int row = static_cast<int>(t / a.cols);
    const int64_t col = t - static_cast<int64_t>(row) * a.cols;
    int64_t kcols = 1;
#pragma unroll
    for (int l = 0; l < kMaxOrder; ++l)
      if (l < a.k && l != a.d.mode) kcols *= a.dims[l];
    inside = row < a.dims[a.d.mode] && col < kcols;
    if (inside) {
      idx[a.d.mode] = row;
      unfold_col_index(a, a.d.mode, col, idx);
    }
    dst_off = static_cast<int64_t>(row) * a.d.ld + col;
  }
  float v = 0.f;
  if (inside) {
    const int64_t so = a.s.mode < 0 ? natural_offset(a, idx) : unfold_offset(a, a.s, idx);
    if (a.src_bf16) {
      const uint16_t bits = reinterpret_cast<const uint16_t*>(a.src)[so];
      v = __uint_as_float(static_cast<uint32_t>(bits) << 16);
    } else {
      v = reinterpret_cast<const float*>(a.src)[so];
    }
  }
  if (a.update)
    a.dst[dst_off] -= a.lr * v;
  else
    a.dst[dst_off] = v;
}

int launch_permute(const PermArgs& a, int64_t total, cudaStream_t st) {
  if (total <= 0) return 0;
  ProfScope ps(K_PERMUTE, st, 0.0, 8.0 * total);
  const unsigned grid = static_cast<unsigned>((total + 255) / 256);
  tensor_permute_kernel<<<grid, 256, 0, st>>>(a, total);
  count_launch();
  return check_cuda(cudaGetLastError(), "tensor_permute_kernel");
}

// Diagonal variant, statistics: h[x] <- beta h[x] + sum_c U[x][c]^2 over the
// row x of the mode's unfolding (one warp per row, float64 sums).
__global__ void row_sumsq_kernel(const float* __restrict__ U, int64_t ld, int n, int64_t K, float beta,
                                 float* __restrict__ h) {
  pdl_launch_dependents();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n) return;
  const float* row = U + static_cast<int64_t>(warp) * ld;
  double acc = 0.0;
  for (int64_t c = lane; c < K; c += 32) {
    const double v = row[c];
    acc += v * v;
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) h[warp] = static_cast<float>(static_cast<double>(beta) * h[warp] + acc);
}

// Diagonal variant, roots: d = (h + eps)^{-1/p}, 0 where h + eps = 0.
__global__ void diag_root_kernel(const float* __restrict__ h, int n, float eps, float inv_p, float* __restrict__ d,
                                 int* flags) {
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= n) return;
  const float v = h[x] + eps;
  const float r = v > 0.f ? powf(v, -inv_p) : 0.f;
  if (!isfinite(r)) raise_flag(flags, DEV_FLAG_NONFINITE);
  d[x] = r;
}

// Diagonal variant, product along the mode: out[x][c] = d[x] cur[x][c] for
// x < n (zero on the padded rows).
__global__ void row_scale_kernel(const float* __restrict__ cur, const float* __restrict__ d, int n, int rows,
                                 int64_t cols, float* __restrict__ out) {
  pdl_launch_dependents();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(rows) * cols) return;
  const int x = static_cast<int>(t / cols);
  out[t] = x < n ? d[x] * cur[t] : 0.f;
}

// Short-mode statistics are summed in K-chunks of 4096 fibres (kGramChunk),
// each chunk's n (n + 1) / 2 pair sums in float64 (at most kGramPairs);
// gram_reduce_kernel then adds the chunks' partials in chunk order and writes
// H <- beta H + sum (both triangles).
constexpr int kGramChunk = 4096;
constexpr int kGramPairs = 32 * 33 / 2;

__global__ void gram_reduce_kernel(const double* __restrict__ partial, int nchunks, int n, float beta,
                                   float* __restrict__ H, int ldh) {
  const int npairs = n * (n + 1) / 2;
  for (int pidx0 = threadIdx.x; pidx0 < npairs; pidx0 += blockDim.x) {
    double sum = 0.0;
    for (int ch = 0; ch < nchunks; ++ch) sum += partial[static_cast<int64_t>(ch) * kGramPairs + pidx0];
    int pidx = pidx0, x = 0;
    while (pidx >= n - x) pidx -= n - x, ++x;
    const int y = x + pidx;
    const float v = static_cast<float>(static_cast<double>(beta) * H[x * ldh + y] + sum);
    H[x * ldh + y] = v;
    H[y * ldh + x] = v;
  }
}

// Statistic of a short mode from the natural layout: the fibres along mode m
// (fixed other indices; element j of fibre f at (f / S) n S + j S + f % S,
// S the product of the later dimensions) are the columns of the mode's
// unfolding, so the Gram sum over fibres is the unfolding's.  Each CTA takes
// one chunk: it stages 128 fibres at a time in shared memory (n rows) and
// accumulates its threads' pairs (x <= y) in float64.  A single 32 x 32 GEMM
// tile would have to sweep all of K (up to 10^6) alone.
__global__ void __launch_bounds__(256) gram_natural_kernel(const void* __restrict__ src, int src_bf16, int n,
                                                           int64_t S, int64_t fibers,
                                                           double* __restrict__ partial) {
  __shared__ float tile[32][129];
  const int chunk = blockIdx.x;
  const int64_t f_begin = static_cast<int64_t>(chunk) * kGramChunk;
  const int64_t f_end = f_begin + kGramChunk < fibers ? f_begin + kGramChunk : fibers;
  const int npairs = n * (n + 1) / 2;
  double acc[3] = {0.0, 0.0, 0.0};
  int px[3], py[3];
#pragma unroll
  for (int q = 0; q < 3; ++q) {
    int pidx = threadIdx.x + 256 * q, x = 0;
    while (pidx >= n - x && x < n) pidx -= n - x, ++x;
    px[q] = x;
    py[q] = x + pidx;
  }
  for (int64_t f0 = f_begin; f0 < f_end; f0 += 128) {
    for (int e = threadIdx.x; e < 32 * 128; e += 256) {
      const int r = e >> 7, c = e & 127;
      const int64_t f = f0 + c;
      float v = 0.f;
      if (r < n && f < f_end) {
        const int64_t o = f / S;
        const int64_t off = o * n * S + static_cast<int64_t>(r) * S + (f - o * S);
        v = src_bf16 ? __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(src)[off]) << 16)
                     : reinterpret_cast<const float*>(src)[off];
      }
      tile[r][c] = v;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      if (threadIdx.x + 256 * q >= npairs) continue;
      double a = 0.0;
      for (int c = 0; c < 128; ++c) a += static_cast<double>(tile[px[q]][c]) * tile[py[q]][c];
      acc[q] += a;
    }
    __syncthreads();
  }
#pragma unroll
  for (int q = 0; q < 3; ++q)
    if (threadIdx.x + 256 * q < npairs) partial[static_cast<int64_t>(chunk) * kGramPairs + threadIdx.x + 256 * q] = acc[q];
}

// The same statistic for modes of at most 8: with a handful of pairs the
// staged tile leaves most threads idle, so here each thread takes every
// blockDim-th fibre of the chunk and keeps all N (N + 1) / 2 pair sums of its
// fibres in float64 registers; the CTA then adds its threads' sums in a fixed
// order (per warp by shuffles, then warp by warp).
template <int N>
__global__ void __launch_bounds__(256) gram_tiny_kernel(const void* __restrict__ src, int src_bf16, int64_t S,
                                                        int64_t fibers, double* __restrict__ partial) {
  constexpr int kPairs = N * (N + 1) / 2;
  __shared__ double red[8][kPairs];
  const int64_t f_begin = static_cast<int64_t>(blockIdx.x) * kGramChunk;
  const int64_t f_end = f_begin + kGramChunk < fibers ? f_begin + kGramChunk : fibers;
  double acc[kPairs];
#pragma unroll
  for (int q = 0; q < kPairs; ++q) acc[q] = 0.0;
  for (int64_t f = f_begin + threadIdx.x; f < f_end; f += blockDim.x) {
    const int64_t o = f / S;
    const int64_t base = o * N * S + (f - o * S);
    double x[N];
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const int64_t off = base + static_cast<int64_t>(j) * S;
      x[j] = src_bf16 ? __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(src)[off]) << 16)
                      : reinterpret_cast<const float*>(src)[off];
    }
    int q = 0;
#pragma unroll
    for (int a = 0; a < N; ++a)
#pragma unroll
      for (int b = a; b < N; ++b) acc[q++] += x[a] * x[b];
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int q = 0; q < kPairs; ++q) {
    double v = acc[q];
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) red[warp][q] = v;
  }
  __syncthreads();
  for (int q = threadIdx.x; q < kPairs; q += blockDim.x) {
    double v = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) v += red[w][q];
    partial[static_cast<int64_t>(blockIdx.x) * kGramPairs + q] = v;
  }
}

int launch_gram_natural(const void* src, int src_bf16, int n, int64_t S, int64_t fibers, double* partial,
                        cudaStream_t st) {
  const unsigned nchunks = static_cast<unsigned>((fibers + kGramChunk - 1) / kGramChunk);
  switch (n) {
#define GRAM_TINY(N) \
  case N: gram_tiny_kernel<N><<<nchunks, 256, 0, st>>>(src, src_bf16, S, fibers, partial); break;
    GRAM_TINY(1) GRAM_TINY(2) GRAM_TINY(3) GRAM_TINY(4) GRAM_TINY(5) GRAM_TINY(6) GRAM_TINY(7) GRAM_TINY(8)
#undef GRAM_TINY
    default: gram_natural_kernel<<<nchunks, 256, 0, st>>>(src, src_bf16, n, S, fibers, partial);
  }
  count_launch();
  return check_cuda(cudaGetLastError(), n <= 8 ? "gram_tiny_kernel" : "gram_natural_kernel");
}

// Product along a short mode in the natural layout: every fibre x (n values,
// stride S) becomes X x, X the mode's n x n root (row stride ldx); with
// `update` the result goes into the weight, dst -= lr X x.  One thread a
// fibre, grid-stride; consecutive threads take consecutive fibres, so every
// load and store is coalesced.
__global__ void __launch_bounds__(256) mode_small_kernel(const void* __restrict__ src, int src_bf16,
                                                         float* __restrict__ dst, int update, float lr,
                                                         const float* __restrict__ X, int ldx, int n, int64_t S,
                                                         int64_t fibers) {
  pdl_launch_dependents();
  __shared__ float xs[32][33];
  for (int e = threadIdx.x; e < 32 * 32; e += blockDim.x) {
    const int r = e >> 5, c = e & 31;
    xs[r][c] = (r < n && c < n) ? X[r * ldx + c] : 0.f;
  }
  __syncthreads();
  for (int64_t f = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; f < fibers;
       f += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t o = f / S;
    const int64_t base = o * n * S + (f - o * S);
    float x[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      x[j] = 0.f;
      if (j < n) {
        const int64_t off = base + static_cast<int64_t>(j) * S;
        x[j] = src_bf16 ? __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(src)[off]) << 16)
                        : reinterpret_cast<const float*>(src)[off];
      }
    }
#pragma unroll 1
    for (int i = 0; i < n; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) acc = fmaf(xs[i][j], x[j], acc);
      float* d = dst + base + static_cast<int64_t>(i) * S;
      if (update)
        *d -= lr * acc;
      else
        *d = acc;
    }
  }
}

struct Mode {
  int n, npad;
  int64_t K;
  int Kpad;
  int diag;          // 1: diagonal variant (h, d vectors instead of H, X)
  int group, slot;   // root group and index in its stacks (matrix modes)
  size_t h_off, d_off;  // state byte offsets of h and d (diagonal modes)
  size_t u_off;      // float offset of U_i in the unfolding area (per parameter)
};

struct Param {
  int k;
  int dims[kMaxOrder];
  int64_t size;
  std::vector<Mode> modes;
  size_t u_floats;   // all modes' unfoldings
};

struct Group {
  int npad, p, count;
  size_t h_off, x_off, valid_off;  // state byte offsets
  std::vector<int> valid;
};

struct Plan {
  std::vector<Param> params;
  std::vector<Group> groups;
  size_t state_status, state_total;
  size_t u_area, v_floats, root_bytes, gram_bytes;
  size_t scratch_u, scratch_v0, scratch_v1, scratch_root, scratch_gram, scratch_total;
};

// A mode whose statistic takes the split-K path.
// A mode handled in the natural layout (no unfolding): at most 32 long and not diagonal.
bool short_mode(const Mode& m) { return !m.diag && m.n <= 32; }

int validate_tensor_config(const shampoo_config* c) {
  if (!c) return set_error(SHAMPOO_ERR_INVALID_ARG, "config is NULL");
  if (!(c->beta >= 0.f) || !(c->beta <= 1.f)) return set_error(SHAMPOO_ERR_INVALID_ARG, "beta must be in [0, 1]");
  if (!(c->eps >= 0.f)) return set_error(SHAMPOO_ERR_INVALID_ARG, "eps must be >= 0");
  if (!(c->lr == c->lr)) return set_error(SHAMPOO_ERR_INVALID_ARG, "lr is NaN");
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
  if (c->momentum != 0.f) return set_error(SHAMPOO_ERR_UNSUPPORTED, "tensor Shampoo takes no momentum");
  if (c->diag_threshold > 1024)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "diag_threshold %d above 1024, the largest root computed",
                     c->diag_threshold);
  return SHAMPOO_OK;
}

int make_plan(const shampoo_config* cfg, int32_t nparams, const int32_t* orders, const int64_t* dims, Plan& P) {
  if (nparams < 1 || nparams > kMaxTensorParams)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "nparams %d: need 1..%d", nparams, kMaxTensorParams);
  if (!orders || !dims) return set_error(SHAMPOO_ERR_INVALID_ARG, "orders/dims is NULL");
  P = Plan();
  const int thr = cfg->diag_threshold > 0 ? cfg->diag_threshold : 1024;
  std::map<std::pair<int, int>, int> gid;
  size_t di = 0;
  for (int j = 0; j < nparams; ++j) {
    Param pr;
    pr.k = orders[j];
    if (pr.k < 2 || pr.k > kMaxOrder) return set_error(SHAMPOO_ERR_INVALID_ARG, "param %d has order %d (2..4)", j, pr.k);
    if (cfg->solver == SHAMPOO_SOLVER_NEWTON_DB && pr.k != 2)
      return set_error(SHAMPOO_ERR_INVALID_ARG, "Newton-DB computes the -1/4 power only (order 2)");
    pr.size = 1;
    for (int l = 0; l < pr.k; ++l) {
      const int64_t d = dims[di + l];
      if (d < 1) return set_error(SHAMPOO_ERR_INVALID_ARG, "param %d dimension %d is %lld", j, l, (long long)d);
      if (d > (1 << 20)) return set_error(SHAMPOO_ERR_UNSUPPORTED, "param %d dimension %d is %lld > 2^20", j, l,
                                          (long long)d);
      pr.dims[l] = static_cast<int>(d);
      pr.size *= d;
    }
    if (pr.size > (int64_t(1) << 31)) return set_error(SHAMPOO_ERR_UNSUPPORTED, "param %d is too large", j);
    di += pr.k;
    const int p = 2 * pr.k;
    pr.u_floats = 0;
    for (int i = 0; i < pr.k; ++i) {
      Mode m;
      m.n = pr.dims[i];
      m.npad = up32(m.n);
      m.K = pr.size / m.n;
      m.Kpad = up32(m.K);
      m.diag = m.n > thr ? 1 : 0;
      m.group = m.slot = -1;
      m.h_off = m.d_off = 0;
      m.u_off = pr.u_floats;
      pr.u_floats += alt(static_cast<size_t>(m.npad) * m.Kpad * 4) / 4;
      if (m.diag) {
        pr.modes.push_back(m);
        continue;
      }
      auto key = std::make_pair(m.npad, p);
      auto it = gid.find(key);
      if (it == gid.end()) {
        Group g;
        g.npad = m.npad;
        g.p = p;
        g.count = 0;
        it = gid.emplace(key, static_cast<int>(P.groups.size())).first;
        P.groups.push_back(g);
      }
      m.group = it->second;
      m.slot = P.groups[m.group].count++;
      P.groups[m.group].valid.push_back(m.n);
      pr.modes.push_back(m);
    }
    P.params.push_back(pr);
  }
  // state: status | per group: valid, H stack, X stack
  size_t o = 0;
  P.state_status = o, o += alt(4);
  for (Group& g : P.groups) {
    const size_t mat = static_cast<size_t>(g.npad) * g.npad * 4;
    g.valid_off = o, o += alt(static_cast<size_t>(g.count) * 4);
    g.h_off = o, o += alt(mat * g.count);
    g.x_off = o, o += alt(mat * g.count);
  }
  for (Param& pr : P.params)
    for (Mode& m : pr.modes)
      if (m.diag) {
        m.h_off = o, o += alt(static_cast<size_t>(m.n) * 4);
        m.d_off = o, o += alt(static_cast<size_t>(m.n) * 4);
      }
  P.state_total = o;
  // scratch: all unfoldings of the largest parameter | two product buffers | root solver
  P.u_area = 0;
  P.v_floats = 0;
  for (const Param& pr : P.params) {
    P.u_area = std::max(P.u_area, pr.u_floats);
    for (const Mode& m : pr.modes) P.v_floats = std::max(P.v_floats, static_cast<size_t>(m.npad) * m.Kpad);
  }
  P.gram_bytes = 0;
  for (const Param& pr : P.params)
    for (const Mode& m : pr.modes)
      if (short_mode(m))
        P.gram_bytes = std::max(P.gram_bytes, static_cast<size_t>((m.K + kGramChunk - 1) / kGramChunk) * kGramPairs * 8);
  P.root_bytes = 0;
  for (const Group& g : P.groups) {
    const size_t per = root_scratch_per_matrix(g.npad, cfg->solver, g.p);
    const size_t want = root_scratch_header() + per * g.count;
    P.root_bytes = std::max(P.root_bytes, std::min(want, std::max(kTensorRootBudget, root_scratch_header() + per)));
  }
  o = 0;
  P.scratch_u = o, o += alt(P.u_area * 4);
  P.scratch_v0 = o, o += alt(P.v_floats * 4);
  P.scratch_v1 = o, o += alt(P.v_floats * 4);
  P.scratch_root = o, o += alt(P.root_bytes);
  P.scratch_gram = o, o += alt(P.gram_bytes);
  P.scratch_total = o;
  return SHAMPOO_OK;
}

bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }

}  // namespace

struct shampoo_tensor_ctx {
  shampoo_config cfg;
  Plan plan;
  char* state = nullptr;
  char* scratch = nullptr;
  int* d_status = nullptr;
  std::vector<StackMaps> mH, mX;  // per group
  int64_t step = 0;
  cudaStream_t last_stream = nullptr;
};

extern "C" {

int shampoo_tensor_query_sizes(const shampoo_config* cfg, int32_t nparams, const int32_t* orders,
                               const int64_t* dims, size_t* state_bytes, size_t* scratch_bytes) {
  int rc = validate_tensor_config(cfg);
  if (rc) return rc;
  Plan P;
  if ((rc = make_plan(cfg, nparams, orders, dims, P))) return rc;
  if (!state_bytes || !scratch_bytes) return set_error(SHAMPOO_ERR_INVALID_ARG, "output pointer is NULL");
  *state_bytes = P.state_total;
  *scratch_bytes = P.scratch_total;
  return SHAMPOO_OK;
}

int shampoo_tensor_init(const shampoo_config* cfg, int32_t nparams, const int32_t* orders, const int64_t* dims,
                        void* d_state, size_t state_bytes, void* d_scratch, size_t scratch_bytes, void* stream,
                        shampoo_tensor_handle* out) {
  int rc = validate_tensor_config(cfg);
  if (rc) return rc;
  if (!out) return set_error(SHAMPOO_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  Plan P;
  if ((rc = make_plan(cfg, nparams, orders, dims, P))) return rc;
  if (!d_state || !d_scratch) return set_error(SHAMPOO_ERR_INVALID_ARG, "state/scratch is NULL");
  if (!aligned256(d_state) || !aligned256(d_scratch))
    return set_error(SHAMPOO_ERR_UNSUPPORTED, "state/scratch must be 256-byte aligned");
  if (state_bytes < P.state_total)
    return set_error(SHAMPOO_ERR_WORKSPACE, "state %zu < %zu bytes", state_bytes, P.state_total);
  if (scratch_bytes < P.scratch_total)
    return set_error(SHAMPOO_ERR_WORKSPACE, "scratch %zu < %zu bytes", scratch_bytes, P.scratch_total);
  shampoo_tensor_ctx* h = new (std::nothrow) shampoo_tensor_ctx;
  if (!h) return set_error(SHAMPOO_ERR_INVALID_ARG, "out of host memory");
  h->cfg = *cfg;
  h->plan = P;
  h->state = static_cast<char*>(d_state);
  h->scratch = static_cast<char*>(d_scratch);
  h->d_status = reinterpret_cast<int*>(h->state + P.state_status);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  rc = check_cuda(cudaMemsetAsync(h->state, 0, P.state_total, st), "zero tensor state");
  for (size_t g = 0; g < P.groups.size() && !rc; ++g) {
    const Group& G = P.groups[g];
    rc = check_cuda(cudaMemcpyAsync(h->state + G.valid_off, G.valid.data(), G.valid.size() * 4,
                                    cudaMemcpyHostToDevice, st),
                    "upload valid extents");
  }
  if (!rc) rc = check_cuda(cudaStreamSynchronize(st), "tensor init sync");
  h->mH.resize(P.groups.size());
  h->mX.resize(P.groups.size());
  for (size_t g = 0; g < P.groups.size() && !rc; ++g) {
    const Group& G = P.groups[g];
    if ((rc = make_stack_maps(h->mH[g], reinterpret_cast<float*>(h->state + G.h_off), G.count, G.npad))) break;
    rc = make_stack_maps(h->mX[g], reinterpret_cast<float*>(h->state + G.x_off), G.count, G.npad);
  }
  if (rc) {
    delete h;
    return rc;
  }
  *out = h;
  return SHAMPOO_OK;
}

int shampoo_tensor_step(shampoo_tensor_handle h, float* const* d_weights, const void* const* d_grads, void* stream) {
  if (!h) return set_error(SHAMPOO_ERR_INVALID_ARG, "handle is NULL");
  if (!d_weights || !d_grads) return set_error(SHAMPOO_ERR_INVALID_ARG, "weights/grads array is NULL");
  const Plan& P = h->plan;
  const shampoo_config& c = h->cfg;
  for (size_t j = 0; j < P.params.size(); ++j)
    if (!d_weights[j] || !d_grads[j]) return set_error(SHAMPOO_ERR_INVALID_ARG, "param %zu has a NULL pointer", j);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  float* U = reinterpret_cast<float*>(h->scratch + P.scratch_u);
  float* V[2] = {reinterpret_cast<float*>(h->scratch + P.scratch_v0),
                 reinterpret_cast<float*>(h->scratch + P.scratch_v1)};
  const bool refresh = h->step % c.refresh_every == 0;
  const int g_exact = c.grad_dtype == SHAMPOO_BF16 ? 1 : 0;
  int rc;
  auto hptr = [&](const Mode& m) {
    const Group& G = P.groups[m.group];
    return reinterpret_cast<float*>(h->state + G.h_off) + static_cast<size_t>(m.slot) * G.npad * G.npad;
  };
  // stride of mode i in the natural layout: the product of the later dimensions
  auto stride_after = [](const Param& pr, int i) {
    int64_t S = 1;
    for (int l = i + 1; l < pr.k; ++l) S *= pr.dims[l];
    return S;
  };
  const int bf16 = c.grad_dtype == SHAMPOO_BF16 ? 1 : 0;
  // 1-2. unfold every long mode of every parameter and accumulate its
  // statistic (one GEMM launch per parameter, one group per mode); short
  // modes sum theirs from the gradient's natural layout.  With a refresh
  // pending, all statistics must be complete before the roots.
  for (size_t j = 0; j < P.params.size(); ++j) {
    const Param& pr = P.params[j];
    std::vector<StackMaps> um(pr.k);
    for (int i = 0; i < pr.k; ++i) {
      const Mode& m = pr.modes[i];
      if (short_mode(m)) continue;
      PermArgs a;
      std::memset(&a, 0, sizeof(a));
      a.k = pr.k;
      for (int l = 0; l < pr.k; ++l) a.dims[l] = pr.dims[l];
      a.src = d_grads[j];
      a.src_bf16 = bf16;
      a.s = PermSide{-1, 0};
      a.dst = U + m.u_off;
      a.d = PermSide{i, m.Kpad};
      a.rows = m.npad;
      a.cols = m.Kpad;
      if ((rc = launch_permute(a, static_cast<int64_t>(m.npad) * m.Kpad, st))) return rc;
      if (!m.diag && (rc = make_rect_maps(um[i], U + m.u_off, 1, m.npad, m.Kpad))) return rc;
    }
    Builder b;
    for (int i = 0; i < pr.k; ++i) {
      const Mode& m = pr.modes[i];
      if (m.diag) {
        ProfScope ps(K_DIAG, st, 0.0, 4.0 * m.n * double(m.Kpad));
        const unsigned blocks = static_cast<unsigned>((static_cast<int64_t>(m.n) * 32 + 255) / 256);
        row_sumsq_kernel<<<blocks, 256, 0, st>>>(U + m.u_off, m.Kpad, m.n, m.K, c.beta,
                                                 reinterpret_cast<float*>(h->state + m.h_off));
        count_launch();
        if ((rc = check_cuda(cudaGetLastError(), "row_sumsq_kernel"))) return rc;
        continue;
      }
      if (short_mode(m)) {
        double* partial = reinterpret_cast<double*>(h->scratch + P.scratch_gram);
        const int nchunks = static_cast<int>((m.K + kGramChunk - 1) / kGramChunk);
        {
          ProfScope ps(K_GRAM, st, 2.0 * m.n * double(m.n) * m.K, (bf16 ? 2.0 : 4.0) * m.n * double(m.K));
          if ((rc = launch_gram_natural(d_grads[j], bf16, m.n, stride_after(pr, i), m.K, partial, st))) return rc;
          gram_reduce_kernel<<<1, 256, 0, st>>>(partial, nchunks, m.n, c.beta, hptr(m), m.npad);
          count_launch();
          if ((rc = check_cuda(cudaGetLastError(), "gram_reduce_kernel"))) return rc;
        }
        continue;
      }
      Epilogue& e = b.add_rect(1, m.npad, m.npad, m.Kpad, um[i], 0, um[i], 0, 2.0 * m.n * double(m.n) * m.K,
                               B_TRANSPOSED);
      b.L.g[b.L.ngroups - 1].a_exact = b.L.g[b.L.ngroups - 1].b_exact = g_exact;
      b.L.g[b.L.ngroups - 1].sym = 1;
      e.beta = c.beta;
      e.C = hptr(m);
      e.D = hptr(m);
      e.flags = h->d_status;
    }
    if (b.L.ngroups > 0 && (rc = b.launch(st))) return rc;
    for (int i = 0; i < pr.k; ++i)
      if (!pr.modes[i].diag && !short_mode(pr.modes[i]) &&
          (rc = launch_mirror_lower(hptr(pr.modes[i]), 1, pr.modes[i].npad, st)))
        return rc;
  }
  // 3. roots X = (H + eps I)^{-1/(2k)}, batched per (npad, k)
  if (refresh) {
    for (size_t g = 0; g < P.groups.size(); ++g) {
      const Group& G = P.groups[g];
      RootJob job;
      job.batch = G.count;
      job.n = G.npad;
      job.p = G.p;
      job.solver = c.solver;
      job.iters = c.iters;
      job.cheb_degree = c.cheb_degree;
      job.eps = c.eps;
      job.tol = c.tol;
      job.cheb_lo = c.cheb_lo;
      job.A = reinterpret_cast<float*>(h->state + G.h_off);
      job.valid = reinterpret_cast<int*>(h->state + G.valid_off);
      job.X = reinterpret_cast<float*>(h->state + G.x_off);
      job.iters_used = nullptr;
      job.flags = h->d_status;
      if ((rc = run_inverse_roots(job, h->scratch + P.scratch_root, P.root_bytes, st))) return rc;
    }
    for (const Param& pr : P.params)
      for (const Mode& m : pr.modes) {
        if (!m.diag) continue;
        ProfScope ps(K_DIAG, st, 0.0, 8.0 * m.n);
        diag_root_kernel<<<static_cast<unsigned>((m.n + 255) / 256), 256, 0, st>>>(
            reinterpret_cast<const float*>(h->state + m.h_off), m.n, c.eps, 1.f / (2 * pr.k),
            reinterpret_cast<float*>(h->state + m.d_off), h->d_status);
        count_launch();
        if ((rc = check_cuda(cudaGetLastError(), "diag_root_kernel"))) return rc;
      }
  }
  // 4. apply: the short modes' products on the natural layout first, then the
  // long modes on unfoldings (mode by mode); the last product updates W.
  auto xptr = [&](const Mode& m) {
    const Group& G = P.groups[m.group];
    return reinterpret_cast<const float*>(h->state + G.x_off) + static_cast<size_t>(m.slot) * G.npad * G.npad;
  };
  for (size_t j = 0; j < P.params.size(); ++j) {
    const Param& pr = P.params[j];
    std::vector<int> shorts, longs;
    for (int i = 0; i < pr.k; ++i) (short_mode(pr.modes[i]) ? shorts : longs).push_back(i);
    const void* src = d_grads[j];  // natural layout of the partial product
    int src_bf16 = bf16;
    for (size_t q = 0; q < shorts.size(); ++q) {
      const Mode& m = pr.modes[shorts[q]];
      const bool last = longs.empty() && q + 1 == shorts.size();
      float* dst = last ? d_weights[j] : (src == V[0] ? V[1] : V[0]);
      const int64_t fibers = pr.size / m.n;
      ProfScope ps(K_MODE_SMALL, st, 2.0 * m.n * double(m.n) * fibers, ((src_bf16 ? 2.0 : 4.0) + (last ? 8.0 : 4.0)) * pr.size);
      const unsigned grid = static_cast<unsigned>(std::min<int64_t>((fibers + 255) / 256, 148 * 8));
      mode_small_kernel<<<grid, 256, 0, st>>>(src, src_bf16, dst, last ? 1 : 0, c.lr, xptr(m), m.npad, m.n,
                                              stride_after(pr, shorts[q]), fibers);
      count_launch();
      if ((rc = check_cuda(cudaGetLastError(), "mode_small_kernel"))) return rc;
      src = dst;
      src_bf16 = 0;
    }
    if (longs.empty()) continue;
    // cur: unfolding of the partial product along the current mode; out: X_i cur.
    // The next mode's permutation reads `out` into `cur`, so the two never trade roles.
    float* cur = src == V[1] ? V[0] : V[1];
    float* out = cur == V[1] ? V[0] : V[1];
    {  // first long mode's unfolding of the natural partial product
      const Mode& m0 = pr.modes[longs[0]];
      PermArgs a;
      std::memset(&a, 0, sizeof(a));
      a.k = pr.k;
      for (int l = 0; l < pr.k; ++l) a.dims[l] = pr.dims[l];
      a.src = src;
      a.src_bf16 = src_bf16;
      a.s = PermSide{-1, 0};
      a.dst = cur;
      a.d = PermSide{longs[0], m0.Kpad};
      a.rows = m0.npad;
      a.cols = m0.Kpad;
      if ((rc = launch_permute(a, static_cast<int64_t>(m0.npad) * m0.Kpad, st))) return rc;
    }
    for (size_t q = 0; q < longs.size(); ++q) {
      const int i = longs[q];
      const Mode& m = pr.modes[i];
      if (q > 0) {  // cur <- mode-i unfolding of the previous product (held in `out` as that mode's)
        const Mode& mp = pr.modes[longs[q - 1]];
        PermArgs a;
        std::memset(&a, 0, sizeof(a));
        a.k = pr.k;
        for (int l = 0; l < pr.k; ++l) a.dims[l] = pr.dims[l];
        a.src = out;
        a.s = PermSide{longs[q - 1], mp.Kpad};
        a.dst = cur;
        a.d = PermSide{i, m.Kpad};
        a.rows = m.npad;
        a.cols = m.Kpad;
        if ((rc = launch_permute(a, static_cast<int64_t>(m.npad) * m.Kpad, st))) return rc;
      }
      if (m.diag) {
        ProfScope ps(K_DIAG, st, 0.0, 8.0 * m.npad * double(m.Kpad));
        const int64_t total = static_cast<int64_t>(m.npad) * m.Kpad;
        row_scale_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(
            cur, reinterpret_cast<const float*>(h->state + m.d_off), m.n, m.npad, m.Kpad, out);
        count_launch();
        if ((rc = check_cuda(cudaGetLastError(), "row_scale_kernel"))) return rc;
        continue;
      }
      StackMaps cm;
      if ((rc = make_rect_maps(cm, cur, 1, m.npad, m.Kpad))) return rc;
      Builder b;
      Epilogue& e = b.add_rect(1, m.npad, m.Kpad, m.npad, h->mX[m.group], m.slot, cm, 0,
                               2.0 * m.n * double(m.n) * m.K, B_MN_MAJOR);
      if (q == 0 && shorts.empty()) b.L.g[0].b_exact = g_exact;  // the raw (widened bf16) gradient
      e.D = out;
      e.flags = h->d_status;
      if ((rc = b.launch(st))) return rc;
    }
    {  // fold the last product (its mode's unfolding) into the weight: W -= lr P
      const Mode& ml = pr.modes[longs.back()];
      PermArgs a;
      std::memset(&a, 0, sizeof(a));
      a.k = pr.k;
      for (int l = 0; l < pr.k; ++l) a.dims[l] = pr.dims[l];
      a.src = out;
      a.s = PermSide{longs.back(), ml.Kpad};
      a.dst = d_weights[j];
      a.d = PermSide{-1, 0};
      a.update = 1;
      a.lr = c.lr;
      if ((rc = launch_permute(a, pr.size, st))) return rc;
    }
  }
  h->step += 1;
  return SHAMPOO_OK;
}

int shampoo_tensor_views(shampoo_tensor_handle h, int32_t param, int32_t mode, float** H, float** X, int32_t* npad,
                         int32_t* diagonal, int64_t* step) {
  if (!h) return set_error(SHAMPOO_ERR_INVALID_ARG, "handle is NULL");
  const Plan& P = h->plan;
  if (param < 0 || param >= static_cast<int>(P.params.size()) || mode < 0 || mode >= P.params[param].k)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "no mode %d of param %d", mode, param);
  const Mode& m = P.params[param].modes[mode];
  if (diagonal) *diagonal = m.diag;
  if (step) *step = h->step;
  if (m.diag) {
    if (H) *H = reinterpret_cast<float*>(h->state + m.h_off);
    if (X) *X = reinterpret_cast<float*>(h->state + m.d_off);
    if (npad) *npad = m.n;
    return SHAMPOO_OK;
  }
  const Group& G = P.groups[m.group];
  const size_t off = static_cast<size_t>(m.slot) * G.npad * G.npad;
  if (H) *H = reinterpret_cast<float*>(h->state + G.h_off) + off;
  if (X) *X = reinterpret_cast<float*>(h->state + G.x_off) + off;
  if (npad) *npad = G.npad;
  if (step) *step = h->step;
  return SHAMPOO_OK;
}

int shampoo_tensor_get_status(shampoo_tensor_handle h, int32_t* status, int32_t reset) {
  if (!h || !status) return set_error(SHAMPOO_ERR_INVALID_ARG, "handle/status is NULL");
  int rc = check_cuda(cudaStreamSynchronize(h->last_stream), "status sync");
  if (rc) return rc;
  int v = 0;
  if ((rc = check_cuda(cudaMemcpy(&v, h->d_status, 4, cudaMemcpyDeviceToHost), "read status"))) return rc;
  *status = v;
  if (reset && (rc = check_cuda(cudaMemset(h->d_status, 0, 4), "reset status"))) return rc;
  return SHAMPOO_OK;
}

void shampoo_tensor_destroy(shampoo_tensor_handle h) { delete h; }

}  // extern "C"
