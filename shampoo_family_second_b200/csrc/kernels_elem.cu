// Memory-bound kernels of the blocked Shampoo step: the block partitioner /
// stacker, the damping + Frobenius pre-scaling prologues of the inverse-root
// solvers, the residual check, the unscale / output pass, and the Chebyshev
// coefficient setup.  All reads and writes are coalesced (transposes go through
// a 32 x 33 shared-memory tile) and each kernel touches each byte once.
#include <algorithm>
#include <cmath>

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace shampoo {

// Kernels executed inside graph loops (added by the loop's check kernel once
// per pass); read by shampoo_launch_count.
__device__ unsigned long long g_graph_kernels = 0;

uint64_t graph_kernel_count() {
  unsigned long long v = 0;
  if (cudaMemcpyFromSymbol(&v, g_graph_kernels, sizeof(v)) != cudaSuccess) return 0;
  return v;
}

namespace {

__device__ __forceinline__ float load_grad(const void* g, size_t idx, int dtype) {
  if (dtype == 1) {
    const uint16_t bits = reinterpret_cast<const uint16_t*>(g)[idx];
    return __uint_as_float(static_cast<uint32_t>(bits) << 16);
  }
  return reinterpret_cast<const float*>(g)[idx];
}

// ---------------------------------------------------------------------------
// A1 partition / stack.  DASH abstract: preconditioner blocks stacked into 3D
// tensors.  Block b of the table {param, row0, col0, r, c} is copied from the
// row-major gradient into Gs[b] (B x B) and its transpose into Gt[b],
// zero-padded beyond (r, c).  Also records where the block's weights live.
// grid (ceil(B/128), B/32, nb), block (32, 8): a CTA moves a 32 x 128 piece.
// Each thread loads 4 x 4 consecutive values (16-byte loads when the row is
// aligned), writes them to Gs directly and through a shared-memory tile to
// Gt; the tile's row stride (132 floats) keeps the 16-byte stores aligned.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float4 load_grad4(const void* g, size_t idx, int dtype, bool vec, int valid_cols) {
  // Values idx .. idx+3 of one row; columns beyond valid_cols read as 0.
  if (vec && valid_cols >= 4) {
    if (dtype == 1) {
      const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(g) + idx);
      return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                         __uint_as_float(u.y & 0xFFFF0000u));
    }
    return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(g) + idx);
  }
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (valid_cols > 0) v.x = load_grad(g, idx + 0, dtype);
  if (valid_cols > 1) v.y = load_grad(g, idx + 1, dtype);
  if (valid_cols > 2) v.z = load_grad(g, idx + 2, dtype);
  if (valid_cols > 3) v.w = load_grad(g, idx + 3, dtype);
  return v;
}

// With a moment stack (M != NULL) the same pass updates it in place,
// M_b <- alpha M_b + gscale G_b: Shampoo's momentum ahead of the
// preconditioner (podcast cue 28; gscale = 1) or Adam's first moment (SOAP;
// alpha = beta1, gscale = 1 - beta1).  The statistics keep the raw G in Gs, Gt.
// Four values exact in bf16 (widened bf16 gradients) as packed bf16: their
// upper halves, element 0 in the low half-word.
__device__ __forceinline__ uint2 pack_bf16x4(float4 v) {
  return make_uint2((__float_as_uint(v.x) >> 16) | (__float_as_uint(v.y) & 0xFFFF0000u),
                    (__float_as_uint(v.z) >> 16) | (__float_as_uint(v.w) & 0xFFFF0000u));
}

__global__ void stack_blocks_kernel(const __grid_constant__ StackArgs args, const int* __restrict__ table, int B,
                                    int dtype, float* __restrict__ Gs, float* __restrict__ Gt,
                                    float* __restrict__ M, float alpha, float gscale, float** blk_wptr,
                                    int* blk_ld, uint16_t* __restrict__ Gs16, uint16_t* __restrict__ Gt16) {
  pdl_launch_dependents();  // a following GEMM may start its prologue
  constexpr int TC = 128, STRIDE = TC + 4;
  __shared__ __align__(16) float tile[32 * STRIDE];
  const int b = blockIdx.z;
  const int r0 = blockIdx.y * 32;      // first row of the piece (block coordinates)
  const int c0 = blockIdx.x * TC;      // first column
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int t = ty * 32 + tx;
  const int param = table[5 * b + 0];
  const int row0 = table[5 * b + 1], col0 = table[5 * b + 2];
  const int r = table[5 * b + 3], c = table[5 * b + 4];
  const void* g = args.g[param];
  const int ld = args.ld[param];
  const bool vec = args.vec[param] != 0;
  const size_t nn = static_cast<size_t>(B) * B;
  const int col = c0 + 4 * tx;  // this thread's 4 columns
  if (col < B) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int row = r0 + ty + 8 * k;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (row < r) v = load_grad4(g, static_cast<size_t>(row0 + row) * ld + col0 + col, dtype, vec, c - col);
      if (Gs16)  // bf16 gradients: the statistics read G as bf16
        *reinterpret_cast<uint2*>(Gs16 + b * nn + static_cast<size_t>(row) * B + col) = pack_bf16x4(v);
      else
        *reinterpret_cast<float4*>(Gs + b * nn + static_cast<size_t>(row) * B + col) = v;
      if (M) {
        float4* mp = reinterpret_cast<float4*>(M + b * nn + static_cast<size_t>(row) * B + col);
        float4 m = *mp;
        m.x = fmaf(alpha, m.x, gscale * v.x);
        m.y = fmaf(alpha, m.y, gscale * v.y);
        m.z = fmaf(alpha, m.z, gscale * v.z);
        m.w = fmaf(alpha, m.w, gscale * v.w);
        *mp = m;
      }
      *reinterpret_cast<float4*>(&tile[(ty + 8 * k) * STRIDE + 4 * tx]) = v;
    }
  }
  __syncthreads();
  // Gt[b][c0 + j][r0 .. r0+31] = tile[0 .. 31][j]: 128 rows of 8 float4 each.
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int idx = t + 256 * k;
    const int j = idx >> 3;         // column of the piece = row of Gt
    const int part = idx & 7;       // 4-row group
    if (c0 + j < B) {
      float4 v;
      v.x = tile[(4 * part + 0) * STRIDE + j];
      v.y = tile[(4 * part + 1) * STRIDE + j];
      v.z = tile[(4 * part + 2) * STRIDE + j];
      v.w = tile[(4 * part + 3) * STRIDE + j];
      if (Gt) *reinterpret_cast<float4*>(Gt + b * nn + static_cast<size_t>(c0 + j) * B + r0 + 4 * part) = v;
      if (Gt16) *reinterpret_cast<uint2*>(Gt16 + b * nn + static_cast<size_t>(c0 + j) * B + r0 + 4 * part) =
          pack_bf16x4(v);
    }
  }
  if (blockIdx.x == 0 && blockIdx.y == 0 && t == 0) {
    blk_wptr[b] = args.w[param] + static_cast<size_t>(row0) * ld + col0;
    blk_ld[b] = ld;
  }
}

// ---------------------------------------------------------------------------
// s_i = ||A_i + eps I||_F over the valid region, and sc_i = s_i^{-1/p}
// (Frobenius pre-scaling; DASH abstract: matrix scaling).  One CTA per matrix,
// float64 accumulation.
// ---------------------------------------------------------------------------
__global__ void frob_norm_kernel(const float* __restrict__ A, int n, const int* __restrict__ valid, float eps,
                                 double inv_p, float* __restrict__ s, float* __restrict__ sc) {
  const int i = blockIdx.x;
  const int v = valid ? valid[i] : n;
  const float* a = A + static_cast<size_t>(i) * n * n;
  double acc = 0.0;
  for (int r = threadIdx.y; r < v; r += blockDim.y) {
    const float* row = a + static_cast<size_t>(r) * n;
    for (int c = threadIdx.x; c < v; c += blockDim.x) {
      const double x = static_cast<double>(row[c]) + ((r == c) ? static_cast<double>(eps) : 0.0);
      acc += x * x;
    }
  }
  __shared__ double red[32];
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  const int tid = threadIdx.y * blockDim.x + threadIdx.x;
  if ((tid & 31) == 0) red[tid >> 5] = acc;
  __syncthreads();
  if (tid < 32) {
    const int nw = (blockDim.x * blockDim.y) >> 5;
    double x = (tid < nw) ? red[tid] : 0.0;
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (tid == 0) {
      double sv = sqrt(x);
      if (!(sv > 0.0)) sv = 1.0;  // all-zero matrix with eps = 0: keep the scale finite
      s[i] = static_cast<float>(sv);
      sc[i] = static_cast<float>(pow(sv, -inv_p));
    }
  }
}

// Coupled-Newton scaling (DASH abstract: matrix scaling).  sf_i =
// ||A_i + eps I||_F over the valid region (float64 accumulation), and
// s_i = min(sf_i, 1.25 lam_i) with lam_i a power-iteration estimate of the
// largest eigenvalue of A_i + eps I: `iters` steps x <- (A + eps I) x / ||.||
// from a fixed start vector, lam = the last norm (a lower estimate of the
// largest eigenvalue, within a few percent after 12 steps on these
// matrices).  sf >= lam_max always; coupled Newton converges for any scaled
// spectrum in (0, p + 1), so an estimate below lam_max stays safe, and the
// largest scaled eigenvalue lands near 0.8 instead of lam_max / sf (0.1 to 0.3
// on Wishart-like statistics), which saves iterations.  sc_i = s_i^{-1/p}.
// One CTA of 512 threads per matrix; x and (A + eps I) x live in shared memory.
// With a vector store (vec != NULL) the last normalised iterate of each matrix
// is kept there, and when *warm != 0 the next call starts from it and runs
// warm_iters steps instead of iters: statistics change little between
// refreshes, so the previous dominant direction is already close.  The store
// and its flag live in the caller's state, so a restored state restarts the
// same way.
__global__ void __launch_bounds__(512) spectral_scale_kernel(const float* __restrict__ A, int n,
                                                             const int* __restrict__ valid, float eps, double inv_p,
                                                             int iters, float* __restrict__ s,
                                                             float* __restrict__ sc, float* __restrict__ sf,
                                                             float* __restrict__ vec, const int* __restrict__ warm,
                                                             int warm_iters) {
  extern __shared__ float xy[];  // x[n], y[n]
  __shared__ double red[16];
  __shared__ double bcast;
  const int i = blockIdx.x;
  const int v = valid ? valid[i] : n;
  const float* a = A + static_cast<size_t>(i) * n * n;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* x = xy;
  float* y = xy + n;
  auto block_sum = [&](double t) -> double {
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) red[warp] = t;
    __syncthreads();
    if (warp == 0) {
      double u = (lane < 16) ? red[lane] : 0.0;
      for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
      if (lane == 0) bcast = u;
    }
    __syncthreads();
    const double r = bcast;
    __syncthreads();
    return r;
  };
  // Frobenius norm of A + eps I (valid region)
  double acc = 0.0;
  for (int r = warp; r < v; r += 16) {
    const float* row = a + static_cast<size_t>(r) * n;
    for (int c = lane; c < v; c += 32) {
      const double t = static_cast<double>(row[c]) + ((r == c) ? static_cast<double>(eps) : 0.0);
      acc += t * t;
    }
  }
  double fro = sqrt(block_sum(acc));
  if (!(fro > 0.0)) fro = 1.0;  // all-zero matrix with eps = 0: keep the scale finite
  // start vector: the stored one (warm), else positive with a fixed irregular pattern
  const bool from_store = vec && warm && *warm;
  float* xs = vec ? vec + static_cast<size_t>(i) * n : nullptr;
  double nx = 0.0;
  for (int j = tid; j < v; j += 512) {
    const float t = from_store ? xs[j] : 1.f + 0.3f * static_cast<float>((j * 7919) % 17) / 17.f;
    x[j] = t;
    nx += static_cast<double>(t) * t;
  }
  nx = sqrt(block_sum(nx));
  if (!(nx > 0.0)) {  // a stored zero vector (all-zero statistics): the fixed start
    nx = 0.0;
    for (int j = tid; j < v; j += 512) {
      const float t = 1.f + 0.3f * static_cast<float>((j * 7919) % 17) / 17.f;
      x[j] = t;
      nx += static_cast<double>(t) * t;
    }
    nx = sqrt(block_sum(nx));
  }
  for (int j = tid; j < v; j += 512) x[j] = static_cast<float>(x[j] / nx);
  __syncthreads();
  double lam = 0.0;
  const int steps = from_store ? warm_iters : iters;
  for (int k = 0; k < steps; ++k) {
    double part = 0.0;
    for (int r = warp; r < v; r += 16) {
      const float* row = a + static_cast<size_t>(r) * n;
      float dot = 0.f;
      for (int c = lane; c < v; c += 32) dot = fmaf(row[c], x[c], dot);
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (lane == 0) {
        const float yr = dot + eps * x[r];
        y[r] = yr;
        part += static_cast<double>(yr) * yr;
      }
    }
    lam = sqrt(block_sum(part));
    if (!(lam > 0.0)) break;
    for (int j = tid; j < v; j += 512) x[j] = static_cast<float>(y[j] / lam);
    __syncthreads();
  }
  if (xs)
    for (int j = tid; j < v; j += 512) xs[j] = x[j];
  if (tid == 0) {
    double sv = fro;
    if (lam > 0.0 && 1.25 * lam < fro) sv = 1.25 * lam;
    s[i] = static_cast<float>(sv);
    sf[i] = static_cast<float>(fro);
    sc[i] = static_cast<float>(pow(sv, -inv_p));
  }
}


// Damping actually applied by the solvers: eps_eff = max(eps, u s) with
// u = 2^-24 and s = ||A + eps I||_F.  Statistics accumulated in fp32 carry
// rounding errors of about u s, which can make A + eps I indefinite when eps
// is below that level; the iterations would then grow the negative
// eigenvalue until it overflows.  A shift of u s is the size of rounding A to
// fp32 and keeps the scaled matrix positive definite.
__device__ __forceinline__ float effective_eps(float eps, float s) { return fmaxf(eps, s * 5.9604645e-8f); }

// ---------------------------------------------------------------------------
// Solver prologues.  A' = (sym(A) + eps_eff I) / s on the valid region; the
// padded region of a ragged block gets the identity (its root is then exactly
// the identity times s^{-1/p} and never slows convergence).
//   kind 0, coupled Newton: out0 = M0 = A', out1 = T0 = ((p+1) I - A') / p,
//                           out2 = X1 = T0.
//   kind 1, Newton-DB:      out0 = Y0 = A', out1 = T0 = (3 I - A') / 2,
//                           out2 = Z1 = T0.
// grid (n/32, n/32, batch), block (32, 8).
// ---------------------------------------------------------------------------
// set_flag (nullable): written 1 by one thread (marks a power-iterate store as
// filled; this kernel runs after the scale kernel that read the flag).
__global__ void root_prologue_kernel(int kind, const float* __restrict__ A, int n, const int* __restrict__ valid,
                                     float eps, int p, const float* __restrict__ s, const float* __restrict__ sf,
                                     float* __restrict__ out0, float* __restrict__ out1, float* __restrict__ out2,
                                     int* set_flag) {
  pdl_launch_dependents();  // a following GEMM may start its prologue
  if (set_flag && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0 && threadIdx.y == 0)
    *set_flag = 1;
  __shared__ float t1[32][33];
  __shared__ float t2[32][33];
  const int i = blockIdx.z;
  const int bi = blockIdx.y, bj = blockIdx.x;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const size_t nn = static_cast<size_t>(n) * n;
  const float* a = A + i * nn;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    t1[ty + 8 * k][tx] = a[static_cast<size_t>(bi * 32 + ty + 8 * k) * n + bj * 32 + tx];
    t2[ty + 8 * k][tx] = a[static_cast<size_t>(bj * 32 + ty + 8 * k) * n + bi * 32 + tx];
  }
  __syncthreads();
  const int v = valid ? valid[i] : n;
  const float inv_s = 1.f / s[i];
  const float eps_eff = effective_eps(eps, sf[i]);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = bi * 32 + ty + 8 * k, c = bj * 32 + tx;
    const float sym = 0.5f * (t1[ty + 8 * k][tx] + t2[tx][ty + 8 * k]);
    const float d = (r == c) ? 1.f : 0.f;
    const float m = (r < v && c < v) ? (sym + d * eps_eff) * inv_s : d;
    float t;
    if (kind == 0)
      t = (static_cast<float>(p + 1) * d - m) / static_cast<float>(p);
    else
      t = 0.5f * (3.f * d - m);
    const size_t idx = i * nn + static_cast<size_t>(r) * n + c;
    out0[idx] = m;
    out1[idx] = t;
    out2[idx] = t;
  }
}

// Second Newton-DB stage (p = 4): its input is the first stage's Y (~A'^{1/2},
// spectrum in (0, 1]); Y0' = Y, T0 = (3 I - Y) / 2, Z1 = T0.  Elementwise.
__global__ void db_stage2_kernel(const float* Y0, const float* Y1, const int* __restrict__ iters, int n,
                                 float* Ynew0, float* __restrict__ T, float* __restrict__ Z1) {
  pdl_launch_dependents();  // a following GEMM may start its prologue
  const int i = blockIdx.y;
  const size_t nn = static_cast<size_t>(n) * n;
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= nn) return;
  const float* src = (iters[i] & 1) ? Y1 : Y0;
  const float y = src[i * nn + idx];
  const int r = static_cast<int>(idx / n), c = static_cast<int>(idx % n);
  const float t = 0.5f * (3.f * ((r == c) ? 1.f : 0.f) - y);
  Ynew0[i * nn + idx] = y;
  T[i * nn + idx] = t;
  Z1[i * nn + idx] = t;
}

// Residual check after an iteration, one CTA for the whole batch.  The
// iteration number is it = counter[0] + 1 (counter[0] then holds it, and
// counter[1] the number of matrices still active).  For an
// active matrix with r = |tr(I - acc)| / valid:
//   r <= tol                        done = 1 (converged);
//   it >= kmin, r >= (1 - 1e-3) r'  done = 2 (stagnated; r' = previous r);
//   it >= cap                       done = 3 (iteration cap reached).
// Both iterations lift an eigenvalue mu << 1 of M by a fixed factor per
// iteration (((p+1)/p)^p for coupled Newton, 9/4 for the square-root
// iteration), so by iteration kmin every eigenvalue above fp32 resolution
// (2^-24) has converged in exact arithmetic; a residual that no longer falls
// from there on is held up by rounding, and more iterations cannot lower it.
// A finished matrix's later GEMM tiles are skipped.  Inside a graph loop
// (set_cond) the loop condition becomes "some matrix still active", and
// graph_kernels (the kernels of one iteration) is added to the device-side
// launch count.
__global__ void __launch_bounds__(1024) check_kernel(float* res, float* prev, int* done, int* iters,
                                                     const int* valid, int batch, int n, float tol, int* counter,
                                                     int cap, int kmin, int* flags, cudaGraphConditionalHandle cond,
                                                     int set_cond, int graph_kernels) {
  pdl_launch_dependents();  // a following GEMM may start its prologue
  __shared__ int active;
  if (threadIdx.x == 0) active = 0;
  __syncthreads();
  const int it = *counter + 1;
  int mine = 0;
  for (int i = threadIdx.x; i < batch; i += blockDim.x) {
    if (done[i]) {
      res[i] = 0.f;
      continue;
    }
    const int v = valid ? valid[i] : n;
    const float r = fabsf(res[i]) / static_cast<float>(v);
    res[i] = 0.f;
    iters[i] = it;
    if (!isfinite(r)) {
      done[i] = 1;
      raise_flag(flags, DEV_FLAG_NONFINITE);
    } else if (r <= tol) {
      done[i] = 1;
    } else if (it >= kmin && r >= 0.999f * prev[i]) {
      done[i] = 2;
      raise_flag(flags, DEV_FLAG_STAGNATED);
    } else if (it >= cap) {
      done[i] = 3;
    } else {
      ++mine;
    }
    prev[i] = r;
  }
  if (mine) atomicAdd(&active, mine);
  __syncthreads();
  if (threadIdx.x == 0) {
    counter[0] = it;
    counter[1] = active;
    if (set_cond) {
      cudaGraphSetConditional(cond, active > 0 ? 1u : 0u);
      atomicAdd(&g_graph_kernels, static_cast<unsigned long long>(graph_kernels));
    }
  }
}

// Output pass: X = sym(final iterate) * s^{-1/p}, with sym(Y) = (Y + Y^T)/2.
// The principal root is symmetric; the iterates pick up a small
// antisymmetric rounding component, which this removes.  The final iterate sits in buffer (iters[i] & 1).
// grid (n/32, n/32, batch), block (32, 8).
__global__ void finalize_kernel(const float* __restrict__ X0, const float* __restrict__ X1,
                                const int* __restrict__ iters, int default_iters, const float* __restrict__ sc, int n,
                                float* __restrict__ out, int* flags) {
  pdl_launch_dependents();  // a following GEMM may start its prologue
  __shared__ float t1[32][33];
  __shared__ float t2[32][33];
  const int i = blockIdx.z;
  const int bi = blockIdx.y, bj = blockIdx.x;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const size_t nn = static_cast<size_t>(n) * n;
  const int it = iters ? iters[i] : default_iters;
  const float* src = ((it & 1) ? X1 : X0) + i * nn;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    t1[ty + 8 * k][tx] = src[static_cast<size_t>(bi * 32 + ty + 8 * k) * n + bj * 32 + tx];
    t2[ty + 8 * k][tx] = src[static_cast<size_t>(bj * 32 + ty + 8 * k) * n + bi * 32 + tx];
  }
  __syncthreads();
  const float f = sc[i];
  bool bad = false;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = bi * 32 + ty + 8 * k, c = bj * 32 + tx;
    const float v = 0.5f * (t1[ty + 8 * k][tx] + t2[tx][ty + 8 * k]) * f;
    bad |= !isfinite(v);
    out[i * nn + static_cast<size_t>(r) * n + c] = v;
  }
  if (bad) raise_flag(flags, DEV_FLAG_NONFINITE);
}

// ---------------------------------------------------------------------------
// Chebyshev setup (DASH abstract names Chebyshev approximation; reading:
// interpolation of x^{-1/p} on [a, 1] at first-kind Chebyshev points, with
// a = lo / s, lo = cheb_lo if > 0 else eps, a >= 1 clamped to 1/2).
// coef layout per matrix: c_0 .. c_d (c_0 halved), then a.  One CTA per matrix,
// float64 arithmetic.
// ---------------------------------------------------------------------------
__global__ void cheb_coef_kernel(const float* __restrict__ s, int degree, int p, float eps, float lo,
                                 float* __restrict__ coef, float* __restrict__ sc) {
  const int i = blockIdx.x;
  const double sv = s[i];
  const double base = (lo > 0.f) ? static_cast<double>(lo) : static_cast<double>(effective_eps(eps, s[i]));
  double a = base / sv;
  if (a >= 1.0) a = 0.5;
  const int d = degree;
  const double pi = 3.14159265358979323846;
  float* ci = coef + static_cast<size_t>(i) * (d + 2);
  for (int k = threadIdx.x; k <= d; k += blockDim.x) {
    double acc = 0.0;
    for (int j = 0; j <= d; ++j) {
      const double th = pi * (j + 0.5) / (d + 1);
      const double x = 0.5 * (1.0 - a) * cos(th) + 0.5 * (1.0 + a);
      acc += pow(x, -1.0 / p) * cos(k * th);
    }
    acc *= 2.0 / (d + 1);
    if (k == 0) acc *= 0.5;
    ci[k] = static_cast<float>(acc);
  }
  if (threadIdx.x == 0) {
    ci[d + 1] = static_cast<float>(a);
    sc[i] = static_cast<float>(pow(sv, -1.0 / p));
  }
}

// Xt = (2 A' - (1 + a) I) / (1 - a) on the valid region (identity on the pad),
// b_d = c_d I and b_{d-1} = 2 c_d Xt + c_{d-1} I (first two Clenshaw terms).
__global__ void cheb_prologue_kernel(const float* __restrict__ A, int n, const int* __restrict__ valid, float eps,
                                     const float* __restrict__ s, const float* __restrict__ coef, int degree,
                                     float* __restrict__ Xt, float* __restrict__ bd, float* __restrict__ bd1) {
  pdl_launch_dependents();  // a following GEMM may start its prologue
  __shared__ float t1[32][33];
  __shared__ float t2[32][33];
  const int i = blockIdx.z;
  const int bi = blockIdx.y, bj = blockIdx.x;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const size_t nn = static_cast<size_t>(n) * n;
  const float* a_in = A + i * nn;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    t1[ty + 8 * k][tx] = a_in[static_cast<size_t>(bi * 32 + ty + 8 * k) * n + bj * 32 + tx];
    t2[ty + 8 * k][tx] = a_in[static_cast<size_t>(bj * 32 + ty + 8 * k) * n + bi * 32 + tx];
  }
  __syncthreads();
  const int v = valid ? valid[i] : n;
  const float inv_s = 1.f / s[i];
  const float eps_eff = effective_eps(eps, s[i]);
  const float* ci = coef + static_cast<size_t>(i) * (degree + 2);
  const float a = ci[degree + 1];
  const float cd = ci[degree], cd1 = ci[degree - 1];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = bi * 32 + ty + 8 * k, c = bj * 32 + tx;
    const float sym = 0.5f * (t1[ty + 8 * k][tx] + t2[tx][ty + 8 * k]);
    const float d = (r == c) ? 1.f : 0.f;
    const float m = (r < v && c < v) ? (sym + d * eps_eff) * inv_s : d;
    const float x = (2.f * m - (1.f + a) * d) / (1.f - a);
    const size_t idx = i * nn + static_cast<size_t>(r) * n + c;
    Xt[idx] = x;
    bd[idx] = cd * d;
    bd1[idx] = 2.f * cd * x + cd1 * d;
  }
}

// Lower blocks of a symmetric result whose GEMM skipped the tiles wholly below
// the diagonal (tile row tm >= 2 tn + 2 of the 128 x 256 tiling): block (bi, bj)
// of 32 x 32 takes the transpose of block (bj, bi), which the GEMM computed.
// grid (n/32, n/32, batch), block (32, 8).
__global__ void mirror_lower_kernel(float* __restrict__ D, int n) {
  pdl_launch_dependents();
  const int i = blockIdx.z, bi = blockIdx.y, bj = blockIdx.x;
  const int tm = bi / (kTileM / 32), tn = bj / (kTileN / 32);
  if (tm < 2 * tn + 2) return;  // computed by the GEMM
  __shared__ float t[32][33];
  const size_t nn = static_cast<size_t>(n) * n;
  float* d = D + i * nn;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    t[threadIdx.y + 8 * k][threadIdx.x] = d[static_cast<size_t>(bj * 32 + threadIdx.y + 8 * k) * n + bi * 32 + threadIdx.x];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k)
    d[static_cast<size_t>(bi * 32 + threadIdx.y + 8 * k) * n + bj * 32 + threadIdx.x] = t[threadIdx.x][threadIdx.y + 8 * k];
}

// X split into three bf16 planes whose sum is X exactly: each plane is the
// nearest bf16 to what the previous ones leave (the remainder of a fp32 value
// after rounding its leading 8 significant bits is exact in fp32, and after
// two such steps at most 8 significant bits are left, which bf16 holds).  The
// roots stay fixed between refreshes, so the first apply product reads them
// in this form on the bf16 MMA, each plane times the bf16 gradient exact in
// fp32.  Grid-stride over float4 groups.
__global__ void split_planes_kernel(const float4* __restrict__ X, int64_t n4, uint2* __restrict__ P) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 x = X[i];
    float r[4] = {x.x, x.y, x.z, x.w};
    uint32_t h[3][4];
#pragma unroll
    for (int q = 0; q < 3; ++q)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __nv_bfloat16 b = __float2bfloat16_rn(r[k]);
        h[q][k] = __bfloat16_as_ushort(b);
        r[k] -= __bfloat162float(b);
      }
#pragma unroll
    for (int q = 0; q < 3; ++q) P[q * n4 + i] = make_uint2(h[q][0] | (h[q][1] << 16), h[q][2] | (h[q][3] << 16));
  }
}

// The 3xTF32 product's operand split (split_tf32, the converter warps' own
// function), stored: hi[i] + lo[i] = X[i].  The roots XR stay fixed between
// refreshes, so the second apply product reads them split from HBM and its
// converters split only T.  Grid-stride over float4 groups.
__global__ void split_tf32_kernel(const float4* __restrict__ X, int64_t n4, float4* __restrict__ hi,
                                  float4* __restrict__ lo) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 x = X[i];
    float4 h, l;
    split_tf32(x.x, h.x, l.x);
    split_tf32(x.y, h.y, l.y);
    split_tf32(x.z, h.z, l.z);
    split_tf32(x.w, h.w, l.w);
    hi[i] = h;
    lo[i] = l;
  }
}

__global__ void fill_int_kernel(int* p, int64_t count, int value) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < count) p[i] = value;
}

}  // namespace

int launch_stack(const StackArgs& args, const int* d_table, int nb, int B, int grad_dtype, float* Gs, float* Gts,
                 float* M, float alpha, float gscale, float** blk_wptr, int* blk_ld, cudaStream_t st,
                 double alg_bytes, uint16_t* Gs16, uint16_t* Gt16) {
  if (nb == 0) return 0;
  if ((Gs16 || Gt16) && grad_dtype != 1)
    return set_error(-1, "bf16 stacks need bf16 gradients (other values are not exact in bf16)");
  ProfScope ps(K_STACK, st, 0.0, alg_bytes);
  dim3 grid((B + 127) / 128, B / 32, nb), block(32, 8);
  stack_blocks_kernel<<<grid, block, 0, st>>>(args, d_table, B, grad_dtype, Gs, Gts, M, alpha, gscale, blk_wptr,
                                              blk_ld, Gs16, Gt16);
  count_launch();
  return check_cuda(cudaGetLastError(), "stack_blocks_kernel");
}

int launch_frob_norm(const float* A, int64_t batch, int n, const int* valid, float eps, int p, float* s, float* sc,
                     cudaStream_t st) {
  if (batch == 0) return 0;
  ProfScope ps(K_NORM, st, 0.0, 4.0 * batch * n * n);
  frob_norm_kernel<<<static_cast<unsigned>(batch), dim3(32, 16), 0, st>>>(A, n, valid, eps, 1.0 / p, s, sc);
  count_launch();
  return check_cuda(cudaGetLastError(), "frob_norm_kernel");
}

int launch_spectral_scale(const float* A, int64_t batch, int n, const int* valid, float eps, int p, int iters,
                          float* s, float* sc, float* sf, float* vec, const int* warm, int warm_iters,
                          int warm_hint, cudaStream_t st) {
  if (batch == 0) return 0;
  ProfScope ps(K_SCALE, st, 0.0, 4.0 * ((warm_hint ? warm_iters : iters) + 1) * batch * n * n);
  spectral_scale_kernel<<<static_cast<unsigned>(batch), 512, 2 * n * sizeof(float), st>>>(
      A, n, valid, eps, 1.0 / p, iters, s, sc, sf, vec, warm, warm_iters);
  count_launch();
  return check_cuda(cudaGetLastError(), "spectral_scale_kernel");
}

int launch_root_prologue(int kind, const float* A, int64_t batch, int n, const int* valid, float eps, int p,
                         const float* s, const float* sf, float* out0, float* out1, float* out2, int* set_flag,
                         cudaStream_t st) {
  if (batch == 0) return 0;
  ProfScope ps(K_PROLOGUE, st, 0.0, 16.0 * batch * n * n);
  dim3 grid(n / 32, n / 32, static_cast<unsigned>(batch)), block(32, 8);
  root_prologue_kernel<<<grid, block, 0, st>>>(kind, A, n, valid, eps, p, s, sf ? sf : s, out0, out1, out2,
                                               set_flag);
  count_launch();
  return check_cuda(cudaGetLastError(), "root_prologue_kernel");
}

int launch_db_stage2_prologue(const float* Y0, const float* Y1, const int* iters, int64_t batch, int n, float* Ynew0,
                              float* T, float* Z1, cudaStream_t st) {
  if (batch == 0) return 0;
  ProfScope ps(K_PROLOGUE, st, 0.0, 16.0 * batch * n * n);
  const size_t nn = static_cast<size_t>(n) * n;
  dim3 grid(static_cast<unsigned>((nn + 255) / 256), static_cast<unsigned>(batch));
  db_stage2_kernel<<<grid, 256, 0, st>>>(Y0, Y1, iters, n, Ynew0, T, Z1);
  count_launch();
  return check_cuda(cudaGetLastError(), "db_stage2_kernel");
}

int launch_check(float* res, float* prev, int* done, int* iters, const int* valid, int64_t batch, int n, float tol,
                 int* counter, int cap, int kmin, int* flags, const GraphLoop* loop, cudaStream_t st) {
  if (batch == 0) return 0;
  ProfScope ps(K_CHECK, st, 0.0, 24.0 * batch);
  check_kernel<<<1, 1024, 0, st>>>(res, prev, done, iters, valid, static_cast<int>(batch), n, tol, counter, cap,
                                   kmin, flags, loop ? loop->cond : cudaGraphConditionalHandle(0), loop ? 1 : 0,
                                   loop ? loop->kernels_per_check : 0);
  count_launch();
  return check_cuda(cudaGetLastError(), "check_kernel");
}

int launch_finalize(const float* X0, const float* X1, const int* iters, int default_iters, const float* sc,
                    int64_t batch, int n, float* out, int* flags, cudaStream_t st) {
  if (batch == 0) return 0;
  ProfScope ps(K_FINALIZE, st, 0.0, 8.0 * batch * n * n);
  dim3 grid(n / 32, n / 32, static_cast<unsigned>(batch)), block(32, 8);
  finalize_kernel<<<grid, block, 0, st>>>(X0, X1, iters, default_iters, sc, n, out, flags);
  count_launch();
  return check_cuda(cudaGetLastError(), "finalize_kernel");
}

int launch_cheb_setup(const float* A, int64_t batch, int n, const int* valid, float eps, int p, int degree, float lo,
                      const float* s, float* coef, float* sc, float* Xt, float* bd, float* bd1, cudaStream_t st) {
  if (batch == 0) return 0;
  {
    ProfScope ps(K_CHEB_COEF, st, 0.0, 8.0 * batch);
    cheb_coef_kernel<<<static_cast<unsigned>(batch), 128, 0, st>>>(s, degree, p, eps, lo, coef, sc);
    count_launch();
    int rc = check_cuda(cudaGetLastError(), "cheb_coef_kernel");
    if (rc) return rc;
  }
  ProfScope ps(K_PROLOGUE, st, 0.0, 16.0 * batch * n * n);
  dim3 grid(n / 32, n / 32, static_cast<unsigned>(batch)), block(32, 8);
  cheb_prologue_kernel<<<grid, block, 0, st>>>(A, n, valid, eps, s, coef, degree, Xt, bd, bd1);
  count_launch();
  return check_cuda(cudaGetLastError(), "cheb_prologue_kernel");
}

int launch_mirror_lower(float* D, int64_t batch, int n, cudaStream_t st) {
  if (batch == 0 || n <= kTileN) return 0;  // one tile column: every tile is computed
  ProfScope ps(K_MIRROR, st, 0.0, 8.0 * batch * n * double(n) * 0.375);
  dim3 grid(n / 32, n / 32, static_cast<unsigned>(batch)), block(32, 8);
  mirror_lower_kernel<<<grid, block, 0, st>>>(D, n);
  count_launch();
  return check_cuda(cudaGetLastError(), "mirror_lower_kernel");
}

int launch_split_planes(const float* X, int64_t count, uint16_t* planes, cudaStream_t st) {
  if (count == 0) return 0;
  if (count % 4 || (reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(planes)) & 15)
    return set_error(-1, "split_planes: %lld values, or unaligned buffers", static_cast<long long>(count));
  ProfScope ps(K_PLANES, st, 0.0, 10.0 * count);
  const int64_t n4 = count / 4;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>((n4 + 255) / 256, 148 * 16));
  split_planes_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const float4*>(X), n4, reinterpret_cast<uint2*>(planes));
  count_launch();
  return check_cuda(cudaGetLastError(), "split_planes_kernel");
}

int launch_split_tf32(const float* X, int64_t count, float* hi, float* lo, cudaStream_t st) {
  if (count == 0) return 0;
  if (count % 4 ||
      (reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(hi) | reinterpret_cast<uintptr_t>(lo)) & 15)
    return set_error(-1, "split_tf32: %lld values, or unaligned buffers", static_cast<long long>(count));
  ProfScope ps(K_PLANES, st, 0.0, 12.0 * count);
  const int64_t n4 = count / 4;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>((n4 + 255) / 256, 148 * 16));
  split_tf32_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const float4*>(X), n4, reinterpret_cast<float4*>(hi),
                                          reinterpret_cast<float4*>(lo));
  count_launch();
  return check_cuda(cudaGetLastError(), "split_tf32_kernel");
}

int launch_fill_iters(int* iters, int64_t batch, int value, cudaStream_t st) {
  if (batch == 0) return 0;
  fill_int_kernel<<<static_cast<unsigned>((batch + 255) / 256), 256, 0, st>>>(iters, batch, value);
  count_launch();
  return check_cuda(cudaGetLastError(), "fill_int_kernel");
}

}  // namespace shampoo

namespace shampoo {
namespace {

// Per-matrix iteration report: out[i] = iterations (+ add[i]); negated when
// the residual never reached tol: the cap was reached (done 0 or 3, raises
// DEV_FLAG_NOT_CONVERGED) or the residual stagnated (done 2, flagged by the
// check).
__global__ void report_kernel(const int* iters, const int* add, const int* done, int batch, int default_iters,
                              int* out, int* flags, int residual) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= batch) return;
  int it = iters ? iters[i] : default_iters;
  if (add) it += add[i];
  const bool capped = residual && done && (done[i] == 0 || done[i] == 3);
  const bool failed = residual && done && done[i] != 1;
  if (capped) raise_flag(flags, DEV_FLAG_NOT_CONVERGED);
  if (out) out[i] = failed ? -it : it;
}

}  // namespace

int launch_report(const int* iters, const int* add, const int* done, int64_t batch, int default_iters, int* out,
                  int* flags, bool residual, cudaStream_t st) {
  if (batch == 0) return 0;
  ProfScope ps(K_CHECK, st, 0.0, 16.0 * batch);
  report_kernel<<<static_cast<unsigned>((batch + 255) / 256), 256, 0, st>>>(
      iters, add, done, static_cast<int>(batch), default_iters, out, flags, residual ? 1 : 0);
  count_launch();
  return check_cuda(cudaGetLastError(), "report_kernel");
}

}  // namespace shampoo
