// Double-precision iterates for the inverse p-th root (coupled Newton with the
// second-degree correction, solver SHAMPOO_SOLVER_NEWTON_CUBIC_F64).
//
// Why: a root computed with fp32-accurate iterates carries an error of about
// (1/p) u kappa relative to the exact root of the same input (u = 2^-24): on
// statistics with kappa >= 1e6 that is a few percent, far above 2e-3.  The
// same iteration run in fp64 keeps the iterates' rounding at 2^-53, so the
// result is the exact root of the (damped) input to the last fp32 bit of the
// output.  The iteration, the scale, the damping and the stopping rule are the
// fp32 solver's (coupled Newton of Guo & Higham 2006 with the degree-2 binomial
// correction); only the arithmetic of the iterates changes.
//
// The products run on the fp64 tensor-core instruction
// mma.sync.aligned.m8n8k4.f64 (tcgen05 has no fp64 kind): a CTA of four warps
// computes a 64 x 64 tile, each warp a 32 x 32 quarter as 4 x 4 m8n8 blocks,
// with operands staged through a three-stage cp.async ring in shared memory
// (rows padded so that every fragment load is two conflict-free wavefronts).
// The epilogue fuses the iteration's affine terms: D = alpha A B + beta C +
// gamma I, optionally E = e_mul D + e_add I (the next I - M) and the trace
// residual tr(I - M) over the valid rows.
#include "../../include/shampoo.h"
#include "common.cuh"
#include "internal.h"

namespace shampoo {
namespace {

constexpr int kDT = 64;                 // CTA tile: 64 x 64 outputs
constexpr int kDK = 16;                 // K per stage
constexpr int kDStages = 3;
constexpr int kDThreads = 128;          // 4 warps, 2 x 2 quarters of 32 x 32
constexpr int kAStride = kDK + 4;       // elements per A row in shared memory
constexpr int kBStride = kDT + 8;       // elements per B row
constexpr int kAStage = kDT * kAStride; // elements per A stage
constexpr int kBStage = kDK * kBStride;
// Operands are fp64, or fp32 widened exactly when fragments are loaded (the
// statistics of fp32 / bf16 gradient stacks).  Both paddings keep every
// fragment load at the minimum number of shared-memory wavefronts.
template <class TIn>
constexpr size_t dsmem_bytes() { return sizeof(TIn) * kDStages * (kAStage + kBStage); }

struct DArgs {
  DGemmGroup g[2];
  int ngroups;
  int n;
  int batch;
  const int* valid;
  const int* skip;
  int* flags;
  int sym;  // symmetric results: tiles wholly below the diagonal are skipped
  double* prof_flops;  // profiling on: executed algorithmic flops accumulate here
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  const int sz = pred ? 16 : 0;  // 0: no bytes read, the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// D(8x8, two values per lane) += A(8x4, one per lane) B(4x8, one per lane).
__device__ __forceinline__ void dmma8x8x4(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};\n"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

// grid (ceil(n/64), ceil(n/64), ngroups * batch), block 128.  Every operand is
// a row-major n x n matrix; the product is the true product A B.
template <class TIn>
__global__ void __launch_bounds__(kDThreads) dgemm_kernel(DArgs args) {
  const int z = blockIdx.z;
  const int gi = z / args.batch, m = z - gi * args.batch;
  if (args.skip && args.skip[m]) return;  // converged matrix: its iterates are final
  if (args.sym && blockIdx.y > blockIdx.x) return;  // mirror_lower_f64_kernel fills it from its transpose
  if (args.prof_flops && threadIdx.x == 0)  // tiles that ran, so skipped matrices add nothing
    atomicAdd(&args.prof_flops[K_GEMM_F64],
              2.0 * min(kDT, args.n - static_cast<int>(blockIdx.y) * kDT) *
                  min(kDT, args.n - static_cast<int>(blockIdx.x) * kDT) * args.n);
  const DGemmGroup& G = args.g[gi];
  const int n = args.n;
  const size_t nn = static_cast<size_t>(n) * n;
  const TIn* A = static_cast<const TIn*>(G.A) + m * nn;
  const TIn* B = static_cast<const TIn*>(G.B) + m * nn;
  const int row0 = blockIdx.y * kDT, col0 = blockIdx.x * kDT;

  extern __shared__ __align__(16) unsigned char dsm_raw[];
  TIn* As = reinterpret_cast<TIn*>(dsm_raw);
  TIn* Bs = As + kDStages * kAStage;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = warp >> 1, wn = warp & 1;
  constexpr int kPer = 16 / sizeof(TIn);      // elements per 16-byte piece
  constexpr int kAPieces = kDK / kPer;        // pieces per A row (8 fp64, 4 fp32)
  constexpr int kBPieces = kDT / kPer;        // pieces per B row (32 fp64, 16 fp32)
  constexpr int kLoads = kDT * kAPieces / kDThreads;  // per thread and operand (4 fp64, 2 fp32)
  static_assert(kDK * kBPieces == kDT * kAPieces, "A and B stages have the same number of pieces");

  auto load_stage = [&](int stage, int kt) {
    const int k0 = kt * kDK;
    TIn* as = As + stage * kAStage;
    TIn* bs = Bs + stage * kBStage;
#pragma unroll
    for (int q = 0; q < kLoads; ++q) {
      const int idx = tid + q * kDThreads;  // 64 rows x kAPieces
      const int r = idx / kAPieces, c = idx % kAPieces;
      const bool ok = row0 + r < n;
      const TIn* src = ok ? A + static_cast<size_t>(row0 + r) * n + k0 + kPer * c : A;
      cp_async16(as + r * kAStride + kPer * c, src, ok);
    }
#pragma unroll
    for (int q = 0; q < kLoads; ++q) {
      const int idx = tid + q * kDThreads;  // 16 rows x kBPieces
      const int k = idx / kBPieces, c = idx % kBPieces;
      const bool ok = col0 + kPer * c < n;
      const TIn* src = ok ? B + static_cast<size_t>(k0 + k) * n + col0 + kPer * c : B;
      cp_async16(bs + k * kBStride + kPer * c, src, ok);
    }
  };

  double acc[4][4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;

  const int KT = n / kDK;
#pragma unroll
  for (int s = 0; s < kDStages - 1; ++s) {
    if (s < KT) load_stage(s, s);
    cp_async_commit();
  }
  const int ar = wm * 32 + (lane >> 2), ak = lane & 3;  // A fragment: row, k
  const int bk = lane & 3, bc = wn * 32 + (lane >> 2);  // B fragment: k, column
  for (int kt = 0; kt < KT; ++kt) {
    cp_async_wait<kDStages - 2>();
    __syncthreads();  // stage kt landed for every thread; stage kt - 1 is free
    if (kt + kDStages - 1 < KT) load_stage((kt + kDStages - 1) % kDStages, kt + kDStages - 1);
    cp_async_commit();
    const TIn* as = As + (kt % kDStages) * kAStage;
    const TIn* bs = Bs + (kt % kDStages) * kBStage;
#pragma unroll
    for (int kk = 0; kk < kDK; kk += 4) {
      double a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = static_cast<double>(as[(ar + 8 * i) * kAStride + kk + ak]);
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = static_cast<double>(bs[(kk + bk) * kBStride + bc + 8 * j]);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) dmma8x8x4(acc[i][j], a[i], b[j]);
    }
  }
  cp_async_wait<0>();

  // Epilogue.  Lane holds D[r][c], D[r][c+1] of each 8 x 8 block with
  // r = lane / 4, c = 2 (lane % 4).
  const int v = args.valid ? args.valid[m] : n;
  double* D = G.D + m * nn;
  const double* C = G.C ? G.C + m * nn : nullptr;
  double* E = G.E ? G.E + m * nn : nullptr;
  double rsum = 0.0;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = row0 + wm * 32 + 8 * i + (lane >> 2);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = col0 + wn * 32 + 8 * j + 2 * (lane & 3);
      if (r >= n || c >= n) continue;
      const size_t off = static_cast<size_t>(r) * n + c;
      double2 cv = make_double2(0.0, 0.0);
      if (C) cv = *reinterpret_cast<const double2*>(C + off);
      double2 out;
      out.x = G.alpha * acc[i][j][0] + G.beta * cv.x + (r == c ? G.gamma : 0.0);
      out.y = G.alpha * acc[i][j][1] + G.beta * cv.y + (r == c + 1 ? G.gamma : 0.0);
      bad |= !isfinite(out.x) || !isfinite(out.y);
      *reinterpret_cast<double2*>(D + off) = out;
      if (E) {
        double2 e;
        e.x = G.e_mul * out.x + (r == c ? G.e_add : 0.0);
        e.y = G.e_mul * out.y + (r == c + 1 ? G.e_add : 0.0);
        *reinterpret_cast<double2*>(E + off) = e;
      }
      if (G.res && r < v) {
        if (r == c) rsum += 1.0 - out.x;
        if (r == c + 1) rsum += 1.0 - out.y;
      }
    }
  }
  if (G.res) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rsum += __shfl_xor_sync(0xffffffffu, rsum, o);
    if (lane == 0 && rsum != 0.0) atomicAdd(&G.res[m], static_cast<float>(rsum));
  }
  if (bad) raise_flag(args.flags, DEV_FLAG_NONFINITE);
}

// Lower part of a symmetric fp64 result whose product skipped the 64 x 64 tiles
// wholly below the diagonal: block (bi, bj) of 32 x 32 in such a tile takes
// the transpose of block (bj, bi), which was computed.  grid (n/32, n/32,
// batch), block (32, 8).
__global__ void mirror_lower_f64_kernel(double* __restrict__ D, int n) {
  const int i = blockIdx.z, bi = blockIdx.y, bj = blockIdx.x;
  if (bi / (kDT / 32) <= bj / (kDT / 32)) return;  // computed by the product
  __shared__ double t[32][33];
  const size_t nn = static_cast<size_t>(n) * n;
  double* d = D + i * nn;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    t[threadIdx.y + 8 * k][threadIdx.x] = d[static_cast<size_t>(bj * 32 + threadIdx.y + 8 * k) * n + bi * 32 + threadIdx.x];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k)
    d[static_cast<size_t>(bi * 32 + threadIdx.y + 8 * k) * n + bj * 32 + threadIdx.x] = t[threadIdx.x][threadIdx.y + 8 * k];
}

// Damping and scaling in fp64, the first plain Newton step, and X1 = T0:
// M0 = (sym(A) + eps_eff I) / s on the valid block and the identity on the
// padding; T0 = ((p+1) I - M0) / p.  A is fp32 (kind 0) or fp64 (kind 1).
// grid (n/32, n/32, batch), block (32, 8).
template <class TA>
__global__ void prologue_f64_kernel(const TA* __restrict__ A, int n, const int* __restrict__ valid, float eps,
                                    float eps_floor_rel, int p, const float* __restrict__ s,
                                    const float* __restrict__ sf, double* __restrict__ M0, double* __restrict__ T,
                                    double* __restrict__ X1, int* set_flag) {
  if (set_flag && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0 && threadIdx.y == 0)
    *set_flag = 1;
  __shared__ double t1[32][33];
  __shared__ double t2[32][33];
  const int i = blockIdx.z;
  const int bi = blockIdx.y, bj = blockIdx.x;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const size_t nn = static_cast<size_t>(n) * n;
  const TA* a = A + i * nn;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    t1[ty + 8 * k][tx] = static_cast<double>(a[static_cast<size_t>(bi * 32 + ty + 8 * k) * n + bj * 32 + tx]);
    t2[ty + 8 * k][tx] = static_cast<double>(a[static_cast<size_t>(bj * 32 + ty + 8 * k) * n + bi * 32 + tx]);
  }
  __syncthreads();
  const int v = valid ? valid[i] : n;
  const double inv_s = 1.0 / static_cast<double>(s[i]);
  const double eps_eff = fmax(static_cast<double>(eps), static_cast<double>(sf[i]) * eps_floor_rel);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = bi * 32 + ty + 8 * k, c = bj * 32 + tx;
    const double sym = 0.5 * (t1[ty + 8 * k][tx] + t2[tx][ty + 8 * k]);
    const double d = (r == c) ? 1.0 : 0.0;
    const double mv = (r < v && c < v) ? (sym + d * eps_eff) * inv_s : d;
    const double t = (static_cast<double>(p + 1) * d - mv) / static_cast<double>(p);
    const size_t idx = i * nn + static_cast<size_t>(r) * n + c;
    M0[idx] = mv;
    T[idx] = t;
    X1[idx] = t;
  }
}

// X = sym(final iterate) s^{-1/p}, rounded once to fp32.  The final iterate
// sits in buffer (iters[i] & 1).  grid (n/32, n/32, batch), block (32, 8).
__global__ void finalize_f64_kernel(const double* __restrict__ X0, const double* __restrict__ X1,
                                    const int* __restrict__ iters, int default_iters, const float* __restrict__ s,
                                    int p, int n, float* __restrict__ out, int* flags) {
  __shared__ double t1[32][33];
  __shared__ double t2[32][33];
  const int i = blockIdx.z;
  const int bi = blockIdx.y, bj = blockIdx.x;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const size_t nn = static_cast<size_t>(n) * n;
  const int it = iters ? iters[i] : default_iters;
  const double* src = ((it & 1) ? X1 : X0) + i * nn;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    t1[ty + 8 * k][tx] = src[static_cast<size_t>(bi * 32 + ty + 8 * k) * n + bj * 32 + tx];
    t2[ty + 8 * k][tx] = src[static_cast<size_t>(bj * 32 + ty + 8 * k) * n + bi * 32 + tx];
  }
  __syncthreads();
  const double f = pow(static_cast<double>(s[i]), -1.0 / p);
  bool bad = false;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = bi * 32 + ty + 8 * k, c = bj * 32 + tx;
    const float val = static_cast<float>(0.5 * (t1[ty + 8 * k][tx] + t2[tx][ty + 8 * k]) * f);
    bad |= !isfinite(val);
    out[i * nn + static_cast<size_t>(r) * n + c] = val;
  }
  if (bad) raise_flag(flags, DEV_FLAG_NONFINITE);
}

// Scale of an fp64 input: s = sf = ||A + eps I||_F over the valid block, an
// upper bound of the largest eigenvalue, in fp64.  One CTA per matrix.
__global__ void frob_f64_kernel(const double* __restrict__ A, int n, const int* __restrict__ valid, float eps,
                                float* __restrict__ s, float* __restrict__ sf) {
  const int i = blockIdx.x;
  const int v = valid ? valid[i] : n;
  const double* a = A + static_cast<size_t>(i) * n * n;
  double acc = 0.0;
  for (int r = threadIdx.y; r < v; r += blockDim.y)
    for (int c = threadIdx.x; c < v; c += blockDim.x) {
      const double x = a[static_cast<size_t>(r) * n + c] + (r == c ? static_cast<double>(eps) : 0.0);
      acc += x * x;
    }
  __shared__ double part[32];
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  const int w = (threadIdx.y * blockDim.x + threadIdx.x) >> 5;
  if ((threadIdx.x & 31) == 0) part[w] = acc;
  __syncthreads();
  if (threadIdx.x == 0 && threadIdx.y == 0) {
    double t = 0.0;
    for (int k = 0; k < static_cast<int>(blockDim.x * blockDim.y / 32); ++k) t += part[k];
    const float f = static_cast<float>(sqrt(t));
    s[i] = f > 0.f ? f : 1.f;  // an all-zero block: any scale
    sf[i] = f;
  }
}

}  // namespace

int launch_frob_f64(const double* A, int64_t batch, int n, const int* valid, float eps, float* s, float* sf,
                    cudaStream_t st) {
  if (batch == 0) return 0;
  ProfScope ps(K_SCALE, st, 0.0, 8.0 * batch * n * n);
  frob_f64_kernel<<<static_cast<unsigned>(batch), dim3(32, 16), 0, st>>>(A, n, valid, eps, s, sf);
  count_launch();
  return check_cuda(cudaGetLastError(), "frob_f64_kernel");
}

int launch_dgemm(const DGemmGroup* groups, int ngroups, int64_t batch, int n, const int* valid, const int* skip,
                 int* flags, cudaStream_t st, bool f32_operands, bool sym) {
  if (batch == 0) return 0;
  if (ngroups < 1 || ngroups > 2 || n % kDK != 0 || batch * ngroups > 65535)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "dgemm: %d groups, n %d, batch %lld", ngroups, n,
                     static_cast<long long>(batch));
  static bool attr_set[64][2] = {};  // per device and operand type
  int dev = 0;
  int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
  if (rc) return rc;
  if (dev < 0 || dev >= 64) return set_error(SHAMPOO_ERR_UNSUPPORTED, "device %d", dev);
  if (!attr_set[dev][f32_operands]) {
    rc = f32_operands ? check_cuda(cudaFuncSetAttribute(dgemm_kernel<float>,
                                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                        static_cast<int>(dsmem_bytes<float>())),
                                   "cudaFuncSetAttribute(dgemm_kernel<float>)")
                      : check_cuda(cudaFuncSetAttribute(dgemm_kernel<double>,
                                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                        static_cast<int>(dsmem_bytes<double>())),
                                   "cudaFuncSetAttribute(dgemm_kernel<double>)");
    if (rc) return rc;
    attr_set[dev][f32_operands] = true;
  }
  DArgs a;
  for (int g = 0; g < ngroups; ++g) a.g[g] = groups[g];
  a.ngroups = ngroups;
  a.n = n;
  a.batch = static_cast<int>(batch);
  a.valid = valid;
  a.skip = skip;
  a.flags = flags;
  a.sym = sym ? 1 : 0;
  a.prof_flops = device_flop_slots();
  const unsigned tiles = static_cast<unsigned>((n + kDT - 1) / kDT);
  // computed fraction: every tile, or those on and above the diagonal
  const double frac = sym ? (tiles + 1.0) / (2.0 * tiles) : 1.0;
  const double flops = 2.0 * n * static_cast<double>(n) * n * batch * ngroups * frac;
  ProfScope ps(K_GEMM_F64, st, flops,
               (f32_operands ? 8.0 : 16.0) * n * static_cast<double>(n) * batch * ngroups +
                   16.0 * frac * n * static_cast<double>(n) * batch * ngroups);
  const dim3 grid(tiles, tiles, static_cast<unsigned>(batch * ngroups));
  if (f32_operands)
    dgemm_kernel<float><<<grid, kDThreads, dsmem_bytes<float>(), st>>>(a);
  else
    dgemm_kernel<double><<<grid, kDThreads, dsmem_bytes<double>(), st>>>(a);
  count_launch();
  return check_cuda(cudaGetLastError(), "dgemm_kernel");
}

int launch_mirror_lower_f64(double* D, int64_t batch, int n, cudaStream_t st) {
  if (batch == 0 || n <= kDT) return 0;  // one tile: computed whole
  const double t = (n + kDT - 1) / kDT;
  ProfScope ps(K_MIRROR, st, 0.0, 16.0 * batch * n * double(n) * (t - 1.0) / (2.0 * t));
  dim3 grid(n / 32, n / 32, static_cast<unsigned>(batch)), block(32, 8);
  mirror_lower_f64_kernel<<<grid, block, 0, st>>>(D, n);
  count_launch();
  return check_cuda(cudaGetLastError(), "mirror_lower_f64_kernel");
}

int launch_prologue_f64(const void* A, int a_is_f64, int64_t batch, int n, const int* valid, float eps,
                        float eps_floor_rel, int p, const float* s, const float* sf, double* M0, double* T,
                        double* X1, int* set_flag, cudaStream_t st) {
  if (batch == 0) return 0;
  ProfScope ps(K_PROLOGUE, st, 0.0, (a_is_f64 ? 8.0 : 4.0) * batch * n * n + 24.0 * batch * n * n);
  dim3 grid(n / 32, n / 32, static_cast<unsigned>(batch)), block(32, 8);
  if (a_is_f64)
    prologue_f64_kernel<double><<<grid, block, 0, st>>>(static_cast<const double*>(A), n, valid, eps, eps_floor_rel,
                                                        p, s, sf, M0, T, X1, set_flag);
  else
    prologue_f64_kernel<float><<<grid, block, 0, st>>>(static_cast<const float*>(A), n, valid, eps, eps_floor_rel, p,
                                                       s, sf, M0, T, X1, set_flag);
  count_launch();
  return check_cuda(cudaGetLastError(), "prologue_f64_kernel");
}

int launch_finalize_f64(const double* X0, const double* X1, const int* iters, int default_iters, const float* s,
                        int p, int64_t batch, int n, float* out, int* flags, cudaStream_t st) {
  if (batch == 0) return 0;
  ProfScope ps(K_FINALIZE, st, 0.0, 12.0 * batch * n * n);
  dim3 grid(n / 32, n / 32, static_cast<unsigned>(batch)), block(32, 8);
  finalize_f64_kernel<<<grid, block, 0, st>>>(X0, X1, iters, default_iters, s, p, n, out, flags);
  count_launch();
  return check_cuda(cudaGetLastError(), "finalize_f64_kernel");
}

}  // namespace shampoo

extern "C" int shampoo_dgemm_batched(const double* d_A, const double* d_B, const double* d_C, double* d_D,
                                     int64_t batch, int32_t n, double alpha, double beta, double gamma,
                                     int32_t* d_status, void* stream) {
  using namespace shampoo;
  if (batch < 0 || batch > 65535 || n < 16 || n > 4096 || n % 16)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "dgemm: batch %lld, n %d", static_cast<long long>(batch), n);
  if (batch == 0) return SHAMPOO_OK;
  if (!d_A || !d_B || !d_D) return set_error(SHAMPOO_ERR_INVALID_ARG, "NULL device pointer");
  if ((reinterpret_cast<uintptr_t>(d_A) | reinterpret_cast<uintptr_t>(d_B) | reinterpret_cast<uintptr_t>(d_C) |
       reinterpret_cast<uintptr_t>(d_D)) & 15)
    return set_error(SHAMPOO_ERR_UNSUPPORTED, "operands must be 16-byte aligned");
  DGemmGroup g;
  g.A = d_A;
  g.B = d_B;
  g.C = d_C;
  g.D = d_D;
  g.alpha = alpha;
  g.beta = d_C ? beta : 0.0;
  g.gamma = gamma;
  return launch_dgemm(&g, 1, batch, n, nullptr, nullptr, d_status, static_cast<cudaStream_t>(stream));
}
