// Internal (host + device) declarations of the blocked Shampoo library.
// Nothing here is part of the public C ABI (include/shampoo.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>
#include <cuda.h>  // CUtensorMap (type only; the driver entry point is fetched at run time)
#include <cuda_runtime.h>

namespace shampoo {

// ---------------------------------------------------------------------------
// Storage format: every stack is plain fp32, (batch, n, n), row-major matrices
// back to back.  The tensor-core GEMM splits its operand tiles into tf32 hi /
// lo parts in shared memory.
// ---------------------------------------------------------------------------
inline size_t plain_floats(int64_t batch, int n) { return static_cast<size_t>(batch) * n * n; }

constexpr int kMaxGroups = 4;
constexpr int kMaxMaps = 2 * kMaxGroups;
constexpr int kMaxParams = 1024;
constexpr int kMaxChebDegree = 64;
constexpr int kMaxSolver = 4;  // SHAMPOO_SOLVER_NEWTON_CUBIC_F64

// Epilogue of one GEMM group.  For matrix i of the group and element (r, c):
//   v = scale_i * (alpha * acc + beta * C_i[r][c] + gamma_i * [r == c])
// with acc = (A_i B_i^T)[r][c], gamma_i = gamma_vec[i * gamma_stride] when
// gamma_vec is set (else gamma) and scale_i = scale_vec[i] (else 1).
// All per-matrix pointers are already offset to the group's first matrix.
struct Epilogue {
  float alpha, beta, gamma;
  const float* gamma_vec;
  int gamma_stride;
  const float* scale_vec;
  const float* C;  // optional input stack
  float* D;        // optional main output stack
  float* E;        // optional second output stack: e_mul * v + e_add * [r == c]
  float e_mul, e_add;
  float* res;        // optional: res[i] += sum over the valid diagonal of (1 - acc): tr(I - acc)
  const int* valid;  // per-matrix valid extent (nullable: n)
  const int* skip;   // per-matrix "done" flags: a set flag skips the matrix
  int* flags;        // device status word (nullable)
  // Weight update: W_i[r * ld_i + c] -= lr * v for r < wrows_i, c < wcols_i,
  // W_i = wptr[i] (a pointer to the block's top-left weight element).
  float* const* wptr;
  const int* wld;
  const int* wrows;
  const int* wcols;
  float lr;
};

struct GemmGroup {
  int batch;       // matrices in this group
  int n;           // columns N of B and D (multiple of 32); square products: also M and K
  int m, k;        // rows M of A and D (multiple of 32), depth K (multiple of 4)
  int a_map, b_map;  // tensor-map slots (A as 128-row boxes, B as 256-row boxes)
  int a_off, b_off;  // matrix index offsets into the mapped stacks
  int a_rows, b_rows;  // box rows of the two maps (min(tile, n))
  int b_mn;            // 1: B is read MN-major (D = A B); 0: K-major (D = A B^T)
  int a_exact, b_exact;  // 1: every value of the operand is exact in tf32 (e.g. widened bf16), so its
                         // lo part is zero: the MMAs with that lo part are skipped and its tiles are
                         // not split
  int bf16;              // 1: both operands are bf16 stacks: kind::f16 MMAs, 32 K per 64-byte stage row
  int a_planes;          // bf16 only: A is the exact sum of this many bf16 planes (0 or 1: one), plane q
                         // at matrix a_off + mat + q * a_plane_stride of A's stack; one MMA per plane
  int a_plane_stride;
  int b_presplit;        // fp32 K-major B given as tf32 hi parts (matrix b_off + mat) and lo parts (matrix
  int b_plane_stride;    // b_off + mat + b_plane_stride) of split_tf32: B's tiles are not split on chip
  int sym;               // 1: D is symmetric (square, e.g. G G^T): only the tiles that reach the
                         // diagonal or above are computed; launch_mirror_lower fills the rest
  int tiles_per;         // tiles computed per matrix (filled by launch_gemm)
  int tiles_m, tiles_n, cta_begin;  // filled by launch_gemm (cta_begin: first tile of the group)
  double flops_per_matrix;          // algorithmic flops (profiling only)
  Epilogue ep;
};

struct GemmLaunch {
  int ngroups;
  int total_tiles;  // filled by launch_gemm
  int profile;  // accumulate executed algorithmic flops into the profiler slot
  int prof_slot;
  GemmGroup g[kMaxGroups];
};

struct TmaMaps {
  CUtensorMap m[kMaxMaps];
};

// GEMM tile geometry (tcgen05 kind::tf32, one CTA per tile).
constexpr int kTileM = 128;
constexpr int kTileN = 256;
constexpr int kTileK = 16;

// Host helpers -------------------------------------------------------------
int encode_stack_map(CUtensorMap* map, const void* base, int64_t batch, int rows, int cols, int box_rows,
                     int mn_layout, int bf16);
int launch_gemm(GemmLaunch& L, const TmaMaps& maps, cudaStream_t st);
Epilogue epilogue_defaults();

// Errors: codes from include/shampoo.h; message kept per thread.
int set_error(int code, const char* fmt, ...);
int check_cuda(cudaError_t e, const char* what);

// Profiler (process-wide).  Kinds index the per-kernel tallies.
enum KernelKind : int {
  K_GEMM = 0,
  K_STACK = 1,
  K_NORM = 2,
  K_PROLOGUE = 3,
  K_CHECK = 4,
  K_FINALIZE = 5,
  K_CHEB_COEF = 6,
  K_SCALE = 7,
  K_MIRROR = 8,
  K_EIGEN = 9,
  K_GEMM_F64 = 10,
  K_PERMUTE = 11,
  K_GRAM = 12,
  K_DIAG = 13,
  K_SOAP = 14,
  K_PLANES = 15,
  K_MODE_SMALL = 16,
  K_COUNT = 17,
};
struct ProfScope {
  ProfScope(int kind, cudaStream_t st, double alg_flops, double alg_bytes);
  ~ProfScope();
  int kind;
  cudaStream_t st;
  double flops, bytes;
  int active;
  int ev;
};
void count_launch();
// While alive, this thread's launches are being recorded into a graph (not
// counted as launches; the graph's own execution is counted on the device).
struct CaptureScope {
  CaptureScope();
  ~CaptureScope();
};
void note_graph_loop_launch();  // a graph loop ran: shampoo_launch_count adds its device-side count
bool profiling_enabled();
double* device_flop_slots();  // device address of the executed-flop accumulators


// A GEMM launch under construction: groups plus the tensor maps they reference.
struct StackMaps {
  CUtensorMap a, b;  // the stack as A (128-row boxes) and as K-major B (256-row boxes)
  CUtensorMap mn;    // as MN-major B: 16 rows of K x 32 columns of N
  float* base;
  int a_rows, b_rows;
  int rows, cols;    // shape of each matrix of the stack
  int bf16;          // 1: a bf16 stack (K-major maps only, 32 columns per box)
};
int make_stack_maps(StackMaps& sm, const float* base, int64_t batch, int n);
// A stack (batch, n, n) of bf16 matrices, as K-major A and B operands of the
// kind::f16 MMA (both operands of a group must be bf16 stacks).
int make_stack_maps_bf16(StackMaps& sm, const void* base, int64_t batch, int n);
// A stack (batch, rows, cols) of row-major matrices (cols a multiple of 4).
int make_rect_maps(StackMaps& sm, const float* base, int64_t batch, int rows, int cols);

// How a group reads its B operand: as B^T (K-major; D = A B^T) or as B
// (MN-major; D = A B).
enum BMode : int { B_TRANSPOSED = 0, B_MN_MAJOR = 1 };

struct Builder {
  GemmLaunch L;
  TmaMaps M;
  int nmaps;
  Builder();
  // Adds a group D_i = epi(A_i B_i^T) (b_mn = 0) or epi(A_i B_i) (b_mn = 1)
  // over matrices a_off.. of `a` and b_off.. of `b`.
  Epilogue& add(int batch, int n, const StackMaps& a, int a_off, const StackMaps& b, int b_off,
                double flops_per_matrix, int bmode = B_TRANSPOSED);
  // Rectangular: D_i (M x N) = epi(A_i op(B_i)), A_i M x K; B_i N x K (B_TRANSPOSED) or K x N
  // (B_MN_MAJOR).  M and N multiples of 32, K a multiple of 4.
  Epilogue& add_rect(int batch, int M, int N, int K, const StackMaps& a, int a_off, const StackMaps& b, int b_off,
                     double flops_per_matrix, int bmode);
  int launch(cudaStream_t st) { return launch_gemm(L, M, st); }
};

int launch_report(const int* iters, const int* add, const int* done, int64_t batch, int default_iters, int* out,
                  int* flags, bool residual, cudaStream_t st);

// Block partition of a parameter set (api.cu): table gets nb x {param, row0,
// col0, r, c}, in (param, block row, block column) order.
int build_block_table(int B, int32_t nparams, const int64_t* rows, const int64_t* cols, std::vector<int>& table);

// Elementwise / reduction kernels (kernels_elem.cu) ---------------------------
struct StackArgs {
  const void* g[kMaxParams];
  float* w[kMaxParams];
  int ld[kMaxParams];
  unsigned char vec[kMaxParams];  // rows of param i start 16-byte (fp32) / 8-byte (bf16) aligned
};
// M (nullable): moment stack, updated in place as M <- alpha M + gscale G_b.
// Gs16 / Gt16 (nullable, bf16 gradients only): G and G^T also as packed bf16
// stacks; with Gs16 the fp32 Gs is not written.
int launch_stack(const StackArgs& args, const int* d_table, int nb, int B, int grad_dtype, float* Gs, float* Gts,
                 float* M, float alpha, float gscale, float** blk_wptr, int* blk_ld, cudaStream_t st,
                 double alg_bytes, uint16_t* Gs16 = nullptr, uint16_t* Gt16 = nullptr);

int launch_frob_norm(const float* A, int64_t batch, int n, const int* valid, float eps, int p, float* s, float* sc,
                     cudaStream_t st);
// kind: 0 = Newton (M0, T0 = ((p+1)I - M0)/p, X1 = T0)
//       1 = Newton-DB (Y0 = A', T0 = (3I - A')/2, Z1 = T0)
// Coupled-Newton scale: s = min(||A + eps I||_F, 1.25 x power-iteration estimate
// of the largest eigenvalue), sc = s^{-1/p}, sf = ||A + eps I||_F.
// vec (nullable): per-matrix store of the power iterate (batch x n floats);
// with *warm != 0 the iteration starts from it for warm_iters steps (the root
// prologue of the refresh's last chunk sets *warm).
int launch_spectral_scale(const float* A, int64_t batch, int n, const int* valid, float eps, int p, int iters,
                          float* s, float* sc, float* sf, float* vec, const int* warm, int warm_iters,
                          int warm_hint, cudaStream_t st);
// sf (nullable: s) sets the damping floor eps_eff = max(eps, 2^-24 sf);
// set_flag (nullable) is set to 1 (a power-iterate store is filled).
int launch_root_prologue(int kind, const float* A, int64_t batch, int n, const int* valid, float eps, int p,
                         const float* s, const float* sf, float* out0, float* out1, float* out2, int* set_flag,
                         cudaStream_t st);
// Second Newton-DB stage: Y0' = Y_par(i) (parity from iters), T0 = (3I - Y0')/2, Z1 = T0.
int launch_db_stage2_prologue(const float* Y0, const float* Y1, const int* iters, int64_t batch, int n,
                              float* Ynew0, float* T, float* Z1, cudaStream_t st);
// A residual-checked iteration loop captured as a CUDA graph WHILE node: the
// check kernel of each pass sets the loop condition.
struct GraphLoop {
  cudaGraphConditionalHandle cond;
  int kernels_per_check;  // kernels of one iteration (the check's own included)
};
// Residual check after an iteration (one CTA): it = *counter + 1; converged
// (done = 1) when the residual is at most tol; stagnated (done = 2) when, from
// iteration kmin on, it failed to improve on the previous one (kept in prev)
// by a relative 1e-3; capped (done = 3) at it = cap.  Inside a graph loop
// (loop != NULL) it also sets the loop condition.
int launch_check(float* res, float* prev, int* done, int* iters, const int* valid, int64_t batch, int n, float tol,
                 int* counter, int cap, int kmin, int* flags, const GraphLoop* loop, cudaStream_t st);
uint64_t graph_kernel_count();  // kernels run inside graph loops so far (synchronous read)
int launch_finalize(const float* X0, const float* X1, const int* iters, int default_iters, const float* sc,
                    int64_t batch, int n, float* out, int* flags, cudaStream_t st);
int launch_cheb_setup(const float* A, int64_t batch, int n, const int* valid, float eps, int p, int degree,
                      float lo, const float* s, float* coef, float* sc, float* Xt, float* bd, float* bd1,
                      cudaStream_t st);
int launch_fill_iters(int* iters, int64_t batch, int value, cudaStream_t st);
// After a GEMM group with sym = 1: copies the transpose of the computed upper
// part into the 32 x 32 blocks of the tiles it skipped (wholly below the diagonal).
int launch_mirror_lower(float* D, int64_t batch, int n, cudaStream_t st);
// planes[q * count + i], q = 0, 1, 2: bf16 values whose sum is X[i] exactly
// (each the nearest bf16 to what the previous planes leave); count % 4 == 0.
int launch_split_planes(const float* X, int64_t count, uint16_t* planes, cudaStream_t st);
// hi[i], lo[i] = split_tf32(X[i]) (the on-chip split of the 3xTF32 product,
// stored); count % 4 == 0.
int launch_split_tf32(const float* X, int64_t count, float* hi, float* lo, cudaStream_t st);

// fp64 products of the fp64-iterate solver (solver_f64.cu): per matrix,
// D = alpha A B + beta C + gamma I (true product, row-major n x n operands),
// optionally E = e_mul D + e_add I and res[m] += sum over the valid diagonal
// of (1 - D).  C may be D itself; A and B must not be written by the launch.
struct DGemmGroup {
  const void* A = nullptr;  // double, or float with f32_operands (widened exactly)
  const void* B = nullptr;
  const double* C = nullptr;
  double* D = nullptr;
  double* E = nullptr;
  double alpha = 1.0, beta = 0.0, gamma = 0.0, e_mul = 0.0, e_add = 0.0;
  float* res = nullptr;
};
// sym: the results are symmetric; tiles wholly below the diagonal are skipped
// (launch_mirror_lower_f64 fills them).
int launch_dgemm(const DGemmGroup* groups, int ngroups, int64_t batch, int n, const int* valid, const int* skip,
                 int* flags, cudaStream_t st, bool f32_operands = false, bool sym = false);
int launch_mirror_lower_f64(double* D, int64_t batch, int n, cudaStream_t st);
// s = sf = ||A + eps I||_F (valid block) of fp64 matrices.
int launch_frob_f64(const double* A, int64_t batch, int n, const int* valid, float eps, float* s, float* sf,
                    cudaStream_t st);
// M0 = (sym(A) + eps_eff I)/s (identity on the padding), T = ((p+1) I - M0)/p,
// X1 = T; eps_eff = max(eps, eps_floor_rel * sf).  A is fp32 or (a_is_f64) fp64.
int launch_prologue_f64(const void* A, int a_is_f64, int64_t batch, int n, const int* valid, float eps,
                        float eps_floor_rel, int p, const float* s, const float* sf, double* M0, double* T,
                        double* X1, int* set_flag, cudaStream_t st);
// out = sym(X_final) s^{-1/p} in fp32; X_final = X1 if (iters or default_iters) is odd, else X0.
int launch_finalize_f64(const double* X0, const double* X1, const int* iters, int default_iters, const float* s,
                        int p, int64_t batch, int n, float* out, int* flags, cudaStream_t st);

// Inverse-root solver (solver.cu) ---------------------------------------------
struct RootJob {
  int64_t batch;
  int n, p, solver, iters, cheb_degree;
  float eps, tol, cheb_lo;
  const float* A;    // plain stack input
  const int* valid;  // device valid extents (nullable)
  float* X;          // output stack
  int* iters_used;   // device per-matrix iterations (nullable)
  int* flags;        // device status word (nullable)
  int plain_launches = 0;  // 1: never build or run a CUDA graph loop (residual-checked loops are
                           // issued as plain launches up to the cap)
  float* power_vec = nullptr;  // coupled Newton's scale: per-matrix power-iterate store (batch x n), or NULL
  int* power_warm = nullptr;   // device flag: power_vec holds the previous refresh's iterates
  int power_warm_hint = 0;     // host's view of that flag, used only for the profiler's byte count
  const double* A64 = nullptr;  // fp64 input stack instead of A (fp64-iterate solver only): scaled by
                                // its Frobenius norm and damped at the fp64 statistics' rounding
};
// inv_root_batched with a switch for plain launches (shared by the public
// entry points of api.cu and noalloc.cu).
int inv_root_batched_impl(const float* d_A, float* d_X, int64_t batch, int n, int p, float eps, int solver, int iters,
                          float tol, int cheb_degree, float cheb_lo, void* d_scratch, size_t scratch_bytes,
                          int* d_iters_used, int* d_status, cudaStream_t st, bool plain_launches);
size_t root_scratch_per_matrix(int n, int solver, int p);
// Batched symmetric eigendecomposition (eigen.cu): Q (columns) and lam
// (nullable) of the valid part of each A_i; warm_start = 0: cyclic Jacobi (at
// most jacobi_sweeps) from scratch, then refine_iters refinement iterations;
// warm_start = 1: Q holds an approximate basis on entry, refinement only.
size_t eig_scratch_per_matrix(int n);
int run_eigh(const float* A, float* Q, float* lam, int64_t batch, int n, const int* valid, int warm_start,
             int jacobi_sweeps, int refine_iters, void* scratch, size_t scratch_bytes, int* flags, cudaStream_t st);
size_t root_scratch_header();
int run_inverse_roots(const RootJob& job, void* scratch, size_t scratch_bytes, cudaStream_t st);

}  // namespace shampoo
