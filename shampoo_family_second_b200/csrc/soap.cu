// SOAP: Adam run in the eigenbasis of Shampoo's preconditioner (pith.science
// record of "SOAP: Improving and Stabilizing Shampoo using Adam": abstract and
// claims; the basis is recomputed at a fixed frequency and kept in between),
// on the same blocks, stacks and statistics as the blocked Shampoo step.
//
// Step t (t from 0), every block (ragged blocks use their r x c part):
//   1. stack     Gs, Gt as for Shampoo; m <- beta1 m + (1 - beta1) G (fused)
//   2. rotate    G' = QL^T G QR and m' = QL^T m QR (two launches, two groups each;
//                QL^T is kept transposed in the state so that every product
//                reads its left operand K-major)
//   3. Adam      v <- beta2 v + (1 - beta2) G'^2,
//                N' = (m' / (1 - beta1^{t+1})) / (sqrt(v / (1 - beta2^{t+1})) + eps)
//   4. back      W <- W - lr QL N' QR^T (the second product's epilogue updates W)
//   5. stats     L <- beta L + G G^T, R <- beta R + G^T G
//   6. refresh   if t % refresh_every == 0: new bases from L and R (batched
//                Jacobi, warm-started from the current ones, the identity before
//                the first refresh; then orthogonalisation steps), and the
//                second moment carried over,
//                v <- (PL o PL) v (PR o PR)^T with P = Q_new^T Q_old.
// The basis of a step is built from statistics without that step's gradient:
// the current gradient never enters its own projection, whose exact zeros
// fp32 would turn into rounding noise that Adam's normalisation amplifies.
#include <algorithm>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/shampoo.h"
#include "common.cuh"
#include "internal.h"

using namespace shampoo;

namespace {

constexpr size_t kAlignS = 256;
constexpr size_t kEigBudget = size_t(16) << 30;
size_t als(size_t x) { return (x + kAlignS - 1) / kAlignS * kAlignS; }

// v <- beta2 v + (1 - beta2) g'^2 and N' = (m' c1) / (sqrt(v c2) + eps) on each
// block's r x c part; zeros elsewhere (v stays zero there).
// grid (B / 32, B / 8, nb), block (32, 8).
__global__ void soap_adam_kernel(const float* __restrict__ Grot, const float* __restrict__ Mrot,
                                 float* __restrict__ V, const int* __restrict__ rows, const int* __restrict__ cols,
                                 int B, float beta2, float c1, float c2, float eps, float* __restrict__ Nrot,
                                 int* flags) {
  pdl_launch_dependents();
  const int b = blockIdx.z;
  const int r = blockIdx.y * 8 + threadIdx.y;
  const int c = blockIdx.x * 32 + threadIdx.x;
  const size_t idx = static_cast<size_t>(b) * B * B + static_cast<size_t>(r) * B + c;
  float out = 0.f;
  if (r < rows[b] && c < cols[b]) {
    const float g = Grot[idx];
    const float v = fmaf(beta2, V[idx], (1.f - beta2) * g * g);
    V[idx] = v;
    out = (Mrot[idx] * c1) / (sqrtf(v * c2) + eps);
    if (!isfinite(out)) raise_flag(flags, DEV_FLAG_NONFINITE);
  }
  Nrot[idx] = out;
}

// P <- P o P (elementwise square), for the second moment's carry-over.
__global__ void square_kernel(float* __restrict__ P, size_t count) {
  pdl_launch_dependents();
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < count) P[i] = P[i] * P[i];
}

// Identity stacks (the basis before the first refresh).
__global__ void identity_kernel(float* __restrict__ Q, int n, size_t count) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= count) return;
  const size_t e = i % (static_cast<size_t>(n) * n);
  Q[i] = (e / n == e % n) ? 1.f : 0.f;
}

__global__ void transpose_stack_kernel(const float* __restrict__ X, int n, float* __restrict__ Xt) {
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

struct SoapState {
  size_t status, table, valid, wrows, wcols, stats, Q, Qt, m, v, total;
};
struct SoapScratch {
  size_t gs, gt, t1, t2, grot, mrot, qold, p, wptr, ld, eig, eig_bytes, total;
};

SoapState soap_state(int nb, int B) {
  SoapState s;
  const size_t one = plain_floats(nb, B) * 4;
  size_t o = 0;
  s.status = o, o += als(4);
  s.table = o, o += als(size_t(nb) * 5 * 4);
  s.valid = o, o += als(size_t(2) * nb * 4);
  s.wrows = o, o += als(size_t(nb) * 4);
  s.wcols = o, o += als(size_t(nb) * 4);
  s.stats = o, o += als(2 * one);
  s.Q = o, o += als(2 * one);
  s.Qt = o, o += als(2 * one);
  s.m = o, o += als(one);
  s.v = o, o += als(one);
  s.total = o;
  return s;
}

SoapScratch soap_scratch(int nb, int B) {
  SoapScratch s;
  const size_t one = plain_floats(nb, B) * 4;
  size_t o = 0;
  s.gs = o, o += als(one);
  s.gt = o, o += als(one);
  s.t1 = o, o += als(one);
  s.t2 = o, o += als(one);
  s.grot = o, o += als(one);
  s.mrot = o, o += als(one);
  s.qold = o, o += als(2 * one);
  s.p = o, o += als(2 * one);
  s.wptr = o, o += als(size_t(nb) * 8);
  s.ld = o, o += als(size_t(nb) * 4);
  s.eig = o;
  const size_t per = eig_scratch_per_matrix(B);
  s.eig_bytes = std::min(per * size_t(2 * nb), std::max(kEigBudget, per));
  o += als(s.eig_bytes);
  s.total = o;
  return s;
}

int validate_soap(const shampoo_config* c, const shampoo_soap_config* sc) {
  if (!c || !sc) return set_error(SHAMPOO_ERR_INVALID_ARG, "config is NULL");
  if (c->block < 32 || c->block > 1024 || c->block % 32)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "block %d: need a multiple of 32 in [32, 1024]", c->block);
  if (!(c->beta >= 0.f) || !(c->beta <= 1.f)) return set_error(SHAMPOO_ERR_INVALID_ARG, "beta must be in [0, 1]");
  if (!(c->lr == c->lr)) return set_error(SHAMPOO_ERR_INVALID_ARG, "lr is NaN");
  if (c->refresh_every < 1) return set_error(SHAMPOO_ERR_INVALID_ARG, "refresh_every must be >= 1");
  if (c->grad_dtype != SHAMPOO_F32 && c->grad_dtype != SHAMPOO_BF16)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "grad_dtype must be SHAMPOO_F32 or SHAMPOO_BF16");
  if (!(sc->beta1 >= 0.f && sc->beta1 < 1.f) || !(sc->beta2 >= 0.f && sc->beta2 < 1.f))
    return set_error(SHAMPOO_ERR_INVALID_ARG, "beta1, beta2 must be in [0, 1)");
  if (!(sc->eps > 0.f)) return set_error(SHAMPOO_ERR_INVALID_ARG, "eps must be > 0");
  if (sc->jacobi_sweeps < 1 || sc->jacobi_sweeps > 100 || sc->refine_iters < 0 || sc->refine_iters > 100)
    return set_error(SHAMPOO_ERR_INVALID_ARG, "jacobi_sweeps in [1, 100], refine_iters in [0, 100]");
  return SHAMPOO_OK;
}

bool aligned256s(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }

}  // namespace

struct shampoo_soap_ctx {
  shampoo_config cfg;
  shampoo_soap_config sc;
  int nparams = 0, nb = 0;
  std::vector<int64_t> rows, cols;
  std::vector<int> table;
  SoapState sl;
  SoapScratch xl;
  char* state = nullptr;
  char* scratch = nullptr;
  int* d_status = nullptr;
  float *stats = nullptr, *Q = nullptr, *Qt = nullptr, *m = nullptr, *v = nullptr;
  float *Gs = nullptr, *Gt = nullptr, *T1 = nullptr, *T2 = nullptr, *Grot = nullptr, *Mrot = nullptr;
  float *Qold = nullptr, *P = nullptr;
  float** blk_wptr = nullptr;
  int* blk_ld = nullptr;
  int *d_valid = nullptr, *d_wrows = nullptr, *d_wcols = nullptr, *d_table = nullptr;
  StackMaps mGs, mGt, mQ, mQt, mM, mT1, mT2, mN, mQold, mP, mV;
  double fl = 0, fr = 0, stack_bytes = 0;
  int64_t step = 0;
  cudaStream_t last_stream = nullptr;
};

extern "C" {

int shampoo_soap_query_sizes(const shampoo_config* cfg, const shampoo_soap_config* sc, int32_t nparams,
                             const int64_t* rows, const int64_t* cols, size_t* state_bytes, size_t* scratch_bytes) {
  int rc = validate_soap(cfg, sc);
  if (rc) return rc;
  std::vector<int> table;
  if ((rc = build_block_table(cfg->block, nparams, rows, cols, table))) return rc;
  if (!state_bytes || !scratch_bytes) return set_error(SHAMPOO_ERR_INVALID_ARG, "output pointer is NULL");
  const int nb = static_cast<int>(table.size() / 5);
  *state_bytes = soap_state(nb, cfg->block).total;
  *scratch_bytes = soap_scratch(nb, cfg->block).total;
  return SHAMPOO_OK;
}

int shampoo_soap_init(const shampoo_config* cfg, const shampoo_soap_config* sc, int32_t nparams, const int64_t* rows,
                      const int64_t* cols, void* d_state, size_t state_bytes, void* d_scratch, size_t scratch_bytes,
                      void* stream, shampoo_soap_handle* out) {
  int rc = validate_soap(cfg, sc);
  if (rc) return rc;
  if (!out) return set_error(SHAMPOO_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  std::vector<int> table;
  if ((rc = build_block_table(cfg->block, nparams, rows, cols, table))) return rc;
  if (!d_state || !d_scratch) return set_error(SHAMPOO_ERR_INVALID_ARG, "state/scratch is NULL");
  if (!aligned256s(d_state) || !aligned256s(d_scratch))
    return set_error(SHAMPOO_ERR_UNSUPPORTED, "state/scratch must be 256-byte aligned");
  const int B = cfg->block, nb = static_cast<int>(table.size() / 5);
  SoapState sl = soap_state(nb, B);
  SoapScratch xl = soap_scratch(nb, B);
  if (state_bytes < sl.total) return set_error(SHAMPOO_ERR_WORKSPACE, "state %zu < %zu bytes", state_bytes, sl.total);
  if (scratch_bytes < xl.total)
    return set_error(SHAMPOO_ERR_WORKSPACE, "scratch %zu < %zu bytes", scratch_bytes, xl.total);
  shampoo_soap_ctx* h = new (std::nothrow) shampoo_soap_ctx;
  if (!h) return set_error(SHAMPOO_ERR_INVALID_ARG, "out of host memory");
  h->cfg = *cfg;
  h->sc = *sc;
  h->nparams = nparams;
  h->nb = nb;
  h->rows.assign(rows, rows + nparams);
  h->cols.assign(cols, cols + nparams);
  h->table = table;
  h->sl = sl;
  h->xl = xl;
  h->state = static_cast<char*>(d_state);
  h->scratch = static_cast<char*>(d_scratch);
  auto S = [&](size_t o) { return reinterpret_cast<float*>(h->state + o); };
  auto X = [&](size_t o) { return reinterpret_cast<float*>(h->scratch + o); };
  h->d_status = reinterpret_cast<int*>(h->state + sl.status);
  h->d_table = reinterpret_cast<int*>(h->state + sl.table);
  h->d_valid = reinterpret_cast<int*>(h->state + sl.valid);
  h->d_wrows = reinterpret_cast<int*>(h->state + sl.wrows);
  h->d_wcols = reinterpret_cast<int*>(h->state + sl.wcols);
  h->stats = S(sl.stats);
  h->Q = S(sl.Q);
  h->Qt = S(sl.Qt);
  h->m = S(sl.m);
  h->v = S(sl.v);
  h->Gs = X(xl.gs);
  h->Gt = X(xl.gt);
  h->T1 = X(xl.t1);
  h->T2 = X(xl.t2);
  h->Grot = X(xl.grot);
  h->Mrot = X(xl.mrot);
  h->Qold = X(xl.qold);
  h->P = X(xl.p);
  h->blk_wptr = reinterpret_cast<float**>(h->scratch + xl.wptr);
  h->blk_ld = reinterpret_cast<int*>(h->scratch + xl.ld);
  std::vector<int> valid(2 * nb), wr(nb), wc(nb);
  for (int b = 0; b < nb; ++b) {
    const double r = table[5 * b + 3], c = table[5 * b + 4];
    valid[b] = wr[b] = table[5 * b + 3];
    valid[nb + b] = wc[b] = table[5 * b + 4];
    h->fl += 2 * r * r * c / nb;
    h->fr += 2 * r * c * c / nb;
    h->stack_bytes += r * c * (cfg->grad_dtype == SHAMPOO_BF16 ? 2 : 4) + 16.0 * B * B;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  const size_t one = plain_floats(nb, B);
  auto up = [&](void* dst, const void* src, size_t bytes) {
    return check_cuda(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, st), "upload block table");
  };
  if (!(rc = up(h->d_table, table.data(), table.size() * 4)) && !(rc = up(h->d_valid, valid.data(), valid.size() * 4)) &&
      !(rc = up(h->d_wrows, wr.data(), wr.size() * 4)) && !(rc = up(h->d_wcols, wc.data(), wc.size() * 4)) &&
      !(rc = check_cuda(cudaMemsetAsync(h->d_status, 0, 4, st), "zero status")) &&
      !(rc = check_cuda(cudaMemsetAsync(h->stats, 0, 2 * one * 4, st), "zero statistics")) &&
      !(rc = check_cuda(cudaMemsetAsync(h->m, 0, one * 4, st), "zero m")) &&
      !(rc = check_cuda(cudaMemsetAsync(h->v, 0, one * 4, st), "zero v"))) {
    const size_t cnt = 2 * one;
    identity_kernel<<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, st>>>(h->Q, B, cnt);
    identity_kernel<<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, st>>>(h->Qt, B, cnt);
    count_launch();
    count_launch();
    rc = check_cuda(cudaGetLastError(), "identity_kernel");
    if (!rc) rc = check_cuda(cudaStreamSynchronize(st), "init sync");
  }
  if (!rc && !((rc = make_stack_maps(h->mGs, h->Gs, nb, B)) || (rc = make_stack_maps(h->mGt, h->Gt, nb, B)) ||
               (rc = make_stack_maps(h->mQ, h->Q, 2 * nb, B)) || (rc = make_stack_maps(h->mQt, h->Qt, 2 * nb, B)) ||
               (rc = make_stack_maps(h->mM, h->m, nb, B)) || (rc = make_stack_maps(h->mT1, h->T1, nb, B)) ||
               (rc = make_stack_maps(h->mT2, h->T2, nb, B)) || (rc = make_stack_maps(h->mN, h->Grot, nb, B)) ||
               (rc = make_stack_maps(h->mQold, h->Qold, 2 * nb, B)) || (rc = make_stack_maps(h->mP, h->P, 2 * nb, B)) ||
               (rc = make_stack_maps(h->mV, h->v, nb, B)))) {
  }
  if (rc) {
    delete h;
    return rc;
  }
  *out = h;
  return SHAMPOO_OK;
}

int shampoo_soap_step(shampoo_soap_handle h, float* const* d_weights, const void* const* d_grads, void* stream) {
  if (!h) return set_error(SHAMPOO_ERR_INVALID_ARG, "handle is NULL");
  if (!d_weights || !d_grads) return set_error(SHAMPOO_ERR_INVALID_ARG, "weights/grads array is NULL");
  const shampoo_config& c = h->cfg;
  const shampoo_soap_config& sc = h->sc;
  const int B = c.block, nb = h->nb;
  StackArgs args;
  for (int i = 0; i < h->nparams; ++i) {
    if (!d_weights[i] || !d_grads[i]) return set_error(SHAMPOO_ERR_INVALID_ARG, "param %d has a NULL pointer", i);
    args.g[i] = d_grads[i];
    args.w[i] = d_weights[i];
    args.ld[i] = static_cast<int>(h->cols[i]);
    const size_t esize = c.grad_dtype == SHAMPOO_BF16 ? 2 : 4;
    args.vec[i] = (h->cols[i] % 4 == 0 && reinterpret_cast<uintptr_t>(d_grads[i]) % (4 * esize) == 0) ? 1 : 0;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  const size_t one = plain_floats(nb, B);
  const double f1 = 2.0 * B * static_cast<double>(B) * B;
  int rc;
  // 1. stack, and m <- beta1 m + (1 - beta1) G
  if ((rc = launch_stack(args, h->d_table, nb, B, c.grad_dtype, h->Gs, h->Gt, h->m, sc.beta1, 1.f - sc.beta1,
                         h->blk_wptr, h->blk_ld, st, h->stack_bytes)))
    return rc;
  const int g_exact = c.grad_dtype == SHAMPOO_BF16 ? 1 : 0;
  {  // 2a. T1 = QL^T G, T2 = QL^T m
    Builder b;
    Epilogue& e1 = b.add(nb, B, h->mQt, 0, h->mGt, 0, h->fl);
    b.L.g[0].b_exact = g_exact;
    e1.D = h->T1;
    e1.flags = h->d_status;
    Epilogue& e2 = b.add(nb, B, h->mQt, 0, h->mM, 0, h->fl, B_MN_MAJOR);
    e2.D = h->T2;
    e2.flags = h->d_status;
    if ((rc = b.launch(st))) return rc;
  }
  {  // 2b. G' = T1 QR, m' = T2 QR
    Builder b;
    Epilogue& e1 = b.add(nb, B, h->mT1, 0, h->mQ, nb, h->fr, B_MN_MAJOR);
    e1.D = h->Grot;
    e1.flags = h->d_status;
    Epilogue& e2 = b.add(nb, B, h->mT2, 0, h->mQ, nb, h->fr, B_MN_MAJOR);
    e2.D = h->Mrot;
    e2.flags = h->d_status;
    if ((rc = b.launch(st))) return rc;
  }
  {  // 3. Adam in the eigenbasis (N' overwrites G')
    const double t = static_cast<double>(h->step + 1);
    const float c1 = static_cast<float>(1.0 / (1.0 - std::pow(static_cast<double>(sc.beta1), t)));
    const float c2 = static_cast<float>(1.0 / (1.0 - std::pow(static_cast<double>(sc.beta2), t)));
    ProfScope ps(K_SOAP, st, 0.0, 20.0 * one);
    soap_adam_kernel<<<dim3(B / 32, B / 8, nb), dim3(32, 8), 0, st>>>(h->Grot, h->Mrot, h->v, h->d_wrows, h->d_wcols,
                                                                     B, sc.beta2, c1, c2, sc.eps, h->Grot,
                                                                     h->d_status);
    count_launch();
    if ((rc = check_cuda(cudaGetLastError(), "soap_adam_kernel"))) return rc;
  }
  {  // 4a. T1 = QL N'
    Builder b;
    Epilogue& e = b.add(nb, B, h->mQ, 0, h->mN, 0, h->fl, B_MN_MAJOR);
    e.D = h->T1;
    e.flags = h->d_status;
    if ((rc = b.launch(st))) return rc;
  }
  {  // 4b. W -= lr T1 QR^T (QR read K-major: D = T1 QR^T), masked to each block
    Builder b;
    Epilogue& e = b.add(nb, B, h->mT1, 0, h->mQ, nb, h->fr, B_TRANSPOSED);
    e.wptr = h->blk_wptr;
    e.wld = h->blk_ld;
    e.wrows = h->d_wrows;
    e.wcols = h->d_wcols;
    e.lr = c.lr;
    e.flags = h->d_status;
    if ((rc = b.launch(st))) return rc;
  }
  {  // 5. statistics
    Builder b;
    Epilogue& eL = b.add(nb, B, h->mGs, 0, h->mGs, 0, h->fl);
    b.L.g[0].a_exact = b.L.g[0].b_exact = g_exact;
    b.L.g[0].sym = 1;
    eL.beta = c.beta;
    eL.C = h->stats;
    eL.D = h->stats;
    eL.flags = h->d_status;
    Epilogue& eR = b.add(nb, B, h->mGt, 0, h->mGt, 0, h->fr);
    b.L.g[1].a_exact = b.L.g[1].b_exact = g_exact;
    b.L.g[1].sym = 1;
    eR.beta = c.beta;
    eR.C = h->stats + one;
    eR.D = h->stats + one;
    eR.flags = h->d_status;
    if ((rc = b.launch(st))) return rc;
    if ((rc = launch_mirror_lower(h->stats, 2 * nb, B, st))) return rc;
  }
  // 6. refresh: new bases, the second moment carried over
  if (h->step % c.refresh_every == 0) {
    if ((rc = check_cuda(cudaMemcpyAsync(h->Qold, h->Q, 2 * one * 4, cudaMemcpyDeviceToDevice, st), "save basis")))
      return rc;
    if ((rc = run_eigh(h->stats, h->Q, nullptr, 2 * nb, B, h->d_valid, 1, sc.jacobi_sweeps, sc.refine_iters,
                       h->scratch + h->xl.eig, h->xl.eig_bytes, h->d_status, st)))
      return rc;
    {
      ProfScope ps(K_SOAP, st, 0.0, 16.0 * one);
      transpose_stack_kernel<<<dim3(B / 32, B / 32, 2 * nb), dim3(32, 8), 0, st>>>(h->Q, B, h->Qt);
      count_launch();
      if ((rc = check_cuda(cudaGetLastError(), "transpose_stack_kernel"))) return rc;
    }
    {  // P = Q_new^T Q_old, both sides
      Builder b;
      Epilogue& e = b.add(2 * nb, B, h->mQt, 0, h->mQold, 0, 2 * f1 / 2, B_MN_MAJOR);
      e.D = h->P;
      e.flags = h->d_status;
      if ((rc = b.launch(st))) return rc;
    }
    {
      ProfScope ps(K_SOAP, st, 0.0, 16.0 * one);
      const size_t cnt = 2 * one;
      square_kernel<<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, st>>>(h->P, cnt);
      count_launch();
      if ((rc = check_cuda(cudaGetLastError(), "square_kernel"))) return rc;
    }
    {  // T2 = PL2 v
      Builder b;
      Epilogue& e = b.add(nb, B, h->mP, 0, h->mV, 0, f1, B_MN_MAJOR);
      e.D = h->T2;
      e.flags = h->d_status;
      if ((rc = b.launch(st))) return rc;
    }
    {  // v = T2 PR2^T
      Builder b;
      Epilogue& e = b.add(nb, B, h->mT2, 0, h->mP, nb, f1, B_TRANSPOSED);
      e.D = h->v;
      e.flags = h->d_status;
      if ((rc = b.launch(st))) return rc;
    }
  }
  h->step += 1;
  return SHAMPOO_OK;
}

int shampoo_soap_views(shampoo_soap_handle h, float** L, float** R, float** QL, float** QR, float** m, float** v,
                       int64_t* step) {
  if (!h) return set_error(SHAMPOO_ERR_INVALID_ARG, "handle is NULL");
  const size_t one = plain_floats(h->nb, h->cfg.block);
  if (L) *L = h->stats;
  if (R) *R = h->stats + one;
  if (QL) *QL = h->Q;
  if (QR) *QR = h->Q + one;
  if (m) *m = h->m;
  if (v) *v = h->v;
  if (step) *step = h->step;
  return SHAMPOO_OK;
}

int shampoo_soap_get_status(shampoo_soap_handle h, int32_t* status, int32_t reset) {
  if (!h || !status) return set_error(SHAMPOO_ERR_INVALID_ARG, "handle/status is NULL");
  int rc = check_cuda(cudaStreamSynchronize(h->last_stream), "status sync");
  if (rc) return rc;
  int v = 0;
  if ((rc = check_cuda(cudaMemcpy(&v, h->d_status, 4, cudaMemcpyDeviceToHost), "read status"))) return rc;
  *status = v;
  if (reset && (rc = check_cuda(cudaMemset(h->d_status, 0, 4), "reset status"))) return rc;
  return SHAMPOO_OK;
}

void shampoo_soap_destroy(shampoo_soap_handle h) { delete h; }

}  // extern "C"
