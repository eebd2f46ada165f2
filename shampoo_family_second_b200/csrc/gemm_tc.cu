// Batched fp32-accurate GEMM on the sm_100a tensor cores (tcgen05, kind::tf32,
// three MMAs per product: hi*hi + hi*lo + lo*hi) with fused epilogues.
//
// Every dense contraction of the blocked Shampoo step runs through this kernel:
//   statistics      L <- beta L + G G^T,  R <- beta R + G^T G
//                   ("Shampoo optimizer" notes, matrix-case listing; podcast
//                   "Preconditioned optimization without the full matrix cost",
//                   cue 20),
//   inverse roots   the products of the coupled-Newton, Newton-DB and Chebyshev
//                   iterations on stacked blocks (DASH abstract: blocks stacked
//                   into 3D tensors, Newton-DB and Chebyshev solvers),
//   apply + update  T = L^{-1/4} G, then W <- W - lr T R^{-1/4} scattered into
//                   the weight (notes' listing, last line).
//
// One CTA computes one 128 x 256 tile of one matrix D_i = epi(A_i B_i^T), or
// epi(A_i B_i) when B is read MN-major (B stored K x N row-major):
//   warp 0      one thread issues TMA loads of the A and B tiles (hi and lo
//               planes) into a 2-stage shared-memory ring;
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 buffers); one
//               thread issues the tcgen05 MMAs (3 per K-step of 8), each K
//               segment of 64 into the next buffer, and commits them to the
//               ring's "empty" barriers and the buffer's "full" barrier;
//   warps 2-9   add each finished segment into fp32 registers (round to
//               nearest; one row x 128 columns per thread), then apply the
//               epilogue and store.  The tensor core's own fp32 additions
//               truncate; summing short segments outside it keeps the product
//               as accurate as a plain fp32 GEMM.
// Every wait is bounded (2 s); a time-out raises DEV_FLAG_TIMEOUT and the CTA
// unwinds, releasing its TMEM.
#include <cstdio>
#include <cstring>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace shampoo {
namespace {

constexpr int BM = kTileM;
constexpr int BN = kTileN;
constexpr int BK = kTileK;
constexpr int STAGES = 2;
constexpr int A_PLANE = BM * BK * 4;                        // 16 KB
constexpr int B_PLANE = BN * BK * 4;                        // 32 KB
constexpr int STAGE_BYTES = 2 * A_PLANE + 2 * B_PLANE;      // 96 KB
constexpr int MN_BLOCK = BK * 32 * 4;                      // 4 KB: 32 K-rows x 32 columns
constexpr int TMEM_COLS = 512;  // two 128 x 256 fp32 accumulators (K-segment double buffer)
constexpr int SEG = 2;           // K chunks (of 32) per accumulation segment
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;

__device__ __forceinline__ void store_row32(float* dst, const float (&v)[32]) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int j = 0; j < 8; ++j) d4[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

__device__ __forceinline__ void store_split_row32(float* hi_dst, float* lo_dst, const float (&v)[32]) {
  float4* h4 = reinterpret_cast<float4*>(hi_dst);
  float4* l4 = reinterpret_cast<float4*>(lo_dst);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float h[4], l[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) split_tf32(v[4 * j + q], h[q], l[q]);
    h4[j] = make_float4(h[0], h[1], h[2], h[3]);
    l4[j] = make_float4(l[0], l[1], l[2], l[3]);
  }
}

// Epilogue for 32 consecutive columns [c0, c0+32) of row r of matrix `mat`;
// acc holds the fp32 products (A B^T or A B) of those columns.
// Returns this thread's residual contribution.
__device__ __forceinline__ float epilogue_chunk(const GemmGroup& G, int mat, int r, int c0, const float* acc,
                                                bool& nonfinite) {
  const Epilogue& E = G.ep;
  const int n = G.n;
  const size_t nn = static_cast<size_t>(n) * n;
  const size_t row_off = static_cast<size_t>(r) * n + c0;
  float v[32];
  float resid = 0.f;
  const int vsz = E.valid ? E.valid[mat] : n;
  if (E.res) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int c = c0 + j;
      float d = acc[j] - ((r == c) ? 1.f : 0.f);
      resid += (r < vsz && c < vsz) ? d * d : 0.f;
    }
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = E.alpha * acc[j];
  if (E.C) {
    if (E.c_split) {
      const float4* h4 = reinterpret_cast<const float4*>(E.C + mat * 2 * nn + row_off);
      const float4* l4 = reinterpret_cast<const float4*>(E.C + mat * 2 * nn + nn + row_off);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 h = h4[j], l = l4[j];
        v[4 * j + 0] += E.beta * (h.x + l.x);
        v[4 * j + 1] += E.beta * (h.y + l.y);
        v[4 * j + 2] += E.beta * (h.z + l.z);
        v[4 * j + 3] += E.beta * (h.w + l.w);
      }
    } else {
      const float4* c4 = reinterpret_cast<const float4*>(E.C + mat * nn + row_off);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 h = c4[j];
        v[4 * j + 0] += E.beta * h.x;
        v[4 * j + 1] += E.beta * h.y;
        v[4 * j + 2] += E.beta * h.z;
        v[4 * j + 3] += E.beta * h.w;
      }
    }
  }
  const float gam = E.gamma_vec ? E.gamma_vec[static_cast<size_t>(mat) * E.gamma_stride] : E.gamma;
  const int dj = r - c0;
  if (dj >= 0 && dj < 32) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j == dj) v[j] += gam;
  }
  if (E.scale_vec) {
    const float sc = E.scale_vec[mat];
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= sc;
  }
  bool bad = false;
#pragma unroll
  for (int j = 0; j < 32; ++j) bad |= !isfinite(v[j]);
  nonfinite |= bad;
  if (E.D) {
    if (E.d_split)
      store_split_row32(E.D + mat * 2 * nn + row_off, E.D + mat * 2 * nn + nn + row_off, v);
    else
      store_row32(E.D + mat * nn + row_off, v);
  }
  if (E.E) {
    float e[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) e[j] = E.e_mul * v[j] + ((j == dj) ? E.e_add : 0.f);
    store_split_row32(E.E + mat * 2 * nn + row_off, E.E + mat * 2 * nn + nn + row_off, e);
  }
  if (E.wptr) {
    const int wr = E.wrows[mat], wc = E.wcols[mat];
    if (r < wr) {
      float* w = E.wptr[mat] + static_cast<size_t>(r) * E.wld[mat];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int c = c0 + j;
        if (c < wc) w[c] -= E.lr * v[j];
      }
    }
  }
  return resid;
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm3x_tf32_kernel(const __grid_constant__ GemmLaunch L, const __grid_constant__ TmaMaps maps,
                       double* prof_flops) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]: a K-segment's partial sums are ready in TMEM buffer b
  uint64_t* acc_empty = acc_full + 2;    // [2]: the epilogue has drained TMEM buffer b
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  // Locate this CTA's group, matrix and tile.
  const int cta = blockIdx.x;
  int gi = 0;
#pragma unroll 1
  while (gi + 1 < L.ngroups && cta >= L.g[gi + 1].cta_begin) ++gi;
  const GemmGroup& G = L.g[gi];
  const int local = cta - G.cta_begin;
  const int tiles = G.tiles_m * G.tiles_n;
  const int mat = local / tiles;
  const int t = local - mat * tiles;
  const int tm = t / G.tiles_n;
  const int tn = t - tm * G.tiles_n;
  if (G.ep.skip && G.ep.skip[mat]) return;  // uniform across the CTA: nothing allocated yet

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n = G.n;
  const int nk = n / BK;
  const int nseg = (nk + SEG - 1) / SEG;
  int* flags = G.ep.flags;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS);
    }
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.m[G.a_map]);
    prefetch_tmap(&maps.m[G.b_map]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const uint32_t tx_bytes = 2u * G.a_rows * BK * 4u + 2u * G.b_rows * BK * 4u;
      const void* amap = &maps.m[G.a_map];
      const void* bmap = &maps.m[G.b_map];
      const int am = G.a_off + mat;
      const int bm = G.b_off + mat;
      int issued = 0;
#pragma unroll 1
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % STAGES;
        if (kc >= STAGES && !mbar_wait_bounded(&empty[s], ((kc / STAGES) - 1) & 1, flags)) break;
        uint8_t* sa = smem + s * STAGE_BYTES;
        uint8_t* sb = sa + 2 * A_PLANE;
        mbar_arrive_expect_tx(&full[s], tx_bytes);
        // One copy per plane, each to its fixed offset (the boxes may hold
        // fewer rows than the tile when n is small).
        tma_load_4d(sa, amap, &full[s], kc * BK, tm * BM, 0, am);
        tma_load_4d(sa + A_PLANE, amap, &full[s], kc * BK, tm * BM, 1, am);
        if (G.b_mn) {
          // B[k][n] row-major: 32 K-rows x 32 N-columns per copy, one copy per
          // 32-column block of the tile, blocks MN_BLOCK bytes apart.
          const int nblk = G.b_rows / 32;
#pragma unroll 1
          for (int q = 0; q < nblk; ++q) {
            tma_load_4d(sb + q * MN_BLOCK, bmap, &full[s], tn * BN + q * 32, kc * BK, 0, bm);
            tma_load_4d(sb + B_PLANE + q * MN_BLOCK, bmap, &full[s], tn * BN + q * 32, kc * BK, 1, bm);
          }
        } else {
          tma_load_4d(sb, bmap, &full[s], kc * BK, tn * BN, 0, bm);
          tma_load_4d(sb + B_PLANE, bmap, &full[s], kc * BK, tn * BN, 1, bm);
        }
        ++issued;
      }
      // Drain: make sure no copy is still landing in shared memory when the
      // CTA retires (bounded; normally these phases completed long ago).
#pragma unroll 1
      for (int kc = (issued > STAGES ? issued - STAGES : 0); kc < issued; ++kc)
        mbar_wait_bounded(&full[kc % STAGES], (kc / STAGES) & 1, flags);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      // K is cut into segments of SEG chunks.  Segment g accumulates from zero
      // into TMEM buffer g & 1; the epilogue warps add each finished segment
      // into fp32 registers with round-to-nearest.  The tensor core's own
      // additions (which truncate) then only ever see one segment's partial
      // sums, which keeps the truncation bias of long products small.
      const uint32_t idesc = idesc_tf32(BM, BN, G.b_mn);
#pragma unroll 1
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % STAGES;
        const int seg = kc / SEG;
        const int b = seg & 1;
        const bool first = (kc % SEG) == 0;
        const uint32_t tbuf = taddr + b * BN;
        if (first && seg >= 2 && !mbar_wait_bounded(&acc_empty[b], ((seg >> 1) - 1) & 1, flags)) break;
        if (!mbar_wait_bounded(&full[s], (kc / STAGES) & 1, flags)) break;
        tc_fence_after();
        const uint32_t a_hi = smem_u32(smem + s * STAGE_BYTES);
        const uint32_t a_lo = a_hi + A_PLANE;
        const uint32_t b_hi = a_hi + 2 * A_PLANE;
        const uint32_t b_lo = b_hi + B_PLANE;
#pragma unroll
        for (int ks = 0; ks < BK / 8; ++ks) {
          const uint32_t off = ks * 32;  // 8 tf32 values = 32 bytes along K (K-major)
          const uint64_t dah = smem_desc_k_sw128(a_hi + off);
          const uint64_t dal = smem_desc_k_sw128(a_lo + off);
          uint64_t dbh, dbl;
          if (G.b_mn) {  // 8 K-rows = 1024 bytes = two 4-row groups
            dbh = smem_desc_mn_sw128_32b(b_hi + ks * 1024, MN_BLOCK);
            dbl = smem_desc_mn_sw128_32b(b_lo + ks * 1024, MN_BLOCK);
          } else {
            dbh = smem_desc_k_sw128(b_hi + off);
            dbl = smem_desc_k_sw128(b_lo + off);
          }
          mma_tf32(tbuf, dah, dbh, idesc, (first && ks == 0) ? 0u : 1u);
          mma_tf32(tbuf, dah, dbl, idesc, 1u);
          mma_tf32(tbuf, dal, dbh, idesc, 1u);
        }
        mma_commit(&empty[s]);
        if ((kc % SEG) == SEG - 1 || kc == nk - 1) mma_commit(&acc_full[b]);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // 8 warps: warp w reads TMEM lane quarter (w & 3) and column half h.
    const int ew = warp - 2;
    const int q = warp & 3;
    const int h = ew >> 2;
    const int r = tm * BM + q * 32 + lane;
    const uint32_t lane_addr = taddr + (static_cast<uint32_t>(q * 32) << 16) + h * (BN / 2);
    float sum[BN / 2];
#pragma unroll
    for (int j = 0; j < BN / 2; ++j) sum[j] = 0.f;
    bool ok = true;
#pragma unroll 1
    for (int seg = 0; seg < nseg; ++seg) {
      const int b = seg & 1;
      if (!mbar_wait_bounded(&acc_full[b], (seg >> 1) & 1, flags)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < BN / 64; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(lane_addr + b * BN + c * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) sum[c * 32 + j] += __uint_as_float(v[j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
    float resid = 0.f;
    bool nonfinite = false;
    if (ok && r < n) {
#pragma unroll
      for (int c = 0; c < BN / 64; ++c) {
        const int c0 = tn * BN + h * (BN / 2) + c * 32;
        if (c0 < n) resid += epilogue_chunk(G, mat, r, c0, &sum[c * 32], nonfinite);
      }
    }
    if (G.ep.res) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) resid += __shfl_xor_sync(0xffffffffu, resid, o);
      if (lane == 0 && resid != 0.f) atomicAdd(&G.ep.res[mat], resid);
    }
    if (nonfinite) raise_flag(flags, DEV_FLAG_NONFINITE);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(taddr, TMEM_COLS);
  }
  if (L.profile && threadIdx.x == 0 && prof_flops)
    atomicAdd(&prof_flops[L.prof_slot], G.flops_per_matrix / tiles);
}

}  // namespace

Epilogue epilogue_defaults() {
  Epilogue e;
  std::memset(&e, 0, sizeof(e));
  e.alpha = 1.f;
  e.gamma_stride = 1;
  return e;
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encoder() {
  if (g_encode) return 0;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
    return set_error(-4, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(e));
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return 0;
}
}  // namespace

// Tensor map over a split stack (batch, 2, n, n) fp32: dimensions (innermost
// first) column = n, row = n, plane = 2, matrix = batch; box {32, box_rows, 1,
// 1} (one plane of a box_rows x 32 tile per copy).  K-major operand tiles use
// the 128-byte swizzle; MN-major tiles (mn_layout) the 128-byte swizzle with
// 32-byte atoms, the only MN-major tf32 layout of the tensor core.
int encode_split_map(CUtensorMap* map, const float* base, int64_t batch, int n, int box_rows, int mn_layout) {
  int rc = get_encoder();
  if (rc) return rc;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return set_error(-2, "stack base not 16-byte aligned");
  const cuuint64_t nn = static_cast<cuuint64_t>(n);
  cuuint64_t dims[4] = {nn, nn, 2, static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[3] = {nn * 4, nn * nn * 4, 2 * nn * nn * 4};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        mn_layout ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(-4, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return 0;
}

int make_stack_maps(StackMaps& sm, float* base, int64_t batch, int n) {
  sm.base = base;
  sm.a_rows = n < BM ? n : BM;
  sm.b_rows = n < BN ? n : BN;
  int rc = encode_split_map(&sm.a, base, batch, n, sm.a_rows);
  if (rc) return rc;
  if ((rc = encode_split_map(&sm.mn, base, batch, n, BK, 1))) return rc;
  return encode_split_map(&sm.b, base, batch, n, sm.b_rows);
}

Builder::Builder() : nmaps(0) {
  std::memset(&L, 0, sizeof(L));
  std::memset(&M, 0, sizeof(M));
}

Epilogue& Builder::add(int batch, int n, const StackMaps& a, int a_off, const StackMaps& b, int b_off,
                       double flops_per_matrix, int b_mn) {
  GemmGroup& g = L.g[L.ngroups++];
  g.batch = batch;
  g.n = n;
  M.m[nmaps] = a.a;
  g.a_map = nmaps++;
  M.m[nmaps] = b_mn ? b.mn : b.b;
  g.b_map = nmaps++;
  g.b_mn = b_mn;
  g.a_off = a_off;
  g.b_off = b_off;
  g.a_rows = a.a_rows;
  g.b_rows = b.b_rows;
  g.flops_per_matrix = flops_per_matrix;
  g.ep = epilogue_defaults();
  return g.ep;
}

int launch_gemm(GemmLaunch& L, const TmaMaps& maps, cudaStream_t st) {
  static unsigned attr_mask = 0;  // devices on which the smem attribute is set
  int dev = 0;
  int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
  if (rc) return rc;
  if (dev < 32 && !(attr_mask & (1u << dev))) {
    rc = check_cuda(cudaFuncSetAttribute(gemm3x_tf32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_BYTES),
                    "cudaFuncSetAttribute(gemm)");
    if (rc) return rc;
    attr_mask |= 1u << dev;
  }
  int64_t total = 0;
  double flops = 0;
  for (int i = 0; i < L.ngroups; ++i) {
    GemmGroup& g = L.g[i];
    g.tiles_m = (g.n + BM - 1) / BM;
    g.tiles_n = (g.n + BN - 1) / BN;
    g.cta_begin = static_cast<int>(total);
    total += static_cast<int64_t>(g.batch) * g.tiles_m * g.tiles_n;
    flops += g.flops_per_matrix * g.batch;
  }
  if (total == 0) return 0;
  if (total > 0x7fffffff) return set_error(-2, "GEMM launch too large (%lld CTAs)", (long long)total);
  L.profile = profiling_enabled() ? 1 : 0;
  L.prof_slot = K_GEMM;
  ProfScope ps(K_GEMM, st, flops, 0.0);
  gemm3x_tf32_kernel<<<static_cast<unsigned>(total), THREADS, SMEM_BYTES, st>>>(L, maps, device_flop_slots());
  count_launch();
  return check_cuda(cudaGetLastError(), "gemm3x_tf32_kernel launch");
}

}  // namespace shampoo
