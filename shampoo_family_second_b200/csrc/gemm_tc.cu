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
// A persistent kernel (one CTA per SM, 16 warps) walks 128 x 256 tiles of the
// matrices D_i = epi(A_i B_i^T), or epi(A_i B_i) when B is read MN-major (B
// stored K x N row-major).  All operands and results are plain fp32 stacks.
//   warp 0      one thread issues TMA loads of the fp32 A and B tiles (16 deep
//               in K) into a 4-stage shared-memory ring;
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 buffers); one
//               thread issues the tcgen05 MMAs (3 per K-step of 8), each K
//               segment of 64 into the next buffer, and commits them to the
//               ring's "empty" barriers and the buffer's "full" barrier;
//   warps 2-7   split each landed tile in place into its tf32 hi part and a
//               separate lo part (split_tf32), then release it to the MMAs;
//   warps 8-15  add each finished segment into fp32 registers (round to
//               nearest; one row x 128 columns per thread), then apply the
//               epilogue through a per-warp 32 x 32 shared-memory tile, so
//               that global loads and stores are whole 128-byte row pieces.
//               The tensor core's own fp32 additions truncate; summing short
//               segments outside it keeps the product as accurate as a plain
//               fp32 GEMM.
// Warps 0-7 hand registers to warps 8-15 (setmaxnreg), whose running sums
// need them.  Every wait is bounded (2 s); a time-out raises
// DEV_FLAG_TIMEOUT, tells the other roles of the CTA to stop waiting, and the
// CTA unwinds, releasing its TMEM.
#include <algorithm>
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
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 4;                  // 8 KB
constexpr int B_BYTES = BN * BK * 4;                  // 16 KB
constexpr int RAW_BYTES = A_BYTES + B_BYTES;          // TMA destination; becomes the hi parts
constexpr int STAGE_BYTES = 2 * RAW_BYTES;            // [A hi | B hi | A lo | B lo]
constexpr int MN_BLOCK = BK * 32 * 4;                 // 2 KB: 16 K-rows x 32 columns
constexpr int TMEM_COLS = 512;  // two 128 x 256 fp32 accumulators (K-segment double buffer)
constexpr int SEG = 4;           // K chunks (of 16) per accumulation segment: 64 deep
constexpr int CONV_WARP0 = 2, CONV_WARPS = 6, CONV_THREADS = 32 * CONV_WARPS;
constexpr int EPI_WARP0 = 8, EPI_WARPS = 8;
constexpr int THREADS = 32 * (EPI_WARP0 + EPI_WARPS);  // 512
constexpr int EPI_TILE_FLOATS = 32 * 32;                // per epilogue warp
constexpr int RING_BYTES = STAGES * STAGE_BYTES;        // 192 KB
constexpr int EPI_BYTES = EPI_WARPS * EPI_TILE_FLOATS * 4;  // 32 KB
constexpr int SMEM_BYTES = RING_BYTES + EPI_BYTES + 1024 + 256;
// Register split: the CTA is launched with 512 x LAUNCH_REGS registers;
// warps 0-7 keep LIGHT_REGS each, warps 8-15 take the rest.
constexpr int LAUNCH_REGS = 128, LIGHT_REGS = 64, HEAVY_REGS = 192;
static_assert(256 * LIGHT_REGS + 256 * HEAVY_REGS == THREADS * LAUNCH_REGS, "register split must match the pool");
static_assert((RAW_BYTES / 16) % CONV_THREADS == 0, "converter work divides evenly");
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

// K per ring chunk (one 64-byte stage row): 16 fp32 values, or 32 bf16; and
// chunks per accumulation segment: 64 deep for fp32 operands, 128 for bf16.
// The bf16 statistics issue one fast MMA per 16 K, and with 64-deep segments
// the epilogue's drains and round-to-nearest adds (32K per segment and tile)
// paced the launch (tensor pipe 13.5% active on the statistics launch of one
// Llama layer); their products are exact, so the longer segment only adds
// truncated fp32 accumulation of exact terms.
__device__ __forceinline__ int chunk_k(const GemmGroup& G) { return G.bf16 ? 2 * BK : BK; }
__device__ __forceinline__ int seg_chunks(const GemmGroup&) { return SEG; }

struct TileCoord {
  int gi, mat, tm, tn;
  bool skip;
};

// Tile `tile` of the launch: group, matrix, tile row and column.  Tiles are
// numbered group by group, matrix by matrix, so the CTAs working at the same
// time share operands of a few matrices through L2.
__device__ __forceinline__ TileCoord tile_coord(const GemmLaunch& L, int tile) {
  TileCoord c;
  int gi = 0;
#pragma unroll 1
  while (gi + 1 < L.ngroups && tile >= L.g[gi + 1].cta_begin) ++gi;
  const GemmGroup& G = L.g[gi];
  const int local = tile - G.cta_begin;
  const int tiles = G.tiles_per;
  c.gi = gi;
  c.mat = local / tiles;
  int t = local - c.mat * tiles;
  if (G.sym) {
    // Symmetric result: tile column tn keeps the tile rows that reach the
    // diagonal or above, tm * BM < (tn + 1) * BN, i.e. tm < 2 tn + 2.
    int tn = 0;
#pragma unroll 1
    while (true) {
      const int cnt = min(2 * tn + 2, G.tiles_m);
      if (t < cnt) break;
      t -= cnt;
      ++tn;
    }
    c.tm = t;
    c.tn = tn;
  } else {
    c.tm = t / G.tiles_n;
    c.tn = t - c.tm * G.tiles_n;
  }
  c.skip = G.ep.skip && G.ep.skip[c.mat];
  return c;
}

// Stages the C rows of the 32 x 32 chunk at (row0, c0) into the warp's shared
// tile with asynchronous 16-byte copies, in the tile's swizzled layout (piece
// k of row R at R * 32 + ((k ^ (R & 7)) << 2)); each 8-lane group copies one
// 128-byte row piece.  The copies are waited for in epilogue_chunk.
__device__ __forceinline__ void stage_c(const Epilogue& E, int m, int n, int mat, int row0, int c0, float* tilebuf,
                                        int lane) {
  const float* base = E.C + static_cast<size_t>(mat) * m * n + static_cast<size_t>(row0) * n + c0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int R = 4 * j + (lane >> 3);
    const int k = lane & 7;
    cp_async_16(tilebuf + R * 32 + ((k ^ (R & 7)) << 2), base + static_cast<size_t>(R) * n + 4 * k);
  }
  cp_async_commit();
}

// Epilogue of one 32 x 32 chunk: rows row0 .. row0+31 (row row0 + lane in this
// thread's registers, acc = its 32 sums for columns c0 .. c0+31).
//   phase 0  (C set) the chunk's C rows arrive in the warp's shared tile by
//            asynchronous copies (issued here, or earlier when c_staged), so
//            all 32 rows are in flight at once and none waits on a register;
//   phase 1  each thread writes alpha * acc + beta C + gamma [r == c] for its
//            row into the warp's shared tile (16-byte pieces XOR-swizzled by
//            the row, so neither phase has bank conflicts; C is read from the
//            same place first) and adds its diagonal term to the residual;
//   phase 2  each quarter-warp takes one row: 8 lanes x 16 bytes = one
//            128-byte piece; the scale, the outputs D, E and the weight update
//            are applied there.
// Each element of C is read before the same thread group's store of that
// element, so C may be the output D (statistics updated in place).
// Epilogue features a launch uses, as a kernel template mask: every line the
// epilogue's four inlined chunk sites carry costs all launches of a kernel
// built with it (with the weight update in every launch, the solver products
// at n = 256 ran 20% slower), so each launch runs the kernel built with only
// the features its groups use.
enum : int {
  F_W = 1,  // weight update (the second apply product)
  F_C = 2,  // C operand (beta C), staged through shared memory
  F_E = 4,  // second output E and the trace residual
};

template <int kF>
__device__ __forceinline__ void epilogue_chunk(const GemmGroup& G, int mat, int row0, int c0, const float* acc,
                                               float* tilebuf, int lane, float& resid, bool& bad, bool c_staged) {
  const Epilogue& E = G.ep;
  const int n = G.n;  // columns (the row stride of C, D, E)
  const int m = G.m;  // rows
  const int r = row0 + lane;
  const int dj = r - c0;  // column of this row's diagonal element within the chunk
  const float gam = E.gamma_vec ? E.gamma_vec[static_cast<size_t>(mat) * E.gamma_stride] : E.gamma;
  if ((kF & F_E) && E.res) {
    const int vsz = E.valid ? E.valid[mat] : n;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j == dj && r < vsz) resid += 1.f - acc[j];
  }
  if ((kF & F_C) && E.C) {
    if (!c_staged) stage_c(E, m, n, mat, row0, c0, tilebuf, lane);
    cp_async_wait_all();
    __syncwarp();
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float4* slot = reinterpret_cast<float4*>(tilebuf + lane * 32 + ((k ^ (lane & 7)) << 2));
    float4 w;
    w.x = E.alpha * acc[4 * k + 0] + ((4 * k + 0 == dj) ? gam : 0.f);
    w.y = E.alpha * acc[4 * k + 1] + ((4 * k + 1 == dj) ? gam : 0.f);
    w.z = E.alpha * acc[4 * k + 2] + ((4 * k + 2 == dj) ? gam : 0.f);
    w.w = E.alpha * acc[4 * k + 3] + ((4 * k + 3 == dj) ? gam : 0.f);
    if ((kF & F_C) && E.C) {
      const float4 c = *slot;
      w.x += E.beta * c.x;
      w.y += E.beta * c.y;
      w.z += E.beta * c.z;
      w.w += E.beta * c.w;
    }
    *slot = w;
  }
  __syncwarp();
  const size_t nn = static_cast<size_t>(m) * n;
  const float sc = E.scale_vec ? E.scale_vec[mat] : 1.f;
  float* wbase = nullptr;
  int wld = 0, wr = 0, wc = 0;
  if ((kF & F_W) && E.wptr) {
    wbase = E.wptr[mat];
    wld = E.wld[mat];
    wr = E.wrows[mat];
    wc = E.wcols[mat];
  }
  const int kq = lane & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int R = 4 * i + (lane >> 3);
    const int gr = row0 + R;
    const int gc = c0 + 4 * kq;
    float4 v = *reinterpret_cast<const float4*>(tilebuf + R * 32 + ((kq ^ (R & 7)) << 2));
    if (gr < m) {
      const size_t off = static_cast<size_t>(mat) * nn + static_cast<size_t>(gr) * n + gc;
      v.x *= sc;
      v.y *= sc;
      v.z *= sc;
      v.w *= sc;
      bad |= !(isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w));
      if (E.D) *reinterpret_cast<float4*>(E.D + off) = v;
      if ((kF & F_E) && E.E) {
        float4 e;
        e.x = E.e_mul * v.x + ((gr == gc + 0) ? E.e_add : 0.f);
        e.y = E.e_mul * v.y + ((gr == gc + 1) ? E.e_add : 0.f);
        e.z = E.e_mul * v.z + ((gr == gc + 2) ? E.e_add : 0.f);
        e.w = E.e_mul * v.w + ((gr == gc + 3) ? E.e_add : 0.f);
        *reinterpret_cast<float4*>(E.E + off) = e;
      }
      if ((kF & F_W) && wbase && gr < wr) {
        float* wrow = wbase + static_cast<size_t>(gr) * wld + gc;
        if (gc + 3 < wc && (reinterpret_cast<uintptr_t>(wrow) & 15) == 0) {
          float4 w4 = *reinterpret_cast<float4*>(wrow);  // one 16-byte read-modify-write
          w4.x -= E.lr * v.x;
          w4.y -= E.lr * v.y;
          w4.z -= E.lr * v.z;
          w4.w -= E.lr * v.w;
          *reinterpret_cast<float4*>(wrow) = w4;
        } else {
          if (gc + 0 < wc) wrow[0] -= E.lr * v.x;
          if (gc + 1 < wc) wrow[1] -= E.lr * v.y;
          if (gc + 2 < wc) wrow[2] -= E.lr * v.z;
          if (gc + 3 < wc) wrow[3] -= E.lr * v.w;
        }
      }
    }
  }
  __syncwarp();
}

// Persistent: one CTA per SM walks the tiles blockIdx.x, blockIdx.x +
// gridDim.x, ...  The shared-memory ring and the two TMEM buffers carry over
// from one tile to the next, so the epilogue of a tile (register sums ->
// global stores) overlaps the MMAs of the next one.
template <int kF>
__global__ void __launch_bounds__(THREADS, 1)
    gemm3x_tf32_kernel(const __grid_constant__ GemmLaunch L, const __grid_constant__ TmaMaps maps,
                       double* prof_flops) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* epi_tiles = reinterpret_cast<float*>(smem + RING_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + RING_BYTES + EPI_BYTES);  // [STAGES]: TMA landed
  uint64_t* conv = full + STAGES;        // [STAGES]: operands split, ready for the MMAs
  uint64_t* empty = conv + STAGES;       // [STAGES]: the MMAs have read the stage
  uint64_t* acc_full = empty + STAGES;   // [2]: a K-segment's partial sums are ready in TMEM buffer b
  uint64_t* acc_empty = acc_full + 2;    // [2]: the epilogue has drained TMEM buffer b
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total = L.total_tiles;
  int* flags = L.g[0].ep.flags;
  pdl_launch_dependents();  // the next launch may take the SMs this one frees

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&conv[s], CONV_WARPS);
      mbar_init(&empty[s], 1);
    }
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane < 2 * L.ngroups) prefetch_tmap(&maps.m[lane]);
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_slot;
  // Everything above overlaps the previous kernel; every global access below
  // (operands, outputs, skip flags) waits for it to complete.
  pdl_wait_prerequisites();

  if (warp < EPI_WARP0) {
    // Warps 0-7 (two whole warpgroups) run the light roles; each warpgroup
    // executes this one setmaxnreg.
    warpgroup_regs_dec<LIGHT_REGS>();
    if (warp == 0) {
      if (lane == 0) {
        // ------------------------------------------------------------ producer
        uint32_t it = 0;  // chunks issued by this CTA (ring position)
        bool ok = true;
#pragma unroll 1
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
          const TileCoord tc = tile_coord(L, tile);
          if (tc.skip) continue;
          const GemmGroup& G = L.g[tc.gi];
          const int ck = chunk_k(G);
          const int nk = (G.k + ck - 1) / ck;
          const int planes = G.a_planes > 1 ? G.a_planes : 1;
          const uint32_t tx_bytes =  // 64 bytes a box row
              static_cast<uint32_t>(G.a_rows * planes + G.b_rows * (G.b_presplit ? 2 : 1)) * BK * 4u;
          const void* amap = &maps.m[G.a_map];
          const void* bmap = &maps.m[G.b_map];
          const int am = G.a_off + tc.mat;
          const int bm = G.b_off + tc.mat;
#pragma unroll 1
          for (int kc = 0; kc < nk; ++kc, ++it) {
            const int s = it % STAGES;
            if (it >= STAGES && !mbar_wait_bounded(&empty[s], ((it / STAGES) - 1) & 1, flags, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t* sa = smem + s * STAGE_BYTES;
            uint8_t* sb = sa + A_BYTES;
            mbar_arrive_expect_tx(&full[s], tx_bytes);
            tma_load_3d(sa, amap, &full[s], kc * ck, tc.tm * BM, am);
            // further bf16 planes of A land in the lo areas (A lo, then the first half of B lo)
            for (int q = 1; q < planes; ++q)
              tma_load_3d(sa + RAW_BYTES + (q - 1) * A_BYTES, amap, &full[s], kc * ck, tc.tm * BM,
                          am + q * G.a_plane_stride);
            if (G.b_mn) {
              // B[k][n] row-major: 16 K-rows x 32 N-columns per copy, one copy per
              // 32-column block of the tile, blocks MN_BLOCK bytes apart.
              const int nblk = G.b_rows / 32;
#pragma unroll 1
              for (int q = 0; q < nblk; ++q)
                tma_load_3d(sb + q * MN_BLOCK, bmap, &full[s], tc.tn * BN + q * 32, kc * BK, bm);
            } else {
              tma_load_3d(sb, bmap, &full[s], kc * ck, tc.tn * BN, bm);
              if (G.b_presplit)  // B's lo parts, split ahead of the launch, straight into the B lo area
                tma_load_3d(sb + RAW_BYTES, bmap, &full[s], kc * ck, tc.tn * BN, bm + G.b_plane_stride);
            }
          }
        }
        // Drain: no copy may still be landing in shared memory when the CTA
        // retires (bounded by time only; normally these phases completed).
#pragma unroll 1
        for (uint32_t k = (it > STAGES ? it - STAGES : 0); k < it; ++k)
          mbar_wait_bounded(&full[k % STAGES], (k / STAGES) & 1, flags, nullptr);
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        // K is cut into segments of SEG chunks.  Segment g (counted across
        // tiles) accumulates from zero into TMEM buffer g & 1; the epilogue warps
        // add each finished segment into fp32 registers with round-to-nearest.
        // The tensor core's own additions (which truncate) then only ever see
        // one segment's partial sums, which keeps long products unbiased.
        uint32_t it = 0, sg = 0;
        bool ok = true;
#pragma unroll 1
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
          const TileCoord tc = tile_coord(L, tile);
          if (tc.skip) continue;
          const GemmGroup& G = L.g[tc.gi];
          const int ck = chunk_k(G), sc = seg_chunks(G);
          const int nk = (G.k + ck - 1) / ck;
          const bool f16 = G.bf16 != 0;
          const uint32_t idesc = f16 ? idesc_bf16(BM, BN) : idesc_tf32(BM, BN, G.b_mn);
#pragma unroll 1
          for (int kc = 0; kc < nk; ++kc, ++it) {
            const int s = it % STAGES;
            const bool first = (kc % sc) == 0;
            const uint32_t b = sg & 1;
            const uint32_t tbuf = taddr + b * BN;
            if (first && sg >= 2 &&
                !mbar_wait_bounded(&acc_empty[b], ((sg >> 1) - 1) & 1, flags, abort_flag)) {
              ok = false;
              break;
            }
            if (!mbar_wait_bounded(&conv[s], (it / STAGES) & 1, flags, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_hi = smem_u32(smem + s * STAGE_BYTES);
            const uint32_t b_hi = a_hi + A_BYTES;
            const uint32_t a_lo = a_hi + RAW_BYTES;
            const uint32_t b_lo = b_hi + RAW_BYTES;
#pragma unroll
            for (int ks = 0; ks < BK / 8; ++ks) {
              const uint32_t off = ks * 32;  // 8 tf32 values = 32 bytes along K (K-major)
              const uint64_t dah = smem_desc_k_sw64(a_hi + off);
              const uint64_t dal = smem_desc_k_sw64(a_lo + off);
              uint64_t dbh, dbl;
              if (G.b_mn) {  // 8 K-rows = 1024 bytes = two 4-row groups
                dbh = smem_desc_mn_sw128_32b(b_hi + ks * 1024, MN_BLOCK);
                dbl = smem_desc_mn_sw128_32b(b_lo + ks * 1024, MN_BLOCK);
              } else {
                dbh = smem_desc_k_sw64(b_hi + off);
                dbl = smem_desc_k_sw64(b_lo + off);
              }
              if (f16) {
                mma_bf16(tbuf, dah, dbh, idesc, (first && ks == 0) ? 0u : 1u);
                if (G.a_planes > 1) {  // A = plane 0 + plane 1 + plane 2, each product exact in fp32
                  mma_bf16(tbuf, dal, dbh, idesc, 1u);
                  mma_bf16(tbuf, smem_desc_k_sw64(a_lo + A_BYTES + off), dbh, idesc, 1u);
                }
              } else {
                mma_tf32(tbuf, dah, dbh, idesc, (first && ks == 0) ? 0u : 1u);
                if (!G.b_exact) mma_tf32(tbuf, dah, dbl, idesc, 1u);
                if (!G.a_exact) mma_tf32(tbuf, dal, dbh, idesc, 1u);
              }
            }
            mma_commit(&empty[s]);
            if ((kc % sc) == sc - 1 || kc == nk - 1) {
              mma_commit(&acc_full[b]);
              ++sg;
            }
          }
        }
      }
    } else {
      // ------------------------------------------------------------ converters
      // Each landed stage (A and B tiles, 24 KB of fp32) is split in place: the
      // hi parts overwrite the fp32 values, the lo parts go RAW_BYTES further.
      // The split is elementwise, so the swizzled layout TMA wrote carries over.
      const int ct = threadIdx.x - 32 * CONV_WARP0;
      uint32_t it = 0;
      bool ok = true;
#pragma unroll 1
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileCoord tc = tile_coord(L, tile);
        if (tc.skip) continue;
        const GemmGroup& G = L.g[tc.gi];
        const int ck = chunk_k(G);
        const int nk = (G.k + ck - 1) / ck;
        // An operand whose values are exact in tf32 needs no split: its hi
        // part is the value as TMA wrote it, and its lo part is never read.
        // A presplit B arrives as its hi and lo parts (two TMA loads).
        const bool keep_a = G.a_exact != 0, keep_b = G.b_exact != 0 || G.b_presplit != 0;
#pragma unroll 1
        for (int kc = 0; kc < nk; ++kc, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait_warp(&full[s], (it / STAGES) & 1, flags, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* base = smem + s * STAGE_BYTES;
#pragma unroll
          for (int i = 0; i < RAW_BYTES / 16 / CONV_THREADS; ++i) {
            const int off = (i * CONV_THREADS + ct) * 16;
            if (off < A_BYTES ? keep_a : keep_b) continue;
            const float4 x = *reinterpret_cast<const float4*>(base + off);
            float4 h, l;
            split_tf32(x.x, h.x, l.x);
            split_tf32(x.y, h.y, l.y);
            split_tf32(x.z, h.z, l.z);
            split_tf32(x.w, h.w, l.w);
            *reinterpret_cast<float4*>(base + off) = h;
            *reinterpret_cast<float4*>(base + RAW_BYTES + off) = l;
          }
          // Each lane orders its stores before the tensor core's reads; the
          // warp then reports once.
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) mbar_arrive(&conv[s]);
        }
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // 8 warps: warp w reads TMEM lane quarter (w & 3) and column half h.
    warpgroup_regs_inc<HEAVY_REGS>();
    const int ew = warp - EPI_WARP0;
    const int q = warp & 3;
    const int h = ew >> 2;
    const uint32_t lane_addr = taddr + (static_cast<uint32_t>(q * 32) << 16) + h * (BN / 2);
    float* tilebuf = epi_tiles + ew * EPI_TILE_FLOATS;
    uint32_t sg = 0;
    bool ok = true;
#pragma unroll 1
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileCoord tc = tile_coord(L, tile);
      if (tc.skip) continue;
      const GemmGroup& G = L.g[tc.gi];
      const int n = G.n;
      const int m = G.m;
      const int ck = chunk_k(G), sc = seg_chunks(G);
      const int nseg = ((G.k + ck - 1) / ck + sc - 1) / sc;
      // C of this warp's first chunk streams into its shared tile while the
      // tile's MMAs run.
      const int row0_first = tc.tm * BM + q * 32;
      const int c0_first = tc.tn * BN + h * (BN / 2);
      const bool staged0 = (kF & F_C) && G.ep.C && row0_first < m && c0_first < n;
      if (staged0) stage_c(G.ep, m, n, tc.mat, row0_first, c0_first, tilebuf, lane);
      float sum[BN / 2];
#pragma unroll
      for (int j = 0; j < BN / 2; ++j) sum[j] = 0.f;
#pragma unroll 1
      for (int seg = 0; seg < nseg; ++seg, ++sg) {
        const uint32_t b = sg & 1;
        if (!mbar_wait_warp(&acc_full[b], (sg >> 1) & 1, flags, abort_flag)) {
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
      if (!ok) {
        cp_async_wait_all();  // no copy may still be landing when the CTA retires
        break;
      }
      float resid = 0.f;
      bool nonfinite = false;
      const int row0 = tc.tm * BM + q * 32;
      if (row0 < m) {
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) {
          const int c0 = tc.tn * BN + h * (BN / 2) + c * 32;
          if (c0 < n)
            epilogue_chunk<kF>(G, tc.mat, row0, c0, &sum[c * 32], tilebuf, lane, resid, nonfinite, c == 0 && staged0);
        }
      }
      if ((kF & F_E) && G.ep.res) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) resid += __shfl_xor_sync(0xffffffffu, resid, o);
        if (lane == 0 && resid != 0.f) atomicAdd(&G.ep.res[tc.mat], resid);
      }
      if (__any_sync(0xffffffffu, nonfinite) && lane == 0) raise_flag(G.ep.flags, DEV_FLAG_NONFINITE);
      if (L.profile && ew == 0 && lane == 0 && prof_flops)
        atomicAdd(&prof_flops[L.prof_slot], G.flops_per_matrix / G.tiles_per);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(taddr, TMEM_COLS);
  }
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

// Tensor map over a stack (batch, rows, cols) of row-major fp32 matrices:
// dimensions (innermost first) column = cols, row = rows, matrix = batch.
// K-major operand tiles (box box_rows x 16) use the 64-byte swizzle; MN-major
// tiles (mn_layout: 16 rows of K x 32 columns) the 128-byte swizzle with
// 32-byte atoms, the only MN-major tf32 layout of the tensor core.  Boxes that
// reach past rows or cols read zeros.
int encode_stack_map(CUtensorMap* map, const void* base, int64_t batch, int rows, int cols, int box_rows,
                     int mn_layout, int bf16) {
  int rc = get_encoder();
  if (rc) return rc;
  const int es = bf16 ? 2 : 4;  // element bytes
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return set_error(-2, "stack base not 16-byte aligned");
  if ((cols * es) % 16 != 0) return set_error(-2, "stack rows of %d elements are not 16-byte multiples", cols);
  const cuuint64_t nr = static_cast<cuuint64_t>(rows), nc = static_cast<cuuint64_t>(cols);
  cuuint64_t dims[3] = {nc, nr, static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {nc * es, nr * nc * es};
  // K-major boxes: 64 bytes of K (BK fp32 or 2 BK bf16 columns) x box_rows
  // rows; MN-major boxes (fp32 only): 32 columns (128 bytes) x box_rows (= BK)
  // rows of K.
  cuuint32_t box[3] = {static_cast<cuuint32_t>(mn_layout ? 32 : 64 / es), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        mn_layout ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(-4, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return 0;
}

int make_rect_maps(StackMaps& sm, const float* base, int64_t batch, int rows, int cols) {
  sm.base = const_cast<float*>(base);
  sm.rows = rows;
  sm.cols = cols;
  sm.a_rows = rows < BM ? rows : BM;
  sm.b_rows = rows < BN ? rows : BN;
  sm.bf16 = 0;
  int rc = encode_stack_map(&sm.a, base, batch, rows, cols, sm.a_rows, 0, 0);
  if (rc) return rc;
  if ((rc = encode_stack_map(&sm.mn, base, batch, rows, cols, BK, 1, 0))) return rc;
  return encode_stack_map(&sm.b, base, batch, rows, cols, sm.b_rows, 0, 0);
}

int make_stack_maps(StackMaps& sm, const float* base, int64_t batch, int n) {
  return make_rect_maps(sm, base, batch, n, n);
}

int make_stack_maps_bf16(StackMaps& sm, const void* base, int64_t batch, int n) {
  std::memset(&sm, 0, sizeof(sm));
  sm.base = nullptr;  // not an fp32 stack
  sm.rows = sm.cols = n;
  sm.a_rows = n < BM ? n : BM;
  sm.b_rows = n < BN ? n : BN;
  sm.bf16 = 1;
  int rc = encode_stack_map(&sm.a, base, batch, n, n, sm.a_rows, 0, 1);
  if (rc) return rc;
  return encode_stack_map(&sm.b, base, batch, n, n, sm.b_rows, 0, 1);
}

Builder::Builder() : nmaps(0) {
  std::memset(&L, 0, sizeof(L));
  std::memset(&M, 0, sizeof(M));
}

Epilogue& Builder::add(int batch, int n, const StackMaps& a, int a_off, const StackMaps& b, int b_off,
                       double flops_per_matrix, int bmode) {
  GemmGroup& g = L.g[L.ngroups++];
  g.batch = batch;
  g.n = n;
  g.m = n;
  g.k = n;
  M.m[nmaps] = a.a;
  g.a_map = nmaps++;
  M.m[nmaps] = bmode == B_MN_MAJOR ? b.mn : b.b;
  g.b_map = nmaps++;
  g.b_mn = bmode == B_MN_MAJOR ? 1 : 0;
  // bf16 stacks (both operands, K-major): kind::f16 MMAs; their values are
  // exact, so nothing is split
  g.bf16 = (a.bf16 && b.bf16 && bmode != B_MN_MAJOR) ? 1 : 0;
  if (g.bf16) g.a_exact = g.b_exact = 1;
  g.a_off = a_off;
  g.b_off = b_off;
  g.a_rows = a.a_rows;
  g.b_rows = b.b_rows;
  g.flops_per_matrix = flops_per_matrix;
  g.ep = epilogue_defaults();
  return g.ep;
}

Epilogue& Builder::add_rect(int batch, int Mr, int N, int K, const StackMaps& a, int a_off, const StackMaps& b,
                            int b_off, double flops_per_matrix, int bmode) {
  Epilogue& e = add(batch, N, a, a_off, b, b_off, flops_per_matrix, bmode);
  GemmGroup& g = L.g[L.ngroups - 1];
  g.m = Mr;
  g.k = K;
  g.a_rows = Mr < BM ? Mr : BM;
  g.b_rows = N < BN ? N : BN;
  return e;
}

// The kernel built for feature mask f (F_W | F_C | F_E).
const void* gemm_kernel(int f) {
  switch (f & 7) {
    case 0: return reinterpret_cast<const void*>(gemm3x_tf32_kernel<0>);
    case 1: return reinterpret_cast<const void*>(gemm3x_tf32_kernel<1>);
    case 2: return reinterpret_cast<const void*>(gemm3x_tf32_kernel<2>);
    case 3: return reinterpret_cast<const void*>(gemm3x_tf32_kernel<3>);
    case 4: return reinterpret_cast<const void*>(gemm3x_tf32_kernel<4>);
    case 5: return reinterpret_cast<const void*>(gemm3x_tf32_kernel<5>);
    case 6: return reinterpret_cast<const void*>(gemm3x_tf32_kernel<6>);
    default: return reinterpret_cast<const void*>(gemm3x_tf32_kernel<7>);
  }
}

int launch_gemm(GemmLaunch& L, const TmaMaps& maps, cudaStream_t st) {
  static unsigned attr_mask = 0;  // devices on which both kernels' attributes are set
  int dev = 0;
  int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
  if (rc) return rc;
  if (dev < 32 && !(attr_mask & (1u << dev))) {
    // The register hand-over inside the kernel (setmaxnreg) balances only if
    // the CTA is launched with exactly LAUNCH_REGS registers per thread; with
    // fewer, the epilogue warps' request could never be met.
    for (int f = 0; f < 8; ++f) {
      const void* k = gemm_kernel(f);
      cudaFuncAttributes fa;
      rc = check_cuda(cudaFuncGetAttributes(&fa, k), "cudaFuncGetAttributes(gemm)");
      if (rc) return rc;
      if (fa.numRegs != LAUNCH_REGS)
        return set_error(-2, "gemm3x_tf32_kernel was built with %d registers per thread; the register split "
                         "needs exactly %d", fa.numRegs, LAUNCH_REGS);
      rc = check_cuda(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES),
                      "cudaFuncSetAttribute(gemm)");
      if (rc) return rc;
    }
    attr_mask |= 1u << dev;
  }
  int features = 0;  // the epilogue features some group uses: the kernel built with those
  for (int i = 0; i < L.ngroups; ++i) {
    const Epilogue& e = L.g[i].ep;
    if (e.wptr) features |= F_W;
    if (e.C) features |= F_C;
    if (e.E || e.res) features |= F_E;
  }
  int64_t total = 0;
  double flops = 0;
  for (int i = 0; i < L.ngroups; ++i) {
    GemmGroup& g = L.g[i];
    g.tiles_m = (g.m + BM - 1) / BM;
    g.tiles_n = (g.n + BN - 1) / BN;
    if (g.sym && g.m != g.n) return set_error(-1, "a symmetric GEMM group must be square");
    // planes 1 and 2 of A land in the stage's lo areas, which only bf16 groups leave unused
    if (g.a_planes > 3 || (g.a_planes > 1 && (!g.bf16 || g.a_rows > BM)))
      return set_error(-1, "A in %d planes needs a bf16 group of at most 3 planes", g.a_planes);
    if (g.b_presplit && (g.bf16 || g.b_mn || g.b_exact || g.b_rows > BN))
      return set_error(-1, "a presplit B needs an fp32 K-major operand with lo parts");
    g.tiles_per = g.tiles_m * g.tiles_n;
    if (g.sym) {
      g.tiles_per = 0;
      for (int tn = 0; tn < g.tiles_n; ++tn) g.tiles_per += std::min(2 * tn + 2, g.tiles_m);
    }
    g.cta_begin = static_cast<int>(total);
    total += static_cast<int64_t>(g.batch) * g.tiles_per;
    flops += g.flops_per_matrix * g.batch;
  }
  if (total == 0) return 0;
  if (total > 0x7fffffff) return set_error(-2, "GEMM launch too large (%lld tiles)", (long long)total);
  static int sm_count[32] = {0};
  if (dev < 32 && sm_count[dev] == 0) {
    rc = check_cuda(cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev), "SM count");
    if (rc) return rc;
  }
  const int sms = (dev < 32 && sm_count[dev] > 0) ? sm_count[dev] : 148;
  L.total_tiles = static_cast<int>(total);
  L.profile = profiling_enabled() ? 1 : 0;
  L.prof_slot = K_GEMM;
  const unsigned grid = static_cast<unsigned>(total < sms ? total : sms);
  ProfScope ps(K_GEMM, st, flops, 0.0);
  // Programmatic stream serialization: the launch may begin (prologue only)
  // while the previous kernel finishes; the kernel waits for it before any
  // global access.
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[3] = {&L, const_cast<TmaMaps*>(&maps), nullptr};
  double* slots = device_flop_slots();
  args[2] = &slots;
  rc = check_cuda(cudaLaunchKernelExC(&cfg, gemm_kernel(features), args), "gemm3x_tf32_kernel launch");
  if (rc) return rc;
  count_launch();
  return check_cuda(cudaGetLastError(), "gemm3x_tf32_kernel launch");
}

}  // namespace shampoo
