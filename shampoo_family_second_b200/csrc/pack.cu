// Block packing for blocks sharded across ranks (DASH abstract: the
// preconditioner blocks are distributed across devices).  One launch moves a
// whole list of r x c blocks between row-strided matrices (weights or
// gradients) and one packed fp32 buffer in which the blocks lie back to back,
// each row-major: the buffer a rank's collectives (reduce-scatter of the
// gradients by block owner, all-gather of the updated blocks) send and receive.
#include "../../include/shampoo.h"
#include "common.cuh"
#include "internal.h"

using namespace shampoo;

namespace {

struct PackArgs {
  void* p[kMaxParams];
  int64_t ld[kMaxParams];
};

// grid (ceil(max_cols / 128), ceil(max_rows / 8), nblocks), block (32, 8):
// each thread moves 4 consecutive elements of one row of one block.
__global__ void pack_blocks_kernel(const __grid_constant__ PackArgs a, const int64_t* __restrict__ table, int dtype,
                                   float* __restrict__ packed, int direction, float scale) {
  const int b = blockIdx.z;
  const int64_t* t = table + 6 * static_cast<int64_t>(b);
  const int param = static_cast<int>(t[0]);
  const int64_t row0 = t[1], col0 = t[2];
  const int r = static_cast<int>(t[3]), c = static_cast<int>(t[4]);
  const int64_t off = t[5];
  const int row = blockIdx.y * 8 + threadIdx.y;
  const int col = blockIdx.x * 128 + 4 * threadIdx.x;
  if (row >= r || col >= c) return;
  const int64_t ld = a.ld[param];
  float* dst_row = packed + off + static_cast<int64_t>(row) * c;
  const int64_t src = (row0 + row) * ld + col0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int j = col + q;
    if (j >= c) break;
    if (direction == 0) {
      float v;
      if (dtype == SHAMPOO_BF16) {
        const uint16_t bits = reinterpret_cast<const uint16_t*>(a.p[param])[src + j];
        v = __uint_as_float(static_cast<uint32_t>(bits) << 16);
      } else {
        v = reinterpret_cast<const float*>(a.p[param])[src + j];
      }
      dst_row[j] = scale * v;
    } else {
      reinterpret_cast<float*>(a.p[param])[src + j] = dst_row[j];
    }
  }
}

}  // namespace

extern "C" {

int shampoo_pack_blocks(const int64_t* d_table, int32_t nblocks, int32_t nparams, void* const* d_params,
                        const int64_t* ld, int32_t dtype, float* d_packed, int32_t direction, float scale,
                        int32_t max_rows, int32_t max_cols, void* stream) {
  if (nblocks < 0 || nblocks > 65535) return set_error(SHAMPOO_ERR_INVALID_ARG, "nblocks %d out of range", nblocks);
  if (nblocks == 0) return SHAMPOO_OK;
  if (nparams < 1 || nparams > kMaxParams) return set_error(SHAMPOO_ERR_INVALID_ARG, "nparams %d out of range", nparams);
  if (!d_table || !d_params || !ld || !d_packed) return set_error(SHAMPOO_ERR_INVALID_ARG, "NULL pointer");
  if (direction != 0 && direction != 1) return set_error(SHAMPOO_ERR_INVALID_ARG, "direction must be 0 or 1");
  if (dtype != SHAMPOO_F32 && dtype != SHAMPOO_BF16) return set_error(SHAMPOO_ERR_INVALID_ARG, "bad dtype");
  if (dtype == SHAMPOO_BF16 && direction == 1)
    return set_error(SHAMPOO_ERR_UNSUPPORTED, "scatter writes fp32 matrices only");
  if (max_rows < 1 || max_cols < 1) return set_error(SHAMPOO_ERR_INVALID_ARG, "max_rows / max_cols must be >= 1");
  PackArgs a;
  for (int i = 0; i < nparams; ++i) {
    if (!d_params[i]) return set_error(SHAMPOO_ERR_INVALID_ARG, "param %d is NULL", i);
    if (ld[i] < 1) return set_error(SHAMPOO_ERR_INVALID_ARG, "param %d has row stride %lld", i, (long long)ld[i]);
    a.p[i] = d_params[i];
    a.ld[i] = ld[i];
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 grid((max_cols + 127) / 128, (max_rows + 7) / 8, nblocks), block(32, 8);
  ProfScope ps(K_STACK, st, 0.0, 0.0);
  pack_blocks_kernel<<<grid, block, 0, st>>>(a, d_table, dtype, d_packed, direction, scale);
  count_launch();
  return check_cuda(cudaGetLastError(), "pack_blocks_kernel");
}

}  // extern "C"
