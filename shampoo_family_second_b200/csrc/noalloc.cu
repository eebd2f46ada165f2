// inv_root_batched_noalloc: the batched inverse-root solver with its scratch in
// a fixed device array owned by this library, for callers that cannot
// allocate device memory.
//
// Who needs it: code that runs where allocation is not allowed or not
// possible, such as inside a region that a framework's memory pool forbids to
// allocate from, a real-time loop that must not call cudaMalloc (it can
// synchronise the device and take unbounded time), or an embedding that owns
// no allocator at all.  Such callers still own their inputs and outputs; only
// the solver's working space comes from here.
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes.  Every
// GPU that loads this library holds that much memory until the process exits.
// Host code cannot use the array's name as a device address, so the first call
// on each device (with that device current) fetches the address with
// cudaGetSymbolAddress; that first call should come before any stream capture.
// All calls share the one array and it keeps the last call's contents: the
// solver clears what it needs zeroed (its residual accumulators) on every call,
// and calls whose work overlaps on the GPU (different streams, or different
// host threads on the same device) race on it.  With tol > 0 the iterations
// run as plain kernel launches up to the cap (the tiles of matrices that have
// finished exit at once) rather than as a CUDA graph loop, because
// instantiating a graph may take device memory.
#include <mutex>

#include "../../include/shampoo.h"
#include "internal.h"

using namespace shampoo;

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};

// Device address of g_noalloc_scratch on the current device (set up once).
int noalloc_scratch(void** out) {
  int dev = 0;
  int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
  if (rc) return rc;
  if (dev < 0 || dev >= 64) return set_error(SHAMPOO_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    rc = check_cuda(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(no-alloc scratch)");
    if (rc) return rc;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SHAMPOO_OK;
}

}  // namespace

extern "C" {

int inv_root_batched_noalloc(const float* d_A, float* d_X, int64_t batch, int32_t n, int32_t p, float eps,
                             int32_t solver, int32_t iters, float tol, int32_t cheb_degree, float cheb_lo,
                             int32_t* d_iters_used, int32_t* d_status, void* stream) {
  if (batch == 0) return SHAMPOO_OK;
  size_t per_matrix = 0;
  int rc = inv_root_scratch_bytes_p(1, n, solver, p, &per_matrix);
  if (rc) return rc;
  if (per_matrix > kNoAllocScratchBytes)
    return set_error(SHAMPOO_ERR_UNSUPPORTED,
                     "inv_root_batched_noalloc: n = %d with solver %d needs %zu bytes of scratch for one matrix; "
                     "the fixed scratch holds %zu bytes (use inv_root_batched with caller-owned scratch)",
                     n, solver, per_matrix, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch))) return rc;
  // The solver works through the batch in chunks that fit the fixed scratch.
  // Residual-checked loops are issued as plain launches: a CUDA graph loop
  // would instantiate a graph, which the runtime may back with device memory.
  return inv_root_batched_impl(d_A, d_X, batch, n, p, eps, solver, iters, tol, cheb_degree, cheb_lo, scratch,
                               kNoAllocScratchBytes, d_iters_used, d_status, static_cast<cudaStream_t>(stream),
                               true);
}

}  // extern "C"
