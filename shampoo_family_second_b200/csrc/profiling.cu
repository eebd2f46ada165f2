// Process-wide launch counter and optional per-kernel event timing.
//
// When profiling is enabled every kernel launch of the library is bracketed by
// two CUDA events recorded on the stream it is launched on, and tallied per
// kernel kind together with its algorithmic flops and bytes.  The GEMM kernels
// (3xTF32 and fp64) add their executed algorithmic flops on the device (tiles
// of converged matrices that exit early add nothing), so achieved TFLOP/s stay
// exact when the residual-checked solvers skip work.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/shampoo.h"
#include "internal.h"

namespace shampoo {

__device__ double g_dev_flops[K_COUNT];

namespace {
std::atomic<uint64_t> g_launches{0};
std::atomic<bool> g_enabled{false};
std::mutex g_mu;
struct Rec {
  int kind;
  cudaEvent_t a, b;
  double flops, bytes;
};
std::vector<Rec> g_open;          // recorded, not yet collected
std::vector<cudaEvent_t> g_pool;  // idle events
int64_t g_count[K_COUNT];
double g_ms[K_COUNT], g_flops[K_COUNT], g_bytes[K_COUNT];
double* g_dev_ptr[64] = {nullptr};
thread_local std::string g_last_error;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

int set_error(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return 0;
  return set_error(SHAMPOO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

namespace {
thread_local int t_capturing = 0;  // > 0 while this thread records launches into a graph
}
CaptureScope::CaptureScope() { ++t_capturing; }
CaptureScope::~CaptureScope() { --t_capturing; }

void count_launch() {
  if (t_capturing == 0) g_launches.fetch_add(1, std::memory_order_relaxed);
}

namespace {
std::atomic<bool> g_graph_loops_used{false};
}
void note_graph_loop_launch() { g_graph_loops_used.store(true, std::memory_order_relaxed); }
bool profiling_enabled() { return g_enabled.load(std::memory_order_relaxed); }

double* device_flop_slots() {
  if (!profiling_enabled()) return nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!g_dev_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_flops) != cudaSuccess) return nullptr;
    g_dev_ptr[dev] = static_cast<double*>(p);
  }
  return g_dev_ptr[dev];
}

ProfScope::ProfScope(int k, cudaStream_t s, double f, double b)
    : kind(k), st(s), flops(f), bytes(b), active(0), ev(-1) {
  if (!profiling_enabled()) return;
  std::lock_guard<std::mutex> lk(g_mu);
  Rec r{k, take_event(), take_event(), f, b};
  cudaEventRecord(r.a, s);
  g_open.push_back(r);
  ev = static_cast<int>(g_open.size()) - 1;
  active = 1;
}

ProfScope::~ProfScope() {
  if (!active) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (ev >= 0 && ev < static_cast<int>(g_open.size())) cudaEventRecord(g_open[ev].b, st);
}

}  // namespace shampoo

using namespace shampoo;

extern "C" {

const char* shampoo_last_error(void) { return g_last_error.c_str(); }

uint64_t shampoo_launch_count(void) {
  // Host-issued launches, plus the kernels graph loops ran on the device
  // (counted there; reading them waits for the device).
  return g_launches.load() + (g_graph_loops_used.load() ? graph_kernel_count() : 0);
}

void shampoo_profile_enable(int32_t on) { g_enabled.store(on != 0); }

void shampoo_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  for (Rec& r : g_open) {
    cudaEventSynchronize(r.b);
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_open.clear();
  for (int k = 0; k < K_COUNT; ++k) g_count[k] = 0, g_ms[k] = g_flops[k] = g_bytes[k] = 0.0;
  double zeros[K_COUNT] = {0};
  cudaMemcpyToSymbol(g_dev_flops, zeros, sizeof(zeros));
}

int shampoo_profile_read(int32_t kind, int64_t* launches, double* total_ms, double* alg_flops, double* alg_bytes) {
  if (kind < 0 || kind >= K_COUNT) return set_error(SHAMPOO_ERR_INVALID_ARG, "profile kind %d out of range", kind);
  std::lock_guard<std::mutex> lk(g_mu);
  for (Rec& r : g_open) {
    cudaError_t e = cudaEventSynchronize(r.b);
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess) return check_cuda(e, "profile event");
    g_count[r.kind] += 1;
    g_ms[r.kind] += ms;
    g_flops[r.kind] += r.flops;
    g_bytes[r.kind] += r.bytes;
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_open.clear();
  double dev[K_COUNT] = {0};
  cudaError_t e = cudaMemcpyFromSymbol(dev, g_dev_flops, sizeof(dev));
  if (e != cudaSuccess) return check_cuda(e, "profile flops");
  if (launches) *launches = g_count[kind];
  if (total_ms) *total_ms = g_ms[kind];
  if (alg_flops) *alg_flops = (kind == K_GEMM || kind == K_GEMM_F64) ? dev[kind] : g_flops[kind];
  if (alg_bytes) *alg_bytes = g_bytes[kind];
  return SHAMPOO_OK;
}

}  // extern "C"
