// static_workspace.cu -- hyena_forward for callers that cannot allocate.
//
// Some callers of this library may not allocate device memory at run time:
// runtimes that have handed the whole device to their own pool allocator and
// forbid allocations behind its back, fixed-budget deployments, and
// latency-critical paths that cannot afford cudaMalloc's implicit device
// synchronisation. For them the long-sequence (four-step) forward runs with
// a scratch buffer that lives in this library's own module memory: a
// file-scope device array of HYENA_STATIC_WORKSPACE_BYTES, reserved on every
// GPU that loads the library and held until the process exits.
//
// The array's name in host code is only a host-side stand-in for the device
// symbol, never a device address; the device address is obtained with
// cudaGetSymbolAddress, once per device, on the first call made while that
// device is current.
#include <atomic>
#include <mutex>

#include "hyena.h"
#include "kernels.cuh"

using namespace hyena;

namespace {

constexpr size_t kStaticBytes = HYENA_STATIC_WORKSPACE_BYTES;
static_assert(kStaticBytes % 256 == 0, "static workspace size");

// Scratch shared by every call on a device. Holds whatever the last call left
// there; the four-step passes write every element they later read, so nothing
// has to be cleared between calls.
static __device__ __align__(256) unsigned char g_static_workspace[kStaticBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_addr[kMaxDevices];
std::mutex g_addr_mu;

// Device address of g_static_workspace on the current device (set up once per device).
cudaError_t static_workspace_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = g_addr[dev].load(std::memory_order_acquire);
  if (p) {
    *out = p;
    return cudaSuccess;
  }
  std::lock_guard<std::mutex> lk(g_addr_mu);
  p = g_addr[dev].load(std::memory_order_relaxed);
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return e;
    g_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" hyena_status hyena_forward_static_workspace(const void* v, const void* const* x, const void* const* hhat,
                                                       int B, int D, int L, int N, hyena_dtype dtype, void* y,
                                                       hyena_stream stream) {
  Layout ly;
  if (!make_layout(L, &ly)) return HYENA_ERR_UNSUPPORTED;
  // Lengths that fit the fused kernel need no scratch at all: hyena_forward
  // with a NULL workspace already allocates nothing there.
  if (!ly.fourstep) return HYENA_ERR_UNSUPPORTED;
  // one channel of the four-step array must fit in the static scratch
  if (sizeof(float2) * (size_t)ly.M > kStaticBytes) return HYENA_ERR_WORKSPACE;
  if (N < 1 || N > kMaxOrder || B < 1 || D < 1 || !x || !hhat) return HYENA_ERR_INVALID_ARG;
  void* ws = nullptr;
  cudaError_t e = static_workspace_address(&ws);
  if (e != cudaSuccess) return report_cuda_error(e);
  return hyena_forward(v, x, hhat, B, D, L, N, dtype, y, ws, kStaticBytes, stream);
}
