// static_workspace.cu -- hyena_forward for callers that cannot allocate.
//
// Some callers of this library may not allocate device memory at run time:
// runtimes that have handed the whole device to their own pool allocator and
// forbid allocations behind its back, fixed-budget deployments, and
// latency-critical paths that cannot afford cudaMalloc's implicit device
// synchronisation. For them the long-sequence (four-step) forward runs with
// a scratch buffer that lives in this library's own module memory: a
// file-scope device array of HYENA_STATIC_WORKSPACE_BYTES, held by every
// context that has loaded this file's module until the process exits (with
// lazy module loading, the module is loaded by the first call of this entry
// point in a context).
//
// The array's name in host code is only a host-side stand-in for the device
// symbol, never a device address; the device address is obtained with
// cudaGetSymbolAddress with the device current. The address belongs to one
// CUDA context: it is looked up once per (device, context) -- keyed by the
// context's unique id, so a context that is destroyed and re-created
// (cudaDeviceReset, or a caller switching to another context) gets a fresh
// lookup instead of a stale address.
#include <cuda.h>

#include <mutex>

#include "hyena.h"
#include "kernels.cuh"

using namespace hyena;

namespace {

constexpr size_t kStaticBytes = HYENA_STATIC_WORKSPACE_BYTES;
static_assert(kStaticBytes % 256 == 0, "static workspace size");

// Scratch shared by every call in a context. Holds whatever the last call left
// there; the four-step passes write every element they later read, so nothing
// has to be cleared between calls.
static __device__ __align__(256) unsigned char g_static_workspace[kStaticBytes];

constexpr int kMaxDevices = 64;
struct AddrEntry {
  unsigned long long ctx_id;   // 0: none cached
  void* addr;
};
AddrEntry g_addr[kMaxDevices];
std::mutex g_addr_mu;

typedef CUresult (*GetCurrentFn)(CUcontext*);
typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);

// Unique id of the current context (driver entry points fetched through the
// runtime, so the library needs no link against the driver library). Returns
// false when the id cannot be read.
bool current_context_id(unsigned long long* id) {
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(f);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_static_workspace in the current context.
cudaError_t static_workspace_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  unsigned long long id = 0;
  if (!current_context_id(&id)) {
    // No context is current yet on this thread: the lookup itself makes the
    // runtime's context current. Cache its result under that context's id
    // when the id can be read; otherwise the next call looks it up again.
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return e;
    *out = p;
    if (current_context_id(&id)) {
      std::lock_guard<std::mutex> lk(g_addr_mu);
      g_addr[dev].ctx_id = id;
      g_addr[dev].addr = p;
    }
    return cudaSuccess;
  }
  std::lock_guard<std::mutex> lk(g_addr_mu);
  if (g_addr[dev].ctx_id != id || g_addr[dev].addr == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return e;
    g_addr[dev].ctx_id = id;
    g_addr[dev].addr = p;
  }
  *out = g_addr[dev].addr;
  return cudaSuccess;
}

bool aligned16(const void* p) { return p && ((reinterpret_cast<uintptr_t>(p) & 15u) == 0); }

}  // namespace

extern "C" hyena_status hyena_forward_static_workspace(const void* v, const void* const* x, const void* const* hhat,
                                                       int B, int D, int L, int N, hyena_dtype dtype, void* y,
                                                       hyena_stream stream) {
  // Every host-side check of hyena_forward runs before the address lookup, so
  // a rejected call touches no module state and loads nothing.
  if (N < 1 || N > kMaxOrder || B < 1 || D < 1) return HYENA_ERR_INVALID_ARG;
  if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
  if (!x || !hhat || !aligned16(v) || !aligned16(y)) return HYENA_ERR_INVALID_ARG;
  for (int n = 0; n < N; ++n)
    if (!aligned16(x[n]) || !aligned16(hhat[n])) return HYENA_ERR_INVALID_ARG;
  if ((long long)B * D > (1LL << 40) / (L > 0 ? L : 1)) return HYENA_ERR_INVALID_ARG;
  Layout ly;
  if (!make_layout(L, &ly)) return HYENA_ERR_UNSUPPORTED;
  // Lengths that fit the fused kernel need no scratch at all: hyena_forward
  // with a NULL workspace already allocates nothing there.
  if (!ly.fourstep) return HYENA_ERR_UNSUPPORTED;
  // one channel of the four-step array must fit in the static scratch
  if (sizeof(float2) * (size_t)ly.M > kStaticBytes) return HYENA_ERR_WORKSPACE;
  void* ws = nullptr;
  cudaError_t e = static_workspace_address(&ws);
  if (e != cudaSuccess) return report_cuda_error(e);
  return hyena_forward(v, x, hhat, B, D, L, N, dtype, y, ws, kStaticBytes, stream);
}
