// api.cu -- C ABI: argument checks, layout, dispatch to the kernels.
#include <mutex>
#include <unordered_map>

#include "hyena.h"
#include "kernels.cuh"

using namespace hyena;

namespace {

thread_local char g_last_cuda_error[256] = "";

hyena_status cuda_fail(cudaError_t e) {
  const char* s = cudaGetErrorString(e);
  size_t i = 0;
  for (; s && s[i] && i + 1 < sizeof(g_last_cuda_error); ++i) g_last_cuda_error[i] = s[i];
  g_last_cuda_error[i] = 0;
  return HYENA_ERR_CUDA;
}

bool aligned16(const void* p) { return p && ((reinterpret_cast<uintptr_t>(p) & 15u) == 0); }

// Four-step channels run in waves through the workspace. The workspace size
// hyena_forward_workspace_bytes asks for depends on the row kernel:
// - rows of 4096 on the tensor cores: a wave whose scratch stays resident in
//   L2 between its passes, 5/8 of the device's L2 (order 2, bf16, D = 256:
//   6.27 / 3.04 ms per forward at L = 2^20 / 2^19 against 6.73 / 3.26 ms at
//   3/4 of L2; at these sizes the wave also cuts DRAM traffic from 89 to
//   56 MB per channel at L = 2^20);
// - the SIMT row kernels, bound by latency rather than DRAM: one wave of up
//   to kWaveMaxBytes, i.e. fewer launches and fewer partly filled last rounds
//   (L = 2^17, bf16: 0.601 against 0.665 ms per forward at 3/4 of L2; L = 2^20,
//   f32: 6.97 against 7.71 ms);
// - the backward's forward transforms: 3/4 of the L2 (as measured for it).
constexpr size_t kWaveL2Num = 6, kWaveL2Den = 8;
constexpr size_t kWaveTcrL2Num = 5, kWaveTcrL2Den = 8;
constexpr size_t kWaveMaxBytes = size_t(1) << 30;
constexpr size_t kWaveFallbackL2 = size_t(126) << 20;
constexpr long long kMaxGridY = 65535;

struct GridKey {
  const void* k;
  int dev;
  int threads;
  size_t smem;
  bool operator==(const GridKey& o) const { return k == o.k && dev == o.dev && threads == o.threads && smem == o.smem; }
};
struct GridKeyHash {
  size_t operator()(const GridKey& g) const {
    return std::hash<const void*>()(g.k) ^ (size_t(g.dev) << 48) ^ (size_t(g.threads) << 32) ^ g.smem;
  }
};
std::mutex g_grid_mu;
std::unordered_map<GridKey, int, GridKeyHash> g_grid_cache;

}  // namespace

hyena_status hyena::report_cuda_error(cudaError_t e) { return cuda_fail(e); }

cudaError_t hyena::persistent_grid(const void* kernel, int threads, size_t smem, int* grid) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  GridKey key{kernel, dev, threads, smem};
  {
    std::lock_guard<std::mutex> lk(g_grid_mu);
    auto it = g_grid_cache.find(key);
    if (it != g_grid_cache.end()) {
      *grid = it->second;
      return cudaSuccess;
    }
  }
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // opt in whenever dynamic shared memory is used: static + dynamic may pass 48 KB
  if (smem > 0) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  *grid = sms * per_sm;
  std::lock_guard<std::mutex> lk(g_grid_mu);
  g_grid_cache[key] = *grid;
  return cudaSuccess;
}

cudaError_t hyena::forward_dispatch(const void* v, const void* const* x, const void* const* hhat, int B, int D,
                                    const Layout& ly, int N, bool bf16, void* y, void* workspace,
                                    size_t workspace_bytes, bool allow_tc, cudaStream_t s, bool spec16) {
  const float2* tables =
      spec16 ? reinterpret_cast<const float2*>(reinterpret_cast<const char*>(hhat[0]) + spec16_tables_offset_bytes(ly, D))
             : reinterpret_cast<const float2*>(hhat[0]) + tables_offset(ly, D);
  if (spec16) allow_tc = false;   // the tensor-core kernels read their own float32 copy
  cudaError_t e = cudaSuccess;
  if (!ly.fourstep) {
    FusedLaunch p{};
    p.v = v;
    for (int n = 0; n < N; ++n) {
      p.x[n] = x[n];
      p.hh.p[n] = reinterpret_cast<const float2*>(hhat[n]);
    }
    p.y = y;
    p.tables = tables;
    p.B = B; p.D = D; p.L = ly.L; p.N = N;
    p.bf16 = bf16;
    p.spec16 = spec16;
    if (allow_tc && p.bf16 && (B % 2) == 0 && (ly.tc || (ly.tcg && N <= kTcgMaxOrder))) {
      // tensor-core kernel on pairs of batch items, reading the tensor-core copy of the spectra
      for (int n = 0; n < N; ++n)
        p.hh.p[n] = reinterpret_cast<const float2*>(hhat[n]) + tc_spectrum_offset(ly, D);
      e = ly.tcg ? launch_tcg_forward(p, s) : launch_tc_forward(p, ly, s);
    } else {
      e = launch_fused_forward(p, ly.logMV, s);
    }
  } else {
    const size_t per = sizeof(float2) * (size_t)ly.M;
    const long long C = (long long)B * D;
    // tensor-core rows when the workspace also holds the per-channel maxima
    bool tcr = allow_tc && bf16 && !spec16 && N <= kTcgMaxOrder && tcr_layout(ly) &&
               workspace_bytes >= per + kTcrChannelExtraBytes;
    long long w = (long long)(workspace_bytes / (tcr ? per + kTcrChannelExtraBytes : per));
    if (w < 1) return cudaErrorInvalidValue;
    if (w > C) w = C;
    if (w > kMaxGridY) w = kMaxGridY;
    FourStepLaunch p{};
    p.tcr = tcr;
    if (tcr) {
      p.xmax = reinterpret_cast<unsigned*>(reinterpret_cast<char*>(workspace) + per * (size_t)w);
      for (int n = 0; n < N; ++n) {
        p.hmax[n] = reinterpret_cast<const float*>(reinterpret_cast<const float2*>(hhat[n]) + hmax_offset(ly, D));
        p.hhalf[n] = reinterpret_cast<const uint32_t*>(reinterpret_cast<const float2*>(hhat[n]) + tcr_half_offset(ly, D));
      }
    }
    p.v = v;
    for (int n = 0; n < N; ++n) {
      p.x[n] = x[n];
      p.hh.p[n] = reinterpret_cast<const float2*>(hhat[n]);
    }
    p.y = y;
    p.tables = tables;
    p.scratch = reinterpret_cast<float2*>(workspace);
    p.B = B; p.D = D; p.L = ly.L; p.N = N;
    p.bf16 = bf16;
    p.spec16 = spec16;
    for (long long c0 = 0; c0 < C && e == cudaSuccess; c0 += w) {
      p.ch0 = c0;
      p.wave = (int)((C - c0) < w ? (C - c0) : w);
      if (tcr) e = cudaMemsetAsync(p.xmax, 0, sizeof(unsigned) * 2 * (size_t)p.wave, s);
      if (e == cudaSuccess) e = launch_fourstep_wave(p, ly, s);
    }
  }
  return e;
}

// L2 capacity of the current device (read once per device)
static size_t device_l2_bytes() {
  static std::mutex mu;
  static std::unordered_map<int, size_t> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return kWaveFallbackL2;
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  int l2 = 0;
  size_t v = kWaveFallbackL2;
  if (cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) == cudaSuccess && l2 > 0) v = (size_t)l2;
  cache[dev] = v;
  return v;
}

size_t hyena::fourstep_wave_bytes(long long channels, const Layout& ly, WaveRule rule) {
  const size_t per = sizeof(float2) * (size_t)ly.M;
  const size_t budget = rule == WaveRule::kTensorRows ? device_l2_bytes() * kWaveTcrL2Num / kWaveTcrL2Den
                        : rule == WaveRule::kSimtRows ? kWaveMaxBytes
                                                      : device_l2_bytes() * kWaveL2Num / kWaveL2Den;
  long long w = (long long)(budget / (per + (tcr_layout(ly) ? kTcrChannelExtraBytes : 0)));
  if (w < 1) w = 1;
  if (w > channels) w = channels;
  if (w > kMaxGridY) w = kMaxGridY;
  return (per + (tcr_layout(ly) ? kTcrChannelExtraBytes : 0)) * (size_t)w;
}

cudaError_t hyena::spectrum_dispatch(const float* h, float2* spec, int rows, const Layout& ly, bool with_tc,
                                     cudaStream_t s) {
  float2* tables = spec + tables_offset(ly, rows);
  cudaError_t e = launch_fill_tables(tables, ly, s);
  if (e != cudaSuccess) return e;
  if (!ly.fourstep) {
    e = launch_fused_spectrum(h, spec, tables, rows, ly.L, ly.logMV, s);
    if (e == cudaSuccess && with_tc && ly.tc)
      e = launch_tc_spectrum(spec, spec + tc_spectrum_offset(ly, rows), tables, rows, ly, s);
    if (e == cudaSuccess && with_tc && ly.tcg)
      e = launch_tcg_spectrum(spec, spec + tc_spectrum_offset(ly, rows), rows, s);
  } else {
    for (long long c0 = 0; c0 < rows && e == cudaSuccess; c0 += kMaxGridY) {
      const int nd = (int)((rows - c0) < kMaxGridY ? (rows - c0) : kMaxGridY);
      e = launch_fourstep_spectrum(h + (size_t)c0 * ly.L, spec + (size_t)c0 * ly.M, tables, nd, ly, s);
    }
    if (e == cudaSuccess && tcr_layout(ly))
      e = launch_tcr_hmax(spec, rows, ly.M, reinterpret_cast<float*>(spec + hmax_offset(ly, rows)), s);
    if (e == cudaSuccess && with_tc && tcr_layout(ly))
      e = launch_tcr_half(spec, reinterpret_cast<const float*>(spec + hmax_offset(ly, rows)), rows, ly.M,
                          reinterpret_cast<uint32_t*>(spec + tcr_half_offset(ly, rows)), s);
  }
  return e;
}

extern "C" {

int hyena_abi_version(void) { return HYENA_ABI_VERSION; }

const char* hyena_status_string(hyena_status s) {
  switch (s) {
    case HYENA_OK: return "ok";
    case HYENA_ERR_INVALID_ARG: return "invalid argument";
    case HYENA_ERR_UNSUPPORTED: return "unsupported length (L must be a power of two in [16, 2^20])";
    case HYENA_ERR_WORKSPACE: return "workspace missing or too small";
    case HYENA_ERR_CUDA: return "CUDA error";
    case HYENA_ERR_TIMEOUT: return "a bounded device wait ran out (results of the affected call are invalid)";
  }
  return "unknown status";
}

const char* hyena_last_cuda_error(void) { return g_last_cuda_error; }

hyena_status hyena_device_timeouts(void) {
  const int b = striped_read_and_clear_timeout();
  if (b < 0) return cuda_fail(cudaGetLastError());
  const int g = tcg_read_and_clear_timeout();
  if (g < 0) return cuda_fail(cudaGetLastError());
  const int f = fourstep_read_and_clear_timeout();
  if (f < 0) return cuda_fail(cudaGetLastError());
  const int r = tcr_read_and_clear_timeout();
  if (r < 0) return cuda_fail(cudaGetLastError());
  return (b || g || f || r) ? HYENA_ERR_TIMEOUT : HYENA_OK;
}

hyena_status hyena_spectrum_layout(int L, int* M, int* M1, int* MV) {
  Layout y;
  if (!make_layout(L, &y)) return HYENA_ERR_UNSUPPORTED;
  if (M) *M = y.M;
  if (M1) *M1 = y.M1;
  if (MV) *MV = y.MV;
  return HYENA_OK;
}

size_t hyena_filter_spectrum_bytes(int D, int L) {
  Layout y;
  if (D < 1 || !make_layout(L, &y)) return 0;
  return sizeof(float2) * spectrum_block_floats2(y, D);
}

hyena_status hyena_filter_generate(const hyena_filter_params* p, int N, int D, int L, float alpha_lo,
                                   float alpha_hi, float* h, hyena_stream stream) {
  if (!p || !h || N < 1 || N > kMaxOrder || D < 1) return HYENA_ERR_INVALID_ARG;
  if (!p->W1 || !p->b1 || !p->W2 || !p->b2 || !p->W3 || !p->b3) return HYENA_ERR_INVALID_ARG;
  if (p->n_bands < 1 || p->n_bands > 32 || p->width < 1 || p->width > 128) return HYENA_ERR_INVALID_ARG;
  if (!aligned16(h)) return HYENA_ERR_INVALID_ARG;
  if ((long long)N * D > (1LL << 30)) return HYENA_ERR_INVALID_ARG;
  Layout y;
  if (!make_layout(L, &y)) return HYENA_ERR_UNSUPPORTED;
  cudaError_t e = launch_filter_generate(p->W1, p->b1, p->W2, p->b2, p->W3, p->b3, p->n_bands, p->width, N, D, L,
                                         alpha_lo, alpha_hi, h, (cudaStream_t)stream);
  return e == cudaSuccess ? HYENA_OK : cuda_fail(e);
}

hyena_status hyena_filter_rfft(const float* h, int D, int L, void* hhat, hyena_stream stream) {
  if (!aligned16(h) || !aligned16(hhat) || D < 1) return HYENA_ERR_INVALID_ARG;
  Layout y;
  if (!make_layout(L, &y)) return HYENA_ERR_UNSUPPORTED;
  const cudaError_t e = spectrum_dispatch(h, reinterpret_cast<float2*>(hhat), D, y, true, (cudaStream_t)stream);
  return e == cudaSuccess ? HYENA_OK : cuda_fail(e);
}

size_t hyena_forward_workspace_bytes(int B, int D, int L, int N, hyena_dtype dtype) {
  Layout y;
  if (B < 1 || D < 1 || N < 1 || N > kMaxOrder || (dtype != HYENA_F32 && dtype != HYENA_BF16)) return 0;
  if (!make_layout(L, &y)) return 0;
  if (!y.fourstep) return 0;
  const bool tensor_rows = dtype == HYENA_BF16 && N <= kTcgMaxOrder && tcr_layout(y);
  return fourstep_wave_bytes((long long)B * D, y, tensor_rows ? WaveRule::kTensorRows : WaveRule::kSimtRows);
}

hyena_status hyena_forward(const void* v, const void* const* x, const void* const* hhat, int B, int D, int L,
                           int N, hyena_dtype dtype, void* y, void* workspace, size_t workspace_bytes,
                           hyena_stream stream) {
  if (N < 1 || N > kMaxOrder || B < 1 || D < 1) return HYENA_ERR_INVALID_ARG;
  if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
  if (!x || !hhat || !aligned16(v) || !aligned16(y)) return HYENA_ERR_INVALID_ARG;
  for (int n = 0; n < N; ++n)
    if (!aligned16(x[n]) || !aligned16(hhat[n])) return HYENA_ERR_INVALID_ARG;
  if ((long long)B * D > (1LL << 40) / (L > 0 ? L : 1)) return HYENA_ERR_INVALID_ARG;
  Layout ly;
  if (!make_layout(L, &ly)) return HYENA_ERR_UNSUPPORTED;
  if (ly.fourstep && (!aligned16(workspace) || workspace_bytes < sizeof(float2) * (size_t)ly.M))
    return HYENA_ERR_WORKSPACE;
  const cudaError_t e = forward_dispatch(v, x, hhat, B, D, ly, N, dtype == HYENA_BF16, y, workspace,
                                         workspace_bytes, true, (cudaStream_t)stream);
  return e == cudaSuccess ? HYENA_OK : cuda_fail(e);
}

size_t hyena_filter_spectrum_bytes_f16(int D, int L) {
  Layout y;
  if (D < 1 || !make_layout(L, &y)) return 0;
  return spec16_block_bytes(y, D);
}

hyena_status hyena_filter_spectrum_to_f16(const void* hhat, int D, int L, void* hhat16, hyena_stream stream) {
  if (!aligned16(hhat) || !aligned16(hhat16) || D < 1) return HYENA_ERR_INVALID_ARG;
  Layout y;
  if (!make_layout(L, &y)) return HYENA_ERR_UNSUPPORTED;
  const cudaError_t e = launch_spectrum_to_f16(reinterpret_cast<const float2*>(hhat),
                                               reinterpret_cast<unsigned char*>(hhat16), D, y, (cudaStream_t)stream);
  return e == cudaSuccess ? HYENA_OK : cuda_fail(e);
}

hyena_status hyena_forward_f16_spectra(const void* v, const void* const* x, const void* const* hhat16, int B, int D,
                                       int L, int N, hyena_dtype dtype, void* y, void* workspace,
                                       size_t workspace_bytes, hyena_stream stream) {
  if (N < 1 || N > kMaxOrder || B < 1 || D < 1) return HYENA_ERR_INVALID_ARG;
  if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
  // f16 bins carry a relative rounding of 2^-11 per stage, far above what
  // float32 I/O promises; only bf16 I/O (whose own rounding is 2^-9) is served
  if (dtype != HYENA_BF16) return HYENA_ERR_UNSUPPORTED;
  if (!x || !hhat16 || !aligned16(v) || !aligned16(y)) return HYENA_ERR_INVALID_ARG;
  for (int n = 0; n < N; ++n)
    if (!aligned16(x[n]) || !aligned16(hhat16[n])) return HYENA_ERR_INVALID_ARG;
  if ((long long)B * D > (1LL << 40) / (L > 0 ? L : 1)) return HYENA_ERR_INVALID_ARG;
  Layout ly;
  if (!make_layout(L, &ly)) return HYENA_ERR_UNSUPPORTED;
  if (ly.fourstep && (!aligned16(workspace) || workspace_bytes < sizeof(float2) * (size_t)ly.M))
    return HYENA_ERR_WORKSPACE;
  const cudaError_t e = forward_dispatch(v, x, hhat16, B, D, ly, N, dtype == HYENA_BF16, y, workspace,
                                         workspace_bytes, false, (cudaStream_t)stream, true);
  return e == cudaSuccess ? HYENA_OK : cuda_fail(e);
}

}  // extern "C"
