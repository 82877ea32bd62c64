// kernels.cuh -- launch parameter structs and launcher prototypes shared by
// the host dispatch (api.cu) and the kernel translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hyena.h"
#include "layout.h"

namespace hyena {

constexpr int kMaxOrder = 8;

template <typename T>
struct GatePtrs {
  const T* p[kMaxOrder];
};

struct SpecPtrs {
  const float2* p[kMaxOrder];   // spectrum blocks of filters 1..N
};

// Entry n of a kernel-parameter pointer array without a runtime-indexed copy
// to local memory (every candidate is read straight from the parameter bank).
template <typename A>
__device__ __forceinline__ auto pick(const A& arr, int n) {
  auto r = arr.p[0];
#pragma unroll
  for (int i = 1; i < kMaxOrder; ++i)
    if (n == i) r = arr.p[i];
  return r;
}

struct FusedLaunch {
  const void* v;
  const void* x[kMaxOrder];
  SpecPtrs hh;
  void* y;
  const float2* tables;
  int B, D, L, N;
  bool bf16;
  bool spec16;       // spectrum blocks in the reduced-precision (__half2) format
};

struct FourStepLaunch {
  const void* v;
  const void* x[kMaxOrder];
  SpecPtrs hh;
  void* y;
  const float2* tables;
  float2* scratch;
  int B, D, L, N;
  bool bf16;
  long long ch0;     // first channel (c-major order) of this wave
  int wave;          // channels in this wave
  bool spec16;       // spectrum blocks in the reduced-precision (__half2) format
  // tensor-core row pass (rows of 4096, bf16, order <= kTcgMaxOrder): two
  // buffers of `wave` per-channel maxima (float bits) of the column pass output
  bool tcr;
  unsigned* xmax;
  const float* hmax[kMaxOrder];   // per filter: the spectrum block's per-channel maxima
  const uint32_t* hhalf[kMaxOrder];   // per filter: the spectrum block's f16 copy (__half2 words)
};

// Records e as this thread's last CUDA error (hyena_last_cuda_error) and
// returns HYENA_ERR_CUDA.
hyena_status report_cuda_error(cudaError_t e);

// The forward on any supported layout: fused kernel (tensor-core kernel for
// bf16 pairs when allow_tc), or four-step waves through the workspace.
// Arguments are assumed checked by the caller.
cudaError_t forward_dispatch(const void* v, const void* const* x, const void* const* hhat, int B, int D,
                             const Layout& ly, int N, bool bf16, void* y, void* workspace, size_t workspace_bytes,
                             bool allow_tc, cudaStream_t s, bool spec16 = false);
// float32 spectrum block -> reduced-precision block (bins and scales; tables copied)
cudaError_t launch_spectrum_to_f16(const float2* spec, unsigned char* out, int D, const Layout& y, cudaStream_t s);
// Workspace of one L2-sized four-step wave over `channels` channels.
// Workspace bytes for one wave of four-step channels (at most `channels`),
// by the rule of the row kernel that will run (api.cu gives the measurements).
enum class WaveRule { kTensorRows, kSimtRows, kBackward };
size_t fourstep_wave_bytes(long long channels, const Layout& ly, WaveRule rule);
// Spectrum block (spectra, optional tensor-core copy, tables) of `rows` real
// rows h [rows][L] float32.
cudaError_t spectrum_dispatch(const float* h, float2* spec, int rows, const Layout& ly, bool with_tc,
                              cudaStream_t s);

// Grid for a persistent kernel: SM count x resident CTAs per SM.
cudaError_t persistent_grid(const void* kernel, int threads, size_t smem, int* grid);

cudaError_t launch_fill_tables(float2* tables, const Layout& y, cudaStream_t s);
cudaError_t launch_fused_forward(const FusedLaunch& p, int logMV, cudaStream_t s);
cudaError_t launch_fused_spectrum(const float* h, float2* spec, const float2* tables, int D, int L, int logMV,
                                  cudaStream_t s);
cudaError_t launch_tc_forward(const FusedLaunch& p, const Layout& y, cudaStream_t s);
cudaError_t launch_tc_spectrum(const float2* nat, float2* tcs, float2* tables, int D, const Layout& y,
                               cudaStream_t s);
// tcgen05 GEMM-level kernel (bf16, L = kTcgL, B even) and its spectrum copy
cudaError_t launch_tcg_forward(const FusedLaunch& p, cudaStream_t s);
cudaError_t launch_tcg_spectrum(const float2* nat, float2* tcs, int D, cudaStream_t s);
int tcg_read_and_clear_timeout();
// StripedHyena-form operator: featurizer length <= kMaxStripedLF, explicit
// inner filter length <= kMaxStripedLG. hG == nullptr: featurize only (q, u).
constexpr int kMaxStripedLF = 16;
constexpr int kMaxStripedLG = 1024;
cudaError_t launch_striped(const void* xq, const void* xk, const void* xv, const float* hT, const float* hH,
                           const float* hK, int lf, const float* hG, int lg, int B, int D, int L, bool bf16, void* y,
                           void* q, void* u, cudaStream_t s);
int striped_read_and_clear_timeout();
cudaError_t launch_exp_sum_filter(const float* R, const float* lam, int d, int D, int L, float* h, cudaStream_t s);
cudaError_t launch_fourstep_wave(const FourStepLaunch& p, const Layout& y, cudaStream_t s);
int fourstep_read_and_clear_timeout();
// tensor-core row pass of one four-step stage (rows of 4096 points)
cudaError_t launch_tcr_rows(float2* scr, const uint32_t* spec16, const float* hmax, const unsigned* xmax,
                            unsigned* xmax_clear, int M1, int B, long long ch0, int wave, cudaStream_t s);
cudaError_t launch_tcr_hmax(const float2* spec, int D, int M, float* hmax, cudaStream_t s);
// f16 copy of a spectrum block's bins for the row pass (after launch_tcr_hmax)
cudaError_t launch_tcr_half(const float2* spec, const float* hmax, int D, int M, uint32_t* out, cudaStream_t s);
int tcr_read_and_clear_timeout();
cudaError_t launch_fourstep_spectrum(const float* h, float2* spec, const float2* tables, int D,
                                     const Layout& y, cudaStream_t s);
cudaError_t launch_filter_generate(const float* W1, const float* b1, const float* W2, const float* b2,
                                   const float* W3, const float* b3, int n_bands, int width, int N, int D,
                                   int L, float alpha_lo, float alpha_hi, float* h, cudaStream_t s);

}  // namespace hyena
