// fused.cu -- Hyena order-N forward for L <= 8192: one CTA per channel at a
// time (persistent over channels), z resident in shared memory across all N
// stages. HBM sees v, x_1..x_N and the filter spectra once and y once.
//
// Stage n (order-N recurrence, "Hyena Hierarchy" digest, 방법 / 프레임워크
// 개요; explainer "Hyena 演算子の形"):
//   z_{n+1} = x_n * (h_n conv z_n), conv = causal, via the 2L-grid FFT.
// Thread tl holds packed points m = tl + r*M/16 (r < 8) of z between stages:
// these are exactly the inputs of the first forward pass and the outputs of
// the last inverse pass, so the gate and the stage hand-off stay in registers.
#include "kernels.cuh"
#include "paired.cuh"

namespace hyena {

// Resident CTAs per SM the register budget is sized for.
#ifndef HYENA_FUSED_THREADS_PER_SM
#define HYENA_FUSED_THREADS_PER_SM 512
#endif
template <int LOGMV>
struct FusedOcc {
  static constexpr int TV = Plan<LOGMV>::TV;
  static constexpr int T = HYENA_FUSED_THREADS_PER_SM;
  static constexpr int value = TV >= 512 ? 1 : (T / TV > 16 ? 16 : (T / TV < 1 ? 1 : T / TV));
};

// Shared memory: z (padded), staged filter spectrum row (bins of type HT),
// staged gate row, staged v row of the next channel. At the longest fused
// length (2^14 points) z alone takes 136 KB, so the spectrum is read from
// global memory instead of being staged, and for float32 rows v is too.
template <int LOGMV, typename T, typename HT = float2>
struct FusedSmem {
  static constexpr int MV = 1 << LOGMV;
  static constexpr bool stage_h = LOGMV <= 13;
  static constexpr bool stage_v = LOGMV <= 13 || sizeof(T) < 4;
  static constexpr size_t z = sizeof(float2) * padded_len(MV);
  static constexpr size_t h = stage_h ? sizeof(HT) * MV : 0;
  static constexpr size_t row = sizeof(T) * MV;      // L <= MV elements, 16-byte multiple
  static constexpr size_t total = z + h + (stage_v ? 2 : 1) * row;
};

// Per-channel factor of a spectrum block: 1 for float32 bins; for __half2
// bins the inverse of the channel's power-of-two scale (exact), applied at the gate.
template <typename HT>
__device__ __forceinline__ float spec_inv_scale(const float2* block, int D, int M, int c) {
  if constexpr (sizeof(HT) == sizeof(float2)) {
    return 1.f;
  } else {
    return __ldg(reinterpret_cast<const float*>(reinterpret_cast<const char*>(block) + (size_t)4 * D * M) + c);
  }
}

template <int LOGMV, typename T, typename HT>
__global__ void __launch_bounds__(Plan<LOGMV>::TV, FusedOcc<LOGMV>::value)
fused_forward_kernel(const T* __restrict__ v, GatePtrs<T> x, SpecPtrs hh, T* __restrict__ y,
                     const float2* __restrict__ tables, int B, int D, int L, int N) {
  using P = Plan<LOGMV>;
  using S = FusedSmem<LOGMV, T, HT>;
  constexpr int MV = P::MV, TV = P::TV, Q8 = MV / 8, Q16 = MV / 16;
  extern __shared__ __align__(16) float2 sm[];
  HT* hs = reinterpret_cast<HT*>(reinterpret_cast<char*>(sm) + S::z);
  T* xs = reinterpret_cast<T*>(reinterpret_cast<char*>(sm) + S::z + S::h);
  T* vs = reinterpret_cast<T*>(reinterpret_cast<char*>(sm) + S::z + S::h + S::row);   // if S::stage_v
  const int tl = threadIdx.x;
  const float2* __restrict__ tw = tables;
  const float2* __restrict__ Wv = tables + MV;
  const long long C = (long long)B * D;
  const bool head = (tl == 0);
  const int jA = head ? 0 : tl;
  const int jB = head ? Q16 : Q8 - tl;
  const float2 one = make_float2(1.f, 0.f);
  const int row_bytes = L * (int)sizeof(T);
  const int h_bytes = MV * (int)sizeof(HT);
  auto spec_row = [&](int n, int c) { return reinterpret_cast<const HT*>(pick(hh, n)) + (size_t)c * MV; };

  // channel order c-major so that CTAs sharing a filter run side by side
  long long ch = blockIdx.x;
  if (ch < C) {
    const int c = (int)(ch / B), b = (int)(ch % B);
    if constexpr (S::stage_v) block_copy_async(vs, v + ((size_t)b * D + c) * (size_t)L, row_bytes, tl, TV);
    if constexpr (S::stage_h) block_copy_async(hs, spec_row(0, c), h_bytes, tl, TV);
    cp_async_commit();
    cp_async_wait_all();
  }
  __syncthreads();

  for (; ch < C; ch += gridDim.x) {
    const int c = (int)(ch / B), b = (int)(ch % B);
    const size_t row = ((size_t)b * D + c) * (size_t)L;
    float2 a[16];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int m = tl + r * Q16;
      if constexpr (S::stage_v)
        a[r] = (2 * m < L) ? IO<T>::load2_smem(vs + 2 * m) : make_float2(0.f, 0.f);
      else
        a[r] = (2 * m < L) ? IO<T>::load2(v + row + 2 * m) : make_float2(0.f, 0.f);
    }
    for (int n = 0; n < N; ++n) {
      // forward: first pass (radix 16, upper half of the input is zero)
      dft16<false, true, false, 0>(a);
      store_block16(sm, tl, a);
      __syncthreads();
      // every thread is past its reads of the gate and v buffers: refill them
      block_copy_async(xs, pick(x, n) + row, row_bytes, tl, TV);
      if (S::stage_v && n == 0 && ch + gridDim.x < C) {
        const long long nx = ch + gridDim.x;
        const int c2 = (int)(nx / B), b2 = (int)(nx % B);
        block_copy_async(vs, v + ((size_t)b2 * D + c2) * (size_t)L, row_bytes, tl, TV);
      }
      cp_async_commit();
      mid_fwd_all<LOGMV>(a, sm, tw, tl);
      // spectrum of stage n, gate of stage n and the next v are resident after this barrier
      cp_async_wait_all();
      __syncthreads();
      // last forward pass + spectral product + first inverse pass
      if constexpr (S::stage_h) {
        paired_pass<LOGMV, kPairConv, true, HT>(sm, sm, jA, jB, head, tw, Wv, one, false, hs, hs, 0.f);
      } else {
        HT* hg = const_cast<HT*>(spec_row(n, c));
        paired_pass<LOGMV, kPairConv, false, HT>(sm, sm, jA, jB, head, tw, Wv, one, false, hg, hg, 0.f);
      }
      __syncthreads();
      // the spectrum buffer is free: stage the next spectrum (next stage or next channel)
      if constexpr (S::stage_h) {
        const HT* hn = nullptr;
        if (n + 1 < N) {
          hn = spec_row(n + 1, c);
        } else if (ch + gridDim.x < C) {
          hn = spec_row(0, (int)((ch + gridDim.x) / B));
        }
        if (hn) block_copy_async(hs, hn, h_bytes, tl, TV);
        cp_async_commit();
      }
      mid_inv_all<LOGMV>(a, sm, tw, tl);
      // last inverse pass (radix 16): only the first half of the outputs is kept
      load_block16(sm, tl, a);
      dft16<true, false, true, 0>(a);
      // gate: z_{n+1}[t] = x_n[t] * conv[t] (times the spectrum block's channel factor)
      const float inv = spec_inv_scale<HT>(pick(hh, n), D, MV, c);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int m = tl + r * Q16;
        const float2 g = (2 * m < L) ? IO<T>::load2_smem(xs + 2 * m) : make_float2(0.f, 0.f);
        a[r] = make_float2(a[r].x * (g.x * inv), a[r].y * (g.y * inv));
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int m = tl + r * Q16;
      if (2 * m < L) IO<T>::store2(y + row + 2 * m, a[r]);
    }
  }
  cp_async_wait_all();
}

// Filter spectrum for the fused layout: H[c][k] = rfft(pad(h_c, 2M))[k] / (4M)
// in natural order k < M, bin 0 holding (H[0], H[M]) (both real).
template <int LOGMV>
__global__ void __launch_bounds__(Plan<LOGMV>::TV)
fused_spectrum_kernel(const float* __restrict__ h, float2* __restrict__ spec, const float2* __restrict__ tables,
                      int D, int L) {
  using P = Plan<LOGMV>;
  constexpr int MV = P::MV, Q8 = MV / 8, Q16 = MV / 16;
  extern __shared__ __align__(16) float2 sm[];
  const int tl = threadIdx.x;
  const float2* __restrict__ tw = tables;
  const float2* __restrict__ Wv = tables + MV;
  const bool head = (tl == 0);
  const int jA = head ? 0 : tl;
  const int jB = head ? Q16 : Q8 - tl;
  const float scale = 1.0f / (8.0f * (float)MV);
  for (int c = blockIdx.x; c < D; c += gridDim.x) {
    const float* __restrict__ hr = h + (size_t)c * L;
    float2 a[16];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int m = tl + r * Q16;
      a[r] = (2 * m < L) ? __ldg(reinterpret_cast<const float2*>(hr + 2 * m)) : make_float2(0.f, 0.f);
    }
    dft16<false, true, false, 0>(a);
    store_block16(sm, tl, a);
    __syncthreads();
    mid_fwd_all<LOGMV>(a, sm, tw, tl);
    float2* H = spec + (size_t)c * MV;
    paired_pass<LOGMV, kPairSpectrum>(sm, sm, jA, jB, head, tw, Wv, make_float2(1.f, 0.f), false, H, H, scale);
    __syncthreads();
  }
}

// ------------------------------------------------------------- launchers --

template <int LOGMV, typename T, typename HT>
static cudaError_t launch_fused_t(const FusedLaunch& p, cudaStream_t s) {
  auto k = fused_forward_kernel<LOGMV, T, HT>;
  const int threads = Plan<LOGMV>::TV;
  const size_t smem = FusedSmem<LOGMV, T, HT>::total;
  int grid = 0;
  cudaError_t e = persistent_grid((const void*)k, threads, smem, &grid);
  if (e != cudaSuccess) return e;
  long long C = (long long)p.B * p.D;
  if ((long long)grid > C) grid = (int)C;
  GatePtrs<T> xp;
  for (int i = 0; i < kMaxOrder; ++i) xp.p[i] = reinterpret_cast<const T*>(p.x[i]);
  k<<<grid, threads, smem, s>>>(reinterpret_cast<const T*>(p.v), xp, p.hh, reinterpret_cast<T*>(p.y),
                                p.tables, p.B, p.D, p.L, p.N);
  return cudaGetLastError();
}

template <int LOGMV>
static cudaError_t launch_fused_l(const FusedLaunch& p, cudaStream_t s) {
  if (p.spec16)
    return p.bf16 ? launch_fused_t<LOGMV, __nv_bfloat16, __half2>(p, s) : launch_fused_t<LOGMV, float, __half2>(p, s);
  return p.bf16 ? launch_fused_t<LOGMV, __nv_bfloat16, float2>(p, s) : launch_fused_t<LOGMV, float, float2>(p, s);
}

cudaError_t launch_fused_forward(const FusedLaunch& p, int logMV, cudaStream_t s) {
  switch (logMV) {
    case 7: return launch_fused_l<7>(p, s);
    case 8: return launch_fused_l<8>(p, s);
    case 9: return launch_fused_l<9>(p, s);
    case 10: return launch_fused_l<10>(p, s);
    case 11: return launch_fused_l<11>(p, s);
    case 12: return launch_fused_l<12>(p, s);
    case 13: return launch_fused_l<13>(p, s);
    case 14: return launch_fused_l<14>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int LOGMV>
static cudaError_t launch_fused_spec_l(const float* h, float2* spec, const float2* tables, int D, int L,
                                       cudaStream_t s) {
  auto k = fused_spectrum_kernel<LOGMV>;
  const int threads = Plan<LOGMV>::TV;
  const size_t smem = sizeof(float2) * padded_len(1 << LOGMV);
  int grid = 0;
  cudaError_t e = persistent_grid((const void*)k, threads, smem, &grid);
  if (e != cudaSuccess) return e;
  if (grid > D) grid = D;
  k<<<grid, threads, smem, s>>>(h, spec, tables, D, L);
  return cudaGetLastError();
}

cudaError_t launch_fused_spectrum(const float* h, float2* spec, const float2* tables, int D, int L, int logMV,
                                  cudaStream_t s) {
  switch (logMV) {
    case 7: return launch_fused_spec_l<7>(h, spec, tables, D, L, s);
    case 8: return launch_fused_spec_l<8>(h, spec, tables, D, L, s);
    case 9: return launch_fused_spec_l<9>(h, spec, tables, D, L, s);
    case 10: return launch_fused_spec_l<10>(h, spec, tables, D, L, s);
    case 11: return launch_fused_spec_l<11>(h, spec, tables, D, L, s);
    case 12: return launch_fused_spec_l<12>(h, spec, tables, D, L, s);
    case 13: return launch_fused_spec_l<13>(h, spec, tables, D, L, s);
    case 14: return launch_fused_spec_l<14>(h, spec, tables, D, L, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hyena
