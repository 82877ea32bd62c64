// nd.cu -- HyenaND: the order-N recurrence with an N-dimensional global
// convolution (HyenaND summary, section 手法: the convolution runs on the
// L_1 x ... x L_N grid through an N-dimensional FFT, circular for periodic
// data, or on the input zero-padded to twice the grid so nothing leaks across
// the boundary).
//
//   z_1 = v,  z_{n+1} = x_n (.) (K_n conv z_n),  y = z_{N+1}
//   circular: (K conv z)[p] = sum_q K[(p - q) mod dims] z[q]
//   zero:     (K conv z)[p] = sum_{0 <= q <= p} K[p - q] z[q]
//
// One CTA per (channel c, batch pair b, b+1): the two real signals of the
// pair are the real and imaginary parts of one complex grid (K is real, so one
// complex convolution carries both), held in shared memory on the padded grid
// P_1 x ... x P_nd (P_a = 2 L_a zero-padded, L_a circular; P = prod P_a <=
// 16384 points, 128 KB). The transform is separable: along every axis,
// in-place decimation-in-frequency radix-4 levels (one radix-2 level first
// when log2 P_a is odd) leave each axis index bit-reversed; the spectrum
// block K^ is stored in that same order, so the product needs no reordering,
// and the inverse runs the levels backwards (decimation in time, conjugate
// twiddles), returning natural order. K^ carries the 1/P of the inverse.
// All N stages stay in shared memory; only v, x_n and y touch HBM, plus K^.
#include <cuda_bf16.h>

#include "fft_engine.cuh"
#include "kernels.cuh"

namespace hyena {

namespace {

constexpr int kNdMaxDims = 3;
constexpr int kNdMaxLogP = 14;      // 16384 complex points: 128 KB of shared memory
constexpr int kNdMaxLogAxis = 10;   // padded axis length <= 1024 (twiddle table <= 512 entries)

struct NdGeom {
  int nd;
  int logP;
  int logn[kNdMaxDims];   // padded axis lengths
  int logs[kNdMaxDims];   // inner stride of each axis on the padded grid
  int logL[kNdMaxDims];   // grid axis lengths
  int logT;               // table length 2^(logT - 1): w_T^k for k < T/2, T = longest padded axis
  int G;                  // grid points prod L_a
  int zero;               // zero-padded boundary
};

__device__ __forceinline__ float ld1(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld1(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }
__device__ __forceinline__ void st1(float* p, float v) { *p = v; }
__device__ __forceinline__ void st1(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// (-i) * a and (+i) * a
__device__ __forceinline__ float2 mul_mi(float2 a) { return make_float2(a.y, -a.x); }
__device__ __forceinline__ float2 mul_pi(float2 a) { return make_float2(-a.y, a.x); }

// Padded-grid position of grid point g (row-major over L_0 x L_1 x L_2).
__device__ __forceinline__ int grid_to_pos(const NdGeom& g, int gi) {
  int pos = 0;
#pragma unroll
  for (int a = kNdMaxDims - 1; a >= 0; --a) {
    if (a < g.nd) {
      const int coord = gi & ((1 << g.logL[a]) - 1);
      gi >>= g.logL[a];
      pos += coord << g.logs[a];
    }
  }
  return pos;
}

// Grid index of padded position pos, or -1 in the padding.
__device__ __forceinline__ int pos_to_grid(const NdGeom& g, int pos) {
  int gi = 0;
#pragma unroll
  for (int a = 0; a < kNdMaxDims; ++a) {
    if (a < g.nd) {
      const int coord = (pos >> g.logs[a]) & ((1 << g.logn[a]) - 1);
      if (coord >> g.logL[a]) return -1;
      gi = (gi << g.logL[a]) + coord;
    }
  }
  return gi;
}

// One radix-2 level (block size 2^logm) along an axis of inner stride 2^logs.
template <bool INV>
__device__ __forceinline__ void level2(float2* s, const float2* tw, int logT, int logm, int logs, int P, int tid,
                                       int nt) {
  const int logh = logm - 1;
  for (int t = tid; t < (P >> 1); t += nt) {
    const int in = t & ((1 << logs) - 1);
    const int r = t >> logs;
    const int j = r & ((1 << logh) - 1);
    const int blk = r >> logh;
    const int i0 = (((blk << logm) + j) << logs) + in;
    const int i1 = i0 + (1 << (logh + logs));
    const float2 w = tw[j << (logT - logm)];
    const float2 a = s[i0], b = s[i1];
    if (!INV) {
      s[i0] = cadd(a, b);
      s[i1] = cmul(csub(a, b), w);
    } else {
      const float2 bw = cmulc(b, w);
      s[i0] = cadd(a, bw);
      s[i1] = csub(a, bw);
    }
  }
}

// Two radix-2 levels (block sizes 2^logm and 2^(logm-1)) fused in registers.
template <bool INV>
__device__ __forceinline__ void level4(float2* s, const float2* tw, int logT, int logm, int logs, int P, int tid,
                                       int nt) {
  const int logq = logm - 2;
  for (int t = tid; t < (P >> 2); t += nt) {
    const int in = t & ((1 << logs) - 1);
    const int r = t >> logs;
    const int j = r & ((1 << logq) - 1);
    const int blk = r >> logq;
    const int i0 = (((blk << logm) + j) << logs) + in;
    const int dq = 1 << (logq + logs);
    const float2 w1 = tw[j << (logT - logm)];        // w_m^j
    const float2 w2 = tw[j << (logT - logm + 1)];    // w_{m/2}^j
    float2 x0 = s[i0], x1 = s[i0 + dq], x2 = s[i0 + 2 * dq], x3 = s[i0 + 3 * dq];
    if (!INV) {
      const float2 a0 = cadd(x0, x2), a2 = cmul(csub(x0, x2), w1);
      const float2 a1 = cadd(x1, x3), a3 = cmul(mul_mi(csub(x1, x3)), w1);
      s[i0] = cadd(a0, a1);
      s[i0 + dq] = cmul(csub(a0, a1), w2);
      s[i0 + 2 * dq] = cadd(a2, a3);
      s[i0 + 3 * dq] = cmul(csub(a2, a3), w2);
    } else {
      const float2 t1 = cmulc(x1, w2), t3 = cmulc(x3, w2);
      const float2 a0 = cadd(x0, t1), a1 = csub(x0, t1);
      const float2 a2 = cadd(x2, t3), a3 = csub(x2, t3);
      const float2 u2 = cmulc(a2, w1), u3 = mul_pi(cmulc(a3, w1));
      s[i0] = cadd(a0, u2);
      s[i0 + 2 * dq] = csub(a0, u2);
      s[i0 + dq] = cadd(a1, u3);
      s[i0 + 3 * dq] = csub(a1, u3);
    }
  }
}

// Forward transform (natural order in, per-axis bit-reversed out) or its
// inverse (bit-reversed in, natural out, scaled by P). Ends with a barrier.
template <bool INV>
__device__ void nd_transform(float2* s, const float2* tw, const NdGeom& g, int tid, int nt) {
  const int P = 1 << g.logP;
  for (int a = 0; a < g.nd; ++a) {
    const int n = g.logn[a], ls = g.logs[a];
    const bool odd = n & 1;
    if (!INV) {
      if (odd) {
        level2<false>(s, tw, g.logT, n, ls, P, tid, nt);
        __syncthreads();
      }
      for (int m = odd ? n - 1 : n; m >= 2; m -= 2) {
        level4<false>(s, tw, g.logT, m, ls, P, tid, nt);
        __syncthreads();
      }
    } else {
      for (int m = 2; m <= (odd ? n - 1 : n); m += 2) {
        level4<true>(s, tw, g.logT, m, ls, P, tid, nt);
        __syncthreads();
      }
      if (odd) {
        level2<true>(s, tw, g.logT, n, ls, P, tid, nt);
        __syncthreads();
      }
    }
  }
}

template <typename T>
struct NdGates {
  const T* p[kMaxOrder];
};

template <typename T>
__global__ void __launch_bounds__(1024) nd_forward_kernel(const T* __restrict__ v, NdGates<T> xs, SpecPtrs kh,
                                                          T* __restrict__ y, NdGeom g, int B, int D, int N) {
  extern __shared__ float4 nd_smem_raw[];
  float2* s = reinterpret_cast<float2*>(nd_smem_raw);
  const int P = 1 << g.logP;
  float2* tw = s + P;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int c = blockIdx.x % D;
  const int b0 = 2 * (blockIdx.x / D);
  const bool has1 = b0 + 1 < B;
  const size_t G = (size_t)g.G;
  const size_t row0 = ((size_t)b0 * D + c) * G;
  const size_t row1 = row0 + (size_t)D * G;

  const float2* tsrc = kh.p[0] + (size_t)D * P;
  for (int i = tid; i < (1 << (g.logT - 1)); i += nt) tw[i] = __ldg(tsrc + i);
  if (g.zero)
    for (int i = tid; i < P; i += nt) s[i] = make_float2(0.f, 0.f);
  __syncthreads();
  for (int gi = tid; gi < g.G; gi += nt)
    s[grid_to_pos(g, gi)] = make_float2(ld1(v + row0 + gi), has1 ? ld1(v + row1 + gi) : 0.f);
  __syncthreads();

  for (int n = 0; n < N; ++n) {
    nd_transform<false>(s, tw, g, tid, nt);
    const float2* __restrict__ H = pick(kh, n) + (size_t)c * P;
    for (int i = tid; i < P; i += nt) s[i] = cmul(s[i], __ldg(H + i));
    __syncthreads();
    nd_transform<true>(s, tw, g, tid, nt);
    const T* __restrict__ x = pick(xs, n);
    if (n + 1 < N) {
      if (g.zero) {
        for (int i = tid; i < P; i += nt) {
          const int gi = pos_to_grid(g, i);
          float2 z = make_float2(0.f, 0.f);
          if (gi >= 0) {
            const float2 u = s[i];
            z = make_float2(u.x * ld1(x + row0 + gi), has1 ? u.y * ld1(x + row1 + gi) : 0.f);
          }
          s[i] = z;
        }
      } else {
        for (int gi = tid; gi < g.G; gi += nt) {
          const int i = grid_to_pos(g, gi);
          const float2 u = s[i];
          s[i] = make_float2(u.x * ld1(x + row0 + gi), has1 ? u.y * ld1(x + row1 + gi) : 0.f);
        }
      }
      __syncthreads();
    } else {
      for (int gi = tid; gi < g.G; gi += nt) {
        const float2 u = s[grid_to_pos(g, gi)];
        const float x0 = ld1(x + row0 + gi);
        const float x1 = has1 ? ld1(x + row1 + gi) : 0.f;
        st1(y + row0 + gi, u.x * x0);
        if (has1) st1(y + row1 + gi, u.y * x1);
      }
    }
  }
}

// Spectrum of one filter: K [D][grid] float32 -> [D][P] float2 (transform
// order, times 1/P), one CTA per channel; the twiddle table follows.
__global__ void __launch_bounds__(1024) nd_spectrum_kernel(const float* __restrict__ K, float2* __restrict__ out,
                                                           NdGeom g, int D) {
  extern __shared__ float4 nd_smem_raw[];
  float2* s = reinterpret_cast<float2*>(nd_smem_raw);
  const int P = 1 << g.logP;
  float2* tw = s + P;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int c = blockIdx.x;
  const float2* tsrc = out + (size_t)D * P;
  for (int i = tid; i < (1 << (g.logT - 1)); i += nt) tw[i] = tsrc[i];
  for (int i = tid; i < P; i += nt) s[i] = make_float2(0.f, 0.f);
  __syncthreads();
  for (int gi = tid; gi < g.G; gi += nt) s[grid_to_pos(g, gi)] = make_float2(__ldg(K + (size_t)c * g.G + gi), 0.f);
  __syncthreads();
  nd_transform<false>(s, tw, g, tid, nt);
  const float inv = 1.0f / (float)P;   // exact: P is a power of two
  for (int i = tid; i < P; i += nt) {
    const float2 u = s[i];
    out[(size_t)c * P + i] = make_float2(u.x * inv, u.y * inv);
  }
}

// w_T^k = exp(-2 pi i k / T), k < T/2, formed in double and rounded once.
__global__ void nd_table_kernel(float2* __restrict__ tw, int logT) {
  const int half = 1 << (logT - 1);
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < half; k += gridDim.x * blockDim.x) {
    double sn, cs;
    sincospi(2.0 * (double)k / (double)(1 << logT), &sn, &cs);
    tw[k] = make_float2((float)cs, (float)-sn);
  }
}

int ilog2_pow2(int x) {
  if (x < 1 || (x & (x - 1))) return -1;
  int l = 0;
  while ((1 << l) < x) ++l;
  return l;
}

// Geometry of (nd, dims, boundary); false when unsupported.
bool nd_geometry(int nd, const int* dims, int boundary, NdGeom* g) {
  if (nd < 1 || nd > kNdMaxDims || !dims || (boundary != 0 && boundary != 1)) return false;
  NdGeom r{};
  r.nd = nd;
  r.zero = boundary == 0;
  int logP = 0, logG = 0, logT = 1;
  for (int a = 0; a < nd; ++a) {
    const int l = ilog2_pow2(dims[a]);
    if (l < 0) return false;
    r.logL[a] = l;
    r.logn[a] = l + (r.zero ? 1 : 0);
    if (r.logn[a] > kNdMaxLogAxis) return false;
    logP += r.logn[a];
    logG += l;
    if (r.logn[a] > logT) logT = r.logn[a];
  }
  if (logP > kNdMaxLogP) return false;
  int acc = 0;
  for (int a = nd - 1; a >= 0; --a) {
    r.logs[a] = acc;
    acc += r.logn[a];
  }
  r.logP = logP;
  r.logT = logT;
  r.G = 1 << logG;
  *g = r;
  return true;
}

int nd_threads(const NdGeom& g) {
  int t = (1 << g.logP) / 16;
  if (t < 64) t = 64;
  if (t > 1024) t = 1024;
  return t;
}

size_t nd_smem(const NdGeom& g) { return sizeof(float2) * ((size_t)(1 << g.logP) + (1 << (g.logT - 1))); }

size_t nd_block_bytes(const NdGeom& g, int D) {
  return sizeof(float2) * ((size_t)D * (1 << g.logP) + (((1 << (g.logT - 1)) + 1) & ~1));
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

bool nd_aligned16(const void* q) { return q && ((reinterpret_cast<uintptr_t>(q) & 15u) == 0); }

}  // namespace

}  // namespace hyena

using namespace hyena;

extern "C" {

size_t hyena_nd_spectrum_bytes(int D, int nd, const int* dims, int boundary) {
  NdGeom g;
  if (D < 1 || !nd_geometry(nd, dims, boundary, &g)) return 0;
  return nd_block_bytes(g, D);
}

hyena_status hyena_nd_filter_spectrum(const float* K, int D, int nd, const int* dims, int boundary, void* khat,
                                      hyena_stream stream) {
  NdGeom g;
  if (D < 1 || !nd_aligned16(K) || !nd_aligned16(khat)) return HYENA_ERR_INVALID_ARG;
  if (!nd_geometry(nd, dims, boundary, &g)) return HYENA_ERR_UNSUPPORTED;
  if ((long long)D > (1LL << 40) / g.G) return HYENA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  float2* out = reinterpret_cast<float2*>(khat);
  nd_table_kernel<<<1, 256, 0, s>>>(out + (size_t)D * (1 << g.logP), g.logT);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = set_smem(nd_spectrum_kernel, nd_smem(g));
  if (e == cudaSuccess) {
    nd_spectrum_kernel<<<D, nd_threads(g), nd_smem(g), s>>>(K, out, g, D);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? HYENA_OK : report_cuda_error(e);
}

hyena_status hyena_nd_forward(const void* v, const void* const* x, const void* const* khat, int B, int D, int nd,
                              const int* dims, int boundary, int N, hyena_dtype dtype, void* y, hyena_stream stream) {
  if (N < 1 || N > kMaxOrder || B < 1 || D < 1) return HYENA_ERR_INVALID_ARG;
  if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
  if (!x || !khat || !nd_aligned16(v) || !nd_aligned16(y)) return HYENA_ERR_INVALID_ARG;
  for (int n = 0; n < N; ++n)
    if (!nd_aligned16(x[n]) || !nd_aligned16(khat[n])) return HYENA_ERR_INVALID_ARG;
  NdGeom g;
  if (!nd_geometry(nd, dims, boundary, &g)) return HYENA_ERR_UNSUPPORTED;
  if ((long long)B * D > (1LL << 40) / g.G) return HYENA_ERR_INVALID_ARG;
  const long long blocks = (long long)D * ((B + 1) / 2);
  if (blocks > 0x7fffffffLL) return HYENA_ERR_INVALID_ARG;
  SpecPtrs kh{};
  for (int n = 0; n < N; ++n) kh.p[n] = reinterpret_cast<const float2*>(khat[n]);
  cudaStream_t s = (cudaStream_t)stream;
  const size_t smem = nd_smem(g);
  cudaError_t e;
  if (dtype == HYENA_BF16) {
    NdGates<__nv_bfloat16> xs{};
    for (int n = 0; n < N; ++n) xs.p[n] = reinterpret_cast<const __nv_bfloat16*>(x[n]);
    e = set_smem(nd_forward_kernel<__nv_bfloat16>, smem);
    if (e == cudaSuccess) {
      nd_forward_kernel<__nv_bfloat16><<<(unsigned)blocks, nd_threads(g), smem, s>>>(
          reinterpret_cast<const __nv_bfloat16*>(v), xs, kh, reinterpret_cast<__nv_bfloat16*>(y), g, B, D, N);
      e = cudaGetLastError();
    }
  } else {
    NdGates<float> xs{};
    for (int n = 0; n < N; ++n) xs.p[n] = reinterpret_cast<const float*>(x[n]);
    e = set_smem(nd_forward_kernel<float>, smem);
    if (e == cudaSuccess) {
      nd_forward_kernel<float><<<(unsigned)blocks, nd_threads(g), smem, s>>>(
          reinterpret_cast<const float*>(v), xs, kh, reinterpret_cast<float*>(y), g, B, D, N);
      e = cudaGetLastError();
    }
  }
  return e == cudaSuccess ? HYENA_OK : report_cuda_error(e);
}

}  // extern "C"
