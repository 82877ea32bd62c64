// striped.cu -- the StripedHyena-form operator ("02. 3つの Hyena 演算子",
// section 2, the operator structure; section 3, the SE / MR / LI variants;
// section 4, the FIR sum y_t = sum_{k < l_h} h_k x_{t-k}):
//   q = h_T * xq,  k = h_H * xk,  v = h_K * xv      short explicit featurizers
//   y = q . (h_G * (k . v))                          inner filter h_G
// (xq, xk, xv are the outputs of the dense projections, which are not part of
// this operator).
//   - SE / MR (explicit inner filter of up to kMaxLG taps): one fused kernel,
//     each CTA one (b, c) row and one time tile, inputs staged with their
//     causal halo in shared memory, the inner sum in a register sliding window.
//   - LI (long implicit inner filter): the featurizer kernel writes q and
//     u = k . v, and y = q . (h_G * u) is an order-1 forward on the FFT path.
// Plus the LI filter h_t = sum_n R_n lambda_n^t (section 3, Hyena-LI; the
// pages' 1-based t - 1 is the 0-based lag t).
#include "fft_engine.cuh"
#include "kernels.cuh"

namespace hyena {

namespace {

constexpr int kStThreads = 256;
constexpr int kStTile = 2048;        // outputs per CTA
constexpr int kStPer = kStTile / kStThreads;   // consecutive outputs per thread (8)

template <typename T>
__device__ __forceinline__ float ld1(const T* p);
template <>
__device__ __forceinline__ float ld1<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }

template <typename T>
__device__ __forceinline__ void st1(T* p, float v);
template <>
__device__ __forceinline__ void st1<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void st1<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// s[i] = x[row + t0 - halo + i] as float, zero before t = 0 and from t = L on
template <typename T>
__device__ __forceinline__ void stage_row(float* s, const T* __restrict__ x, size_t row, int t0, int halo, int n, int L,
                                          int tid) {
  for (int i = tid; i < n; i += kStThreads) {
    const int t = t0 - halo + i;
    s[i] = (t >= 0 && t < L) ? ld1<T>(x + row + t) : 0.f;
  }
}

// Featurize q (optional) and u = (hH * xk)(hK * xv) for the rows' outputs.
template <typename T, bool FUSED>
__global__ void __launch_bounds__(kStThreads)
striped_kernel(const T* __restrict__ xq, const T* __restrict__ xk, const T* __restrict__ xv,
               const float* __restrict__ hT, const float* __restrict__ hH, const float* __restrict__ hK, int lf,
               const float* __restrict__ hG, int lg, int D, int L, T* __restrict__ y, T* __restrict__ qout,
               T* __restrict__ uout) {
  extern __shared__ float st[];
  const int tid = threadIdx.x;
  const int tiles = (L + kStTile - 1) / kStTile;
  const long long rowi = blockIdx.x / tiles;
  const int c = (int)(rowi % D);
  const size_t row = (size_t)rowi * L;
  const int t0 = (int)(blockIdx.x % tiles) * kStTile;
  const int n_out = min(kStTile, L - t0);
  const int hg = FUSED ? lg - 1 : 0;           // halo of u for the inner filter
  const int hf = lf - 1;                        // halo of the featurizers
  const int nu = n_out + hg;                    // u values this tile needs
  const int nx = nu + hf;                       // xk, xv values
  float* fT = st;                               // [lf]
  float* fH = fT + 16;
  float* fK = fH + 16;
  float* fG = fK + 16;                          // [lg]
  const int S = kStTile + lg + 16;              // staged-row capacity (>= nx)
  float* sk = fG + (FUSED ? lg : 0);            // [nx]
  float* sv = sk + S;
  float* su = sv + S;                           // [nu]
  float* sq = su + S;                           // [n_out + hf]
  for (int i = tid; i < lf; i += kStThreads) {
    fT[i] = hT[(size_t)c * lf + i];
    fH[i] = hH[(size_t)c * lf + i];
    fK[i] = hK[(size_t)c * lf + i];
  }
  if (FUSED)
    for (int i = tid; i < lg; i += kStThreads) fG[i] = hG[(size_t)c * lg + i];
  stage_row<T>(sk, xk, row, t0, hg + hf, nx, L, tid);
  stage_row<T>(sv, xv, row, t0, hg + hf, nx, L, tid);
  stage_row<T>(sq, xq, row, t0, hf, n_out + hf, L, tid);
  __syncthreads();
  // u[i] = k . v at t = t0 - hg + i (zero before t = 0)
  for (int i = tid; i < nu; i += kStThreads) {
    float a = 0.f, b = 0.f;
    for (int j = 0; j < lf; ++j) {
      a = fmaf(fH[j], sk[i + hf - j], a);
      b = fmaf(fK[j], sv[i + hf - j], b);
    }
    su[i] = (t0 - hg + i >= 0) ? a * b : 0.f;
  }
  __syncthreads();
  // outputs t0 + base + p, p < kStPer
  const int base = tid * kStPer;
  if (base >= n_out) return;
  float acc[kStPer];
  if (FUSED) {
    // inner sum w[t] = sum_j hG[j] u[t - j] as a sliding window: win[p] = u at (t_p - j)
#pragma unroll
    for (int p = 0; p < kStPer; ++p) acc[p] = 0.f;
    float win[kStPer];
#pragma unroll
    for (int p = 0; p < kStPer; ++p) win[p] = su[hg + base + p];   // j = 0
    for (int j = 0; j < lg; ++j) {
      const float g = fG[j];
#pragma unroll
      for (int p = 0; p < kStPer; ++p) acc[p] = fmaf(g, win[p], acc[p]);
      // slide: index (base + p + hg) - (j + 1)
#pragma unroll
      for (int p = kStPer - 1; p > 0; --p) win[p] = win[p - 1];
      win[0] = (j + 1 < lg) ? su[hg + base - j - 1] : 0.f;
    }
  }
#pragma unroll
  for (int p = 0; p < kStPer; ++p) {
    const int i = base + p;
    if (i >= n_out) break;
    float q = 0.f;
    for (int j = 0; j < lf; ++j) q = fmaf(fT[j], sq[i + hf - j], q);
    if (FUSED) {
      st1<T>(y + row + t0 + i, q * acc[p]);
    } else {
      st1<T>(qout + row + t0 + i, q);
      st1<T>(uout + row + t0 + i, su[i]);
    }
  }
}

// h[c][t] = sum_n R[c][n] lambda[c][n]^t
__global__ void exp_sum_filter_kernel(const float* __restrict__ R, const float* __restrict__ lam, int d, int D, int L,
                                      float* __restrict__ h) {
  const size_t n = (size_t)D * L;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int c = (int)(i / L), t = (int)(i % L);
    float acc = 0.f;
    for (int k = 0; k < d; ++k) acc = fmaf(R[(size_t)c * d + k], powf(lam[(size_t)c * d + k], (float)t), acc);
    h[i] = acc;
  }
}

size_t striped_smem(bool fused, int lg) {
  return sizeof(float) * (size_t)(16 * 3 + (fused ? lg : 0) + 4 * (kStTile + lg + 16));
}

template <typename T, bool FUSED>
cudaError_t launch_striped_t(const void* xq, const void* xk, const void* xv, const float* hT, const float* hH,
                             const float* hK, int lf, const float* hG, int lg, int B, int D, int L, void* y, void* q,
                             void* u, cudaStream_t s) {
  auto k = striped_kernel<T, FUSED>;
  const size_t smem = striped_smem(FUSED, lg);
  cudaError_t e = cudaFuncSetAttribute((const void*)k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long blocks = (long long)((L + kStTile - 1) / kStTile) * B * D;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  k<<<(unsigned)blocks, kStThreads, smem, s>>>(reinterpret_cast<const T*>(xq), reinterpret_cast<const T*>(xk),
                                   reinterpret_cast<const T*>(xv), hT, hH, hK, lf, hG, lg, D, L,
                                   reinterpret_cast<T*>(y), reinterpret_cast<T*>(q), reinterpret_cast<T*>(u));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_striped(const void* xq, const void* xk, const void* xv, const float* hT, const float* hH,
                           const float* hK, int lf, const float* hG, int lg, int B, int D, int L, bool bf16, void* y,
                           void* q, void* u, cudaStream_t s) {
  const bool fused = (hG != nullptr);
  if (bf16)
    return fused ? launch_striped_t<__nv_bfloat16, true>(xq, xk, xv, hT, hH, hK, lf, hG, lg, B, D, L, y, q, u, s)
                 : launch_striped_t<__nv_bfloat16, false>(xq, xk, xv, hT, hH, hK, lf, hG, lg, B, D, L, y, q, u, s);
  return fused ? launch_striped_t<float, true>(xq, xk, xv, hT, hH, hK, lf, hG, lg, B, D, L, y, q, u, s)
               : launch_striped_t<float, false>(xq, xk, xv, hT, hH, hK, lf, hG, lg, B, D, L, y, q, u, s);
}

cudaError_t launch_exp_sum_filter(const float* R, const float* lam, int d, int D, int L, float* h, cudaStream_t s) {
  const size_t n = (size_t)D * L;
  size_t blocks = (n + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  exp_sum_filter_kernel<<<(int)blocks, 256, 0, s>>>(R, lam, d, D, L, h);
  return cudaGetLastError();
}

}  // namespace hyena

using namespace hyena;

namespace {
bool st_aligned16(const void* q) { return q && ((reinterpret_cast<uintptr_t>(q) & 15u) == 0); }

hyena_status striped_check(const void* xq, const void* xk, const void* xv, const float* hT, const float* hH,
                           const float* hK, int lf, int B, int D, int L, hyena_dtype dtype) {
  if (B < 1 || D < 1 || L < 1 || lf < 1 || lf > kMaxStripedLF) return HYENA_ERR_INVALID_ARG;
  if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
  if (!st_aligned16(xq) || !st_aligned16(xk) || !st_aligned16(xv) || !st_aligned16(hT) || !st_aligned16(hH) ||
      !st_aligned16(hK))
    return HYENA_ERR_INVALID_ARG;
  if ((long long)B * D > (1LL << 40) / L) return HYENA_ERR_INVALID_ARG;
  return HYENA_OK;
}
}  // namespace

extern "C" {

hyena_status hyena_striped_forward(const void* xq, const void* xk, const void* xv, const float* hT, const float* hH,
                                   const float* hK, int lf, const float* hG, int lg, int B, int D, int L,
                                   hyena_dtype dtype, void* y, hyena_stream stream) {
  hyena_status st = striped_check(xq, xk, xv, hT, hH, hK, lf, B, D, L, dtype);
  if (st != HYENA_OK) return st;
  if (!st_aligned16(hG) || !st_aligned16(y) || lg < 1 || lg > kMaxStripedLG) return HYENA_ERR_INVALID_ARG;
  const cudaError_t e = launch_striped(xq, xk, xv, hT, hH, hK, lf, hG, lg, B, D, L, dtype == HYENA_BF16, y, nullptr,
                                       nullptr, (cudaStream_t)stream);
  return e == cudaSuccess ? HYENA_OK : report_cuda_error(e);
}

hyena_status hyena_striped_featurize(const void* xq, const void* xk, const void* xv, const float* hT,
                                     const float* hH, const float* hK, int lf, int B, int D, int L,
                                     hyena_dtype dtype, void* q, void* u, hyena_stream stream) {
  hyena_status st = striped_check(xq, xk, xv, hT, hH, hK, lf, B, D, L, dtype);
  if (st != HYENA_OK) return st;
  if (!st_aligned16(q) || !st_aligned16(u)) return HYENA_ERR_INVALID_ARG;
  const cudaError_t e = launch_striped(xq, xk, xv, hT, hH, hK, lf, nullptr, 0, B, D, L, dtype == HYENA_BF16, nullptr,
                                       q, u, (cudaStream_t)stream);
  return e == cudaSuccess ? HYENA_OK : report_cuda_error(e);
}

hyena_status hyena_filter_exponential(const float* R, const float* lambda, int d, int D, int L, float* h,
                                      hyena_stream stream) {
  if (!st_aligned16(R) || !st_aligned16(lambda) || !st_aligned16(h) || d < 1 || d > 64 || D < 1 || L < 1)
    return HYENA_ERR_INVALID_ARG;
  if ((long long)D * L > (1LL << 40)) return HYENA_ERR_INVALID_ARG;
  const cudaError_t e = launch_exp_sum_filter(R, lambda, d, D, L, h, (cudaStream_t)stream);
  return e == cudaSuccess ? HYENA_OK : report_cuda_error(e);
}

}  // extern "C"
