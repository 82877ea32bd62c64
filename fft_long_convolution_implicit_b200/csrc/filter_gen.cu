// filter_gen.cu -- implicit Hyena filter (glossary "Hyena（ハイエナ）", section
// 暗黙的畳み込みフィルタ: h(t) = Window(t) * FFN(t/L, sin, cos)):
//   e(t)  = [t/L, sin(2 pi k t/L) k=1..K, cos(2 pi k t/L) k=1..K]
//   s1    = sin(W1 e + b1), s2 = sin(W2 s1 + b2), o = W3 s2 + b3
//   h_n[c][t] = o[n D + c] * exp(-alpha_c t / L), alpha_c = lo + (hi - lo) c / (D - 1)
// One CTA per tile of 32 taps: the two hidden layers are computed once per
// tap and shared by all N*D outputs of the last layer.
#include "kernels.cuh"

namespace hyena {

constexpr int kFgTaps = 32;
constexpr int kFgThreads = 256;

__global__ void __launch_bounds__(kFgThreads)
filter_gen_kernel(const float* __restrict__ W1, const float* __restrict__ b1, const float* __restrict__ W2,
                  const float* __restrict__ b2, const float* __restrict__ W3, const float* __restrict__ b3,
                  int K, int H, int N, int D, int L, float alpha_lo, float alpha_hi, float* __restrict__ h) {
  extern __shared__ float fs[];
  const int E = 1 + 2 * K;
  float* e = fs;                        // [32][E]
  float* s1 = e + kFgTaps * E;          // [32][H]
  float* s2 = s1 + kFgTaps * H;         // [32][H + 1]
  const int t0 = blockIdx.x * kFgTaps;
  const int tid = threadIdx.x;

  for (int idx = tid; idx < kFgTaps * E; idx += blockDim.x) {
    const int tt = idx / E, i = idx % E;
    const int t = t0 + tt;
    float val = 0.f;
    if (t < L) {
      if (i == 0) {
        val = (float)t / (float)L;
      } else {
        const int k = (i <= K) ? i : i - K;
        // angle 2 pi k t / L = pi * x with x = (2 k t mod 2L) / L, formed exactly
        const long long num = (2LL * k * t) % (2LL * L);
        float s, c;
        sincospif((float)num / (float)L, &s, &c);
        val = (i <= K) ? s : c;
      }
    }
    e[idx] = val;
  }
  __syncthreads();
  for (int idx = tid; idx < kFgTaps * H; idx += blockDim.x) {
    const int tt = idx / H, o = idx % H;
    float acc = __ldg(&b1[o]);
    for (int i = 0; i < E; ++i) acc = fmaf(__ldg(&W1[o * E + i]), e[tt * E + i], acc);
    s1[idx] = sinf(acc);
  }
  __syncthreads();
  for (int idx = tid; idx < kFgTaps * H; idx += blockDim.x) {
    const int tt = idx / H, o = idx % H;
    float acc = __ldg(&b2[o]);
    for (int i = 0; i < H; ++i) acc = fmaf(__ldg(&W2[o * H + i]), s1[tt * H + i], acc);
    s2[tt * (H + 1) + o] = sinf(acc);
  }
  __syncthreads();
  // last layer + window: warp w takes outputs w, w + 8, ...; lane = tap
  const int lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int t = t0 + lane;
  const float tl = (float)t / (float)L;
  const float* srow = s2 + lane * (H + 1);
  for (int o = warp; o < N * D; o += nwarps) {
    float acc = __ldg(&b3[o]);
    const float* w = W3 + (size_t)o * H;
    for (int i = 0; i < H; ++i) acc = fmaf(__ldg(&w[i]), srow[i], acc);
    const int c = o % D;
    const float alpha = (D > 1) ? alpha_lo + (alpha_hi - alpha_lo) * (float)c / (float)(D - 1) : alpha_lo;
    if (t < L) h[(size_t)o * L + t] = acc * expf(-alpha * tl);
  }
}

cudaError_t launch_filter_generate(const float* W1, const float* b1, const float* W2, const float* b2,
                                   const float* W3, const float* b3, int n_bands, int width, int N, int D,
                                   int L, float alpha_lo, float alpha_hi, float* h, cudaStream_t s) {
  const int E = 1 + 2 * n_bands;
  const size_t smem = sizeof(float) * (size_t)kFgTaps * (E + width + width + 1);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute((const void*)filter_gen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int grid = (L + kFgTaps - 1) / kFgTaps;
  filter_gen_kernel<<<grid, kFgThreads, smem, s>>>(W1, b1, W2, b2, W3, b3, n_bands, width, N, D, L, alpha_lo,
                                                   alpha_hi, h);
  return cudaGetLastError();
}

}  // namespace hyena
