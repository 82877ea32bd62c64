// filter_gen.cu -- implicit Hyena filter (glossary "Hyena（ハイエナ）", section
// 暗黙的畳み込みフィルタ: h(t) = Window(t) * FFN(t/L, sin, cos)):
//   e(t)  = [t/L, sin(2 pi k t/L) k=1..K, cos(2 pi k t/L) k=1..K]
//   s1    = sin(W1 e + b1), s2 = sin(W2 s1 + b2), o = W3 s2 + b3
//   h_n[c][t] = o[n D + c] * exp(-alpha_c t / L), alpha_c = lo + (hi - lo) c / (D - 1)
// One CTA per tile of taps: the two hidden layers are computed once per tap
// and shared by all N*D outputs of the last layer (any width; the standard
// width 64 runs the register-tiled kernel below).
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

// Width-64 FFN (the standard width): the same computation with both 64-wide
// layers as register-tiled products. A CTA takes 64 taps; layer 2 gives each
// thread a 4 x 4 tile (taps x hidden units), the last layer an 8 x 8 tile
// (taps x outputs) of 8 x 4 per block of 128 outputs, with W3 staged through shared
// memory in chunks of 16 inputs, so an FMA costs about 1.1 instructions. The
// sums run over the same terms in float32 (in a different order).
constexpr int kFgT = 64;          // taps per CTA
constexpr int kFgH = 64;          // hidden width of this kernel
constexpr int kFgOB = 128;        // outputs per block of the last layer
constexpr int kFgKC = 16;         // inputs per staged W3 chunk
constexpr int kFgW3S = kFgOB + 4; // row stride of the staged chunk (2-way bank conflicts at most on its stores)

__global__ void __launch_bounds__(256, 2)
filter_gen64_kernel(const float* __restrict__ W1, const float* __restrict__ b1, const float* __restrict__ W2,
                    const float* __restrict__ b2, const float* __restrict__ W3, const float* __restrict__ b3,
                    int K, int N, int D, int L, float alpha_lo, float alpha_hi, float* __restrict__ h) {
  extern __shared__ __align__(16) float fs[];
  const int E = 1 + 2 * K;
  float* e = fs;                                  // [kFgT][E]
  float* s1T = e + kFgT * E;                      // [kFgH][kFgT]: s1 transposed (tap fastest)
  float* s2T = s1T + kFgH * kFgT;                 // [kFgH][kFgT]
  float* w2T = s2T + kFgH * kFgT;                 // [kFgH][kFgH]: W2 transposed (output fastest)
  float* w3c = w2T + kFgH * kFgH;                 // [kFgKC][kFgW3S]: chunk of W3 transposed
  const int t0 = blockIdx.x * kFgT;
  const int tid = threadIdx.x;
  const int NO = N * D;

  for (int idx = tid; idx < kFgT * E; idx += 256) {
    const int tt = idx / E, i = idx % E;
    const int t = t0 + tt;
    float val = 0.f;
    if (t < L) {
      if (i == 0) {
        val = (float)t / (float)L;
      } else {
        const int k = (i <= K) ? i : i - K;
        const long long num = (2LL * k * t) % (2LL * L);
        float s, c;
        sincospif((float)num / (float)L, &s, &c);
        val = (i <= K) ? s : c;
      }
    }
    e[idx] = val;
  }
  for (int idx = tid; idx < kFgH * kFgH; idx += 256) {
    const int o = idx / kFgH, i = idx % kFgH;
    w2T[i * kFgH + o] = __ldg(&W2[idx]);
  }
  __syncthreads();
  // layer 1 (E inputs, small): one (tap, unit) per thread per step
  for (int idx = tid; idx < kFgT * kFgH; idx += 256) {
    const int o = idx / kFgT, tt = idx % kFgT;
    float acc = __ldg(&b1[o]);
    for (int i = 0; i < E; ++i) acc = fmaf(__ldg(&W1[o * E + i]), e[tt * E + i], acc);
    s1T[o * kFgT + tt] = sinf(acc);
  }
  __syncthreads();
  // layer 2: thread (ty, tx) takes taps 4 tx .. 4 tx + 3 and units 4 ty .. 4 ty + 3
  {
    const int tx = tid % 16, ty = tid / 16;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = __ldg(&b2[4 * ty + b]);
#pragma unroll 8
    for (int i = 0; i < kFgH; ++i) {
      const float4 sv = *reinterpret_cast<const float4*>(s1T + i * kFgT + 4 * tx);
      const float4 wv = *reinterpret_cast<const float4*>(w2T + i * kFgH + 4 * ty);
      const float s4[4] = {sv.x, sv.y, sv.z, sv.w}, w4[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(w4[b], s4[a], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) s2T[(4 * ty + b) * kFgT + 4 * tx + a] = sinf(acc[a][b]);
  }
  // last layer + window: thread (ty, tx) takes taps 8 tx .. 8 tx + 7 and
  // outputs ob + 4 ty .. ob + 4 ty + 3 of each block of 128 outputs
  const int tx = tid % 8, ty = tid / 8;
  const int tb = t0 + 8 * tx;
  for (int ob = 0; ob < NO; ob += kFgOB) {
    float acc[8][4];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
    for (int k0 = 0; k0 < kFgH; k0 += kFgKC) {
      __syncthreads();   // s2T complete (first chunk); previous chunk consumed
      for (int idx = tid; idx < kFgKC * kFgOB; idx += 256) {
        const int oo = idx / kFgKC, kk = idx % kFgKC;
        const int o = ob + oo;
        w3c[kk * kFgW3S + oo] = (o < NO) ? __ldg(&W3[(size_t)o * kFgH + k0 + kk]) : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < kFgKC; ++kk) {
        const float4 s0 = *reinterpret_cast<const float4*>(s2T + (k0 + kk) * kFgT + 8 * tx);
        const float4 s1v = *reinterpret_cast<const float4*>(s2T + (k0 + kk) * kFgT + 8 * tx + 4);
        const float4 w0 = *reinterpret_cast<const float4*>(w3c + kk * kFgW3S + 4 * ty);
        const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1v.x, s1v.y, s1v.z, s1v.w};
        const float wv[4] = {w0.x, w0.y, w0.z, w0.w};
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(wv[b], sv[a], acc[a][b]);
      }
    }
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int o = ob + 4 * ty + b;
      if (o >= NO) break;
      const int c = o % D;
      const float alpha = (D > 1) ? alpha_lo + (alpha_hi - alpha_lo) * (float)c / (float)(D - 1) : alpha_lo;
      const float bias = __ldg(&b3[o]);
      float out[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) out[a] = (acc[a][b] + bias) * expf(-alpha * ((float)(tb + a) / (float)L));
      float* dst = h + (size_t)o * L + tb;
      if (tb + 8 <= L) {
        reinterpret_cast<float4*>(dst)[0] = make_float4(out[0], out[1], out[2], out[3]);
        reinterpret_cast<float4*>(dst)[1] = make_float4(out[4], out[5], out[6], out[7]);
      } else {
        for (int a = 0; a < 8; ++a)
          if (tb + a < L) dst[a] = out[a];
      }
    }
  }
}

cudaError_t launch_filter_generate(const float* W1, const float* b1, const float* W2, const float* b2,
                                   const float* W3, const float* b3, int n_bands, int width, int N, int D,
                                   int L, float alpha_lo, float alpha_hi, float* h, cudaStream_t s) {
  const int E = 1 + 2 * n_bands;
  if (width == kFgH && L % 8 == 0) {
    const size_t smem64 = sizeof(float) * ((size_t)kFgT * E + 2 * kFgH * kFgT + kFgH * kFgH + kFgKC * kFgW3S);
    cudaError_t e = cudaFuncSetAttribute((const void*)filter_gen64_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem64);
    if (e != cudaSuccess) return e;
    const int grid64 = (L + kFgT - 1) / kFgT;
    filter_gen64_kernel<<<grid64, 256, smem64, s>>>(W1, b1, W2, b2, W3, b3, n_bands, N, D, L, alpha_lo, alpha_hi, h);
    return cudaGetLastError();
  }
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
