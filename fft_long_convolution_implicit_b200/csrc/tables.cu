// tables.cu -- FFT tables kept at the end of every filter spectrum block.
//
//  tw_v[i]: twiddles of the MV-point Stockham plan (see fft_engine.cuh):
//           pass (Ns, R) keeps w_{Ns R}^{jm r} at (Ns - 1) + (r - 1) Ns + jm.
//  w_v[k]:  w_{2 MV}^k, k < MV (real-FFT unpack twiddle of the row transform).
//  tw_1[i]: twiddles of the M1-point column plan (radix 16, then radix M1/16).
// Values are formed in double with sincospi and rounded once to float.
#include <cuda_fp16.h>

#include "kernels.cuh"

namespace hyena {

struct PlanRadices {
  int n;
  int r[8];
};

static PlanRadices mv_plan(int logMV) {
  PlanRadices p{};
  const int mid = logMV - 7;
  p.r[p.n++] = 16;
  for (int i = 0; i < mid / 4; ++i) p.r[p.n++] = 16;
  if (mid % 4) p.r[p.n++] = 1 << (mid % 4);
  p.r[p.n++] = 8;
  return p;
}

static PlanRadices col_plan(int mb) {
  PlanRadices p{};
  p.r[p.n++] = 16;
  if (mb > 1) p.r[p.n++] = mb;
  return p;
}

__device__ float2 plan_entry(const PlanRadices& pl, int i) {
  int ns = 1;
  for (int q = 0; q < pl.n; ++q) {
    const int R = pl.r[q];
    if (ns > 1 && i >= ns - 1 && i < ns * R - 1) {
      const int off = i - (ns - 1);
      const int r = off / ns + 1, jm = off % ns;
      double s, c;
      sincospi(2.0 * (double)jm * (double)r / (double)(ns * R), &s, &c);
      return make_float2((float)c, (float)(-s));
    }
    ns *= R;
  }
  return make_float2(1.f, 0.f);
}

__global__ void fill_tables_kernel(float2* __restrict__ tab, PlanRadices pv, PlanRadices p1, int MV, int M1,
                                   int tw_v, int w_v, int tw_1, int table_len) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < MV) {
    tab[tw_v + i] = plan_entry(pv, i);
    double s, c;
    sincospi((double)i / (double)MV, &s, &c);
    tab[w_v + i] = make_float2((float)c, (float)(-s));
  }
  if (M1 > 1 && i < M1) tab[tw_1 + i] = plan_entry(p1, i);
  // padding entries
  const int used = tw_1 + (M1 > 1 ? M1 : 0);
  if (i < table_len - used) tab[used + i] = make_float2(0.f, 0.f);
}

cudaError_t launch_fill_tables(float2* tables, const Layout& y, cudaStream_t s) {
  const PlanRadices pv = mv_plan(y.logMV);
  const PlanRadices p1 = col_plan(y.fourstep ? y.mb : 0);
  const int n = y.MV > y.M1 ? y.MV : y.M1;
  fill_tables_kernel<<<(n + 255) / 256, 256, 0, s>>>(tables, pv, p1, y.MV, y.fourstep ? y.M1 : 0, y.tw_v, y.w_v,
                                                     y.tw_1, y.table_len);
  return cudaGetLastError();
}

}  // namespace hyena

namespace hyena {

// Reduced-precision copy of a spectrum block, one CTA per channel: bins as
// __half2 after multiplying by the power of two f_c that brings every
// component below 2^15 (the f16 range stops at 65504), and 1 / f_c per channel.
__global__ void spectrum_to_f16_kernel(const float2* __restrict__ spec, __half2* __restrict__ out,
                                       float* __restrict__ inv_scale, int M) {
  __shared__ float red[8];
  const int c = blockIdx.x, tid = threadIdx.x;
  const float2* __restrict__ row = spec + (size_t)c * M;
  float mx = 0.f;
  for (int i = tid; i < M; i += blockDim.x) mx = fmaxf(mx, fmaxf(fabsf(row[i].x), fabsf(row[i].y)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  __syncthreads();
  mx = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[w]);
  int e = (int)((__float_as_uint(mx) >> 23) & 0xff);    // mx < 2^(e - 126)
  e = e < 15 ? 15 : (e > 254 ? 254 : e);
  float f = __uint_as_float((unsigned)(268 - e) << 23);  // 2^(141 - e): mx f < 2^15
  float inv = __uint_as_float((unsigned)(e - 14) << 23); // 2^(e - 141)
  if (mx == 0.f) { f = 1.f; inv = 1.f; }
  for (int i = tid; i < M; i += blockDim.x)
    out[(size_t)c * M + i] = __floats2half2_rn(row[i].x * f, row[i].y * f);
  if (tid == 0) inv_scale[c] = inv;
}

cudaError_t launch_spectrum_to_f16(const float2* spec, unsigned char* out, int D, const Layout& y, cudaStream_t s) {
  spectrum_to_f16_kernel<<<D, 256, 0, s>>>(spec, reinterpret_cast<__half2*>(out),
                                           reinterpret_cast<float*>(out + spec16_scales_offset_bytes(y, D)), y.M);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the table region is copied as it is
  return cudaMemcpyAsync(out + spec16_tables_offset_bytes(y, D), spec + tables_offset(y, D),
                         sizeof(float2) * (size_t)y.table_len, cudaMemcpyDeviceToDevice, s);
}

}  // namespace hyena
