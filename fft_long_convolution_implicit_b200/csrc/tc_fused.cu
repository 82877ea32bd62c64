// tc_fused.cu -- Hyena order-N forward on tensor cores for bf16 I/O,
// L in {1024, 2048}, B even.
//
// Two batch items b, b+1 of one channel c share the filter h_c, so their
// causal convolutions are the real and imaginary parts of one complex
// convolution: c[t] = z_b[t] + i z_{b+1}[t] on the 2L zero-padded grid
// (glossary "Hyena（ハイエナ）", section 計算効率; "Native Multi-Dimensional
// Subquadratic Operators via Input Dependent Long Convolutions", section 境界の処理).
// Its 2L-point transform is split 2L = R0 * 256, m = 256 n0 + m', bin
// k = k0 + R0 k':
//   outer  (fp32 SIMT, thread m'): DFT_R0 over n0, twiddle w_{2L}^{m' k0};
//   inner  (warp, tensor cores):   256-point DFT over m' for each k0, as
//          16 x 16 DFT-matrix products (mma.sync m16n8k16, f16 in, f32 out):
//          T = F16 X, twiddle w_256^{k1 m2}, Y = T F16; the stage-one
//          accumulators are the stage-two A operand without leaving registers;
//   product with the filter spectrum (fp32), the inverse 256-point DFT as the
//          forward one of the conjugate (one 8x8 movmatrix transpose per tile),
//          and the outer inverse over k0 keeping n0 < R0/2 (t < L).
// The gate x_n multiplies real and imaginary parts separately, and the output
// of the last outer inverse pass is exactly the input of the next stage's outer
// forward pass, so z stays in registers between stages.
// f16 operands are scaled per warp by a power of two (maximum magnitude 2^10)
// and unscaled exactly after each 256-point transform.
#include <cuda_fp16.h>

#include "fft_engine.cuh"
#include "kernels.cuh"
#include "tc_dft.cuh"

namespace hyena {

constexpr int kTcThreads = 256;

template <int R0>
struct TcCfg {
  static constexpr int L = 128 * R0;
  static constexpr int XS = 18;            // padded row stride (float2) of a 16 x 16 block
  static constexpr int XBLK = 16 * XS;     // float2 per k0 block
  static constexpr int KPW = R0 / 8;       // 256-point transforms per warp
  static constexpr size_t x_bytes = sizeof(float2) * R0 * XBLK;
  static constexpr size_t h_bytes = sizeof(float2) * (L + 2);   // bins, (1/f_c, 0), padding
  static constexpr size_t row_bytes = sizeof(__nv_bfloat16) * 2 * L;   // rows b and b+1
  // two spectrum and two gate buffers (job parity), one input buffer
  static constexpr size_t total = x_bytes + 2 * h_bytes + 3 * row_bytes;
};

__device__ __forceinline__ float2 bf2_to_f2(unsigned int u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
__device__ __forceinline__ float bf_to_f(unsigned short u) { return __uint_as_float((unsigned)u << 16); }

template <int R0>
__device__ __forceinline__ void outer_dft_fwd(float2 (&a)[R0]) {
  if constexpr (R0 == 16) {
    dft16<false, true, false, 0>(a);
  } else {
    a[4] = a[5] = a[6] = a[7] = make_float2(0.f, 0.f);
    dft8<false, 0>(a);
  }
}
// forward DFT_R0 keeping outputs n0 < R0/2 (the inverse of conjugated data)
template <int R0>
__device__ __forceinline__ void outer_dft_fwd_half_out(float2 (&a)[R0]) {
  if constexpr (R0 == 16) dft16<false, false, true, 0>(a);
  else dft8<false, 0>(a);
}


template <int R0>
__global__ void __launch_bounds__(kTcThreads, 2)
tc_forward_kernel(const __nv_bfloat16* __restrict__ v, GatePtrs<__nv_bfloat16> x, SpecPtrs hh,
                  __nv_bfloat16* __restrict__ y, const float2* __restrict__ otw, int B, int D, int N,
                  long long npairs) {
  using Cfg = TcCfg<R0>;
  constexpr int L = Cfg::L, XS = Cfg::XS, XBLK = Cfg::XBLK, HROW = L + 2;
  extern __shared__ __align__(16) float2 sm[];
  __shared__ float red[kTcThreads / 32];
  float2* X = sm;
  float2* Hbuf = sm + R0 * XBLK;                                          // [2][HROW]
  unsigned short* xbuf = reinterpret_cast<unsigned short*>(Hbuf + 2 * HROW);   // [2][2][L] gate rows
  unsigned short* vs = xbuf + 4 * L;                                      // [2][L] input rows
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int mp = tid;                                   // m' of the outer passes
  float2* Xo = X + (mp >> 4) * XS + (mp & 15);

  Dft16Frags F;
  build_frags(F, g, t);
  Tw256 tw;
  build_tw256(tw, g, t);

  const int Bh = B >> 1;
  const int row_bytes = L * 2;
  auto pair_rows = [&](long long pp, size_t& r0, size_t& r1, int& c) {
    c = (int)(pp / Bh);
    const int b0 = 2 * (int)(pp % Bh);
    r0 = ((size_t)b0 * D + c) * (size_t)L;
    r1 = r0 + (size_t)D * L;
  };
  // A job is one stage of one pair; its spectrum row and gate rows are staged
  // into the buffers of its parity during the previous job.
  auto stage_job = [&](long long pp, int n, int par) {
    size_t q0, q1;
    int qc;
    pair_rows(pp, q0, q1, qc);
    block_copy_async(Hbuf + par * HROW, pick(hh, n) + (size_t)qc * HROW, HROW * (int)sizeof(float2), tid,
                     kTcThreads);
    block_copy_async(xbuf + par * 2 * L, pick(x, n) + q0, row_bytes, tid, kTcThreads);
    block_copy_async(xbuf + par * 2 * L + L, pick(x, n) + q1, row_bytes, tid, kTcThreads);
  };
  long long p = blockIdx.x;
  int par = 0;
  if (p < npairs) {
    size_t r0, r1;
    int c;
    pair_rows(p, r0, r1, c);
    block_copy_async(vs, v + r0, row_bytes, tid, kTcThreads);
    block_copy_async(vs + L, v + r1, row_bytes, tid, kTcThreads);
    stage_job(p, 0, 0);
    cp_async_commit();
    cp_async_wait_all();
  }
  __syncthreads();

  for (; p < npairs; p += gridDim.x) {
    size_t r0, r1;
    int c;
    pair_rows(p, r0, r1, c);
    float2 a[R0];
    float zm = 0.f;
#pragma unroll
    for (int n0 = 0; n0 < R0 / 2; ++n0) {
      a[n0] = make_float2(bf_to_f(vs[256 * n0 + mp]), bf_to_f(vs[L + 256 * n0 + mp]));
      zm = fmaxf(zm, fmaxf(fabsf(a[n0].x), fabsf(a[n0].y)));
    }
    zm = warp_max(zm);
    if (lane == 0) red[warp] = zm;
    __syncthreads();

    for (int n = 0; n < N; ++n, par ^= 1) {
      const float2* Hs = Hbuf + par * HROW;
      const unsigned short* xs = xbuf + par * 2 * L;
      // scale bringing the outer transform's output below 2^10 (|X| <= R0 max|z|)
      float zmax = red[0];
#pragma unroll
      for (int w = 1; w < kTcThreads / 32; ++w) zmax = fmaxf(zmax, red[w]);
      float s, inv_s;
      pow2_scale((float)R0 * zmax, s, inv_s);
#pragma unroll
      for (int n0 = 0; n0 < R0 / 2; ++n0) a[n0] = make_float2(a[n0].x * s, a[n0].y * s);
#pragma unroll
      for (int n0 = R0 / 2; n0 < R0; ++n0) a[n0] = make_float2(0.f, 0.f);
      // ---- outer forward: DFT_R0 over n0, twiddle, to X[k0][m']
      outer_dft_fwd<R0>(a);
#pragma unroll
      for (int k0 = 1; k0 < R0; ++k0) a[k0] = cmul(a[k0], __ldg(otw + k0 * 256 + mp));
#pragma unroll
      for (int k0 = 0; k0 < R0; ++k0) Xo[k0 * XBLK] = a[k0];
      cp_async_wait_all();       // this job's spectrum and gate rows (staged last job) have landed
      __syncthreads();
      // the next pair's input rows (free: read at this pair's start) in their own group
      if (n == 0) {
        if (p + gridDim.x < npairs) {
          size_t q0, q1;
          int qc;
          pair_rows(p + gridDim.x, q0, q1, qc);
          block_copy_async(vs, v + q0, row_bytes, tid, kTcThreads);
          block_copy_async(vs + L, v + q1, row_bytes, tid, kTcThreads);
        }
        cp_async_commit();
      }
      // stage the next job into the other buffers (free: last read by the previous job)
      if (n + 1 < N) {
        stage_job(p, n + 1, par ^ 1);
      } else if (p + gridDim.x < npairs) {
        stage_job(p + gridDim.x, 0, par ^ 1);
      }
      cp_async_commit();
      const float inv_f = Hs[L].x;   // the spectrum copy is scaled by f_c, |H f_c| < 2^-9

      // ---- inner: 256-point transforms on tensor cores, spectral product, inverse
#pragma unroll
      for (int q = 0; q < Cfg::KPW; ++q) {
        const int k0 = warp + 8 * q;
        float2* Xb = X + k0 * XBLK;
        float2 vin[4][2];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int m1 = 2 * t + (qq & 1) + 8 * (qq >> 1);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) vin[qq][nt] = Xb[m1 * XS + 8 * nt + g];
        }
        float Dm[4][4];
        dft256_fwd(F, tw, vin, Dm);

        // spectral product with the cached filter spectrum (tensor-core order,
        // [k0][k1][k2 < 8]; bins k2 >= 8 are conjugate mirrors). |Y| < 2^10.
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int k1 = g + 8 * i;
          const float4 hd4 = *reinterpret_cast<const float4*>(Hs + k0 * 128 + k1 * 8 + 2 * t);
          float2 hd0 = make_float2(hd4.x, hd4.y), hd1 = make_float2(hd4.z, hd4.w);
          float2 hm0, hm1;
          if (k0 != 0 || k1 != 0) {
            const int mrow = (k0 != 0) ? ((R0 - k0) * 128 + (15 - k1) * 8) : ((16 - k1) * 8);
            const float4 q4 = *reinterpret_cast<const float4*>(Hs + mrow + 6 - 2 * t);
            hm0 = make_float2(q4.z, -q4.w);
            hm1 = make_float2(q4.x, -q4.y);
          } else {
            const float2 h0 = Hs[0];
            const float2 hn0 = Hs[8 - 2 * t];
            const float2 hn1 = Hs[7 - 2 * t];
            hm0 = (t == 0) ? make_float2(h0.y, 0.f) : make_float2(hn0.x, -hn0.y);
            hm1 = make_float2(hn1.x, -hn1.y);
            if (t == 0) hd0 = make_float2(h0.x, 0.f);
          }
          const float2 hb[2][2] = {{hd0, hd1}, {hm0, hm1}};
#pragma unroll
          for (int jn = 0; jn < 2; ++jn)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float re = Dm[jn][2 * i + e], im = Dm[2 + jn][2 * i + e];
              const float2 hv = hb[jn][e];
              Dm[jn][2 * i + e] = re * hv.x - im * hv.y;
              Dm[2 + jn][2 * i + e] = re * hv.y + im * hv.x;
            }
        }
        float G[2][2][4];
        dft256_inv(F, tw, Dm, G);
        // G = conj(x) (scaled by s f_c) back to X[k0][16 m1 + m2]
#pragma unroll
        for (int np = 0; np < 2; ++np)
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int m1 = g + 8 * i;
            *reinterpret_cast<float4*>(Xb + m1 * XS + 8 * np + 2 * t) =
                make_float4(G[0][np][2 * i], G[1][np][2 * i], G[0][np][2 * i + 1], G[1][np][2 * i + 1]);
          }
      }
      __syncthreads();
      // ---- outer inverse over k0 (t < L only), on conjugated data, and the gate
#pragma unroll
      for (int k0 = 0; k0 < R0; ++k0) a[k0] = Xo[k0 * XBLK];
#pragma unroll
      for (int k0 = 1; k0 < R0; ++k0) a[k0] = cmul(a[k0], __ldg(otw + k0 * 256 + mp));
      outer_dft_fwd_half_out<R0>(a);
      const float u = inv_s * inv_f;
      zm = 0.f;
#pragma unroll
      for (int n0 = 0; n0 < R0 / 2; ++n0) {
        const int tt = 256 * n0 + mp;
        a[n0] = make_float2(a[n0].x * (u * bf_to_f(xs[tt])), a[n0].y * (-u * bf_to_f(xs[L + tt])));
        zm = fmaxf(zm, fmaxf(fabsf(a[n0].x), fabsf(a[n0].y)));
      }
      zm = warp_max(zm);
      if (lane == 0) red[warp] = zm;
      // before the next pair reads its input rows: every group but the newest
      // (the next job's staging) is complete
      if (n + 1 == N) cp_async_wait_all_but_newest();
      __syncthreads();           // X, the gate rows and red are reused by the next stage
    }
#pragma unroll
    for (int n0 = 0; n0 < R0 / 2; ++n0) {
      const int tt = 256 * n0 + mp;
      y[r0 + tt] = __float2bfloat16_rn(a[n0].x);
      y[r1 + tt] = __float2bfloat16_rn(a[n0].y);
    }
  }
  cp_async_wait_all();
}

// Tensor-core copy of one channel's spectrum (one CTA per channel):
// S[k0][k1][k2 < 8] = 2 f_c nat[k0 + R0 (k1 + 16 k2)] (the natural copy holds
// rfft / (4L), this one rfft / (2L)), entry 0 packing (H[0], H[L]), then
// (1 / f_c, 0) and a zero pad. f_c is the power of two that brings every
// component of the scaled spectrum below 2^-9.
__global__ void tc_spectrum_kernel(const float2* __restrict__ nat, float2* __restrict__ tcs, int R0, int M) {
  __shared__ float red[256 / 32];
  const int L = 128 * R0, c = blockIdx.x, tid = threadIdx.x;
  const float2* __restrict__ nr = nat + (size_t)c * M;
  float2* __restrict__ row = tcs + (size_t)c * (L + 2);
  float mx = 0.f;
  for (int i = tid; i < L; i += blockDim.x) mx = fmaxf(mx, fmaxf(fabsf(nr[i].x), fabsf(nr[i].y)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  __syncthreads();
  mx = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[w]);
  const float hc = 2.f * mx;                                  // component bound of 2 * nat
  int e = (int)((__float_as_uint(hc) >> 23) & 0xff);          // hc < 2^(e - 126)
  e = e < 1 ? 1 : (e > 243 ? 243 : e);
  float f = __uint_as_float((unsigned)(244 - e) << 23);       // 2^(117 - e)
  float inv_f = __uint_as_float((unsigned)(e + 10) << 23);    // 2^(e - 117)
  if (hc == 0.f) { f = 1.f; inv_f = 1.f; }
  for (int r = tid; r < L; r += blockDim.x) {
    const int k0 = r >> 7, k1 = (r >> 3) & 15, k2 = r & 7;
    const float2 h = nr[k0 + R0 * (k1 + 16 * k2)];
    row[r] = make_float2(2.f * f * h.x, 2.f * f * h.y);
  }
  if (tid == 0) {
    row[L] = make_float2(inv_f, 0.f);
    row[L + 1] = make_float2(0.f, 0.f);
  }
}

// w_{256 R0}^{m k0} for k0 < R0, m < 256
__global__ void tc_otw_kernel(float2* __restrict__ otw, int R0) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R0 * 256) return;
  const int k0 = i / 256, m = i % 256;
  double s, c;
  sincospi(-2.0 * (double)((m * k0) % (256 * R0)) / (double)(256 * R0), &s, &c);
  otw[i] = make_float2((float)c, (float)s);
}

template <int R0>
static cudaError_t launch_tc_r(const FusedLaunch& p, const float2* otw, cudaStream_t s) {
  auto k = tc_forward_kernel<R0>;
  const size_t smem = TcCfg<R0>::total;
  int grid = 0;
  cudaError_t e = persistent_grid((const void*)k, kTcThreads, smem, &grid);
  if (e != cudaSuccess) return e;
  const long long npairs = (long long)(p.B / 2) * p.D;
  if ((long long)grid > npairs) grid = (int)npairs;
  GatePtrs<__nv_bfloat16> xp;
  for (int i = 0; i < kMaxOrder; ++i) xp.p[i] = reinterpret_cast<const __nv_bfloat16*>(p.x[i]);
  k<<<grid, kTcThreads, smem, s>>>(reinterpret_cast<const __nv_bfloat16*>(p.v), xp, p.hh,
                                   reinterpret_cast<__nv_bfloat16*>(p.y), otw, p.B, p.D, p.N, npairs);
  return cudaGetLastError();
}

cudaError_t launch_tc_forward(const FusedLaunch& p, const Layout& y, cudaStream_t s) {
  const float2* otw = p.tables + y.tc_otw;
  if (y.R0 == 8) return launch_tc_r<8>(p, otw, s);
  if (y.R0 == 16) return launch_tc_r<16>(p, otw, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_tc_spectrum(const float2* nat, float2* tcs, float2* tables, int D, const Layout& y,
                               cudaStream_t s) {
  tc_spectrum_kernel<<<D, 256, 0, s>>>(nat, tcs, y.R0, y.M);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  tc_otw_kernel<<<(y.R0 * 256 + 255) / 256, 256, 0, s>>>(tables + y.tc_otw, y.R0);
  return cudaGetLastError();
}

}  // namespace hyena
