// fourstep.cu -- Hyena order-N forward for 8192 < L <= 2^20.
//
// The packed M-point transform (M = L) is split M = M1 * MV, input index
// m = MV n1 + n2, output bin k = k1 + M1 k2:
//   column pass: M1-point DFTs over n1 for each n2  -> A[k1][n2]
//   row pass:    twiddle w_M^{n2 k1}, MV-point FFT over n2 -> bins k1 + M1 k2;
//                rows k1 and M1-k1 hold mirror bins, so one CTA takes both,
//                forms the spectral product and runs the inverse row FFT and
//                conjugate twiddle in place             -> E[k1][n2]
//   column pass: inverse M1-point DFTs over k1, keep n1 < M1/2 (first L real
//                outputs), gate with x_n, and -- between stages -- the next
//                stage's forward column DFTs on the same column.
// A channel's A/E array lives in a caller workspace and is visited by
// 2N + 1 launches per wave of channels; waves are sized by the workspace so
// that the array stays resident in L2.
#include "kernels.cuh"
#include "mbar.cuh"
#include "paired.cuh"

namespace hyena {

// Row pass spectrum rows fed by bulk copies into shared memory (issued when
// the CTA starts, waited for before the paired pass) for rows of up to
// 2^HYENA_ROW_BULK_MAX_LOG points, else read from global memory inside the
// paired pass. Measured: rows of 1024 (L = 2^17) 0.702 -> 0.683 ms per
// forward with the copies; rows of 4096 (L = 2^20) 7.69 -> 7.95 ms, where the
// 64 KB of staged rows leave the one resident CTA less L1 for its scratch rows.
#ifndef HYENA_ROW_BULK_MAX_LOG
#define HYENA_ROW_BULK_MAX_LOG 10
#endif

__device__ int g_fourstep_timeout;

enum ColMode { kColFirst = 0, kColMid = 1, kColLast = 2, kColSpecFirst = 3 };

template <int MB>
struct ColCfg {
  static constexpr int M1 = 16 * MB;
  // columns per CTA: 16 once the columns reach 64 points (two resident CTAs of
  // 16 x MB threads overlap each other's barriers; 3 % faster than 32 at
  // L = 2^17 and 2^20), and 128 B of every row per CTA either way
  static constexpr int CW = MB == 1 ? 128 : (MB == 2 ? 64 : 16);
  static constexpr int THREADS = CW * MB;
  static constexpr int VEC = padded_len(M1) + 1;                  // smem stride of one column
  static constexpr size_t SMEM = MB == 1 ? 0 : sizeof(float2) * (size_t)CW * VEC;
};

// exp(-2 pi i e / M) for an integer exponent e in [0, M)
__device__ __forceinline__ float2 expi_neg(int e, int M) {
  float s, c;
  sincospif(2.0f * (float)e / (float)M, &s, &c);
  return make_float2(c, -s);
}

// Column pass. Thread (j, col): column n2 = tile*CW + col; in the 16-point
// stage it owns rows n1 = j + r*MB; in the MB-point stage butterflies
// jj = j + q*MB (bins jj + 16 r).
template <int MB, int MODE, typename T>
__global__ void __launch_bounds__(ColCfg<MB>::THREADS)
col_kernel(const T* __restrict__ zin, const T* __restrict__ gate, T* __restrict__ yout, float2* __restrict__ scr,
           const float2* __restrict__ tw1, int B, int D, int L, int MV, long long ch0,
           const float* __restrict__ inv_scale, unsigned* __restrict__ xmax) {
  using Cfg = ColCfg<MB>;
  constexpr int M1 = Cfg::M1, CW = Cfg::CW, NQ = 16 / MB;
  extern __shared__ float2 sm[];
  const int tid = threadIdx.x;
  const int col = tid % CW, j = tid / CW;
  const int n2 = blockIdx.x * CW + col;
  const long long ch = ch0 + blockIdx.y;
  const int c = (int)(ch / B), b = (int)(ch % B);
  const size_t row = ((size_t)b * D + c) * (size_t)L;
  float2* __restrict__ S = scr + (size_t)blockIdx.y * ((size_t)M1 * MV);
  float2* csm = sm + col * Cfg::VEC;
  float2 a[16];

  if constexpr (MODE == kColFirst || MODE == kColSpecFirst) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const size_t m = (size_t)MV * (j + r * MB) + n2;
      a[r] = IO<T>::load2_stream(zin + row + 2 * m);
    }
  } else {
    if constexpr (MB == 1) {
#pragma unroll
      for (int r = 0; r < 16; ++r) a[r] = S[(size_t)r * MV + n2];
    } else {
#pragma unroll
      for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int r = 0; r < MB; ++r) a[q * MB + r] = S[(size_t)(j + q * MB + 16 * r) * MV + n2];
      dft_blocks<MB, true>(a);
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int jj = j + q * MB;
#pragma unroll
        for (int r = 1; r < MB; ++r) a[q * MB + r] = cmulc(a[q * MB + r], __ldg(&tw1[15 + (r - 1) * 16 + jj]));
#pragma unroll
        for (int r = 0; r < MB; ++r) csm[pidx(jj + 16 * r)] = a[q * MB + r];
      }
      __syncthreads();
#pragma unroll
      for (int r = 0; r < 16; ++r) a[r] = csm[pidx(16 * j + r)];
    }
    dft16<true, false, true, 0>(a);          // outputs n1 = j + r*MB, r < 8
    // reduced-precision spectra: the channel's exact inverse scale joins the gate
    const float inv = inv_scale ? __ldg(inv_scale + c) : 1.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const size_t m = (size_t)MV * (j + r * MB) + n2;
      const float2 g = IO<T>::load2_stream(gate + row + 2 * m);
      a[r] = make_float2(a[r].x * (g.x * inv), a[r].y * (g.y * inv));
    }
    if constexpr (MODE == kColLast) {
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const size_t m = (size_t)MV * (j + r * MB) + n2;
        IO<T>::store2(yout + row + 2 * m, a[r]);
      }
      return;
    }
  }
  // forward column transform (upper half of the column is zero)
  dft16<false, true, false, 0>(a);
  // largest component of the channel's column outputs (float bits order as
  // unsigned integers for non-negative values), for the tensor-core row pass
  auto record_max = [&]() {
    if (xmax == nullptr) return;
    float mx = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r) mx = fmaxf(mx, fmaxf(fabsf(a[r].x), fabsf(a[r].y)));
    const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
    if ((threadIdx.x & 31) == 0) atomicMax(xmax + blockIdx.y, m);
  };
  if constexpr (MB == 1) {
#pragma unroll
    for (int r = 0; r < 16; ++r) S[(size_t)r * MV + n2] = a[r];
    record_max();
  } else {
#pragma unroll
    for (int r = 0; r < 16; ++r) csm[pidx(16 * j + r)] = a[r];
    __syncthreads();
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int jj = j + q * MB;
#pragma unroll
      for (int r = 0; r < MB; ++r) a[q * MB + r] = csm[pidx(jj + 16 * r)];
#pragma unroll
      for (int r = 1; r < MB; ++r) a[q * MB + r] = cmul(a[q * MB + r], __ldg(&tw1[15 + (r - 1) * 16 + jj]));
    }
    dft_blocks<MB, false>(a);
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
      for (int r = 0; r < MB; ++r) S[(size_t)(j + q * MB + 16 * r) * MV + n2] = a[q * MB + r];
    record_max();
  }
}

// Row pass on rows kA and kB (kA + kB = M1, or the self-mirrored rows 0 and
// M1/2 in CTA 0). Threads [0, TV) work on row kA, [TV, 2 TV) on row kB.
// The two spectrum rows of the pair are fetched by one thread with two bulk
// copies into shared memory while the forward row FFT runs (byte-counted on
// an mbarrier, bounded wait before the paired pass).
// Resident row-pair CTAs per SM the register budget is sized for: 512 threads
// per SM (rows of 1024 points: 4 CTAs of 128 threads at <= 128 registers,
// measured 8 % faster than the unbounded 137 registers and 3 CTAs).
template <int LOGMV>
constexpr int row_blocks() {
  return 512 / (2 * Plan<LOGMV>::TV) > 1 ? 512 / (2 * Plan<LOGMV>::TV) : 1;
}

template <int LOGMV, int MODE, typename HT>
struct RowSmem {
  static constexpr int MV = 1 << LOGMV;
  static constexpr bool bulk = LOGMV <= HYENA_ROW_BULK_MAX_LOG && MODE == kPairConv;
  static constexpr size_t data = sizeof(float2) * 2 * (size_t)padded_len(MV);
  static constexpr size_t spec_row = sizeof(HT) * (size_t)MV;   // bytes of one staged spectrum row
  static constexpr size_t total = data + (bulk ? 2 * spec_row : 0);
};

template <int LOGMV, int MODE, typename HT = float2>
__global__ void __launch_bounds__(2 * Plan<LOGMV>::TV, row_blocks<LOGMV>())
row_kernel(float2* __restrict__ scr, const float2* __restrict__ spec, const float2* __restrict__ tables, int M1,
           int B, long long ch0) {
  using P = Plan<LOGMV>;
  using RS = RowSmem<LOGMV, MODE, HT>;
  constexpr int MV = P::MV, TV = P::TV, Q8 = MV / 8, Q16 = MV / 16, VEC = padded_len(MV);
  extern __shared__ __align__(16) float2 sm[];
  __shared__ __align__(8) uint64_t hbar;
  const int M = M1 * MV;
  const float2* __restrict__ tw = tables;
  const float2* __restrict__ Wv = tables + MV;
  const int p = blockIdx.x;
  const int kA = p, kB = (p == 0) ? M1 / 2 : M1 - p;
  float2* S = scr + (size_t)blockIdx.y * M;
  HT* H;
  if constexpr (MODE == kPairConv) {
    const long long ch = ch0 + blockIdx.y;
    H = reinterpret_cast<HT*>(const_cast<float2*>(spec)) + (size_t)(ch / B) * M;
  } else {
    H = S;   // spectrum block of channel blockIdx.y, transformed in place
  }
  const int t = threadIdx.x;
  const int vec = t / TV, tl = t % TV;
  const int krow = vec ? kB : kA;
  float2* base = sm + vec * VEC;
  float2* src = S + (size_t)krow * MV;
  HT* hs = reinterpret_cast<HT*>(reinterpret_cast<char*>(sm) + RS::data);   // staged rows kA, kB
  if constexpr (RS::bulk) {
    if (t == 0) {
      const uint32_t bar = smem_u32(&hbar);
      mbar_init(bar, 1);
      mbar_init_fence();
      mbar_arrive_expect_tx(bar, (uint32_t)(2 * RS::spec_row));
      const uint64_t pol = l2_policy_evict_first();   // spectrum rows are read once per stage
      bulk_g2s_policy(smem_u32(hs), H + (size_t)kA * MV, (uint32_t)RS::spec_row, bar, pol);
      bulk_g2s_policy(smem_u32(hs + MV), H + (size_t)kB * MV, (uint32_t)RS::spec_row, bar, pol);
    }
    // the barrier after the first forward pass publishes the initialised mbarrier
  }

  // four-step twiddle w_M^{krow n2}, n2 = tl + r*Q16
  const float2 tw0 = expi_neg((int)(((long long)krow * tl) % M), M);
  const float2 tstep = expi_neg((int)(((long long)krow * Q16) % M), M);
  float2 a[16];
#pragma unroll
  for (int r = 0; r < 16; ++r) a[r] = src[tl + r * Q16];
  {
    float2 cur = tw0;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      a[r] = cmul(a[r], cur);
      cur = cmul(cur, tstep);
    }
  }
  dft16<false, false, false, 0>(a);
  store_block16(base, tl, a);
  __syncthreads();
  mid_fwd_all<LOGMV>(a, base, tw, tl);

  {
    float2 *bA, *bB;
    HT *HA, *HB;
    int jA, jB;
    bool head = false, has_rho = true;
    float2 rho;
    if (p != 0) {
      bA = sm; bB = sm + VEC;
      jA = t; jB = Q8 - 1 - t;
      float s, c;
      sincospif((float)kA / (float)M, &s, &c);
      rho = make_float2(c, -s);
      HA = RS::bulk ? hs : H + (size_t)kA * MV;
      HB = RS::bulk ? hs + MV : H + (size_t)kB * MV;
    } else if (t < Q16) {
      bA = bB = sm;
      head = (t == 0);
      jA = head ? 0 : t; jB = head ? Q16 : Q8 - t;
      rho = make_float2(1.f, 0.f); has_rho = false;
      HA = HB = RS::bulk ? hs : H;
    } else {
      const int t2 = t - Q16;
      bA = bB = sm + VEC;
      jA = t2; jB = Q8 - 1 - t2;
      float s, c;
      sincospif((float)(M1 / 2) / (float)M, &s, &c);
      rho = make_float2(c, -s);
      HA = HB = RS::bulk ? hs + MV : H + (size_t)(M1 / 2) * MV;
    }
    if constexpr (RS::bulk) {
      if (!mbar_wait(smem_u32(&hbar), 0)) {
        atomicExch(&g_fourstep_timeout, 1);
        mbar_wait(smem_u32(&hbar), 0, 1000000000ull);   // bounded second wait for the copies in flight
      }
      paired_pass<LOGMV, MODE, true, HT>(bA, bB, jA, jB, head, tw, Wv, rho, has_rho, HA, HB, 1.0f / (8.0f * (float)M));
    } else {
      paired_pass<LOGMV, MODE, false, HT>(bA, bB, jA, jB, head, tw, Wv, rho, has_rho, HA, HB,
                                          1.0f / (8.0f * (float)M));
    }
  }
  if (MODE == kPairSpectrum) return;
  __syncthreads();
  mid_inv_all<LOGMV>(a, base, tw, tl);
  load_block16(base, tl, a);
  dft16<true, false, false, 0>(a);
  {
    float2 cur = tw0;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      a[r] = cmulc(a[r], cur);
      cur = cmul(cur, tstep);
    }
  }
#pragma unroll
  for (int r = 0; r < 16; ++r) src[tl + r * Q16] = a[r];
}

// ------------------------------------------------------------- launchers --

template <typename K>
static cudaError_t prep(K kernel, size_t smem) {
  if (smem > 48 * 1024) return cudaFuncSetAttribute((const void*)kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  return cudaSuccess;
}

template <int MB, int MODE, typename T>
static cudaError_t launch_col(const T* zin, const T* gate, T* yout, float2* scr, const float2* tw1, int B, int D,
                              int L, int MV, long long ch0, int nch, cudaStream_t s,
                              const float* inv_scale = nullptr, unsigned* xmax = nullptr) {
  using Cfg = ColCfg<MB>;
  auto k = col_kernel<MB, MODE, T>;
  cudaError_t e = prep(k, Cfg::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid(MV / Cfg::CW, nch);
  k<<<grid, Cfg::THREADS, Cfg::SMEM, s>>>(zin, gate, yout, scr, tw1, B, D, L, MV, ch0, inv_scale, xmax);
  return cudaGetLastError();
}

template <int LOGMV, int MODE, typename HT = float2>
static cudaError_t launch_row(float2* scr, const float2* spec, const float2* tables, int M1, int B, long long ch0,
                              int nch, cudaStream_t s) {
  auto k = row_kernel<LOGMV, MODE, HT>;
  const size_t smem = RowSmem<LOGMV, MODE, HT>::total;
  cudaError_t e = prep(k, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(M1 / 2, nch);
  k<<<grid, 2 * Plan<LOGMV>::TV, smem, s>>>(scr, spec, tables, M1, B, ch0);
  return cudaGetLastError();
}

template <int LOGMV, int MB, typename T, typename HT>
static cudaError_t wave_t(const FourStepLaunch& p, const Layout& y, cudaStream_t s) {
  const float2* tw1 = p.tables + y.tw_1;
  const int MV = y.MV;
  // tensor-core rows: stage n reads the column maxima in buffer n & 1 and
  // clears the other for the column pass that feeds stage n + 1
  unsigned* xm[2] = {p.tcr ? p.xmax : nullptr, p.tcr ? p.xmax + p.wave : nullptr};
  cudaError_t e = launch_col<MB, kColFirst, T>(reinterpret_cast<const T*>(p.v), nullptr, nullptr, p.scratch, tw1,
                                               p.B, p.D, p.L, MV, p.ch0, p.wave, s, nullptr, xm[0]);
  for (int n = 0; n < p.N && e == cudaSuccess; ++n) {
    if (p.tcr)
      e = launch_tcr_rows(p.scratch, p.hhalf[n], p.hmax[n], xm[n & 1], xm[(n + 1) & 1], y.M1, p.B, p.ch0, p.wave,
                          s);
    else
      e = launch_row<LOGMV, kPairConv, HT>(p.scratch, p.hh.p[n], p.tables, y.M1, p.B, p.ch0, p.wave, s);
    if (e != cudaSuccess) break;
    const float* inv = nullptr;
    if (sizeof(HT) != sizeof(float2))
      inv = reinterpret_cast<const float*>(reinterpret_cast<const char*>(p.hh.p[n]) + spec16_scales_offset_bytes(y, p.D));
    const T* g = reinterpret_cast<const T*>(p.x[n]);
    if (n + 1 < p.N)
      e = launch_col<MB, kColMid, T>(nullptr, g, nullptr, p.scratch, tw1, p.B, p.D, p.L, MV, p.ch0, p.wave, s, inv,
                                     xm[(n + 1) & 1]);
    else
      e = launch_col<MB, kColLast, T>(nullptr, g, reinterpret_cast<T*>(p.y), p.scratch, tw1, p.B, p.D, p.L, MV,
                                      p.ch0, p.wave, s, inv);
  }
  return e;
}

template <int LOGMV, int MB>
static cudaError_t wave_lm(const FourStepLaunch& p, const Layout& y, cudaStream_t s) {
  if (p.spec16)
    return p.bf16 ? wave_t<LOGMV, MB, __nv_bfloat16, __half2>(p, y, s) : wave_t<LOGMV, MB, float, __half2>(p, y, s);
  return p.bf16 ? wave_t<LOGMV, MB, __nv_bfloat16, float2>(p, y, s) : wave_t<LOGMV, MB, float, float2>(p, y, s);
}

template <int LOGMV>
static cudaError_t wave_l(const FourStepLaunch& p, const Layout& y, cudaStream_t s) {
  switch (y.mb) {
    case 1: return wave_lm<LOGMV, 1>(p, y, s);
    case 2: return wave_lm<LOGMV, 2>(p, y, s);
    case 4: return wave_lm<LOGMV, 4>(p, y, s);
    case 8: return wave_lm<LOGMV, 8>(p, y, s);
    case 16: return wave_lm<LOGMV, 16>(p, y, s);
    default: return cudaErrorInvalidValue;
  }
}

// Row lengths make_layout produces: 1024 (L <= 2^18) and 4096 points.
cudaError_t launch_fourstep_wave(const FourStepLaunch& p, const Layout& y, cudaStream_t s) {
  switch (y.logMV) {
    case 10: return wave_l<10>(p, y, s);
    case 12: return wave_l<12>(p, y, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int LOGMV, int MB>
static cudaError_t spec_lm(const float* h, float2* spec, const float2* tables, int D, const Layout& y,
                           cudaStream_t s) {
  cudaError_t e = launch_col<MB, kColSpecFirst, float>(h, nullptr, nullptr, spec, tables + y.tw_1, 1, D, y.L, y.MV,
                                                       0, D, s);
  if (e != cudaSuccess) return e;
  return launch_row<LOGMV, kPairSpectrum>(spec, spec, tables, y.M1, 1, 0, D, s);
}

template <int LOGMV>
static cudaError_t spec_l(const float* h, float2* spec, const float2* tables, int D, const Layout& y,
                          cudaStream_t s) {
  switch (y.mb) {
    case 1: return spec_lm<LOGMV, 1>(h, spec, tables, D, y, s);
    case 2: return spec_lm<LOGMV, 2>(h, spec, tables, D, y, s);
    case 4: return spec_lm<LOGMV, 4>(h, spec, tables, D, y, s);
    case 8: return spec_lm<LOGMV, 8>(h, spec, tables, D, y, s);
    case 16: return spec_lm<LOGMV, 16>(h, spec, tables, D, y, s);
    default: return cudaErrorInvalidValue;
  }
}

int fourstep_read_and_clear_timeout() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_fourstep_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_fourstep_timeout, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

cudaError_t launch_fourstep_spectrum(const float* h, float2* spec, const float2* tables, int D, const Layout& y,
                                     cudaStream_t s) {
  switch (y.logMV) {
    case 10: return spec_l<10>(h, spec, tables, D, y, s);
    case 12: return spec_l<12>(h, spec, tables, D, y, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hyena
