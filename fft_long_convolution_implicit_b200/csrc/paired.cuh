// paired.cuh -- the pass where spectrum bins k and M-k meet.
//
// The last forward Stockham pass (radix 8, span MV/8) leaves butterfly j
// holding bins j + r*MV/8. Butterfly j of one row and butterfly j' of the
// mirror row hold mirror bins, so a thread that owns both can unpack the real
// transform, multiply by the filter spectrum and repack without touching
// shared memory; the first inverse (transposed) pass then runs on the same
// registers. Mirror pairs are (a[r], b[7-r]) for every layout except the
// head thread of row 0, whose butterflies 0 and MV/16 are each self-mirrored.
#pragma once

#include <cuda_fp16.h>

#include "fft_engine.cuh"

namespace hyena {

enum PairMode { kPairConv = 0, kPairSpectrum = 1 };

// Filter spectrum reads: from global memory as streaming loads (each bin is
// read once per forward, so it is marked evict-first and does not displace
// the four-step scratch from L2), or from a shared-memory copy staged by the
// caller (H_SMEM); bins stored as float2, or as __half2 (the reduced-precision
// block, scaled per channel by a power of two that the caller removes at the
// gate).
template <bool H_SMEM, typename HT = float2>
struct HRead;
template <>
struct HRead<false, float2> {
  static __device__ __forceinline__ float2 at(const float2* p, int i) { return __ldcs(p + i); }
};
template <>
struct HRead<true, float2> {
  static __device__ __forceinline__ float2 at(const float2* p, int i) { return p[i]; }
};
template <>
struct HRead<false, __half2> {
  static __device__ __forceinline__ float2 at(const __half2* p, int i) { return __half22float2(__ldcs(p + i)); }
};
template <>
struct HRead<true, __half2> {
  static __device__ __forceinline__ float2 at(const __half2* p, int i) { return __half22float2(p[i]); }
};

// W for bin kA of row A: w_{2M}^{k1 + M1 k2} = rho * w_{2 MV}^{k2}.
__device__ __forceinline__ float2 pair_w(const float2* __restrict__ Wv, int k2, float2 rho, bool has_rho) {
  float2 w = __ldg(&Wv[k2]);
  return has_rho ? cmul(rho, w) : w;
}

// MODE kPairConv: HA/HB are the spectrum rows of row A and row B (read);
//   data is transformed in place in shared memory.
// MODE kPairSpectrum: the unpacked spectrum 2 Z[k] * scale is written to HA/HB
//   (library order, packed DC/Nyquist in bin 0 of row 0); shared memory is not
//   written back.
template <int LOGMV, int MODE, bool H_SMEM = false, typename HT = float2>
__device__ __forceinline__ void paired_pass(float2* baseA, float2* baseB, int jA, int jB, bool head,
                                            const float2* __restrict__ tw, const float2* __restrict__ Wv,
                                            float2 rho, bool has_rho, HT* HA, HT* HB, float scale) {
  constexpr int MV = 1 << LOGMV, Q8 = MV / 8, Q16 = MV / 16, NS = Q8;
  static_assert(MODE == kPairConv || sizeof(HT) == sizeof(float2), "spectra are written as float2");
  auto hload = [](const HT* p, int i) { return HRead<H_SMEM, HT>::at(p, i); };
  float2 a[8], b[8];
  float2* pa = baseA + pidx(jA);
  float2* pb = baseB + pidx(jB);
  static_assert(Q8 % 16 == 0, "paired pass needs MV >= 128");
  constexpr int QS = Q8 + Q8 / 16;   // padded stride between the bins of one butterfly
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    a[r] = pa[r * QS];
    b[r] = pb[r * QS];
  }
  const float2* __restrict__ twa = tw + (NS - 1) + jA;
  const float2* __restrict__ twb = tw + (NS - 1) + jB;
#pragma unroll
  for (int r = 1; r < 8; ++r) {
    a[r] = cmul(a[r], __ldg(twa + (r - 1) * NS));
    b[r] = cmul(b[r], __ldg(twb + (r - 1) * NS));
  }
  dft8<false, 0>(a);
  dft8<false, 0>(b);

  if (!head) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int kA = jA + r * Q8;
      const float2 W = pair_w(Wv, kA, rho, has_rho);
      if constexpr (MODE == kPairConv) {
        spectral_pair(a[r], b[7 - r], hload(HA, kA), hload(HB, jB + (7 - r) * Q8), W);
      } else {
        float2 za, zb;
        unpack_pair(a[r], b[7 - r], W, za, zb);
        HA[kA] = make_float2(za.x * scale, za.y * scale);
        HB[jB + (7 - r) * Q8] = make_float2(zb.x * scale, zb.y * scale);
      }
    }
  } else {
    // butterfly 0 of row 0: bins r*Q8. Bin 0 pairs with bin M (packed Nyquist),
    // bin M/2 with itself, and r with 8-r otherwise.
    {
      const float2 one = make_float2(1.f, 0.f);
      if constexpr (MODE == kPairConv) {
        float2 c0 = a[0], c0b = a[0];
        const float2 h0 = hload(HA, 0);
        spectral_pair(c0, c0b, make_float2(h0.x, 0.f), make_float2(h0.y, 0.f), one);
        a[0] = c0;
      } else {
        float2 za, zb;
        unpack_pair(a[0], a[0], one, za, zb);
        HA[0] = make_float2(za.x * scale, zb.x * scale);
      }
    }
#pragma unroll
    for (int r = 1; r < 4; ++r) {
      const float2 W = __ldg(&Wv[r * Q8]);
      if constexpr (MODE == kPairConv) {
        spectral_pair(a[r], a[8 - r], hload(HA, r * Q8), hload(HA, (8 - r) * Q8), W);
      } else {
        float2 za, zb;
        unpack_pair(a[r], a[8 - r], W, za, zb);
        HA[r * Q8] = make_float2(za.x * scale, za.y * scale);
        HA[(8 - r) * Q8] = make_float2(zb.x * scale, zb.y * scale);
      }
    }
    {
      const float2 W = __ldg(&Wv[4 * Q8]);
      if constexpr (MODE == kPairConv) {
        float2 c4 = a[4], c4b = a[4];
        const float2 h4 = hload(HA, 4 * Q8);
        spectral_pair(c4, c4b, h4, h4, W);
        a[4] = c4;
      } else {
        float2 za, zb;
        unpack_pair(a[4], a[4], W, za, zb);
        HA[4 * Q8] = make_float2(za.x * scale, za.y * scale);
      }
    }
    // butterfly MV/16: bins Q16 + r*Q8, pairs r <-> 7-r
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float2 W = __ldg(&Wv[Q16 + r * Q8]);
      if constexpr (MODE == kPairConv) {
        spectral_pair(b[r], b[7 - r], hload(HA, Q16 + r * Q8), hload(HA, Q16 + (7 - r) * Q8), W);
      } else {
        float2 za, zb;
        unpack_pair(b[r], b[7 - r], W, za, zb);
        HA[Q16 + r * Q8] = make_float2(za.x * scale, za.y * scale);
        HA[Q16 + (7 - r) * Q8] = make_float2(zb.x * scale, zb.y * scale);
      }
    }
  }

  if constexpr (MODE == kPairConv) {
    dft8<true, 0>(a);
    dft8<true, 0>(b);
#pragma unroll
    for (int r = 1; r < 8; ++r) {
      a[r] = cmulc(a[r], __ldg(twa + (r - 1) * NS));
      b[r] = cmulc(b[r], __ldg(twb + (r - 1) * NS));
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      pa[r * QS] = a[r];
      pb[r * QS] = b[r];
    }
  }
}

}  // namespace hyena
