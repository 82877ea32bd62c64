// tc_rows.cu -- the row pass of the four-step forward on the 5th-generation
// tensor cores, for rows of MV = 4096 points (bf16 I/O, order <= 3).
//
// The four-step path (fourstep.cu) splits the packed M-point transform into
// M1-point columns and MV-point rows; rows kA and kB = M1 - kA hold mirror
// bins, k = kA + M1 j pairs with M - k = kB + M1 (MV - 1 - j), which the
// real-FFT unpack and the spectral product need together (glossary
// "Hyena（ハイエナ）", section 計算効率: the long convolution through the FFT).
// Here one CTA item is one row pair: both 4096-point transforms run as three
// DFT-matrix GEMM levels per direction, 4096 = 16 x 16 x 16 with
// n = n1 + 16 n2 + 256 n3 and j = k3 + 16 k2 + 256 k1:
//   F1 rows (n1, n2): DFT over n3 -> k3, twiddle w_4096^{(n1 + 16 n2) k3};
//   F2 rows (n1, k3): DFT over n2 -> k2, twiddle w_256^{n1 k2};
//   F3 rows (k3, k2): DFT over n1 -> k1;
//   inverse: I3 rows (k3, k2) over k1 -> n1, twiddle w_256^{-n1 k2}; I2 rows
//   (n1, k3) over k2 -> n2, twiddle w_4096^{-(n1 + 16 n2) k3}; I1 rows
//   (n1, n2) over k3 -> n3.
// Row B is transformed as x'_B[n] = conj(x_B[n]) w_M^{kA n} (the same
// four-step twiddle as row A), whose DFT at j is conj of row B's spectrum at
// MV - 1 - j: the mirror partner of row A's bin j lands in the same TMEM row
// and column, so the unpack and product stay in one thread. The inverse runs
// the same levels on conj(C'_B) and conjugates at the end. The self-mirrored
// rows 0 and M1/2 are two extra items whose B transform is their own row
// (row 0 pairs j with MV - j, its bin 0 holding the packed DC/Nyquist pair).
//
// Scaling (powers of two): the column pass records each channel's largest
// component (xmax), which scales the F1 operands below 2^6; every DFT matrix
// carries 2^-4; the product is scaled by the channel's largest spectrum
// component (hmax), so every f16 operand stays below 2^15 for any input.
//
// The spectrum rows of an item come from the block's f16 copy (f_c H, f_c the
// power of two that puts the channel's largest component in [2^14, 2^15)):
// one thread issues a bulk copy of both rows (16 KB each) into shared memory
// when the item starts, and the product reads them from there after three
// levels; the scale of the product absorbs 1 / f_c. The copies fill L2 as
// evict-first, which keeps the wave's scratch resident in L2 between the
// passes (at L = 2^20: 6.19 against 5.73 ms per forward without the hint).
#include <cuda_fp16.h>

#include "fft_engine.cuh"
#include "kernels.cuh"
#include "mbar.cuh"
#include "tcgen05.cuh"

namespace hyena {

namespace {

constexpr int kRT = 128;                  // threads per CTA (4 warps: one per TMEM lane quarter)
constexpr int kRMV = 4096;
constexpr uint32_t kRCols = 128;          // TMEM columns per CTA (4 tiles x 32)
// A operand: 4 tiles (row A: tiles 0, 1; row B: tiles 2, 3) of 128 rows x 16
// complex, K-major canonical (core matrices of 8 rows x 16 B; LBO 128, SBO 512)
constexpr uint32_t kRLbo = 128, kRSbo = 512, kRTile = 16 * 512;
constexpr uint32_t kRABytes = 4 * kRTile;
constexpr uint32_t kRBF = 0, kRBI = 2048;   // forward / inverse 16-point DFT, N 32 x K 32
constexpr uint32_t kRBBytes = 4096;
constexpr uint32_t kRRowH = 4 * kRMV;     // one f16 spectrum row (bytes)
constexpr uint32_t kROffA = 0, kROffB = kRABytes, kROffH = kROffB + kRBBytes, kROffMisc = kROffH + 2 * kRRowH;
constexpr uint32_t kRSmem = kROffMisc + 64;

__device__ int g_tcr_timeout;

// w_n^e for 0 <= |e| < n, n a power of two (exact arguments)
__device__ __forceinline__ float2 r_root(long long e, long long n) {
  float s, c;
  sincospif(-2.0f * (float)e / (float)n, &s, &c);
  return make_float2(c, s);
}

// Power of two s with mx * s < 2^emax (>= 2^(emax - 1) for a normal mx > 0),
// and 1 / s; both clamped to normal floats.
__device__ __forceinline__ void r_scale(float mx, int emax, float& s, float& inv_s) {
  const int e = (int)((__float_as_uint(mx) >> 23) & 0xff);   // mx < 2^(e - 126)
  int es = emax + 253 - e;                                   // exponent field of 2^(emax - (e - 126))
  es = es < 1 ? 1 : (es > 253 ? 253 : es);
  s = __uint_as_float((unsigned)es << 23);
  inv_s = __uint_as_float((unsigned)(254 - es) << 23);
  if (mx == 0.f) { s = 1.f; inv_s = 1.f; }
}

}  // namespace

// Resident CTAs per SM the register budget is sized for: three (168
// registers, no spills) measured 7.43 ms per forward at L = 2^20 against
// 7.95 ms for four (128 registers, 168 bytes of spills).
#ifndef HYENA_TCR_CTAS_PER_SM
#define HYENA_TCR_CTAS_PER_SM 3
#endif
__global__ void __launch_bounds__(kRT, HYENA_TCR_CTAS_PER_SM)
tcr_row_kernel(float2* __restrict__ scr, const uint32_t* __restrict__ spec16, const float* __restrict__ hmax,
               const unsigned* __restrict__ xmax, unsigned* __restrict__ xmax_clear, int M1, int B,
               long long ch0, int wave) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
  unsigned char* sA = sm + kROffA;
  unsigned char* sB = sm + kROffB;
  const uint32_t* sH = reinterpret_cast<const uint32_t*>(sm + kROffH);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kROffMisc);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kROffMisc + 16);
  const uint32_t aA = smem_u32(sA), aB = smem_u32(sB), aH = smem_u32(sm + kROffH);
  const uint32_t abar = smem_u32(bar), hbar = smem_u32(bar + 1);
  const int M = M1 * kRMV;

  if (w == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(kRCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  if (tid == 0) {
    mbar_init(abar, 1);
    mbar_init(hbar, 1);
    mbar_init_fence();
  }
  g_build_dft(sB, kRBF, 16, 16, 16, false, 0x1p-4f, tid, kRT);
  g_build_dft(sB, kRBI, 16, 16, 16, true, 0x1p-4f, tid, kRT);
  // the next column pass accumulates its maxima into the other buffer
  if (blockIdx.x == 0)
    for (int i = tid; i < wave; i += kRT) xmax_clear[i] = 0u;

  // ---- per-thread rows (t = 0, 1 selects the tile within a transform)
  // F1 / I1 rows (n1, n2): n1 = (l & 7) + 8 t, n2 = ((l >> 3) & 3) + 4 w
  const int n2f = ((l >> 3) & 3) + 4 * w;
  const int m0 = (l & 7) + 16 * n2f;                  // m' of row t = m0 + 8 t
  const float2 tw1a = r_root(m0, kRMV), tw1b = r_root(m0 + 8, kRMV);
  // F2 rows (n1, k3): n1 = ((l >> 3) & 3) + 4 w, k3 = ((l & 7) ^ (n1 & 7)) + 8 t
  const int n1f2 = ((l >> 3) & 3) + 4 * w;
  const int k3f2 = (l & 7) ^ (n1f2 & 7);
  const float2 tw2 = r_root(n1f2, 256);
  // F3 / I3 rows (k3, k2): k3 = (l & 7) + 8 t, k2 = ((l >> 3) & 3) + 4 w
  const int k2f3 = ((l >> 3) & 3) + 4 * w;
  const float2 wj0a = r_root((l & 7) + 16 * k2f3, 2 * kRMV), wj0b = r_root((l & 7) + 8 + 16 * k2f3, 2 * kRMV);
  const float2 tw3 = r_root(-k2f3, 256);
  // I2 rows (n1, k3): k3 = ((l >> 3) & 3) + 4 (w & 1) + 8 t, n1 = ((l & 7) ^ (k3 & 7)) + 8 (w >> 1)
  const int k3i2 = ((l >> 3) & 3) + 4 * (w & 1);       // k3 of row t = k3i2 + 8 t
  const int n1i2 = ((l & 7) ^ k3i2) + 8 * (w >> 1);
  const float2 st2a = r_root(-(n1i2 * k3i2), kRMV), st2b = r_root(-(n1i2 * (k3i2 + 8)), kRMV);
  const float2 sp2a = r_root(-k3i2, 256), sp2b = r_root(-(k3i2 + 8), 256);

  // byte offsets (A region) of this thread's stores; tau (row A / B) adds 2 tiles
  const uint32_t own = (uint32_t)((l & 7) * 16 + (4 * w + (l >> 3)) * kRSbo);   // own row in tile t: + t * tile + c * 128
  const uint32_t f12 = (uint32_t)((n2f & 3) * 4 + (n2f >> 2) * 128);         // + n1 * 512 + (k3 >> 3) tile + xor term
  const uint32_t f23 = (uint32_t)(k3f2 * 16 + (n1f2 & 3) * 4 + (n1f2 >> 2) * 128);   // + t tile + k2 * 512
  const uint32_t i32 = (uint32_t)((k2f3 & 3) * 4 + (k2f3 >> 2) * 128 + (l & 7) * 512);  // + t tile + n1 terms
  const uint32_t i21 = (uint32_t)((n1i2 >> 3) * kRTile + (n1i2 & 7) * 16 + (k3i2 & 3) * 4 + (k3i2 >> 2) * 128);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tslot;
  const uint32_t tlane = tmem + ((uint32_t)(32 * w) << 16);

  uint32_t phase = 0, hphase = 0;
  bool ok = true, h_pending = false;
  auto level = [&](uint32_t bmat) -> bool {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    const int bad = __syncthreads_or(ok ? 0 : 1);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (bad) return false;
    if (tid == 0) {
      const uint64_t da = g_desc(aA, kRLbo, kRSbo), db = g_desc(aB + bmat, 128, 512);
#pragma unroll
      for (int T = 0; T < 4; ++T)
#pragma unroll
        for (int s = 0; s < 2; ++s)
          g_mma(tmem + 32u * T, da + ((T * kRTile + s * 2 * kRLbo) >> 4), db + (s * 256 >> 4), g_idesc(32),
                s > 0 ? 1u : 0u);
      g_commit(abar);
    }
    ok = mbar_wait(abar, phase);
    phase ^= 1;
    if (!ok) atomicExch(&g_tcr_timeout, 1);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    return true;
  };
  // TMEM column of tile (tau, t)
  auto col = [](int tau, int t) { return 32u * (uint32_t)(2 * tau + t); };

  const int per = M1 / 2 + 1;
  const long long nitems = (long long)wave * per;
  for (long long it = blockIdx.x; it < nitems; it += gridDim.x) {
    const int chl = (int)(it / per), q = (int)(it % per);
    const long long ch = ch0 + chl;
    const int c = (int)(ch / B);
    // item kinds: normal pair (kA, M1 - kA); row 0 with itself (mirror j <-> MV - j);
    // row M1/2 with itself (mirror j <-> MV - 1 - j)
    int kA, kB, kind;
    if (q < M1 / 2 - 1) { kA = q + 1; kB = M1 - kA; kind = 0; }
    else if (q == M1 / 2 - 1) { kA = 0; kB = 0; kind = 1; }
    else { kA = M1 / 2; kB = M1 / 2; kind = 2; }
    float2* S = scr + (size_t)chl * M;
    float2* xA = S + (size_t)kA * kRMV;
    float2* xB = S + (size_t)kB * kRMV;
    // the item's f16 spectrum rows into shared memory (row B only for a
    // mirror pair of two rows); every thread's reads of the previous item's
    // rows are ordered before this by the level barriers since then
    // (L2 evict-first: read once per stage, they must not evict the scratch)
    if (tid == 0) {
      const uint32_t* H = spec16 + (size_t)c * M;
      const uint64_t pol = l2_policy_evict_first();
      mbar_arrive_expect_tx(hbar, kind == 0 ? 2 * kRRowH : kRRowH);
      bulk_g2s_policy(aH, H + (size_t)kA * kRMV, kRRowH, hbar, pol);
      if (kind == 0) bulk_g2s_policy(aH + kRRowH, H + (size_t)kB * kRMV, kRRowH, hbar, pol);
    }
    h_pending = true;
    float s_in, inv_s, s2, inv_s2, f_c, inv_fc;
    r_scale(__uint_as_float(xmax[chl]), 6, s_in, inv_s);
    const float hm = __ldg(hmax + c);
    r_scale(hm, 4, s2, inv_s2);
    r_scale(hm, 15, f_c, inv_fc);   // the scale of the f16 copy
    s2 *= inv_fc;
    // four-step twiddle w_M^{kA n}, n = m' + 256 n3: row t starts at w_M^{kA m'}, steps w_M^{256 kA}
    const float2 tin_a = r_root(((long long)kA * m0) % M, M), tin_b = r_root(((long long)kA * (m0 + 8)) % M, M);
    const float2 tin_s = r_root((256LL * kA) % M, M);

    // ---- input: x'_A = x_A w, x'_B = conj(x_B) w (scaled), own F1 rows, K = n3
#pragma unroll 1
    for (int tau = 0; tau < 2; ++tau) {
      const float2* X = tau ? xB : xA;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const float2* xr = X + m0 + 8 * t;
        float2 v[16];
#pragma unroll
        for (int n3 = 0; n3 < 16; ++n3) v[n3] = xr[256 * n3];
        float2 cur = g_opaque(t ? tin_b : tin_a);
        const float2 stp = g_opaque(tin_s);
        cur = make_float2(cur.x * s_in, cur.y * s_in);
        uint32_t pk[16];
#pragma unroll
        for (int n3 = 0; n3 < 16; ++n3) {
          const float2 x = tau ? make_float2(v[n3].x, -v[n3].y) : v[n3];
          const float2 y = g_cmul(x, cur);
          pk[n3] = g_pack(y.x, y.y);
          cur = g_cmul(cur, stp);
        }
        const uint32_t base = own + (uint32_t)(2 * tau + t) * kRTile;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          *reinterpret_cast<uint4*>(sA + base + cc * 128) =
              make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
      }
    }
    if (!level(kRBF)) goto done;
    // ---- F1 out: twiddle w_4096^{m' k3}, to F2 rows (n1, k3) at K = n2
    g_pipe4<32>([&](int ch4) { return tlane + col(ch4 >> 1, ch4 & 1); },
                [&](int ch4, const uint32_t (&r)[32]) {
                  const int tau = ch4 >> 1, t = ch4 & 1;
                  const int n1 = (l & 7) + 8 * t;
                  const float2 twb = g_opaque(t ? tw1b : tw1a);
                  float2 cur = make_float2(1.f, 0.f);
                  const uint32_t base = f12 + (uint32_t)(n1 * 512 + tau * 2 * kRTile);
#pragma unroll
                  for (int k3 = 0; k3 < 16; ++k3) {
                    const float2 vv = g_cmul(g_cval(r, k3), cur);
                    const uint32_t off = base + (uint32_t)((k3 >> 3) * kRTile) + ((uint32_t)((l & 7) ^ (k3 & 7)) << 4);
                    *reinterpret_cast<uint32_t*>(sA + off) = g_pack(vv.x, vv.y);
                    cur = g_cmul(cur, twb);
                  }
                });
    if (!level(kRBF)) goto done;
    // ---- F2 out: twiddle w_256^{n1 k2}, to F3 rows (k3, k2) at K = n1
    g_pipe4<32>([&](int ch4) { return tlane + col(ch4 >> 1, ch4 & 1); },
                [&](int ch4, const uint32_t (&r)[32]) {
                  const int tau = ch4 >> 1, t = ch4 & 1;
                  const float2 twb = g_opaque(tw2);
                  float2 cur = make_float2(1.f, 0.f);
                  const uint32_t base = f23 + (uint32_t)((2 * tau + t) * kRTile);
#pragma unroll
                  for (int k2 = 0; k2 < 16; ++k2) {
                    const float2 vv = g_cmul(g_cval(r, k2), cur);
                    *reinterpret_cast<uint32_t*>(sA + base + k2 * 512) = g_pack(vv.x, vv.y);
                    cur = g_cmul(cur, twb);
                  }
                });
    if (!level(kRBF)) goto done;
    // ---- F3 out: the unpack and spectral product of the mirror pair at bin
    // j = k3 + 16 k2 + 256 k1, scaled by s2; own rows as the I3 operands;
    // the spectrum rows from shared memory (row B of a self-mirrored item is
    // row A)
    if (!mbar_wait(hbar, hphase)) {
      ok = false;   // the next level barrier ends the kernel
      atomicExch(&g_tcr_timeout, 1);
      mbar_wait(hbar, hphase, 1000000000ull);   // bounded second wait for the copies in flight
    }
    hphase ^= 1;
    h_pending = false;
    {
      const uint32_t* HA = sH;
      const uint32_t* HB = sH + (kind == 0 ? kRMV : 0);
      const float2 rho = r_root(kA, 2LL * M);   // w_{2M}^{kA}
      const float2 w32 = make_float2(0.98078528040323044913f, -0.19509032201612826785f);   // w_32
#pragma unroll 1
      for (int t = 0; t < 2; ++t) {
        const int k3 = (l & 7) + 8 * t;
        const int j0 = k3 + 16 * k2f3;
        float2 W = g_cmul(rho, g_opaque(t ? wj0b : wj0a));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float2 ha[8], hb[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = j0 + 256 * (8 * h + e);
            ha[e] = __half22float2(*reinterpret_cast<const __half2*>(HA + j));
            hb[e] = __half22float2(*reinterpret_cast<const __half2*>(
                (kind == 1) ? HA + ((kRMV - j) & (kRMV - 1)) : HB + (kRMV - 1 - j)));
          }
          uint32_t ra[16], rb[16];
          g_ld16(tlane + col(0, t) + 16u * h, ra);
          g_ld16(tlane + col(1, t) + 16u * h, rb);
          g_wait16(ra);
          g_wait16(rb);
          uint32_t pa[8], pb[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float2 Ca = g_cval(ra, e);
            const float2 bv = g_cval(rb, e);
            float2 Cb = make_float2(bv.x, -bv.y);
            float2 Ha = ha[e], Hb = hb[e], Wk = W;
            if (kind == 1 && j0 == 0 && h == 0 && e == 0) {   // bin 0: packed DC and Nyquist
              Ha = make_float2(ha[0].x, 0.f);
              Hb = make_float2(ha[0].y, 0.f);
              Wk = make_float2(1.f, 0.f);
            }
            spectral_pair(Ca, Cb, Ha, Hb, Wk);
            pa[e] = g_pack(Ca.x * s2, Ca.y * s2);
            pb[e] = g_pack(Cb.x * s2, -Cb.y * s2);
            W = g_cmul(W, w32);
          }
          const uint32_t oa = own + (uint32_t)t * kRTile + h * 256;
          const uint32_t ob = oa + 2 * kRTile;
          *reinterpret_cast<uint4*>(sA + oa) = make_uint4(pa[0], pa[1], pa[2], pa[3]);
          *reinterpret_cast<uint4*>(sA + oa + 128) = make_uint4(pa[4], pa[5], pa[6], pa[7]);
          *reinterpret_cast<uint4*>(sA + ob) = make_uint4(pb[0], pb[1], pb[2], pb[3]);
          *reinterpret_cast<uint4*>(sA + ob + 128) = make_uint4(pb[4], pb[5], pb[6], pb[7]);
        }
      }
    }
    if (!level(kRBI)) goto done;
    // ---- I3 out: twiddle w_256^{-n1 k2}, to I2 rows (n1, k3) at K = k2
    g_pipe4<32>([&](int ch4) { return tlane + col(ch4 >> 1, ch4 & 1); },
                [&](int ch4, const uint32_t (&r)[32]) {
                  const int tau = ch4 >> 1, t = ch4 & 1;
                  const float2 twb = g_opaque(tw3);
                  float2 cur = make_float2(1.f, 0.f);
                  const uint32_t base = i32 + (uint32_t)((2 * tau + t) * kRTile);
#pragma unroll
                  for (int n1 = 0; n1 < 16; ++n1) {
                    const float2 vv = g_cmul(g_cval(r, n1), cur);
                    const uint32_t off =
                        base + (uint32_t)(8 * (n1 >> 3) * 512) + ((uint32_t)((n1 & 7) ^ (l & 7)) << 4);
                    *reinterpret_cast<uint32_t*>(sA + off) = g_pack(vv.x, vv.y);
                    cur = g_cmul(cur, twb);
                  }
                });
    if (!level(kRBI)) goto done;
    // ---- I2 out: twiddle w_4096^{-(n1 + 16 n2) k3}, to I1 rows (n1, n2) at K = k3
    g_pipe4<32>([&](int ch4) { return tlane + col(ch4 >> 1, ch4 & 1); },
                [&](int ch4, const uint32_t (&r)[32]) {
                  const int tau = ch4 >> 1, t = ch4 & 1;
                  const float2 twb = g_opaque(t ? sp2b : sp2a);
                  float2 cur = g_opaque(t ? st2b : st2a);
                  const uint32_t base = i21 + (uint32_t)(tau * 2 * kRTile + t * 2 * 128);
#pragma unroll
                  for (int n2 = 0; n2 < 16; ++n2) {
                    const float2 vv = g_cmul(g_cval(r, n2), cur);
                    *reinterpret_cast<uint32_t*>(sA + base + n2 * 512) = g_pack(vv.x, vv.y);
                    cur = g_cmul(cur, twb);
                  }
                });
    if (!level(kRBI)) goto done;
    // ---- I1 out: times the conjugate four-step twiddle and the inverse of
    // the scales; row B conjugated; back to the scratch rows
    {
      const float u = inv_s * inv_s2 * 0x1p24f;
      // (one chunk at a time: a pipelined read here held twice the registers)
#pragma unroll 1
      for (int ch4 = 0; ch4 < 4; ++ch4) {
        const int tau = ch4 >> 1, t = ch4 & 1;
        if (tau == 1 && kind != 0) break;   // a self-mirrored row's partner copy
        uint32_t r[32];
        g_ld32(tlane + col(tau, t), r);
        g_wait32(r);
        {
                    float2* xr = (tau ? xB : xA) + m0 + 8 * t;
                    float2 cur = g_opaque(t ? tin_b : tin_a);
                    const float2 stp = g_opaque(tin_s);
                    cur = make_float2(cur.x * u, -cur.y * u);      // conj, times u
#pragma unroll
                    for (int n3 = 0; n3 < 16; ++n3) {
                      const float2 vv = g_cmul(g_cval(r, n3), cur);
                      xr[256 * n3] = tau ? make_float2(vv.x, -vv.y) : vv;
                      cur = cmulc(cur, stp);
                    }
        }
      }
    }
    // the next item's first level overwrites TMEM: order these reads before it
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  }
done:
  if (!ok) mbar_wait(abar, phase ^ 1, 1000000000ull);
  if (h_pending) mbar_wait(hbar, hphase, 1000000000ull);   // a staging copy still in flight
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (w == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kRCols));
}

// Largest component of each channel's spectrum block rows: kHmaxSplit CTAs
// per channel, 16-byte loads, the maximum merged as float bits (non-negative
// floats order as unsigned integers) into hmax, which starts at zero.
constexpr int kHmaxSplit = 16;
__global__ void tcr_hmax_kernel(const float2* __restrict__ spec, int M, unsigned* __restrict__ hmax) {
  const int c = blockIdx.x / kHmaxSplit, part = blockIdx.x % kHmaxSplit;
  const int n4 = M / 2 / kHmaxSplit;   // float4 (two bins) per CTA
  const float4* r = reinterpret_cast<const float4*>(spec + (size_t)c * M) + (size_t)part * n4;
  float mx = 0.f;
#pragma unroll 4
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 v = __ldcs(r + i);
    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
  if ((threadIdx.x & 31) == 0) atomicMax(hmax + c, m);
}

cudaError_t launch_tcr_rows(float2* scr, const uint32_t* spec16, const float* hmax, const unsigned* xmax,
                            unsigned* xmax_clear, int M1, int B, long long ch0, int wave, cudaStream_t s) {
  auto k = tcr_row_kernel;
  cudaError_t e = cudaFuncSetAttribute((const void*)k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRSmem);
  if (e != cudaSuccess) return e;
  // three CTAs of 68 KB need the largest shared-memory carveout
  e = cudaFuncSetAttribute((const void*)k, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  // at most four CTAs per SM (registers): their TMEM allocations (128 columns
  // each) stay within the SM's 512 columns, so no allocation waits on another CTA
  static_assert(HYENA_TCR_CTAS_PER_SM * kRCols <= 512, "TMEM columns of the resident CTAs");
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  long long grid = (long long)HYENA_TCR_CTAS_PER_SM * sms;
  const long long items = (long long)wave * (M1 / 2 + 1);
  if (grid > items) grid = items;
  k<<<(int)grid, kRT, kRSmem, s>>>(scr, spec16, hmax, xmax, xmax_clear, M1, B, ch0, wave);
  return cudaGetLastError();
}

cudaError_t launch_tcr_hmax(const float2* spec, int D, int M, float* hmax, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(hmax, 0, sizeof(float) * (size_t)D, s);
  if (e != cudaSuccess) return e;
  tcr_hmax_kernel<<<D * kHmaxSplit, 256, 0, s>>>(spec, M, reinterpret_cast<unsigned*>(hmax));
  return cudaGetLastError();
}

// f16 copy of a spectrum block's bins: channel c times the power of two f_c
// that puts hmax[c] in [2^14, 2^15), rounded to nearest; kHmaxSplit CTAs per
// channel, two bins per thread and step.
__global__ void tcr_half_kernel(const float2* __restrict__ spec, const float* __restrict__ hmax, int M,
                                uint2* __restrict__ out) {
  const int c = blockIdx.x / kHmaxSplit, part = blockIdx.x % kHmaxSplit;
  const int n4 = M / 2 / kHmaxSplit;
  float f_c, inv_fc;
  r_scale(hmax[c], 15, f_c, inv_fc);
  const size_t base = (size_t)c * (M / 2) + (size_t)part * n4;
  const float4* r = reinterpret_cast<const float4*>(spec) + base;
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 v = __ldcs(r + i);
    const __half2 a = __floats2half2_rn(v.x * f_c, v.y * f_c), b = __floats2half2_rn(v.z * f_c, v.w * f_c);
    out[base + i] = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
  }
}

cudaError_t launch_tcr_half(const float2* spec, const float* hmax, int D, int M, uint32_t* out, cudaStream_t s) {
  tcr_half_kernel<<<D * kHmaxSplit, 256, 0, s>>>(spec, hmax, M, reinterpret_cast<uint2*>(out));
  return cudaGetLastError();
}

int tcr_read_and_clear_timeout() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tcr_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_tcr_timeout, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

}  // namespace hyena
