// tc_gemm.cu -- Hyena order-N forward for bf16 I/O at L = 8192, B even, with
// every DFT level of the transform as a GEMM on the 5th-generation tensor
// cores (tcgen05.mma: f16 operands in shared memory, f32 accumulators in TMEM).
//
// Two batch items b, b+1 of channel c share the filter h_c, so their causal
// convolutions are the real and imaginary parts of one complex convolution of
// c[m] = z_b[m] + i z_{b+1}[m] on the 2L zero-padded grid (glossary
// "Hyena（ハイエナ）", section 計算効率; "Native Multi-Dimensional Subquadratic
// Operators via Input Dependent Long Convolutions", section 境界の処理).
// With P = 2L = 16384 = 16 * 32 * 32, m = m'' + 32 n2 + 1024 n3 and
// k = k3 + 16 k2 + 512 k1 (a Cooley-Tukey split written as three levels):
//   F1  rows m' = m'' + 32 n2 (1024): 16-point DFT over n3 (n3 < 8 nonzero),
//       then the twiddle w_P^{m' k3};
//   F2  rows (k3, m'') (512): 32-point DFT over n2, twiddle w_1024^{m'' k2};
//   F3  rows (k3, k2) (512): 32-point DFT over m'' -> C[k];
//   the product with the filter spectrum (an f16 copy in F3-row order);
//   I3  rows (k3, k2): inverse 32-point DFT over k1 -> m'', twiddle w_1024^{-m'' k2};
//   I2  rows (k3, m''): inverse 32-point DFT over k2 -> n2, twiddle w_P^{-m' k3};
//   I1  rows m': inverse 16-point DFT over k3, outputs n3 < 8 only (t < L).
// Each level is D[rows x 2R] = A[rows x 2K] B[2R x 2K]^T with complex values
// interleaved (re, im) along K and N, so the real form of the DFT matrix in B
// carries the complex arithmetic. A thread owns fixed TMEM rows in every level
// (warp w reads lanes 32 (w % 4) .. + 31 of the tiles of parity w / 4): it
// reads its rows of D (tcgen05.ld), applies the twiddles in fp32 (powers by
// recurrence from per-thread bases) and writes the values into the rows of the
// next level's A operand; the row numberings and the operand strides are chosen
// so that every one of these stores is free of shared-memory bank conflicts.
// The output rows of I1 are the input rows of F1, so z stays in registers
// between the N stages. One thread issues the MMAs; completion arrives on an
// mbarrier through tcgen05.commit; every wait is bounded in time.
//
// Scaling (exact powers of two): z is scaled so max |component| < 2^6; the
// DFT matrices carry 2^-4 (F1), 2^-8 (F2, F3) and 2^-5 (I3, I2), which keeps
// every f16 operand below 2^15 for any input (each level grows a bound by at
// most its length) while every nonzero matrix entry stays an f16 normal; the
// spectrum copy is scaled per channel to [2^14, 2^15). All factors (2^-30 in
// all) are removed at the gate.
#include <cuda_fp16.h>

#include "fft_engine.cuh"
#include "kernels.cuh"
#include "mbar.cuh"
#include "tcgen05.cuh"

namespace hyena {

namespace {

constexpr int kGT = 256;                  // threads per CTA
constexpr int kGL = 8192;                 // L
constexpr int kGP = 2 * kGL;              // transform length
constexpr uint32_t kGCols = 256;          // TMEM columns per CTA
// A operand (K-major, no swizzle, core matrices of 8 rows x 16 B): byte
// address of complex element kappa of row r within a 128-row tile is
//   (r & 7) * 16 + (kappa & 3) * 4 + (kappa >> 2) * LBO + (r >> 3) * SBO.
constexpr uint32_t kF1Lbo = 128, kF1Sbo = 256, kF1Tile = 16 * 256;        // rows of 8 complex
constexpr uint32_t kCLbo = 128, kCSbo = 1024, kCTile = 16 * 1024;         // rows of 32 complex (F2, I3, I2)
constexpr uint32_t kF3Lbo = 2064, kF3Sbo = 128, kF3Tile = 8 * 2064;       // F3: K chunks 2064 B apart
constexpr uint32_t kI1Lbo = 2080, kI1Sbo = 128, kI1Tile = 4 * 2080;       // I1: K chunks 2080 B apart
constexpr uint32_t kABytes = 66560;
static_assert(4 * kF3Tile <= kABytes && 8 * kI1Tile <= kABytes && 4 * kCTile <= kABytes, "A region");
// B operands (DFT matrices, K-major canonical: LBO 128, SBO = K / 8 * 128)
constexpr uint32_t kBF1 = 0;              // forward 16-point, inputs < 8: N 32 x K 16
constexpr uint32_t kBF32 = 1024;          // forward 32-point: N 64 x K 64
constexpr uint32_t kBI32 = 9216;          // inverse 32-point: N 64 x K 64
constexpr uint32_t kBI1 = 17408;          // inverse 16-point, outputs < 8: N 16 x K 32
constexpr uint32_t kBBytes = 18432;
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kABytes;
constexpr uint32_t kOffMisc = kOffB + kBBytes;   // mbarrier, TMEM address, 8 partial maxima
constexpr uint32_t kOffPtr = kOffMisc + 64;      // gate and spectrum pointers of the N stages
constexpr uint32_t kGSmem = kOffPtr + 16 * kMaxOrder;
// spectrum copy row: 2L f16x2 bins in F3-row order, then 1 / f_c (float), padding
constexpr size_t kGHRowBytes = (size_t)4 * kGP + 16;

__device__ int g_tcg_timeout;

}  // namespace

__global__ void __launch_bounds__(kGT, 2)
tcg_forward_kernel(const __nv_bfloat16* __restrict__ v, GatePtrs<__nv_bfloat16> x, SpecPtrs hh,
                   __nv_bfloat16* __restrict__ y, int B, int D, int N, long long npairs) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const int tid = threadIdx.x, w = tid >> 5, l = tid & 31, q = w & 3, hw = w >> 2;
  unsigned char* sA = sm + kOffA;
  unsigned char* sB = sm + kOffB;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kOffMisc);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kOffMisc + 8);
  float* red = reinterpret_cast<float*>(sm + kOffMisc + 16);
  const __nv_bfloat16** xptr = reinterpret_cast<const __nv_bfloat16**>(sm + kOffPtr);
  const unsigned char** hptr = reinterpret_cast<const unsigned char**>(sm + kOffPtr + 8 * kMaxOrder);
  const uint32_t aA = smem_u32(sA), aB = smem_u32(sB), abar = smem_u32(bar);

  if (w == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(kGCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  if (tid < kMaxOrder) {
    xptr[tid] = x.p[tid];
    hptr[tid] = reinterpret_cast<const unsigned char*>(hh.p[tid]);
  }
  if (tid == 0) {
    mbar_init(abar, 1);
    mbar_init_fence();
  }
  g_build_dft(sB, kBF1, 16, 16, 8, false, 0x1p-4f, tid, kGT);
  g_build_dft(sB, kBF32, 32, 32, 32, false, 0x1p-8f, tid, kGT);
  g_build_dft(sB, kBI32, 32, 32, 32, true, 0x1p-5f, tid, kGT);
  g_build_dft(sB, kBI1, 16, 8, 16, true, 1.f, tid, kGT);

  // ---- per-thread row ownership, twiddle bases and store addresses
  // F1 / I1 rows i: m' = l + 128 w + 32 i (tile 2i + hw); time t = m' + 1024 n3
  // (rows i > 0: tw1 * w_512^i)
  const float2 tw1 = g_root(l + 128 * w, kGP);
  // F2 rows t: (k3 = q + 4 hw + 8 t, m'' = l); twiddle base w_1024^{l}
  const float2 tw2 = g_root(l, 1024);
  // F3 / I3 rows t: (k3 = 8 hw + (l >> 2), k2 = (l & 3) + 4 q + 16 t); I3 twiddle base w_1024^{-k2}
  const float2 tw3a = g_root(-((l & 3) + 4 * q), 1024), tw3b = g_root(-((l & 3) + 4 * q + 16), 1024);
  // I2 rows t: (k3 = l & 15, m'' = (l >> 4) + 2 q + 8 hw + 16 t);
  // twiddle w_P^{-(m'' + 32 n2) k3} = start_t * base^{n2}
  const int k3i2 = l & 15;
  const float2 st2a = g_root(-(((l >> 4) + 2 * q + 8 * hw) * k3i2), kGP);
  const float2 st2b = g_root(-(((l >> 4) + 2 * q + 8 * hw + 16) * k3i2), kGP);
  const float2 tw2i = g_root(-32 * k3i2, kGP);

  // byte offsets (A region) of this thread's stores
  const uint32_t f1_base = (uint32_t)((l & 7) * 16 + (16 * hw + 4 * q + (l >> 3)) * kF1Sbo);   // + c*128 + i*8192
  const uint32_t f12_base = (uint32_t)((l & 7) * 16 + w * 128 + (l >> 3) * 1024);           // + 4096 k3
  // row t of each level adds t times the second constant
  const uint32_t f23_base = (uint32_t)(64 * (q & 1) + 128 * ((q >> 1) + 2 * hw) + (l & 3) * 4 + (l >> 2) * kF3Lbo);
  constexpr uint32_t f23_step = kF3Tile;
  const uint32_t i3_base = (uint32_t)((l & 7) * 16 + (16 * hw + 4 * q + (l >> 3)) * kCSbo);   // + c*128
  constexpr uint32_t i3_step = 32 * kCSbo;
  const uint32_t i32_base = (uint32_t)((l >> 2) * 16 + (l & 3) * 4 + q * 128 + hw * 1024);
  constexpr uint32_t i32_step = 4 * 128;
  const uint32_t i21_base = (uint32_t)((((l >> 4) + 2 * q) * 16) + (k3i2 & 3) * 4 + (k3i2 >> 2) * kI1Lbo + hw * 128);
  constexpr uint32_t i21_step = 2 * 128;
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tslot;
  const uint32_t tlane = tmem + ((uint32_t)(32 * q) << 16);

  uint32_t phase = 0;
  bool ok = true;       // this thread's last wait completed
  // One MMA level: every thread's operand stores are made visible to the
  // tensor core, thread 0 issues `issue`, all wait for completion.
  auto level = [&](auto issue) -> bool {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    const int bad = __syncthreads_or(ok ? 0 : 1);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (bad) return false;
    if (tid == 0) {
      issue();
      g_commit(abar);
    }
    ok = mbar_wait(abar, phase);
    phase ^= 1;
    if (!ok) atomicExch(&g_tcg_timeout, 1);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    return true;
  };
  // MMA issue (thread 0): the start-address field of a descriptor is its low
  // 14 bits (address / 16), so a base descriptor plus offset / 16 addresses
  // every tile and K step (all offsets stay inside shared memory).
  auto issue_f1 = [&]() {
    const uint64_t da = g_desc(aA, kF1Lbo, kF1Sbo), db = g_desc(aB + kBF1, 128, 256);
#pragma unroll
    for (int T = 0; T < 8; ++T) g_mma(tmem + 32u * T, da + (T * kF1Tile >> 4), db, g_idesc(32), 0u);
  };
  auto issue_c = [&](uint32_t tile, uint32_t lbo, uint32_t sbo, uint32_t bmat) {
    const uint64_t da = g_desc(aA, lbo, sbo), db = g_desc(aB + bmat, 128, 1024);
#pragma unroll
    for (int T = 0; T < 4; ++T)
#pragma unroll
      for (int s = 0; s < 4; ++s)
        g_mma(tmem + 64u * T, da + ((T * tile + s * 2 * lbo) >> 4), db + (s * 256 >> 4), g_idesc(64), s > 0 ? 1u : 0u);
  };
  auto issue_i1 = [&]() {
    const uint64_t da = g_desc(aA, kI1Lbo, kI1Sbo), db = g_desc(aB + kBI1, 128, 512);
#pragma unroll
    for (int T = 0; T < 8; ++T)
#pragma unroll
      for (int s = 0; s < 2; ++s)
        g_mma(tmem + 16u * T, da + ((T * kI1Tile + s * 2 * kI1Lbo) >> 4), db + (s * 256 >> 4), g_idesc(16),
              s > 0 ? 1u : 0u);
  };

  const int Bh = B >> 1;
  // Between stages a thread keeps, for its 32 times t = l + 128 w + 32 i + 1024 n3,
  // the bf16 pair (item b, item b + 1) that multiplies the stage output: the
  // input v before stage 0, the gate x_n after stage n; the convolution itself
  // stays in TMEM (the output of I1) and is read again where it is needed.
  uint32_t zp[4][8];
  float u = 0.f;   // unscale factor of the I1 output
  // z of row i (8 values n3) from the I1 output r (or from v before stage 0)
  // z of row i (8 values n3) times `scale`: I1 output r times (u * scale) times
  // the gate pair, or (before stage 0) the input pair times scale
  auto z_of = [&](int i, const uint32_t (&r)[16], bool first, float scale, float2 (&zz)[8]) {
    const float us = first ? scale : u * scale;
#pragma unroll
    for (int n3 = 0; n3 < 8; ++n3) {
      const float g0 = __uint_as_float(zp[i][n3] << 16) * us, g1 = __uint_as_float(zp[i][n3] & 0xffff0000u) * us;
      zz[n3] = first ? make_float2(g0, g1)
                     : make_float2(__uint_as_float(r[2 * n3]) * g0, __uint_as_float(r[2 * n3 + 1]) * g1);
    }
  };
  auto i1_addr = [&](int i) { return tlane + 16u * (2 * i + hw); };
  // bf16 pairs of rows r0, r1 at this thread's 32 times
  auto load_pairs = [&](const __nv_bfloat16* base, size_t r0, size_t r1, size_t tb) {
    const unsigned short* g0p = reinterpret_cast<const unsigned short*>(base + r0 + tb);
    const unsigned short* g1p = reinterpret_cast<const unsigned short*>(base + r1 + tb);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int n3 = 0; n3 < 8; ++n3)
        zp[i][n3] = (uint32_t)__ldcs(g0p + 32 * i + 1024 * n3) | ((uint32_t)__ldcs(g1p + 32 * i + 1024 * n3) << 16);
  };
  for (long long p = blockIdx.x; p < npairs; p += gridDim.x) {
    const int c = (int)(p / Bh);
    const int b0 = 2 * (int)(p % Bh);
    const size_t r0 = ((size_t)b0 * D + c) * (size_t)kGL;
    const size_t r1 = r0 + (size_t)D * kGL;
    const size_t tb = (size_t)(l + 128 * w);
    load_pairs(v, r0, r1, tb);

    for (int n = 0; n < N; ++n) {
      const unsigned char* hrow = hptr[n] + (size_t)c * kGHRowBytes;
      const uint32_t* hw32 = reinterpret_cast<const uint32_t*>(hrow);
      const float inv_fc = __ldg(reinterpret_cast<const float*>(hrow + 4 * kGP));
      // L2 prefetch (bulk, no shared-memory destination) of what this stage
      // reads from HBM later: its spectrum row, its gate rows, and after the
      // last stage the next pair's input rows
      if (tid == 0) {
        bulk_prefetch_l2(hrow, (uint32_t)kGHRowBytes);
        bulk_prefetch_l2(xptr[n] + r0, 2 * kGL);
        bulk_prefetch_l2(xptr[n] + r1, 2 * kGL);
        if (n + 1 == N && p + gridDim.x < npairs) {
          const long long pn = p + gridDim.x;
          const size_t q0 = ((size_t)(2 * (int)(pn % Bh)) * D + (size_t)(pn / Bh)) * (size_t)kGL;
          bulk_prefetch_l2(v + q0, 2 * kGL);
          bulk_prefetch_l2(v + q0 + (size_t)D * kGL, 2 * kGL);
        }
      }
      const bool first = (n == 0);
      // ---- input scale: CTA max |component| of z
      float zm = 0.f;
      {
        auto proc = [&](int i, const uint32_t (&r)[16]) {
          float2 zz[8];
          z_of(i, r, first, 1.f, zz);
#pragma unroll
          for (int n3 = 0; n3 < 8; ++n3) zm = fmaxf(zm, fmaxf(fabsf(zz[n3].x), fabsf(zz[n3].y)));
        };
        if (first) {
          uint32_t r[16];
#pragma unroll
          for (int i = 0; i < 4; ++i) proc(i, r);
        } else {
          g_pipe4<16>(i1_addr, proc);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) zm = fmaxf(zm, __shfl_xor_sync(0xffffffffu, zm, o));
      if (l == 0) red[w] = zm;
      __syncthreads();
      zm = red[0];
#pragma unroll
      for (int k = 1; k < 8; ++k) zm = fmaxf(zm, red[k]);
      float s_in, inv_s;
      g_scale_in(zm, s_in, inv_s);
      // ---- F1 operand: own rows, K = n3 < 8
      {
        auto proc = [&](int i, const uint32_t (&r)[16]) {
          float2 zz[8];
          z_of(i, r, first, s_in, zz);
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint4 q4;
            q4.x = g_pack(zz[4 * cc].x, zz[4 * cc].y);
            q4.y = g_pack(zz[4 * cc + 1].x, zz[4 * cc + 1].y);
            q4.z = g_pack(zz[4 * cc + 2].x, zz[4 * cc + 2].y);
            q4.w = g_pack(zz[4 * cc + 3].x, zz[4 * cc + 3].y);
            *reinterpret_cast<uint4*>(sA + f1_base + cc * 128 + i * 8192) = q4;
          }
        };
        if (first) {
          uint32_t r[16];
#pragma unroll
          for (int i = 0; i < 4; ++i) proc(i, r);
        } else {
          g_pipe4<16>(i1_addr, proc);
        }
      }
      if (!level(issue_f1)) goto done;
      // ---- F1 out: twiddle w_P^{m' k3}, to F2 rows (k3, m'' = l) at K = 4w + i.
      // Chunks: k3 half hf (8 outputs) of row i, the four rows of one half
      // before the next; one 16-byte store per k3 gathers the four rows.
      {
        float2 cur[4], tw1i[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          cur[i] = make_float2(1.f, 0.f);
          // w_512^i, i < 4
          const float2 w512 = i == 0 ? make_float2(1.f, 0.f)
                              : i == 1 ? make_float2(0.99992470183914454f, -0.01227153828571993f)
                              : i == 2 ? make_float2(0.99969881869620425f, -0.02454122852291229f)
                                       : make_float2(0.99932238458834954f, -0.03680722294135883f);
          tw1i[i] = g_cmul(g_opaque(tw1), w512);
        }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[4][8];
          g_pipe4<16>([&](int i) { return tlane + 32u * (2 * i + hw) + 16u * hf; },
                      [&](int i, const uint32_t (&r)[16]) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                          const float2 vv = g_cmul(g_cval(r, j), cur[i]);
                          pk[i][j] = g_pack(vv.x, vv.y);
                          cur[i] = g_cmul(cur[i], tw1i[i]);
                        }
                      });
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(sA + f12_base + 4096 * (8 * hf + j)) =
                make_uint4(pk[0][j], pk[1][j], pk[2][j], pk[3][j]);
        }
      }
      if (!level([&]() { issue_c(kCTile, kCLbo, kCSbo, kBF32); })) goto done;
      // ---- F2 out: twiddle w_1024^{m'' k2}, to F3 rows (k3, k2) at K = m'' = l.
      // Chunk 2 t + hf: outputs k2 = 16 hf .. 16 hf + 15 of row t.
      {
        const float2 twb = g_opaque(tw2);
        float2 cur = make_float2(1.f, 0.f);
        g_pipe4<32>([&](int ch) { return tlane + 64u * (hw + 2 * (ch >> 1)) + 32u * (ch & 1); },
                    [&](int ch, const uint32_t (&r)[32]) {
                      const int t = ch >> 1, hf = ch & 1;
                      if (hf == 0) cur = make_float2(1.f, 0.f);
#pragma unroll
                      for (int j = 0; j < 16; ++j) {
                        const int k2 = 16 * hf + j;
                        const float2 vv = g_cmul(g_cval(r, j), cur);
                        cur = g_cmul(cur, twb);
                        const uint32_t off =
                            (uint32_t)(2 * (k2 >> 4) * kF3Tile + (k2 & 3) * 16 + 512 * ((k2 >> 2) & 3));
                        *reinterpret_cast<uint32_t*>(sA + (f23_base + t * f23_step) + off) = g_pack(vv.x, vv.y);
                      }
                    });
      }
      // ---- F3 out: 2^-20 C[k3 + 16 k2 + 512 k1] times the spectrum copy;
      // own rows as the I3 operand (K = k1). Chunk 2 t + hf holds bins
      // k1 = 16 hf .. 16 hf + 15 of row t; its 64 spectrum bytes are loaded
      // one chunk ahead (the first before the level's wait).
      {
        const uint4* hp0 = reinterpret_cast<const uint4*>(hw32 + (size_t)(128 * hw + 32 * q + l) * 32);
        constexpr int kRowStep = 256 * 32 / 4;   // uint4 from row t = 0 to row t = 1
        uint4 hcur[4], hnext[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) hcur[k] = __ldcs(hp0 + k);
        if (!level([&]() { issue_c(kF3Tile, kF3Lbo, kF3Sbo, kBF32); })) goto done;
        g_pipe4<32>([&](int ch) { return tlane + 64u * (hw + 2 * (ch >> 1)) + 32u * (ch & 1); },
                    [&](int ch, const uint32_t (&r)[32]) {
                      const int t = ch >> 1, hf = ch & 1;
                      if (ch < 3) {
                        const int tn = (ch + 1) >> 1, hn = (ch + 1) & 1;
#pragma unroll
                        for (int k = 0; k < 4; ++k) hnext[k] = __ldcs(hp0 + tn * kRowStep + 4 * hn + k);
                      }
#pragma unroll
                      for (int k = 0; k < 4; ++k) {
                        const uint32_t hu[4] = {hcur[k].x, hcur[k].y, hcur[k].z, hcur[k].w};
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                          const float2 hf2 = __half22float2(*reinterpret_cast<const __half2*>(&hu[e]));
                          const float2 cv = g_cval(r, 4 * k + e);
                          const float2 yv = g_cmul(cv, hf2);
                          o[e] = g_pack(yv.x, yv.y);
                        }
                        *reinterpret_cast<uint4*>(sA + (i3_base + t * i3_step) + (4 * hf + k) * 128) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                      }
#pragma unroll
                      for (int k = 0; k < 4; ++k) hcur[k] = hnext[k];
                    });
      }
      if (!level([&]() { issue_c(kCTile, kCLbo, kCSbo, kBI32); })) goto done;
      // ---- I3 out: twiddle w_1024^{-m'' k2}, to I2 rows (k3, m'') at K = k2
      {
        float2 cur = make_float2(1.f, 0.f), twb = make_float2(1.f, 0.f);
        g_pipe4<32>([&](int ch) { return tlane + 64u * (hw + 2 * (ch >> 1)) + 32u * (ch & 1); },
                    [&](int ch, const uint32_t (&r)[32]) {
                      const int t = ch >> 1, hf = ch & 1;
                      if (hf == 0) {
                        cur = make_float2(1.f, 0.f);
                        twb = g_opaque(t ? tw3b : tw3a);
                      }
#pragma unroll
                      for (int j = 0; j < 16; ++j) {
                        const int mpp = 16 * hf + j;
                        const float2 vv = g_cmul(g_cval(r, j), cur);
                        cur = g_cmul(cur, twb);
                        const uint32_t off = (uint32_t)((16 * (mpp >> 3) + 2 * (mpp & 1) + 4 * ((mpp >> 1) & 3)) * 1024);
                        *reinterpret_cast<uint32_t*>(sA + (i32_base + t * i32_step) + off) = g_pack(vv.x, vv.y);
                      }
                    });
      }
      if (!level([&]() { issue_c(kCTile, kCLbo, kCSbo, kBI32); })) goto done;
      // ---- I2 out: twiddle w_P^{-(m'' + 32 n2) k3}, to I1 rows m' at K = k3
      {
        const float2 twb = g_opaque(tw2i);
        float2 cur = make_float2(1.f, 0.f);
        g_pipe4<32>([&](int ch) { return tlane + 64u * (hw + 2 * (ch >> 1)) + 32u * (ch & 1); },
                    [&](int ch, const uint32_t (&r)[32]) {
                      const int t = ch >> 1, hf = ch & 1;
                      if (hf == 0) cur = g_opaque(t ? st2b : st2a);
#pragma unroll
                      for (int j = 0; j < 16; ++j) {
                        const int n2 = 16 * hf + j;
                        const float2 vv = g_cmul(g_cval(r, j), cur);
                        const int jj = n2 >> 2, ii = n2 & 3;
                        const uint32_t off = (uint32_t)((2 * ii + (jj >> 2)) * kI1Tile + 512 * (jj & 3));
                        *reinterpret_cast<uint32_t*>(sA + (i21_base + t * i21_step) + off) = g_pack(vv.x, vv.y);
                        cur = g_cmul(cur, twb);
                      }
                    });
      }
      // gate rows of this stage, loaded while the last level runs
      load_pairs(xptr[n], r0, r1, tb);
      if (!level(issue_i1)) goto done;
      u = 0x1p16f * inv_s * inv_fc;
    }
    // ---- y: the last stage's I1 output, unscaled and gated
    {
      __nv_bfloat16* y0 = y + r0 + tb;
      __nv_bfloat16* y1 = y + r1 + tb;
      g_pipe4<16>(i1_addr, [&](int i, const uint32_t (&r)[16]) {
        float2 zz[8];
        z_of(i, r, false, 1.f, zz);
#pragma unroll
        for (int n3 = 0; n3 < 8; ++n3) {
          y0[32 * i + 1024 * n3] = __float2bfloat16_rn(zz[n3].x);
          y1[32 * i + 1024 * n3] = __float2bfloat16_rn(zz[n3].y);
        }
      });
    }
    // the next pair's first level overwrites TMEM: order these reads before it
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  }
done:
  // after a timeout: wait (bounded, 1 s) for the MMAs of the last issued level
  if (!ok) mbar_wait(abar, phase ^ 1, 1000000000ull);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (w == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kGCols));
}

// Spectrum copy for tcg_forward_kernel, one CTA per channel: 2L f16x2 bins of
// f_c H[k] in F3-row order (word r * 32 + k1 for row r = (k3, k2) and bin
// k = k3 + 16 k2 + 512 k1, H the 2L-point spectrum of the zero-padded filter),
// then 1 / f_c. The natural copy holds H / (4L) for k < L, bin 0 packing
// (H[0], H[L]); bins above L are conjugate mirrors. f_c is the power of two
// that brings the largest component of f_c H into [2^14, 2^15).
__global__ void tcg_spectrum_kernel(const float2* __restrict__ nat, unsigned char* __restrict__ out) {
  __shared__ float redm[8];
  const int c = blockIdx.x, tid = threadIdx.x;
  const float2* __restrict__ nr = nat + (size_t)c * kGL;
  unsigned char* row = out + (size_t)c * kGHRowBytes;
  float mx = 0.f;
  for (int i = tid; i < kGL; i += blockDim.x) mx = fmaxf(mx, fmaxf(fabsf(nr[i].x), fabsf(nr[i].y)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) redm[tid >> 5] = mx;
  __syncthreads();
  mx = redm[0];
  for (int k = 1; k < (int)(blockDim.x >> 5); ++k) mx = fmaxf(mx, redm[k]);
  mx *= (float)(2 * kGP);                                        // largest component of H
  int e = (int)((__float_as_uint(mx) >> 23) & 0xff);             // mx < 2^(e - 126)
  e = e < 15 ? 15 : (e > 254 ? 254 : e);
  const float fH = __uint_as_float((unsigned)(268 - e > 254 ? 254 : 268 - e) << 23);   // 2^(141 - e)
  float inv_f = __uint_as_float((unsigned)(e - 14) << 23);                              // 2^(e - 141)
  float f = fH * (float)(2 * kGP);                               // applied to the natural copy
  if (mx == 0.f) { f = 1.f; inv_f = 1.f; }
  uint32_t* wds = reinterpret_cast<uint32_t*>(row);
  for (int idx = tid; idx < kGP; idx += blockDim.x) {
    const int r = idx >> 5, k1 = idx & 31;
    const int T = r >> 7, p = r & 127;
    // row r = 128 T + p of F3: k3 = 8 (T & 1) + ((p >> 2) & 7), k2 = (p & 3) + 4 (p >> 5) + 16 (T >> 1)
    const int k3 = 8 * (T & 1) + ((p >> 2) & 7);
    const int k2 = (p & 3) + 4 * (p >> 5) + 16 * (T >> 1);
    const int k = k3 + 16 * k2 + 512 * k1;
    float2 hv;
    if (k == 0) hv = make_float2(nr[0].x, 0.f);
    else if (k == kGL) hv = make_float2(nr[0].y, 0.f);
    else if (k < kGL) hv = nr[k];
    else { const float2 m = nr[kGP - k]; hv = make_float2(m.x, -m.y); }
    wds[idx] = g_pack(f * hv.x, f * hv.y);
  }
  if (tid == 0) {
    float* tail = reinterpret_cast<float*>(row + 4 * kGP);
    tail[0] = inv_f;
    tail[1] = 0.f;
    tail[2] = 0.f;
    tail[3] = 0.f;
  }
}

cudaError_t launch_tcg_forward(const FusedLaunch& p, cudaStream_t s) {
  auto k = tcg_forward_kernel;
  cudaError_t e = cudaFuncSetAttribute((const void*)k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute((const void*)k, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  // Two CTAs per SM: shared memory admits at most two, and their TMEM
  // allocations (256 columns each) fill the SM's 512 columns exactly, so no
  // allocation ever waits on another CTA.
  static_assert(2 * kGCols <= 512 && 3 * (kGSmem + 1024) > 228 * 1024, "at most two resident CTAs per SM");
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  int grid = 2 * sms;
  const long long npairs = (long long)(p.B / 2) * p.D;
  if ((long long)grid > npairs) grid = (int)npairs;
  GatePtrs<__nv_bfloat16> xp;
  for (int i = 0; i < kMaxOrder; ++i) xp.p[i] = reinterpret_cast<const __nv_bfloat16*>(p.x[i]);
  k<<<grid, kGT, kGSmem, s>>>(reinterpret_cast<const __nv_bfloat16*>(p.v), xp, p.hh,
                              reinterpret_cast<__nv_bfloat16*>(p.y), p.B, p.D, p.N, npairs);
  return cudaGetLastError();
}

cudaError_t launch_tcg_spectrum(const float2* nat, float2* tcs, int D, cudaStream_t s) {
  tcg_spectrum_kernel<<<D, 256, 0, s>>>(nat, reinterpret_cast<unsigned char*>(tcs));
  return cudaGetLastError();
}

int tcg_read_and_clear_timeout() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tcg_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_tcg_timeout, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

}  // namespace hyena
