// tc05.cu -- Hyena order-N forward on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in TMEM) for bf16 I/O, L = 2048, B even.
// Built when HYENA_TC05 is defined to 1 (the default build serves this shape
// with the mma.sync kernel of tc_fused.cu, which measured faster: 60 us
// against 79 us per forward on the order-2, B=4, D=768 workload).
//
// As in the mma.sync kernel, batch items b, b+1 of channel c share h_c, so
// their causal convolutions are the real and imaginary parts of one complex
// convolution of c[n] = z_b[n] + i z_{b+1}[n] on the 2L zero-padded grid
// (glossary "Hyena（ハイエナ）", section 計算効率; "Native Multi-Dimensional
// Subquadratic Operators via Input Dependent Long Convolutions", section 境界の処理).
// The 4096-point transform runs as three radix-16 DFT passes, each one GEMM
// D[256 x 32] = A[256 x K] B[32 x K]^T on the tensor cores:
//   n = 256 a + 16 b + c,  k = d + 16 e + 256 f
//   P1 over a (rows (b,c), a < 8 nonzero), twiddle w_4096^{(16b+c) d}
//   P2 over b (rows (d,c)),               twiddle w_256^{c e}
//   P3 over c (rows (d,e))                -> X[d + 16 e + 256 f]
// then the product with the filter spectrum, and the inverse passes in the
// mirrored order (over f, e, d), keeping a < 8 (t < L) in the last one.
// Complex values are interleaved (re, im) along K and N, so the planar DFT
// matrix B carries the complex arithmetic and each thread moves one packed
// f16x2 word per value. Thread r owns TMEM lane row r in every pass (tile
// r / 128 in TMEM columns 32 (r / 128) ...): between passes it reads its row
// of D (tcgen05.ld), applies the twiddles in fp32 and writes the values into
// the rows of the next pass's A operand in shared memory (one transpose per
// pass). One elected thread issues the MMAs; completion arrives on an
// mbarrier (tcgen05.commit). z stays in registers between the N stages.
// Operands are scaled by exact powers of two (|f16| < 2^15) and unscaled
// exactly at the end.
#include <cuda_fp16.h>

#include "fft_engine.cuh"
#include "kernels.cuh"

namespace hyena {

namespace {

constexpr int kT5Threads = 256;
constexpr int kT5L = 2048;
constexpr uint32_t kT5Cols = 64;          // TMEM columns per CTA (two 128-row tiles x 32)
// A operand: K-major, no swizzle, core matrices 8 rows x 16 B; K chunks at
// kLBO, 8-row groups at kSBO (strides chosen for conflict-free transposes)
constexpr uint32_t kLBO = 144, kSBO = 608;
constexpr uint32_t kABytes = 32 * kSBO;   // 256 rows
constexpr uint32_t kTileA = 16 * kSBO;    // rows 128..255
// B operands (K-major, canonical strides LBO = 128, SBO = (K / 8) * 128)
constexpr uint32_t kB1 = 0;               // forward P1: N 32 x K 16
constexpr uint32_t kB16 = 1024;           // forward radix 16: N 32 x K 32
constexpr uint32_t kB16i = 3072;          // inverse radix 16
constexpr uint32_t kB1i = 5120;           // inverse P1': N 16 x K 32
constexpr uint32_t kBBytes = 6144;
constexpr uint32_t kTw2Bytes = 256 * 8;   // w_256^{j x}, [j][x]
constexpr uint32_t kHRow = 4096 * 4 + 16; // spectrum copy row: 4096 f16x2 + (1/f_c) + pad
constexpr uint32_t kGateRow = kT5L * 2;   // one bf16 row
// byte offsets in dynamic shared memory
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kABytes;
constexpr uint32_t kOffTw = kOffB + kBBytes;
constexpr uint32_t kOffH = kOffTw + kTw2Bytes;             // [kHRow] (single buffer)
constexpr uint32_t kOffX = kOffH + kHRow;                   // [2][2][kGateRow]
constexpr uint32_t kOffV = kOffX + 4 * kGateRow;            // [2][kGateRow]
constexpr uint32_t kOffMisc = kOffV + 2 * kGateRow;         // mbarrier, TMEM slot, reductions
constexpr uint32_t kSmemBytes = kOffMisc + 128;

// idesc: f32 accumulate, f16 A and B, both K-major, M = 128
__host__ __device__ constexpr uint32_t idesc_f16(int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46);
}

// byte offset of complex element q (packed f16x2) of A-operand row m
__device__ __forceinline__ uint32_t a_off(int m, int q) {
  return (uint32_t)((m & 7) * 16 + (q & 3) * 4 + (q >> 2) * kLBO + (m >> 3) * kSBO);
}

__device__ __forceinline__ uint32_t pack_h2u(float re, float im) {
  const __half2 v = __floats2half2_rn(re, im);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void mma_f16(uint32_t dtmem, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(dtmem),
      "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0));
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// Bounded wait for the mbarrier phase; false after the iteration limit.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase) {
  for (int it = 0; it < (1 << 24); ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P1;\n\t}\n"
        : "=r"(done)
        : "r"(bar), "r"(phase)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ void tmem_ld32(uint32_t addr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld16(uint32_t addr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(addr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ float2 cmul2(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}

__device__ __forceinline__ float bfu(unsigned short u) { return __uint_as_float((unsigned)u << 16); }

// Power of two s with bound * s < 2^12 (and 1/s), from a bound >= 0.
__device__ __forceinline__ void scale12(float mx, float& s, float& inv_s) {
  int e = (int)((__float_as_uint(mx) >> 23) & 0xff);   // mx < 2^(e - 126)
  e = e < 14 ? 14 : (e > 254 ? 254 : e);
  s = __uint_as_float((unsigned)(265 - e) << 23);      // 2^(138 - e)
  inv_s = __uint_as_float((unsigned)(e - 11) << 23);   // 2^(e - 138)
  if (mx == 0.f) { s = 1.f; inv_s = 1.f; }
}

__device__ int g_tc05_timeout;

}  // namespace

// The planar DFT matrices (f16, K-major canonical layout) and the w_256
// twiddle table, built once per CTA.
__device__ __forceinline__ void tc05_build_constants(unsigned char* sm, int tid) {
  // B element (n, k) of a K-major operand with K f16 columns
  auto put = [&](uint32_t base, int K, int n, int k, float val) {
    const uint32_t o = base + (uint32_t)((n & 7) * 16 + (k & 7) * 2 + (k >> 3) * 128 + (n >> 3) * (K / 8) * 128);
    *reinterpret_cast<__half*>(sm + kOffB + o) = __float2half_rn(val);
  };
  // forward: F[i][o] = w16^{i o}; inverse: conjugate. rows 2o + rho, cols 2i + sigma
  for (int idx = tid; idx < 16 * 16 * 2; idx += kT5Threads) {
    const int inv = idx >> 8, o = (idx >> 4) & 15, i = idx & 15;
    float sn, cs;
    sincospif(-(float)((i * o) & 15) / 8.0f, &sn, &cs);   // w16^{io} = cs + i sn
    const float Fr = cs, Fi = inv ? -sn : sn;
    const uint32_t base = inv ? kB16i : kB16;
    put(base, 32, 2 * o, 2 * i, Fr);
    put(base, 32, 2 * o, 2 * i + 1, -Fi);
    put(base, 32, 2 * o + 1, 2 * i, Fi);
    put(base, 32, 2 * o + 1, 2 * i + 1, Fr);
    if (!inv && i < 8) {   // forward P1: inputs a < 8 only
      put(kB1, 16, 2 * o, 2 * i, Fr);
      put(kB1, 16, 2 * o, 2 * i + 1, -Fi);
      put(kB1, 16, 2 * o + 1, 2 * i, Fi);
      put(kB1, 16, 2 * o + 1, 2 * i + 1, Fr);
    }
    if (inv && o < 8) {    // inverse P1': outputs a < 8 only
      put(kB1i, 32, 2 * o, 2 * i, Fr);
      put(kB1i, 32, 2 * o, 2 * i + 1, -Fi);
      put(kB1i, 32, 2 * o + 1, 2 * i, Fi);
      put(kB1i, 32, 2 * o + 1, 2 * i + 1, Fr);
    }
  }
  float2* tw2 = reinterpret_cast<float2*>(sm + kOffTw);
  for (int idx = tid; idx < 256; idx += kT5Threads) {
    const int j = idx >> 4, x = idx & 15;
    float sn, cs;
    sincospif(-(float)((j * x) & 255) / 128.0f, &sn, &cs);
    tw2[idx] = make_float2(cs, sn);
  }
}

__global__ void __launch_bounds__(kT5Threads, 3)
tc05_forward_kernel(const __nv_bfloat16* __restrict__ v, GatePtrs<__nv_bfloat16> x, SpecPtrs hh,
                    __nv_bfloat16* __restrict__ y, int B, int D, int N, long long npairs) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const int r = threadIdx.x, warp = r >> 5, lane = r & 31;
  const int hi = r >> 4, lo = r & 15;   // row r = 16 hi + lo
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kOffMisc);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kOffMisc + 8);
  float* red = reinterpret_cast<float*>(sm + kOffMisc + 16);   // [8]
  unsigned char* sA = sm + kOffA;
  const uint32_t aA = smem_u32(sA), aB = smem_u32(sm + kOffB), abar = smem_u32(bar);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(kT5Cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  if (r == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(abar), "r"(1));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc05_build_constants(sm, r);
  // per-thread twiddle generators (powers formed by fp32 recurrence, <= 15 steps):
  //   forward P1, row (b,c) = r:      w4096^{r d} = om^d,        om = w4096^r
  //   inverse P2', row (d,c) = (hi,lo): w4096^{-(16 b + lo) hi} = be sg^b,
  //                                    be = w4096^{-lo hi}, sg = w256^{-hi}
  float2 om, be, sg;
  {
    float sn, cs;
    sincospif(-(float)r / 2048.0f, &sn, &cs);
    om = make_float2(cs, sn);
    sincospif((float)((lo * hi) & 4095) / 2048.0f, &sn, &cs);
    be = make_float2(cs, sn);
    sincospif((float)hi / 128.0f, &sn, &cs);
    sg = make_float2(cs, sn);
  }
  // A-operand store bases of the two transposes (row 16 z + lo at K = hi, and
  // row 16 hi + z at K = lo); z adds compile-time offsets
  const uint32_t baseA = (uint32_t)((lo & 7) * 16 + (hi & 3) * 4 + (hi >> 2) * kLBO + (lo >> 3) * kSBO);
  const uint32_t baseB = (uint32_t)((lo & 3) * 4 + (lo >> 2) * kLBO + hi * 2 * kSBO);
  const uint32_t baseS = (uint32_t)((r & 7) * 16 + (r >> 3) * kSBO);   // own row
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tslot;
  const uint32_t tld = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + 32u * (uint32_t)(warp >> 2);
  const float2* tw2 = reinterpret_cast<const float2*>(sm + kOffTw);
  uint32_t phase = 0;
  bool ok = true;

  const int Bh = B >> 1;
  auto pair_rows = [&](long long pp, size_t& r0, size_t& r1, int& c) {
    c = (int)(pp / Bh);
    const int b0 = 2 * (int)(pp % Bh);
    r0 = ((size_t)b0 * D + c) * (size_t)kT5L;
    r1 = r0 + (size_t)D * kT5L;
  };
  unsigned char* hbuf = sm + kOffH;
  unsigned char* xbuf = sm + kOffX;
  unsigned char* vbuf = sm + kOffV;
  auto stage_job = [&](long long pp, int n, int par) {
    size_t q0, q1;
    int qc;
    pair_rows(pp, q0, q1, qc);
    block_copy_async(xbuf + par * 2 * kGateRow, pick(x, n) + q0, kGateRow, r, kT5Threads);
    block_copy_async(xbuf + par * 2 * kGateRow + kGateRow, pick(x, n) + q1, kGateRow, r, kT5Threads);
  };

  auto stage_spectrum = [&](long long pp, int n) {
    const int qc = (int)(pp / Bh);
    block_copy_async(hbuf, reinterpret_cast<const unsigned char*>(pick(hh, n)) + (size_t)qc * kHRow, kHRow, r,
                     kT5Threads);
  };

  // one MMA round: operands are in shared memory; every thread has fenced its
  // writes to the async proxy. Returns false (on every thread) after a timeout.
  auto round = [&](uint32_t bdesc_base, uint32_t bsbo, int ksteps, uint32_t idesc) -> bool {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (r == 0) {
#pragma unroll 1
      for (int t = 0; t < 2; ++t)
#pragma unroll 1
        for (int s = 0; s < ksteps; ++s)
          mma_f16(tmem + 32u * t, smem_desc(aA + t * kTileA + s * 2 * kLBO, kLBO, kSBO),
                  smem_desc(aB + bdesc_base + s * 256, 128, bsbo), idesc, s > 0 ? 1u : 0u);
      mma_commit(abar);
    }
    const bool done = mbar_wait(abar, phase);
    phase ^= 1;
    if (!done && lane == 0) atomicExch(&g_tc05_timeout, 1);
    // every thread leaves together when any wait ran out
    ok = __syncthreads_and(done) != 0;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    return ok;
  };

  long long p = blockIdx.x;
  int par = 0;
  if (p < npairs) {
    size_t r0, r1;
    int c;
    pair_rows(p, r0, r1, c);
    block_copy_async(vbuf, v + r0, kGateRow, r, kT5Threads);
    block_copy_async(vbuf + kGateRow, v + r1, kGateRow, r, kT5Threads);
    stage_job(p, 0, 0);
    stage_spectrum(p, 0);
  }
  cp_async_commit();

  float2 za[8];
  for (; p < npairs && ok; p += gridDim.x) {
    size_t r0, r1;
    int c;
    pair_rows(p, r0, r1, c);
    for (int n = 0; n < N && ok; ++n, par ^= 1) {
      cp_async_wait_all();          // this job's spectrum and gate rows (and this pair's v)
      __syncthreads();
      if (n == 0) {
        const unsigned short* vs = reinterpret_cast<const unsigned short*>(vbuf);
#pragma unroll
        for (int a = 0; a < 8; ++a) za[a] = make_float2(bfu(vs[256 * a + r]), bfu(vs[kT5L + 256 * a + r]));
      }
      // CTA max |z| -> power-of-two input scale
      float zm = 0.f;
#pragma unroll
      for (int a = 0; a < 8; ++a) zm = fmaxf(zm, fmaxf(fabsf(za[a].x), fabsf(za[a].y)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) zm = fmaxf(zm, __shfl_xor_sync(0xffffffffu, zm, o));
      if (lane == 0) red[warp] = zm;
      __syncthreads();              // also: every thread is past its reads of v
      zm = red[0];
#pragma unroll
      for (int w = 1; w < kT5Threads / 32; ++w) zm = fmaxf(zm, red[w]);
      float s0, inv_s0;
      scale12(zm, s0, inv_s0);
      // stage the next job (its buffers were last read by the previous job)
      if (n == 0 && p + gridDim.x < npairs) {
        size_t q0, q1;
        int qc;
        pair_rows(p + gridDim.x, q0, q1, qc);
        block_copy_async(vbuf, v + q0, kGateRow, r, kT5Threads);
        block_copy_async(vbuf + kGateRow, v + q1, kGateRow, r, kT5Threads);
      }
      if (n + 1 < N) stage_job(p, n + 1, par ^ 1);
      else if (p + gridDim.x < npairs) stage_job(p + gridDim.x, 0, par ^ 1);
      cp_async_commit();

      // ---- P1 (over a): own row r = (b,c), complex K index a < 8
      {
        uint32_t w[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) w[a] = pack_h2u(za[a].x * s0, za[a].y * s0);
        *reinterpret_cast<uint4*>(sA + baseS) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(sA + baseS + kLBO) = make_uint4(w[4], w[5], w[6], w[7]);
      }
      if (!round(kB1, 256, 1, idesc_f16(32))) break;
      float dv[32];
      tmem_ld32(tld, dv);
      // twiddle w4096^{r d}; to P2 rows (d, c = lo) at K = b (= hi)
      {
        float2 cur = make_float2(1.f, 0.f);
#pragma unroll
        for (int d = 0; d < 16; ++d) {
          const float2 q = cmul2(make_float2(dv[2 * d], dv[2 * d + 1]), cur);
          *reinterpret_cast<uint32_t*>(sA + baseA + d * 2 * kSBO) = pack_h2u(q.x, q.y);
          cur = cmul2(cur, om);
        }
      }
      if (!round(kB16, 512, 2, idesc_f16(32))) break;
      tmem_ld32(tld, dv);
      // scale 2^-4, twiddle w256^{c e} (c = lo); to P3 rows (d = hi, e) at K = c
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float2 q = cmul2(make_float2(dv[2 * e] * 0.0625f, dv[2 * e + 1] * 0.0625f), tw2[e * 16 + lo]);
        *reinterpret_cast<uint32_t*>(sA + baseB + (e & 7) * 16 + (e >> 3) * kSBO) = pack_h2u(q.x, q.y);
      }
      if (!round(kB16, 512, 2, idesc_f16(32))) break;
      tmem_ld32(tld, dv);
      // X[d + 16 e + 256 f] (row (d, e) = (hi, lo)) times the filter spectrum
      const unsigned char* hs = hbuf;
      const uint32_t* hrow = reinterpret_cast<const uint32_t*>(hs);
      const float inv_fc = *reinterpret_cast<const float*>(hs + 4096 * 4);
#pragma unroll
      for (int qd = 0; qd < 4; ++qd) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int f = 4 * qd + j;
          const uint32_t hu = hrow[f * 256 + r];
          const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hu));
          const float2 q = cmul2(make_float2(dv[2 * f], dv[2 * f + 1]), hf);
          w[j] = pack_h2u(q.x, q.y);
        }
        *reinterpret_cast<uint4*>(sA + baseS + qd * kLBO) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      // ---- inverse: P3' over f (rows (d, e) = (hi, lo)), outputs c
      if (!round(kB16i, 512, 2, idesc_f16(32))) break;
      // every thread is past its reads of the spectrum row: stage the next job's
      if (n + 1 < N) stage_spectrum(p, n + 1);
      else if (p + gridDim.x < npairs) stage_spectrum(p + gridDim.x, 0);
      cp_async_commit();
      tmem_ld32(tld, dv);
      // scale 2^-4, twiddle w256^{-e c} (e = lo); to P2' rows (d = hi, c) at K = e
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) {
        const float2 t = tw2[cc * 16 + lo];
        const float2 q = cmul2(make_float2(dv[2 * cc] * 0.0625f, dv[2 * cc + 1] * 0.0625f), make_float2(t.x, -t.y));
        *reinterpret_cast<uint32_t*>(sA + baseB + (cc & 7) * 16 + (cc >> 3) * kSBO) = pack_h2u(q.x, q.y);
      }
      if (!round(kB16i, 512, 2, idesc_f16(32))) break;
      tmem_ld32(tld, dv);
      // P2' rows (d, c) = (hi, lo), outputs b: scale 2^-4, twiddle w4096^{-(16b+c) d};
      // to P1' rows (b, c) at K = d
      {
        float2 cur = be;
#pragma unroll
        for (int b = 0; b < 16; ++b) {
          const float2 q = cmul2(make_float2(dv[2 * b] * 0.0625f, dv[2 * b + 1] * 0.0625f), cur);
          *reinterpret_cast<uint32_t*>(sA + baseA + b * 2 * kSBO) = pack_h2u(q.x, q.y);
          cur = cmul2(cur, sg);
        }
      }
      if (!round(kB1i, 512, 2, idesc_f16(16))) break;
      float ov[16];
      tmem_ld16(tld, ov);
      // P1' rows (b, c) = r: outputs a < 8 -> t = 256 a + r; unscale, gate
      const float u = 4096.f * inv_s0 * inv_fc;
      const unsigned short* xs = reinterpret_cast<const unsigned short*>(xbuf + par * 2 * kGateRow);
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const int t = 256 * a + r;
        za[a] = make_float2(ov[2 * a] * u * bfu(xs[t]), ov[2 * a + 1] * u * bfu(xs[kT5L + t]));
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    }
    if (!ok) break;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      const int t = 256 * a + r;
      y[r0 + t] = __float2bfloat16_rn(za[a].x);
      y[r1 + t] = __float2bfloat16_rn(za[a].y);
    }
  }
  cp_async_wait_all();
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kT5Cols));
}

// Spectrum copy for this kernel, one CTA per channel: row c holds, for thread
// row r and f < 16, f16x2 of f_c H[k] / 4096 at [f][r] with k = (r >> 4) +
// 16 (r & 15) + 256 f (H the 4096-point spectrum of the zero-padded filter;
// the natural copy holds H / 8192 for k <= 2048, bin 0 packing (H[0], H[2048])),
// then 1 / f_c as a float. f_c is the power of two that brings every
// component below 2^-5, so that |X H f_c| < 2^15 for |X| < 2^19 sqrt(2).
__global__ void tc05_spectrum_kernel(const float2* __restrict__ nat, unsigned char* __restrict__ out, int M) {
  __shared__ float redm[8];
  const int c = blockIdx.x, tid = threadIdx.x;
  const float2* __restrict__ nr = nat + (size_t)c * M;
  unsigned char* row = out + (size_t)c * kHRow;
  float mx = 0.f;
  for (int i = tid; i < kT5L; i += blockDim.x) mx = fmaxf(mx, fmaxf(fabsf(nr[i].x), fabsf(nr[i].y)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) redm[tid >> 5] = mx;
  __syncthreads();
  mx = redm[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, redm[w]);
  const float hc = 2.f * mx;                                   // component bound of H / 4096
  int e = (int)((__float_as_uint(hc) >> 23) & 0xff);           // hc < 2^(e - 126)
  e = e < 1 ? 1 : (e > 248 ? 248 : e);
  float f = __uint_as_float((unsigned)(248 - e) << 23);        // 2^(121 - e): hc f < 2^-5
  float inv_f = __uint_as_float((unsigned)(e + 6) << 23);      // 2^(e - 121)
  if (hc == 0.f) { f = 1.f; inv_f = 1.f; }
  uint32_t* w = reinterpret_cast<uint32_t*>(row);
  for (int i = tid; i < 4096; i += blockDim.x) {
    const int fq = i >> 8, rr = i & 255;
    const int k = (rr >> 4) + 16 * (rr & 15) + 256 * fq;
    float2 h;
    if (k == 0) h = make_float2(nr[0].x, 0.f);
    else if (k == kT5L) h = make_float2(nr[0].y, 0.f);
    else if (k < kT5L) h = nr[k];
    else { const float2 m = nr[2 * kT5L - k]; h = make_float2(m.x, -m.y); }
    const __half2 v2 = __floats2half2_rn(2.f * f * h.x, 2.f * f * h.y);
    w[i] = *reinterpret_cast<const uint32_t*>(&v2);
  }
  if (tid == 0) {
    reinterpret_cast<float*>(row + 4096 * 4)[0] = inv_f;
    reinterpret_cast<float*>(row + 4096 * 4)[1] = 0.f;
    reinterpret_cast<float*>(row + 4096 * 4)[2] = 0.f;
    reinterpret_cast<float*>(row + 4096 * 4)[3] = 0.f;
  }
}

cudaError_t launch_tc05_forward(const FusedLaunch& p, cudaStream_t s) {
  auto k = tc05_forward_kernel;
  cudaError_t e = cudaFuncSetAttribute((const void*)k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute((const void*)k, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  // Resident CTAs per SM from the shared-memory and register budgets
  // (__launch_bounds__(256, 3)): the occupancy query reports one CTA per SM
  // for this kernel, while three fit and run side by side (measured 1.5x with
  // two, 1.6x with three). Three CTAs x 64 TMEM columns stay within the SM's
  // 512, so no allocation waits on another CTA.
  int dev = 0, sms = 0, smem_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess)
    return e;
  int per_sm = smem_sm / (int)(kSmemBytes + 1024);
  if (per_sm > 3) per_sm = 3;
  if (per_sm < 1) per_sm = 1;
  static_assert(3 * kT5Cols <= 512, "TMEM columns of the resident CTAs");
  long long grid = (long long)per_sm * sms;
  const long long npairs = (long long)(p.B / 2) * p.D;
  if (grid > npairs) grid = npairs;
  GatePtrs<__nv_bfloat16> xp;
  for (int i = 0; i < kMaxOrder; ++i) xp.p[i] = reinterpret_cast<const __nv_bfloat16*>(p.x[i]);
  k<<<(int)grid, kT5Threads, kSmemBytes, s>>>(reinterpret_cast<const __nv_bfloat16*>(p.v), xp, p.hh,
                                              reinterpret_cast<__nv_bfloat16*>(p.y), p.B, p.D, p.N, npairs);
  return cudaGetLastError();
}

cudaError_t launch_tc05_spectrum(const float2* nat, float2* tcs, int D, int M, cudaStream_t s) {
  tc05_spectrum_kernel<<<D, 256, 0, s>>>(nat, reinterpret_cast<unsigned char*>(tcs), M);
  return cudaGetLastError();
}

int tc05_read_and_clear_timeout() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc05_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (v) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_tc05_timeout, &zero, sizeof(int));
  }
  return v;
}

}  // namespace hyena
