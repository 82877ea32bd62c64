// tcgen05.cuh -- helpers of the tcgen05 (5th-generation tensor core) kernels:
// instruction and shared-memory descriptors for kind::f16 MMAs with f32
// accumulators in TMEM, TMEM loads whose wait is tied to the loaded
// registers, a one-ahead pipelined TMEM reader, f16 packing, complex
// arithmetic, and the real form of DFT matrices as K-major B operands.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace hyena {

// instruction descriptor: f32 accumulate, f16 A and B, both K-major, M = 128
__host__ __device__ constexpr uint32_t g_idesc(int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}


__device__ __forceinline__ uint64_t g_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46);
}

__device__ __forceinline__ void g_mma(uint32_t dtmem, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(dtmem),
      "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0));
}

__device__ __forceinline__ void g_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

#define G_LD_REGS16(r, o)                                                                                      \
  "=r"(r[o + 0]), "=r"(r[o + 1]), "=r"(r[o + 2]), "=r"(r[o + 3]), "=r"(r[o + 4]), "=r"(r[o + 5]),              \
      "=r"(r[o + 6]), "=r"(r[o + 7]), "=r"(r[o + 8]), "=r"(r[o + 9]), "=r"(r[o + 10]), "=r"(r[o + 11]),        \
      "=r"(r[o + 12]), "=r"(r[o + 13]), "=r"(r[o + 14]), "=r"(r[o + 15])

// 32 consecutive TMEM columns of this thread's lane (not yet waited for)
__device__ __forceinline__ void g_ld32(uint32_t addr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : G_LD_REGS16(r, 0), G_LD_REGS16(r, 16)
      : "r"(addr));
}
__device__ __forceinline__ void g_ld16(uint32_t addr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : G_LD_REGS16(r, 0)
      : "r"(addr));
}
// Wait for this thread's TMEM loads. The loaded registers are operands of the
// wait, so no use of them can be scheduled before it.
#define G_RW_REGS16(r, o)                                                                                      \
  "+r"(r[o + 0]), "+r"(r[o + 1]), "+r"(r[o + 2]), "+r"(r[o + 3]), "+r"(r[o + 4]), "+r"(r[o + 5]),              \
      "+r"(r[o + 6]), "+r"(r[o + 7]), "+r"(r[o + 8]), "+r"(r[o + 9]), "+r"(r[o + 10]), "+r"(r[o + 11]),        \
      "+r"(r[o + 12]), "+r"(r[o + 13]), "+r"(r[o + 14]), "+r"(r[o + 15])
__device__ __forceinline__ void g_wait32(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : G_RW_REGS16(r, 0), G_RW_REGS16(r, 16)::"memory");
}
__device__ __forceinline__ void g_wait16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : G_RW_REGS16(r, 0)::"memory");
}
#undef G_RW_REGS16
#undef G_LD_REGS16

__device__ __forceinline__ uint32_t g_pack(float re, float im) {
  const __half2 v = __floats2half2_rn(re, im);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// a * b: (a.x b.x - a.y b.y, a.x b.y + a.y b.x), two FMUL and two FFMA
__device__ __forceinline__ float2 g_cmul(float2 a, float2 b) {
  return make_float2(fmaf(a.x, b.x, -(a.y * b.y)), fmaf(a.x, b.y, a.y * b.x));
}

// The twiddle powers of a recurrence depend only on per-thread constants; a
// compiler that hoists them out of the pair and stage loops holds dozens of
// them in registers for the whole kernel. Passing the base through an opaque
// move keeps each recurrence where its powers are used.
__device__ __forceinline__ float2 g_opaque(float2 a) {
  float2 b;
  asm volatile("mov.b32 %0, %2;\n\tmov.b32 %1, %3;" : "=f"(b.x), "=f"(b.y) : "f"(a.x), "f"(a.y));
  return b;
}

template <int R>
__device__ __forceinline__ float2 g_cval(const uint32_t (&r)[R], int j) {
  return make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
}

// Four TMEM chunks of C columns (C = 16 or 32) read one ahead of their use:
// chunk j + 1 is loading while chunk j is processed.
template <int C, typename Addr, typename Proc>
__device__ __forceinline__ void g_pipe4(Addr addr, Proc proc) {
  uint32_t ra[C], rb[C];
  auto ld = [](uint32_t a, uint32_t (&r)[C]) {
    if constexpr (C == 32) g_ld32(a, r); else g_ld16(a, r);
  };
  auto wt = [](uint32_t (&r)[C]) {
    if constexpr (C == 32) g_wait32(r); else g_wait16(r);
  };
  ld(addr(0), ra);
  wt(ra);
  ld(addr(1), rb);
  proc(0, ra);
  wt(rb);
  ld(addr(2), ra);
  proc(1, rb);
  wt(ra);
  ld(addr(3), rb);
  proc(2, ra);
  wt(rb);
  proc(3, rb);
}

// w_n^{e} = exp(-2 pi i e / n) for an exact integer e (|e| < n)
__device__ __forceinline__ float2 g_root(int e, int n) {
  float s, c;
  sincospif(-2.0f * (float)e / (float)n, &s, &c);
  return make_float2(c, s);
}

// Power of two s with mx * s < 2^6 (>= 2^5 for mx > 0), and 1 / s.
__device__ __forceinline__ void g_scale_in(float mx, float& s, float& inv_s) {
  int e = (int)((__float_as_uint(mx) >> 23) & 0xff);   // mx < 2^(e - 126)
  e = e < 6 ? 6 : (e > 254 ? 254 : e);
  s = __uint_as_float((unsigned)(259 - e > 254 ? 254 : 259 - e) << 23);   // 2^(132 - e)
  inv_s = __uint_as_float((unsigned)(e - 5) << 23);                        // 2^(e - 132)
  if (mx == 0.f) { s = 1.f; inv_s = 1.f; }
}

// DFT-matrix operand element (n, k) of a K-major canonical B operand with K f16 columns.
__device__ __forceinline__ void g_put(unsigned char* sB, uint32_t base, int K, int n, int k, float v) {
  const uint32_t o = base + (uint32_t)((n & 7) * 16 + (k & 7) * 2 + (k >> 3) * 128 + (n >> 3) * (K / 8) * 128);
  *reinterpret_cast<__half*>(sB + o) = __float2half_rn(v);
}

// Real form of scale * F[o][i], F[o][i] = w_n^{sign o i} (outputs o < no,
// inputs i < ni) at `base`: rows 2o + rho, columns 2i + sigma: [[Fr, -Fi], [Fi, Fr]].
// scale is a power of two small enough to keep every nonzero entry an f16 normal.
inline __device__ void g_build_dft(unsigned char* sB, uint32_t base, int n, int no, int ni, bool inverse, float scale,
                                   int tid, int nthreads) {
  const int K = 2 * ni;
  for (int idx = tid; idx < no * ni; idx += nthreads) {
    const int o = idx / ni, i = idx % ni;
    const int e = (o * i) % n;
    float2 w = g_root(e, n);
    if (inverse) w.y = -w.y;
    w.x *= scale;
    w.y *= scale;
    g_put(sB, base, K, 2 * o, 2 * i, w.x);
    g_put(sB, base, K, 2 * o, 2 * i + 1, -w.y);
    g_put(sB, base, K, 2 * o + 1, 2 * i, w.y);
    g_put(sB, base, K, 2 * o + 1, 2 * i + 1, w.x);
  }
}


}  // namespace hyena
