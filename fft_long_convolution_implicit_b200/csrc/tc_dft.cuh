// tc_dft.cuh -- warp-level 256-point DFTs on the tensor cores (mma.sync,
// f16 operands, f32 accumulation), shared by the tensor-core kernels.
//
// A 256-point DFT of x[16 m1 + m2] is two 16-point DFT-matrix products with a
// twiddle between them (the FFT's Cooley-Tukey split 256 = 16 x 16 written as
// matrix products): T = F16 X (DFT over m1 for every m2), T *= w_256^{k1 m2},
// Y = T F16 (DFT over m2 for every k1); bin k1 + 16 k2 of Y sits in row k1,
// column k2. Complex matrices are multiplied in their real planar forms, so
// one 16-point complex DFT is a 32 x 32 real product. The stage-one
// accumulators are the stage-two A operand without leaving registers.
//
// Register layouts of one warp (g = lane / 4, t = lane % 4):
//  - vin layout:  vin[q][nt] = x[m1][m2], m1 = {2t, 2t+1, 2t+8, 2t+9}[q],
//                 m2 = 8 nt + g (the B-operand layout of the first product);
//  - D layout:    D[nt][e], nt 0,1 real / 2,3 imaginary parts of bin
//                 k1 + 16 k2, k1 = g + 8 (e >> 1), k2 = 8 (nt & 1) + 2t + (e & 1);
//  - C layout:    C[p][np][e], p 0 real / 1 imaginary part of x[16 m1 + m2],
//                 m1 = g + 8 (e >> 1), m2 = 8 np + 2t + (e & 1) (accumulator
//                 layout of an m16n8 product over two n-tiles).
// In the D layout the bin 255 - k of the value in (lane, nt, e) sits in
// (31 - lane, nt ^ 1, e ^ 3).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace hyena {

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// d += A * B, m16n8k16, f16 operands, f32 accumulators
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// transpose of an 8x8 b16 matrix held one row-pair per lane
__device__ __forceinline__ uint32_t movt(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// F16[a][b] = exp(-2 pi i a b / 16) as (cos, sin)
__device__ __forceinline__ void f16_entry(int a, int b, float& re, float& im) {
  sincospif(-(float)((a * b) & 15) / 8.0f, &im, &re);
}

// Planar real forms of the 16-point DFT matrix:
//   A[r][c] = [[Fr, -Fi], [Fi, Fr]]   (left factor:  [Tr; Ti] = A [Xr; Xi])
//   B[r][c] = [[Fr,  Fi], [-Fi, Fr]]  (right factor: [Yr | Yi] = [Tr | Ti] B)
__device__ __forceinline__ float planar_left(int r, int c) {
  float re, im;
  f16_entry(r & 15, c & 15, re, im);
  if (r < 16) return c < 16 ? re : -im;
  return c < 16 ? im : re;
}
__device__ __forceinline__ float planar_right(int r, int c) {
  float re, im;
  f16_entry(r & 15, c & 15, re, im);
  if (r < 16) return c < 16 ? re : im;
  return c < 16 ? -im : re;
}

struct Dft16Frags {
  uint32_t A[2][2][4];   // left factor, [m-tile][k-tile]
  uint32_t B[2][4][2];   // right factor, [k-tile][n-tile]
};

__device__ __forceinline__ void build_frags(Dft16Frags& f, int g, int t) {
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) {
      const int r0 = 16 * mt + g, r1 = r0 + 8, c0 = 16 * kt + 2 * t, c1 = c0 + 8;
      f.A[mt][kt][0] = pack_h2(planar_left(r0, c0), planar_left(r0, c0 + 1));
      f.A[mt][kt][1] = pack_h2(planar_left(r1, c0), planar_left(r1, c0 + 1));
      f.A[mt][kt][2] = pack_h2(planar_left(r0, c1), planar_left(r0, c1 + 1));
      f.A[mt][kt][3] = pack_h2(planar_left(r1, c1), planar_left(r1, c1 + 1));
    }
#pragma unroll
  for (int kt = 0; kt < 2; ++kt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int n = 8 * nt + g, k0 = 16 * kt + 2 * t;
      f.B[kt][nt][0] = pack_h2(planar_right(k0, n), planar_right(k0 + 1, n));
      f.B[kt][nt][1] = pack_h2(planar_right(k0 + 8, n), planar_right(k0 + 9, n));
    }
}

// Inner twiddles w_256^{k1 m2} of the thread's fragment positions as pairs of
// adjacent columns: re/im of (k1 = g + 8 i, m2 = 8 nt + 2t + {0, 1}).
struct Tw256 {
  float2 re[2][2], im[2][2];   // [i][nt]
};

// (re, im) *= (wr, wi) on two columns at once (packed f32x2 arithmetic)
__device__ __forceinline__ void cmul_pair(float& r0, float& r1, float& i0, float& i1, float2 wr, float2 wi) {
  const float2 re = make_float2(r0, r1), im = make_float2(i0, i1);
  const float2 t = __fmul2_rn(im, wi);
  const float2 nr = __ffma2_rn(re, wr, make_float2(-t.x, -t.y));
  const float2 ni = __ffma2_rn(re, wi, __fmul2_rn(im, wr));
  r0 = nr.x; r1 = nr.y; i0 = ni.x; i1 = ni.y;
}

// Forward 256-point DFT of the warp's vector x[16 m1 + m2].
// vin[q][nt] = s * x[m1 = {2t, 2t+1, 2t+8, 2t+9}[q]][m2 = 8 nt + g].
// Out: D[nt][e], nt 0,1 real / 2,3 imaginary parts of Y[k1 + 16 k2],
// k1 = g + 8 (e >> 1), k2 = 8 (nt & 1) + 2t + (e & 1).
__device__ __forceinline__ void dft256_fwd(const Dft16Frags& F, const Tw256& tw, const float2 (&vin)[4][2],
                                           float (&D)[4][4]) {
  uint32_t bx[2][2][2];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    bx[0][nt][0] = pack_h2(vin[0][nt].x, vin[1][nt].x);
    bx[0][nt][1] = pack_h2(vin[2][nt].x, vin[3][nt].x);
    bx[1][nt][0] = pack_h2(vin[0][nt].y, vin[1][nt].y);
    bx[1][nt][1] = pack_h2(vin[2][nt].y, vin[3][nt].y);
  }
  float C[2][2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) C[mt][nt][e] = 0.f;
#pragma unroll
      for (int kt = 0; kt < 2; ++kt) mma_f16(C[mt][nt], F.A[mt][kt], bx[kt][nt][0], bx[kt][nt][1]);
    }
  // twiddle T[k1][m2] *= w_256^{k1 m2}
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 2; ++i)
      cmul_pair(C[0][nt][2 * i], C[0][nt][2 * i + 1], C[1][nt][2 * i], C[1][nt][2 * i + 1], tw.re[i][nt], tw.im[i][nt]);
  uint32_t A[2][4];
#pragma unroll
  for (int kt = 0; kt < 2; ++kt) {
    A[kt][0] = pack_h2(C[kt][0][0], C[kt][0][1]);
    A[kt][1] = pack_h2(C[kt][0][2], C[kt][0][3]);
    A[kt][2] = pack_h2(C[kt][1][0], C[kt][1][1]);
    A[kt][3] = pack_h2(C[kt][1][2], C[kt][1][3]);
  }
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) D[nt][e] = 0.f;
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) mma_f16(D[nt], A[kt], F.B[kt][nt][0], F.B[kt][nt][1]);
  }
}

// Unnormalised inverse 256-point DFT of s * Y (D layout as produced above),
// computed as conj(DFT(conj(Y))). Out: G[mt][nt'][e] = real (mt 0) and
// imaginary (mt 1) parts of conj(x)[16 m1 + m2], m1 = g + 8 (e >> 1),
// m2 = 8 nt' + 2t + (e & 1).
__device__ __forceinline__ void dft256_inv(const Dft16Frags& F, const Tw256& tw, const float (&D)[4][4],
                                           float (&G)[2][2][4]) {
  uint32_t A[2][4];
  A[0][0] = pack_h2(D[0][0], D[0][1]);
  A[0][1] = pack_h2(D[0][2], D[0][3]);
  A[0][2] = pack_h2(D[1][0], D[1][1]);
  A[0][3] = pack_h2(D[1][2], D[1][3]);
  A[1][0] = pack_h2(-D[2][0], -D[2][1]);
  A[1][1] = pack_h2(-D[2][2], -D[2][3]);
  A[1][2] = pack_h2(-D[3][0], -D[3][1]);
  A[1][3] = pack_h2(-D[3][2], -D[3][3]);
  float E[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) E[nt][e] = 0.f;
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) mma_f16(E[nt], A[kt], F.B[kt][nt][0], F.B[kt][nt][1]);
  }
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 2; ++i)
      cmul_pair(E[nt][2 * i], E[nt][2 * i + 1], E[nt + 2][2 * i], E[nt + 2][2 * i + 1], tw.re[i][nt], tw.im[i][nt]);
  uint32_t Bt[2][2][2];
#pragma unroll
  for (int np = 0; np < 2; ++np)
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) {
      const float* src = E[np + 2 * kt];
      Bt[kt][np][0] = movt(pack_h2(src[0], src[1]));
      Bt[kt][np][1] = movt(pack_h2(src[2], src[3]));
    }
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int np = 0; np < 2; ++np) {
#pragma unroll
      for (int e = 0; e < 4; ++e) G[mt][np][e] = 0.f;
#pragma unroll
      for (int kt = 0; kt < 2; ++kt) mma_f16(G[mt][np], F.A[mt][kt], Bt[kt][np][0], Bt[kt][np][1]);
    }
}

// Power-of-two scale s with bound * s < 2^10 (and 1/s), from a bound >= 0.
__device__ __forceinline__ void pow2_scale(float mx, float& s, float& inv_s) {
  int e = (int)((__float_as_uint(mx) >> 23) & 0xff);   // mx < 2^(e - 126)
  e = e < 10 ? 10 : (e > 254 ? 254 : e);
  s = __uint_as_float((unsigned)(263 - e > 254 ? 254 : 263 - e) << 23);   // 2^(136 - e)
  inv_s = __uint_as_float((unsigned)(e - 9) << 23);                        // 2^(e - 136)
  if (mx == 0.f) { s = 1.f; inv_s = 1.f; }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Inner twiddles of a lane (w_256^{k1 m2} at the fragment positions).
__device__ __forceinline__ void build_tw256(Tw256& tw, int g, int t) {
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float w[2][2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k1 = g + 8 * i, m2 = 8 * nt + 2 * t + e;
        sincospif(-(float)((k1 * m2) & 255) / 128.0f, &w[e][1], &w[e][0]);
      }
      tw.re[i][nt] = make_float2(w[0][0], w[1][0]);
      tw.im[i][nt] = make_float2(w[0][1], w[1][1]);
    }
}

// Forward 256-point DFT of s * x given in the C layout (cin[p][np][e] = real
// (p 0) / imaginary (p 1) part of s * x[16 m1 + m2], m1 = g + 8 (e >> 1),
// m2 = 8 np + 2t + (e & 1)). Each 8 x 8 block is moved into the B-operand
// layout of the first product by one movmatrix transpose. Output as
// dft256_fwd (D layout).
__device__ __forceinline__ void dft256_fwd_c(const Dft16Frags& F, const Tw256& tw, const float (&cin)[2][2][4],
                                             float (&D)[4][4]) {
  uint32_t bx[2][2][2];
#pragma unroll
  for (int p = 0; p < 2; ++p)
#pragma unroll
    for (int np = 0; np < 2; ++np)
#pragma unroll
      for (int i = 0; i < 2; ++i) bx[p][np][i] = movt(pack_h2(cin[p][np][2 * i], cin[p][np][2 * i + 1]));
  float C[2][2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) C[mt][nt][e] = 0.f;
#pragma unroll
      for (int kt = 0; kt < 2; ++kt) mma_f16(C[mt][nt], F.A[mt][kt], bx[kt][nt][0], bx[kt][nt][1]);
    }
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 2; ++i)
      cmul_pair(C[0][nt][2 * i], C[0][nt][2 * i + 1], C[1][nt][2 * i], C[1][nt][2 * i + 1], tw.re[i][nt], tw.im[i][nt]);
  uint32_t A[2][4];
#pragma unroll
  for (int kt = 0; kt < 2; ++kt) {
    A[kt][0] = pack_h2(C[kt][0][0], C[kt][0][1]);
    A[kt][1] = pack_h2(C[kt][0][2], C[kt][0][3]);
    A[kt][2] = pack_h2(C[kt][1][0], C[kt][1][1]);
    A[kt][3] = pack_h2(C[kt][1][2], C[kt][1][3]);
  }
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) D[nt][e] = 0.f;
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) mma_f16(D[nt], A[kt], F.B[kt][nt][0], F.B[kt][nt][1]);
  }
}

}  // namespace hyena
