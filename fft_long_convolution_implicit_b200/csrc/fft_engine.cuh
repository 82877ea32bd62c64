// fft_engine.cuh -- register/shared-memory FFT building blocks for the Hyena
// order-N forward on sm_100a.
//
// The causal long convolution of the Hyena operator is evaluated by FFT on
// a 2L zero-padded grid (glossary "Hyena（ハイエナ）", section 計算効率;
// "Native Multi-Dimensional Subquadratic Operators via Input Dependent Long
// Convolutions", section 境界の処理). A length-2L real sequence z is packed as
// M = L complex points c[m] = z[2m] + i z[2m+1]; its upper half is zero.
// The M-point complex FFT is an in-place Stockham autosort FFT in shared
// memory: forward pass p with radix R and span Ns reads butterfly j at
// j + r*M/R, multiplies by w_{Ns R}^{(j mod Ns) r}, applies DFT_R and writes
// at (j/Ns)*Ns*R + (j mod Ns) + r*Ns. The inverse runs the transposed passes
// in reverse order with conjugated twiddles, so both directions share one
// twiddle table and natural-order data.
//
// Twiddle table of an M-point plan: pass p keeps w_{Ns R}^{jm r}, r = 1..R-1,
// jm = 0..Ns-1, at offset (Ns - 1) + (r - 1) Ns + jm (M - 1 entries in all).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hyena {

// ------------------------------------------------------------------ complex --
// Complex sums and differences as one packed f32x2 instruction each (exactly
// rounded per component, the same values as two scalar operations; the
// difference is a - b = fma(b, -1, a), exact too), which halves the issue
// slots of the butterflies' additions.
#ifndef HYENA_PACKED_ADD
#define HYENA_PACKED_ADD 1
#endif
#if HYENA_PACKED_ADD
__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.f, -1.f), a); }
#else
__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
#endif
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}
// a * conj(b)
__device__ __forceinline__ float2 cmulc(float2 a, float2 b) {
  return make_float2(a.x * b.x + a.y * b.y, a.y * b.x - a.x * b.y);
}
__device__ __forceinline__ float2 cconj(float2 a) { return make_float2(a.x, -a.y); }
// multiply by -i (forward) or +i (inverse)
template <bool INV>
__device__ __forceinline__ float2 rot(float2 a) {
  return INV ? make_float2(-a.y, a.x) : make_float2(a.y, -a.x);
}
// forward: a * exp(-i th); inverse: a * exp(+i th), with (c, s) = (cos th, sin th)
template <bool INV>
__device__ __forceinline__ float2 crot(float2 a, float c, float s) {
  return INV ? make_float2(a.x * c - a.y * s, a.y * c + a.x * s)
             : make_float2(a.x * c + a.y * s, a.y * c - a.x * s);
}
// multiply by a table twiddle w (forward) or conj(w) (inverse)
template <bool INV>
__device__ __forceinline__ float2 twmul(float2 a, float2 w) {
  return INV ? cmulc(a, w) : cmul(a, w);
}

// cos(pi/8), sin(pi/8), cos(pi/4)
#define HY_C8 0.92387953251128675613f
#define HY_S8 0.38268343236508977173f
#define HY_R2 0.70710678118654752440f

// ------------------------------------------------------------- small DFTs --
// All DFTs are in place on a register array at compile-time offset O, natural
// order in and out, unnormalised, sign -1 (forward) or +1 (INV).

template <bool INV, int O, int N>
__device__ __forceinline__ void dft2(float2 (&a)[N]) {
  float2 t = a[O];
  a[O] = cadd(t, a[O + 1]);
  a[O + 1] = csub(t, a[O + 1]);
}

template <bool INV>
__device__ __forceinline__ void dft4v(float2& a0, float2& a1, float2& a2, float2& a3) {
  float2 t0 = cadd(a0, a2), t1 = csub(a0, a2), t2 = cadd(a1, a3), t3 = rot<INV>(csub(a1, a3));
  a0 = cadd(t0, t2);
  a2 = csub(t0, t2);
  a1 = cadd(t1, t3);
  a3 = csub(t1, t3);
}
// inputs a2 = a3 = 0 (not read)
template <bool INV>
__device__ __forceinline__ void dft4v_in2(float2& a0, float2& a1, float2& a2, float2& a3) {
  float2 r1 = rot<INV>(a1);
  float2 x0 = a0;
  a2 = csub(x0, a1);
  a3 = csub(x0, r1);
  a0 = cadd(x0, a1);
  a1 = cadd(x0, r1);
}
// only outputs 0 and 1 are produced
template <bool INV>
__device__ __forceinline__ void dft4v_out2(float2& a0, float2& a1, float2 a2, float2 a3) {
  float2 t0 = cadd(a0, a2), t1 = csub(a0, a2), t2 = cadd(a1, a3), t3 = rot<INV>(csub(a1, a3));
  a0 = cadd(t0, t2);
  a1 = cadd(t1, t3);
}

template <bool INV, int O, int N>
__device__ __forceinline__ void dft4(float2 (&a)[N]) {
  dft4v<INV>(a[O], a[O + 1], a[O + 2], a[O + 3]);
}

template <bool INV, int O, int N>
__device__ __forceinline__ void dft8(float2 (&a)[N]) {
  // split even/odd, DFT4 each, combine with w8^k
  float2 e0 = a[O], e1 = a[O + 2], e2 = a[O + 4], e3 = a[O + 6];
  float2 o0 = a[O + 1], o1 = a[O + 3], o2 = a[O + 5], o3 = a[O + 7];
  dft4v<INV>(e0, e1, e2, e3);
  dft4v<INV>(o0, o1, o2, o3);
  o1 = crot<INV>(o1, HY_R2, HY_R2);    // w8^1
  o2 = rot<INV>(o2);                   // w8^2
  o3 = crot<INV>(o3, -HY_R2, HY_R2);   // w8^3
  a[O + 0] = cadd(e0, o0); a[O + 4] = csub(e0, o0);
  a[O + 1] = cadd(e1, o1); a[O + 5] = csub(e1, o1);
  a[O + 2] = cadd(e2, o2); a[O + 6] = csub(e2, o2);
  a[O + 3] = cadd(e3, o3); a[O + 7] = csub(e3, o3);
}

// 16-point DFT as 4 x 4: X[k1 + 4 k2] = sum_n2 w4^{n2 k2} w16^{n2 k1} sum_n1 x[4 n1 + n2] w4^{n1 k1}.
// HALF_IN: inputs 8..15 are zero (not read). HALF_OUT: only outputs 0..7 are formed.
template <bool INV, bool HALF_IN, bool HALF_OUT, int O, int N>
__device__ __forceinline__ void dft16(float2 (&a)[N]) {
  float2 b[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) b[i] = a[O + i];
#pragma unroll
  for (int n2 = 0; n2 < 4; ++n2) {
    if (HALF_IN) dft4v_in2<INV>(b[n2], b[4 + n2], b[8 + n2], b[12 + n2]);
    else dft4v<INV>(b[n2], b[4 + n2], b[8 + n2], b[12 + n2]);
  }
  // b[4 k1 + n2] *= w16^{n2 k1}
  b[5] = crot<INV>(b[5], HY_C8, HY_S8);
  b[6] = crot<INV>(b[6], HY_R2, HY_R2);
  b[7] = crot<INV>(b[7], HY_S8, HY_C8);
  b[9] = crot<INV>(b[9], HY_R2, HY_R2);
  b[10] = rot<INV>(b[10]);
  b[11] = crot<INV>(b[11], -HY_R2, HY_R2);
  b[13] = crot<INV>(b[13], HY_S8, HY_C8);
  b[14] = crot<INV>(b[14], -HY_R2, HY_R2);
  b[15] = crot<INV>(b[15], -HY_C8, -HY_S8);
#pragma unroll
  for (int k1 = 0; k1 < 4; ++k1) {
    if (HALF_OUT) dft4v_out2<INV>(b[4 * k1], b[4 * k1 + 1], b[4 * k1 + 2], b[4 * k1 + 3]);
    else dft4v<INV>(b[4 * k1], b[4 * k1 + 1], b[4 * k1 + 2], b[4 * k1 + 3]);
  }
  // X[k1 + 4 k2] sits in b[4 k1 + k2]
#pragma unroll
  for (int k2 = 0; k2 < (HALF_OUT ? 2 : 4); ++k2)
#pragma unroll
    for (int k1 = 0; k1 < 4; ++k1) a[O + k1 + 4 * k2] = b[4 * k1 + k2];
}

template <int R, bool INV, int O, int N>
__device__ __forceinline__ void dftR(float2 (&a)[N]) {
  if constexpr (R == 2) dft2<INV, O>(a);
  else if constexpr (R == 4) dft4<INV, O>(a);
  else if constexpr (R == 8) dft8<INV, O>(a);
  else if constexpr (R == 16) dft16<INV, false, false, O>(a);
  else static_assert(R == 2 || R == 4 || R == 8 || R == 16, "radix");
}

// ------------------------------------------------------------ async copy --
// 16-byte global -> shared copies that complete asynchronously (cp.async,
// L2 only); completion is awaited with the hardware group wait, no polling.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
// all committed groups except the newest one are complete
__device__ __forceinline__ void cp_async_wait_all_but_newest() {
  asm volatile("cp.async.wait_group 1;\n" ::: "memory");
}

// Copy nbytes (multiple of 16, both addresses 16-byte aligned) with all
// threads of the block; returns without waiting.
__device__ __forceinline__ void block_copy_async(void* smem_dst, const void* gmem_src, int nbytes, int tid,
                                                 int nthreads) {
  char* d = reinterpret_cast<char*>(smem_dst);
  const char* g = reinterpret_cast<const char*>(gmem_src);
  for (int off = tid * 16; off < nbytes; off += nthreads * 16) cp_async16(d + off, g + off);
}

// ----------------------------------------------------------- smem padding --
// one float2 of padding after every 16: removes the bank conflicts of the
// stride-16 block writes of radix-16 passes
__device__ __forceinline__ int pidx(int i) { return i + (i >> 4); }
__host__ __device__ constexpr int padded_len(int m) { return m + m / 16; }
// pidx(i + r*STEP) from p = pidx(i): a compile-time offset when STEP is a
// multiple of 16 (adding whole 16-element groups moves the padding exactly).
template <int STEP>
__device__ __forceinline__ int pidx_step(int p, int i, int r) {
  if constexpr (STEP % 16 == 0) return p + r * (STEP + STEP / 16);
  else return pidx(i + r * STEP);
}

// ---------------------------------------------------------------- plans ----
// Pass plan of an MV-point FFT (MV = 2^LOGMV, LOGMV >= 7), 16 points per
// thread: first pass radix 16 (span 1), middle passes radix 16 and at most
// one of radix 2/4/8, last pass radix 8 (span MV/8), which is the pass where
// spectrum bins k and MV-k meet in one thread.
template <int LOGMV>
struct Plan {
  static_assert(LOGMV >= 7, "plan needs at least 128 points");
  static constexpr int MV = 1 << LOGMV;
  static constexpr int TV = MV / 16;                  // threads per vector
  static constexpr int MID_BITS = LOGMV - 7;
  static constexpr int N16 = MID_BITS / 4;
  static constexpr int SMALL = MID_BITS % 4;
  static constexpr int NMID = N16 + (SMALL ? 1 : 0);
  static constexpr int radix(int i) { return i < N16 ? 16 : (1 << SMALL); }
  static constexpr int span(int i) {  // Ns of middle pass i
    int s = 16;
    for (int q = 0; q < i; ++q) s *= radix(q);
    return s;
  }
};

// DFT_R on each of the 16/R consecutive blocks of a 16-point register array.
template <int R, bool INV, int Q = 0>
__device__ __forceinline__ void dft_blocks(float2 (&a)[16]) {
  if constexpr (Q * R < 16) {
    dftR<R, INV, Q * R>(a);
    dft_blocks<R, INV, Q + 1>(a);
  }
}

// Middle pass I of the forward transform: load, twiddle, DFT_R, barrier, store, barrier.
template <int LOGMV, int I>
__device__ __forceinline__ void mid_fwd(float2 (&a)[16], float2* base, const float2* __restrict__ tw, int tl) {
  using P = Plan<LOGMV>;
  constexpr int MV = P::MV, TV = P::TV, R = P::radix(I), NS = P::span(I), NB = 16 / R, S = MV / R;
  const int ptl = pidx(tl);
#pragma unroll
  for (int q = 0; q < NB; ++q) {
    const int j = tl + q * TV;
    const int pj = pidx_step<TV>(ptl, tl, q);
#pragma unroll
    for (int r = 0; r < R; ++r) a[q * R + r] = base[pidx_step<S>(pj, j, r)];
    const float2* __restrict__ t = tw + (NS - 1) + (j & (NS - 1));
#pragma unroll
    for (int r = 1; r < R; ++r) a[q * R + r] = cmul(a[q * R + r], __ldg(t + (r - 1) * NS));
  }
  dft_blocks<R, false>(a);
  __syncthreads();
#pragma unroll
  for (int q = 0; q < NB; ++q) {
    const int j = tl + q * TV;
    const int o = (j / NS) * NS * R + (j & (NS - 1));
    const int po = pidx(o);
#pragma unroll
    for (int r = 0; r < R; ++r) base[pidx_step<NS>(po, o, r)] = a[q * R + r];
  }
  __syncthreads();
}

// Transposed middle pass I (inverse direction): load at block positions, DFT_R^-1,
// conjugate twiddle, barrier, store at strided positions, barrier.
template <int LOGMV, int I>
__device__ __forceinline__ void mid_inv(float2 (&a)[16], float2* base, const float2* __restrict__ tw, int tl) {
  using P = Plan<LOGMV>;
  constexpr int MV = P::MV, TV = P::TV, R = P::radix(I), NS = P::span(I), NB = 16 / R, S = MV / R;
#pragma unroll
  for (int q = 0; q < NB; ++q) {
    const int j = tl + q * TV;
    const int o = (j / NS) * NS * R + (j & (NS - 1));
    const int po = pidx(o);
#pragma unroll
    for (int r = 0; r < R; ++r) a[q * R + r] = base[pidx_step<NS>(po, o, r)];
  }
  dft_blocks<R, true>(a);
#pragma unroll
  for (int q = 0; q < NB; ++q) {
    const float2* __restrict__ t = tw + (NS - 1) + ((tl + q * TV) & (NS - 1));
#pragma unroll
    for (int r = 1; r < R; ++r) a[q * R + r] = cmulc(a[q * R + r], __ldg(t + (r - 1) * NS));
  }
  __syncthreads();
  const int ptl = pidx(tl);
#pragma unroll
  for (int q = 0; q < NB; ++q) {
    const int j = tl + q * TV;
    const int pj = pidx_step<TV>(ptl, tl, q);
#pragma unroll
    for (int r = 0; r < R; ++r) base[pidx_step<S>(pj, j, r)] = a[q * R + r];
  }
  __syncthreads();
}

// First forward pass output / last inverse pass input of thread tl: the 16
// positions 16 tl + r, padded index 17 tl + r.
__device__ __forceinline__ void store_block16(float2* base, int tl, const float2 (&a)[16]) {
  float2* p = base + 17 * tl;
#pragma unroll
  for (int r = 0; r < 16; ++r) p[r] = a[r];
}
__device__ __forceinline__ void load_block16(const float2* base, int tl, float2 (&a)[16]) {
  const float2* p = base + 17 * tl;
#pragma unroll
  for (int r = 0; r < 16; ++r) a[r] = p[r];
}

template <int LOGMV, int I = 0>
__device__ __forceinline__ void mid_fwd_all(float2 (&a)[16], float2* base, const float2* __restrict__ tw, int tl) {
  if constexpr (I < Plan<LOGMV>::NMID) {
    mid_fwd<LOGMV, I>(a, base, tw, tl);
    mid_fwd_all<LOGMV, I + 1>(a, base, tw, tl);
  }
}

template <int LOGMV, int I = Plan<LOGMV>::NMID - 1>
__device__ __forceinline__ void mid_inv_all(float2 (&a)[16], float2* base, const float2* __restrict__ tw, int tl) {
  if constexpr (I >= 0) {
    mid_inv<LOGMV, I>(a, base, tw, tl);
    mid_inv_all<LOGMV, I - 1>(a, base, tw, tl);
  }
}

// ------------------------------------------------------- spectral product --
// Real-FFT unpack, product with the filter spectrum and repack, for one bin
// pair (k, M-k) of the M-point packed transform C of z:
//   2 Ze = Ca + conj Cb, 2 Zo = (Ca - conj Cb) / i,
//   2 Z[k] = 2Ze + W 2Zo, 2 Z[M-k] = conj(2Ze - W 2Zo),        W = w_{2M}^k
//   Y = H Z (per bin),
//   C'[k] = S + i Dd, C'[M-k] = conj(S) + i conj(Dd),
//   S = Ya + conj Yb, Dd = (Ya - conj Yb) conj(W).
// With H stored as rfft(pad(h, 2L)) / (4L) the unnormalised inverse M-point
// transform of C' is y[2m] + i y[2m+1].
__device__ __forceinline__ void spectral_pair(float2& Ca, float2& Cb, float2 Ha, float2 Hb, float2 W) {
  const float2 cb = cconj(Cb);
  const float2 P = cadd(Ca, cb);
  const float2 Q = rot<false>(csub(Ca, cb));
  const float2 WQ = cmul(W, Q);
  const float2 Za = cadd(P, WQ);
  const float2 Zb = cconj(csub(P, WQ));
  const float2 Ya = cmul(Ha, Za), Yb = cmul(Hb, Zb);
  const float2 yb = cconj(Yb);
  const float2 S = cadd(Ya, yb);
  const float2 Dd = cmulc(csub(Ya, yb), W);
  Ca = make_float2(S.x - Dd.y, S.y + Dd.x);
  Cb = make_float2(S.x + Dd.y, Dd.x - S.y);
}

// Forward-only half (spectrum computation): returns 2 Z[k] and 2 Z[M-k].
__device__ __forceinline__ void unpack_pair(float2 Ca, float2 Cb, float2 W, float2& Za, float2& Zb) {
  const float2 cb = cconj(Cb);
  const float2 P = cadd(Ca, cb);
  const float2 Q = rot<false>(csub(Ca, cb));
  const float2 WQ = cmul(W, Q);
  Za = cadd(P, WQ);
  Zb = cconj(csub(P, WQ));
}

// -------------------------------------------------------------- I/O ------
template <typename T>
struct IO;
template <>
struct IO<float> {
  static __device__ __forceinline__ float2 load2(const float* p) { return __ldg(reinterpret_cast<const float2*>(p)); }
  static __device__ __forceinline__ float2 load2_stream(const float* p) {
    return __ldcs(reinterpret_cast<const float2*>(p));
  }
  static __device__ __forceinline__ void store2(float* p, float2 v) { __stcs(reinterpret_cast<float2*>(p), v); }
  static __device__ __forceinline__ float2 load2_smem(const float* p) { return *reinterpret_cast<const float2*>(p); }
};
template <>
struct IO<__nv_bfloat16> {
  static __device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
    unsigned int u = __ldg(reinterpret_cast<const unsigned int*>(p));
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
  static __device__ __forceinline__ float2 load2_stream(const __nv_bfloat16* p) {
    unsigned int u = __ldcs(reinterpret_cast<const unsigned int*>(p));
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
  static __device__ __forceinline__ float2 load2_smem(const __nv_bfloat16* p) {
    unsigned int u = *reinterpret_cast<const unsigned int*>(p);
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
  static __device__ __forceinline__ void store2(__nv_bfloat16* p, float2 v) {
    __nv_bfloat162 b = __floats2bfloat162_rn(v.x, v.y);  // round to nearest even
    __stcs(reinterpret_cast<unsigned int*>(p), *reinterpret_cast<unsigned int*>(&b));
  }
};

}  // namespace hyena
