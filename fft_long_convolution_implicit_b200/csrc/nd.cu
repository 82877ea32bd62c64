// nd.cu -- HyenaND: the order-N recurrence with an N-dimensional global
// convolution (page "Native Multi-Dimensional Subquadratic Operators via
// Input Dependent Long Convolutions", section 手法: the convolution runs on
// the L_1 x ... x L_N grid through an N-dimensional FFT, circular for
// periodic data, or on the input zero-padded to twice the grid so nothing
// leaks across the boundary).
//
//   z_1 = v,  z_{n+1} = x_n (.) (K_n conv z_n),  y = z_{N+1}
//   circular: (K conv z)[p] = sum_q K[(p - q) mod dims] z[q]
//   zero:     (K conv z)[p] = sum_{0 <= q <= p} K[p - q] z[q]
//
// One CTA per (channel c, batch pair b, b+1): the two real signals of the
// pair are the real and imaginary parts of one complex grid (K is real, so one
// complex convolution carries both), held in shared memory on the padded grid
// P_1 x ... x P_nd (P_a = 2 L_a zero-padded, L_a circular; P = prod P_a <=
// 16384 points, 128 KB plus one spare slot per 16 points against bank
// conflicts). The transform is separable: along every axis, in-place
// decimation-in-frequency steps of radix 2^k (k <= 4, DFT_R in registers,
// then the twiddles w_m^{j r}, output r stored at the bit-reversed slot)
// leave each axis index bit-reversed, exactly as 2-point levels would; the
// spectrum block K^ is stored in that order, so the product needs no
// reordering, and the inverse undoes the steps in reverse (decimation in
// time, conjugate twiddles), returning natural order. K^ carries the 1/P of
// the inverse. Register-resident fusions: the last forward step, the product
// and the first inverse step share one pass; the last inverse step, the gate
// x_n and the next stage's first forward step (same positions) share another.
// All N stages stay in shared memory; only v, x_n and y touch HBM, plus K^.
#include <cuda_bf16.h>

#include "fft_engine.cuh"
#include "kernels.cuh"

namespace hyena {

namespace {

constexpr int kNdMaxDims = 3;
constexpr int kNdMaxLogP = 14;      // 16384 complex points: 128 KB of shared memory
constexpr int kNdMaxLogAxis = 10;   // padded axis length <= 1024 (twiddle table <= 512 entries)

constexpr int kNdMaxSteps = 9;      // <= 3 radix steps per axis (padded axis <= 2^10)

struct NdGeom {
  int nd;
  int logP;
  int logn[kNdMaxDims];   // padded axis lengths
  int logs[kNdMaxDims];   // inner stride of each axis on the padded grid
  int logL[kNdMaxDims];   // grid axis lengths
  int logT;               // twiddle table w_T^k, k < T, T = longest padded axis (at least 2)
  int G;                  // grid points prod L_a
  int zero;               // zero-padded boundary
  // forward radix steps, axis 0 first; step i works along axis st_a[i] on
  // blocks of 2^st_logm[i] points with radix 2^st_logR[i]
  int nsteps;
  signed char st_a[kNdMaxSteps], st_logm[kNdMaxSteps], st_logR[kNdMaxSteps];
  // zero padding: step i skips the butterflies whose offset along the later
  // axes lies in their padding (bit st_p1/st_p2 of the offset set; -1 = none),
  // and the first step of an axis reads only the lower half of that axis
  signed char st_p1[kNdMaxSteps], st_p2[kNdMaxSteps], st_first[kNdMaxSteps];
};

__device__ __forceinline__ float ld1(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld1(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }
__device__ __forceinline__ void st1(float* p, float v) { *p = v; }
__device__ __forceinline__ void st1(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Padded-grid position of grid point g (row-major over L_0 x L_1 x L_2).
__device__ __forceinline__ int grid_to_pos(const NdGeom& g, int gi) {
  int pos = 0;
#pragma unroll
  for (int a = kNdMaxDims - 1; a >= 0; --a) {
    if (a < g.nd) {
      const int coord = gi & ((1 << g.logL[a]) - 1);
      gi >>= g.logL[a];
      pos += coord << g.logs[a];
    }
  }
  return pos;
}

// Grid index of padded position pos, or -1 in the padding.
__device__ __forceinline__ int pos_to_grid(const NdGeom& g, int pos) {
  int gi = 0;
#pragma unroll
  for (int a = 0; a < kNdMaxDims; ++a) {
    if (a < g.nd) {
      const int coord = (pos >> g.logs[a]) & ((1 << g.logn[a]) - 1);
      if (coord >> g.logL[a]) return -1;
      gi = (gi << g.logL[a]) + coord;
    }
  }
  return gi;
}

template <typename T>
struct NdGates {
  const T* p[kMaxOrder];
};

// Shared-memory slot of padded-grid position pos: one spare slot after every
// 16 points keeps the radix steps along the contiguous axis free of bank
// conflicts.
__device__ __forceinline__ int spad(int pos) { return pos + (pos >> 4); }

__host__ __device__ constexpr int brev_bits(int r, int bits) {
  int o = 0;
  for (int i = 0; i < bits; ++i) o |= ((r >> i) & 1) << (bits - 1 - i);
  return o;
}

template <int R>
constexpr int log2_of() {
  return R == 2 ? 1 : R == 4 ? 2 : R == 8 ? 3 : 4;
}

// Step i: blocks of 2^logm points, 2^logq butterflies per block, along an
// axis of inner stride 2^logs (read once per pass from the shared geometry).
struct StepGeo {
  int logs, logq, logm;
  int nskip, p1, p2;   // skipped offset bits (ascending), their count
  bool half_in;        // forward: inputs of the upper half of the axis are zero
};
// ZP: zero-padded boundary (pruning on); circular grids compile without it.
template <bool ZP>
__device__ __forceinline__ StepGeo step_geo(const NdGeom& g, int i) {
  StepGeo q;
  q.logm = g.st_logm[i];
  q.logq = q.logm - g.st_logR[i];
  q.logs = g.logs[g.st_a[i]];
  q.p1 = ZP ? g.st_p1[i] : -1;
  q.p2 = ZP ? g.st_p2[i] : -1;
  q.nskip = ZP ? (q.p1 >= 0) + (q.p2 >= 0) : 0;
  q.half_in = ZP && g.zero && g.st_first[i];
  return q;
}

// Butterfly index of the tc-th butterfly that is not skipped: zero bits
// inserted at the skipped positions (lower one first).
__device__ __forceinline__ int ins0(int x, int p) { return ((x >> p) << (p + 1)) | (x & ((1 << p) - 1)); }
__device__ __forceinline__ int expand_t(const StepGeo& q, int tc) {
  if (q.p1 >= 0) tc = ins0(tc, q.p1);
  if (q.p2 >= 0) tc = ins0(tc, q.p2);
  return tc;
}

// Butterfly t: positions base + r * stride (r < R) in the padded grid;
// in = offset along the inner axes, j = offset inside its block.
struct StepIdx {
  int base, stride, j, logm, in;
};
__device__ __forceinline__ StepIdx step_index(const StepGeo& q, int t) {
  const int in = t & ((1 << q.logs) - 1);
  const int r = t >> q.logs;
  const int j = r & ((1 << q.logq) - 1);
  const int blk = r >> q.logq;
  return {(((blk << q.logm) + j) << q.logs) + in, 1 << (q.logq + q.logs), j, q.logm, in};
}

// Grid index of the inner-axes offset `in` of a step along axis 0 (the
// flattened axes 1 .. nd-1 of the padded grid), or -1 in the padding.
__device__ __forceinline__ int inner_to_grid(const NdGeom& g, int in) {
  int gi = 0;
#pragma unroll
  for (int a = 1; a < kNdMaxDims; ++a) {
    if (a < g.nd) {
      const int coord = (in >> g.logs[a]) & ((1 << g.logn[a]) - 1);
      if (coord >> g.logL[a]) return -1;
      gi = (gi << g.logL[a]) + coord;
    }
  }
  return gi;
}

// a[r] *= w_m^{j r} (forward) or its conjugate (inverse); w_m^k = tw[k T / m].
// Powers come from w^j (and w^{8j}) by at most three products.
template <int R, bool INV>
__device__ __forceinline__ void step_twiddle(float2 (&a)[R], const float2* tw, int logT, int logm, int j) {
  const int sh = logT - logm;
  float2 w[R];
  w[0] = make_float2(1.f, 0.f);
  w[1] = tw[j << sh];
  if constexpr (R >= 4) {
    w[2] = cmul(w[1], w[1]);
    w[3] = cmul(w[2], w[1]);
  }
  if constexpr (R >= 8) {
    w[4] = cmul(w[2], w[2]);
    w[5] = cmul(w[4], w[1]);
    w[6] = cmul(w[4], w[2]);
    w[7] = cmul(w[4], w[3]);
  }
  if constexpr (R >= 16) {
    w[8] = tw[(8 * j) << sh];
#pragma unroll
    for (int r = 9; r < 16; ++r) w[r] = cmul(w[8], w[r - 8]);
  }
#pragma unroll
  for (int r = 1; r < R; ++r) a[r] = INV ? cmulc(a[r], w[r]) : cmul(a[r], w[r]);
}

// Decimation-in-frequency step: a (natural order over r) -> DFT_R, twiddles;
// output r belongs at position base + bitrev(r) * stride.
template <int R>
__device__ __forceinline__ void dif(float2 (&a)[R], const float2* tw, int logT, const StepIdx& x) {
  dftR<R, false, 0>(a);
  step_twiddle<R, false>(a, tw, logT, x.logm, x.j);
}
// Its inverse (times R): a[r] from position base + bitrev(r) * stride ->
// natural order over r.
template <int R>
__device__ __forceinline__ void dit(float2 (&a)[R], const float2* tw, int logT, const StepIdx& x) {
  step_twiddle<R, true>(a, tw, logT, x.logm, x.j);
  dftR<R, true, 0>(a);
}

template <int R, bool INV, bool ZP>
__device__ void plain_step(float2* s, const float2* tw, const NdGeom& g, int i, int tid, int nt) {
  constexpr int LR = log2_of<R>();
  const StepGeo q = step_geo<ZP>(g, i);
  const int nb = ((1 << g.logP) >> LR) >> q.nskip, logT = g.logT;
  for (int tc = tid; tc < nb; tc += nt) {
    const StepIdx x = step_index(q, expand_t(q, tc));
    float2 a[R];
    if (!INV) {
#pragma unroll
      for (int r = 0; r < R; ++r)
        a[r] = (q.half_in && r >= R / 2) ? make_float2(0.f, 0.f) : s[spad(x.base + r * x.stride)];
      dif<R>(a, tw, logT, x);
#pragma unroll
      for (int r = 0; r < R; ++r) s[spad(x.base + brev_bits(r, LR) * x.stride)] = a[r];
    } else {
#pragma unroll
      for (int r = 0; r < R; ++r) a[r] = s[spad(x.base + brev_bits(r, LR) * x.stride)];
      dit<R>(a, tw, logT, x);
#pragma unroll
      for (int r = 0; r < R; ++r) s[spad(x.base + r * x.stride)] = a[r];
    }
  }
}

// The last forward step, the product with the spectrum and the first inverse
// step in registers (the two steps cover the same positions). The last step
// runs along the innermost axis with one butterfly per block, so its R points
// are contiguous (stride 1): their spectrum values are fetched first, as
// 16-byte loads, to overlap the forward DFT.
template <int R, bool ZP>
__device__ void turn_step(float2* s, const float2* tw, const NdGeom& g, int i, const float2* __restrict__ H, int tid,
                          int nt) {
  constexpr int LR = log2_of<R>();
  const StepGeo q = step_geo<ZP>(g, i);   // innermost axis: nothing to skip
  const int nb = (1 << g.logP) >> LR, logT = g.logT;
  for (int t = tid; t < nb; t += nt) {
    const StepIdx x = step_index(q, t);
    float2 hk[R];
    const float4* __restrict__ h4 = reinterpret_cast<const float4*>(H + x.base);
#pragma unroll
    for (int k = 0; k < R / 2; ++k) {
      const float4 u = __ldg(h4 + k);
      hk[2 * k] = make_float2(u.x, u.y);
      hk[2 * k + 1] = make_float2(u.z, u.w);
    }
    float2 a[R];
#pragma unroll
    for (int r = 0; r < R; ++r) a[r] = (q.half_in && r >= R / 2) ? make_float2(0.f, 0.f) : s[spad(x.base + r)];
    dif<R>(a, tw, logT, x);
#pragma unroll
    for (int r = 0; r < R; ++r) a[r] = cmul(a[r], hk[brev_bits(r, LR)]);
    dit<R>(a, tw, logT, x);
#pragma unroll
    for (int r = 0; r < R; ++r) s[spad(x.base + r)] = a[r];
  }
}

// Gate (or v) values of the pair's two rows: from shared-memory copies made
// with cp.async while earlier passes ran, or straight from global memory.
template <typename T, bool STAGED>
struct PairSrc {
  const T* r0;
  const T* r1;
  bool has1;
  __device__ __forceinline__ float2 at(int gi) const {
    if constexpr (STAGED) {
      return make_float2(to_f(r0[gi]), has1 ? to_f(r1[gi]) : 0.f);
    } else {
      return make_float2(ld1(r0 + gi), has1 ? ld1(r1 + gi) : 0.f);
    }
  }
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
};

// Steps 0 run along axis 0 over whole axes (one block), so butterfly t holds
// axis-0 coordinates j + r q at the inner offset in: the grid index is
// (j + r q) * (G / L_0) + inner_to_grid(in) inside the grid.
// First forward step of stage 1 straight from v.
template <int R, typename T, bool STAGED, bool ZP>
__device__ void entry_step(float2* s, const float2* tw, const NdGeom& g, PairSrc<T, STAGED> src, int tid, int nt) {
  constexpr int LR = log2_of<R>();
  const StepGeo q = step_geo<ZP>(g, 0);
  const int nb = ((1 << g.logP) >> LR) >> q.nskip, logT = g.logT;
  const int L0 = 1 << g.logL[0], gstride = g.G >> g.logL[0], qn = 1 << q.logq;
  for (int tc = tid; tc < nb; tc += nt) {
    const StepIdx x = step_index(q, expand_t(q, tc));
    const int gin = inner_to_grid(g, x.in);
    float2 a[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int c0 = x.j + r * qn;
      a[r] = (gin < 0 || c0 >= L0) ? make_float2(0.f, 0.f) : src.at(c0 * gstride + gin);
    }
    dif<R>(a, tw, logT, x);
#pragma unroll
    for (int r = 0; r < R; ++r) s[spad(x.base + brev_bits(r, LR) * x.stride)] = a[r];
  }
}

// Last inverse step of a stage, the gate x_n, then either the next stage's
// first forward step (same positions) or the store of y.
template <int R, bool LAST, typename T, bool STAGED, bool ZP>
__device__ void exit_step(float2* s, const float2* tw, const NdGeom& g, PairSrc<T, STAGED> xg, T* __restrict__ y,
                          size_t row0, size_t row1, int tid, int nt) {
  constexpr int LR = log2_of<R>();
  const StepGeo q = step_geo<ZP>(g, 0);
  const int nb = ((1 << g.logP) >> LR) >> q.nskip, logT = g.logT;
  const int L0 = 1 << g.logL[0], gstride = g.G >> g.logL[0], qn = 1 << q.logq;
  for (int tc = tid; tc < nb; tc += nt) {
    const StepIdx x = step_index(q, expand_t(q, tc));
    const int gin = inner_to_grid(g, x.in);
    float2 a[R];
#pragma unroll
    for (int r = 0; r < R; ++r) a[r] = s[spad(x.base + brev_bits(r, LR) * x.stride)];
    dit<R>(a, tw, logT, x);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int c0 = x.j + r * qn;
      if (gin < 0 || c0 >= L0) {
        a[r] = make_float2(0.f, 0.f);
      } else {
        const int gi = c0 * gstride + gin;
        const float2 xv = xg.at(gi);
        a[r] = make_float2(a[r].x * xv.x, a[r].y * xv.y);
        if (LAST) {
          st1(y + row0 + gi, a[r].x);
          if (xg.has1) st1(y + row1 + gi, a[r].y);
        }
      }
    }
    if (!LAST) {
      dif<R>(a, tw, logT, x);
#pragma unroll
      for (int r = 0; r < R; ++r) s[spad(x.base + brev_bits(r, LR) * x.stride)] = a[r];
    }
  }
}

#define ND_RADIX_SWITCH(LOGR, CALL) \
  switch (LOGR) {                   \
    case 1: { constexpr int R = 2; CALL; } break;  \
    case 2: { constexpr int R = 4; CALL; } break;  \
    case 3: { constexpr int R = 8; CALL; } break;  \
    default: { constexpr int R = 16; CALL; } break; \
  }

// Copy the pair's two rows (G elements each) into shared memory with cp.async
// (16-byte pieces; rows are 16-byte aligned when staging is enabled).
template <typename T>
__device__ __forceinline__ void stage_rows(T* dst, const T* __restrict__ src, size_t row0, size_t row1, bool has1,
                                           int G, int tid, int nt) {
  const int nbytes = G * (int)sizeof(T);
  block_copy_async(dst, src + row0, nbytes, tid, nt);
  if (has1) block_copy_async(dst + G, src + row1, nbytes, tid, nt);
  cp_async_commit();
}

template <typename T, bool STAGED, bool ZP>
__global__ void __launch_bounds__(512) nd_forward_kernel(const T* __restrict__ v, NdGates<T> xs, SpecPtrs kh,
                                                         T* __restrict__ y, NdGeom gp, int B, int D, int N) {
  // the step tables are indexed at run time: read them from shared memory
  __shared__ NdGeom g;
  if (threadIdx.x == 0) g = gp;
  extern __shared__ float4 nd_smem_raw[];
  float2* s = reinterpret_cast<float2*>(nd_smem_raw);
  const int P = 1 << gp.logP;
  float2* tw = s + spad(P) + 1;
  // staged rows (STAGED): [2][G] elements after the table, 16-byte aligned
  T* xb = reinterpret_cast<T*>(reinterpret_cast<char*>(nd_smem_raw) +
                               ((sizeof(float2) * ((size_t)spad(P) + 1 + ((size_t)1 << gp.logT)) + 15) & ~(size_t)15));
  const int tid = threadIdx.x, nt = blockDim.x;
  const int c = blockIdx.x % D;
  const int b0 = 2 * (blockIdx.x / D);
  const int G = gp.G;
  const size_t row0 = ((size_t)b0 * D + c) * (size_t)G;
  const size_t row1 = row0 + (size_t)D * (size_t)G;
  const bool has1 = b0 + 1 < B;
  const int F = gp.nsteps;

  if (STAGED) stage_rows(xb, v, row0, row1, has1, G, tid, nt);
  const float2* tsrc = kh.p[0] + (size_t)D * P;
  for (int i = tid; i < (1 << gp.logT); i += nt) tw[i] = __ldg(tsrc + i);
  if (STAGED) cp_async_wait_all();
  __syncthreads();

  auto src_of = [&](const T* gsrc) {
    PairSrc<T, STAGED> r;
    r.r0 = STAGED ? xb : gsrc + row0;
    r.r1 = STAGED ? xb + G : gsrc + row1;
    r.has1 = has1;
    return r;
  };

  if (F >= 2) {
    ND_RADIX_SWITCH(g.st_logR[0], (entry_step<R, T, STAGED, ZP>(s, tw, g, src_of(v), tid, nt)));
  } else {
    const PairSrc<T, STAGED> vs = src_of(v);
    for (int i = tid; i < P; i += nt) {
      const int gi = pos_to_grid(g, i);
      s[spad(i)] = gi < 0 ? make_float2(0.f, 0.f) : vs.at(gi);
    }
  }
  __syncthreads();

  for (int n = 0; n < N; ++n) {
    const float2* __restrict__ H = pick(kh, n) + (size_t)c * P;
    const T* __restrict__ x_n = pick(xs, n);
    const bool last = n + 1 == N;
    // the gate rows arrive while the transform runs
    if (STAGED) stage_rows(xb, x_n, row0, row1, has1, G, tid, nt);
    for (int i = 1; i + 1 < F; ++i) {
      ND_RADIX_SWITCH(g.st_logR[i], (plain_step<R, false, ZP>(s, tw, g, i, tid, nt)));
      __syncthreads();
    }
    if (F >= 1) {
      ND_RADIX_SWITCH(g.st_logR[F - 1], (turn_step<R, ZP>(s, tw, g, F - 1, H, tid, nt)));
    } else {
      for (int i = tid; i < P; i += nt) s[spad(i)] = cmul(s[spad(i)], __ldg(H + i));
    }
    __syncthreads();
    for (int i = F - 2; i >= 1; --i) {
      ND_RADIX_SWITCH(g.st_logR[i], (plain_step<R, true, ZP>(s, tw, g, i, tid, nt)));
      __syncthreads();
    }
    if (STAGED) {
      cp_async_wait_all();
      __syncthreads();
    }
    const PairSrc<T, STAGED> xg = src_of(x_n);
    if (F >= 2) {
      if (last) {
        ND_RADIX_SWITCH(g.st_logR[0], (exit_step<R, true, T, STAGED, ZP>(s, tw, g, xg, y, row0, row1, tid, nt)));
      } else {
        ND_RADIX_SWITCH(g.st_logR[0], (exit_step<R, false, T, STAGED, ZP>(s, tw, g, xg, y, row0, row1, tid, nt)));
      }
    } else {
      for (int i = tid; i < P; i += nt) {
        const int gi = pos_to_grid(g, i);
        float2 u = make_float2(0.f, 0.f);
        if (gi >= 0) {
          const float2 a = s[spad(i)];
          const float2 xv = xg.at(gi);
          u = make_float2(a.x * xv.x, a.y * xv.y);
          if (last) {
            st1(y + row0 + gi, u.x);
            if (has1) st1(y + row1 + gi, u.y);
          }
        }
        s[spad(i)] = u;
      }
    }
    __syncthreads();
  }
}

// Spectrum of one filter: K [D][grid] float32 -> [D][P] float2 (transform
// order, times 1/P), one CTA per channel, with the forward kernel's radix
// steps and shared-memory layout; the twiddle table follows the spectra.
__global__ void __launch_bounds__(512) nd_spectrum_kernel(const float* __restrict__ K, float2* __restrict__ out,
                                                          NdGeom gp, int D) {
  __shared__ NdGeom g;
  if (threadIdx.x == 0) g = gp;
  extern __shared__ float4 nd_smem_raw[];
  float2* s = reinterpret_cast<float2*>(nd_smem_raw);
  const int P = 1 << gp.logP;
  float2* tw = s + spad(P) + 1;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int c = blockIdx.x;
  const float2* tsrc = out + (size_t)D * P;
  for (int i = tid; i < (1 << gp.logT); i += nt) tw[i] = tsrc[i];
  for (int i = tid; i < P; i += nt) {
    const int gi = pos_to_grid(gp, i);
    s[spad(i)] = make_float2(gi < 0 ? 0.f : __ldg(K + (size_t)c * gp.G + gi), 0.f);
  }
  __syncthreads();
  for (int i = 0; i < gp.nsteps; ++i) {
    ND_RADIX_SWITCH(g.st_logR[i], (plain_step<R, false, true>(s, tw, g, i, tid, nt)));
    __syncthreads();
  }
  const float inv = 1.0f / (float)P;   // exact: P is a power of two
  for (int i = tid; i < P; i += nt) {
    const float2 u = s[spad(i)];
    out[(size_t)c * P + i] = make_float2(u.x * inv, u.y * inv);
  }
}

// w_T^k = exp(-2 pi i k / T), k < T, formed in double and rounded once.
__global__ void nd_table_kernel(float2* __restrict__ tw, int logT) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < (1 << logT); k += gridDim.x * blockDim.x) {
    double sn, cs;
    sincospi(2.0 * (double)k / (double)(1 << logT), &sn, &cs);
    tw[k] = make_float2((float)cs, (float)-sn);
  }
}

int ilog2_pow2(int x) {
  if (x < 1 || (x & (x - 1))) return -1;
  int l = 0;
  while ((1 << l) < x) ++l;
  return l;
}

// Geometry of (nd, dims, boundary); false when unsupported.
bool nd_geometry(int nd, const int* dims, int boundary, NdGeom* g) {
  if (nd < 1 || nd > kNdMaxDims || !dims || (boundary != 0 && boundary != 1)) return false;
  NdGeom r{};
  r.zero = boundary == 0;
  int logP = 0, logG = 0, logT = 1;   // the table has at least 2 entries
  // axes of one point without padding change nothing and are dropped, so
  // that step 0 always runs along the first kept axis
  r.nd = 0;
  for (int a = 0; a < nd; ++a) {
    const int l = ilog2_pow2(dims[a]);
    if (l < 0) return false;
    const int ln = l + (r.zero ? 1 : 0);
    if (ln > kNdMaxLogAxis) return false;
    if (ln == 0) continue;
    r.logL[r.nd] = l;
    r.logn[r.nd] = ln;
    ++r.nd;
    logP += ln;
    logG += l;
    if (ln > logT) logT = ln;
  }
  nd = r.nd;
  if (logP > kNdMaxLogP) return false;
  int acc = 0;
  for (int a = nd - 1; a >= 0; --a) {
    r.logs[a] = acc;
    acc += r.logn[a];
  }
  r.logP = logP;
  r.logT = logT;
  r.G = 1 << logG;
  // radix steps: ceil(log2 P_a / 4) per axis, the levels spread evenly
  r.nsteps = 0;
  for (int a = 0; a < nd; ++a) {
    const int L = r.logn[a];
    const int k = (L + 3) / 4;
    int logm = L;
    for (int q = 0; q < k; ++q) {
      const int lr = L / k + (q < L % k ? 1 : 0);
      r.st_a[r.nsteps] = (signed char)a;
      r.st_logm[r.nsteps] = (signed char)logm;
      r.st_logR[r.nsteps] = (signed char)lr;
      r.st_first[r.nsteps] = (signed char)(q == 0);
      int p[2] = {-1, -1}, np = 0;
      if (r.zero)
        for (int b = nd - 1; b > a; --b) p[np++] = r.logs[b] + r.logL[b];   // ascending
      r.st_p1[r.nsteps] = (signed char)p[0];
      r.st_p2[r.nsteps] = (signed char)p[1];
      ++r.nsteps;
      logm -= lr;
    }
  }
  // the spectral product runs on the last step, which must hold R contiguous
  // points (one butterfly per block on an axis of inner stride 1)
  if (r.nsteps > 0) {
    const int l = r.nsteps - 1;
    if (r.st_logm[l] != r.st_logR[l] || r.logs[r.st_a[l]] != 0) return false;
  }
  *g = r;
  return true;
}

int nd_threads(const NdGeom& g) {
  int t = (1 << g.logP) / 32;
  if (t < 64) t = 64;
  if (t > 512) t = 512;
  return t;
}

// forward kernel: padded grid (+1 spare), the twiddle table, then (staged)
// the pair's two rows of one input
size_t nd_smem(const NdGeom& g, size_t elem, bool staged) {
  const size_t P = (size_t)1 << g.logP;
  const size_t base = (sizeof(float2) * (P + P / 16 + 1 + ((size_t)1 << g.logT)) + 15) & ~(size_t)15;
  return base + (staged ? 2 * elem * (size_t)g.G : 0);
}
// staging wants 16-byte rows and room for them next to the grid
bool nd_staged(const NdGeom& g, size_t elem) {
  return (elem * (size_t)g.G) % 16 == 0 && nd_smem(g, elem, true) + sizeof(NdGeom) <= (size_t)227 * 1024;
}
// spectrum kernel: the forward kernel's grid and table
size_t nd_spec_smem(const NdGeom& g) { return nd_smem(g, 0, false); }

size_t nd_block_bytes(const NdGeom& g, int D) {
  return sizeof(float2) * ((size_t)D * (1 << g.logP) + ((size_t)1 << g.logT));
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

bool nd_aligned16(const void* q) { return q && ((reinterpret_cast<uintptr_t>(q) & 15u) == 0); }

template <typename T>
cudaError_t launch_nd(const void* v, const void* const* x, const SpecPtrs& kh, void* y, const NdGeom& g, int B, int D,
                      int N, unsigned blocks, cudaStream_t s) {
  NdGates<T> xs{};
  for (int n = 0; n < N; ++n) xs.p[n] = reinterpret_cast<const T*>(x[n]);
  const bool staged = nd_staged(g, sizeof(T));
  const size_t smem = nd_smem(g, sizeof(T), staged);
  auto kern = g.zero ? (staged ? nd_forward_kernel<T, true, true> : nd_forward_kernel<T, false, true>)
                     : (staged ? nd_forward_kernel<T, true, false> : nd_forward_kernel<T, false, false>);
  cudaError_t e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  kern<<<blocks, nd_threads(g), smem, s>>>(reinterpret_cast<const T*>(v), xs, kh, reinterpret_cast<T*>(y), g, B, D, N);
  return cudaGetLastError();
}

}  // namespace

}  // namespace hyena

using namespace hyena;

extern "C" {

size_t hyena_nd_spectrum_bytes(int D, int nd, const int* dims, int boundary) {
  NdGeom g;
  if (D < 1 || !nd_geometry(nd, dims, boundary, &g)) return 0;
  return nd_block_bytes(g, D);
}

hyena_status hyena_nd_filter_spectrum(const float* K, int D, int nd, const int* dims, int boundary, void* khat,
                                      hyena_stream stream) {
  NdGeom g;
  if (D < 1 || !nd_aligned16(K) || !nd_aligned16(khat)) return HYENA_ERR_INVALID_ARG;
  if (!nd_geometry(nd, dims, boundary, &g)) return HYENA_ERR_UNSUPPORTED;
  if ((long long)D > (1LL << 40) / g.G) return HYENA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  float2* out = reinterpret_cast<float2*>(khat);
  nd_table_kernel<<<1, 256, 0, s>>>(out + (size_t)D * (1 << g.logP), g.logT);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = set_smem(nd_spectrum_kernel, nd_spec_smem(g));
  if (e == cudaSuccess) {
    nd_spectrum_kernel<<<D, nd_threads(g), nd_spec_smem(g), s>>>(K, out, g, D);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? HYENA_OK : report_cuda_error(e);
}

hyena_status hyena_nd_forward(const void* v, const void* const* x, const void* const* khat, int B, int D, int nd,
                              const int* dims, int boundary, int N, hyena_dtype dtype, void* y, hyena_stream stream) {
  if (N < 1 || N > kMaxOrder || B < 1 || D < 1) return HYENA_ERR_INVALID_ARG;
  if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
  if (!x || !khat || !nd_aligned16(v) || !nd_aligned16(y)) return HYENA_ERR_INVALID_ARG;
  for (int n = 0; n < N; ++n)
    if (!nd_aligned16(x[n]) || !nd_aligned16(khat[n])) return HYENA_ERR_INVALID_ARG;
  NdGeom g;
  if (!nd_geometry(nd, dims, boundary, &g)) return HYENA_ERR_UNSUPPORTED;
  if ((long long)B * D > (1LL << 40) / g.G) return HYENA_ERR_INVALID_ARG;
  const long long blocks = (long long)D * ((B + 1) / 2);
  if (blocks > 0x7fffffffLL) return HYENA_ERR_INVALID_ARG;
  SpecPtrs kh{};
  for (int n = 0; n < N; ++n) kh.p[n] = reinterpret_cast<const float2*>(khat[n]);
  const cudaError_t e = dtype == HYENA_BF16 ? launch_nd<__nv_bfloat16>(v, x, kh, y, g, B, D, N, (unsigned)blocks,
                                                                       (cudaStream_t)stream)
                                            : launch_nd<float>(v, x, kh, y, g, B, D, N, (unsigned)blocks,
                                                               (cudaStream_t)stream);
  return e == cudaSuccess ? HYENA_OK : report_cuda_error(e);
}

}  // extern "C"
