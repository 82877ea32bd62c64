// striped.cu -- the StripedHyena-form operator ("02. 3つの Hyena 演算子",
// section 2, the operator structure; section 3, the SE / MR / LI variants;
// section 4, the FIR sum y_t = sum_{k < l_h} h_k x_{t-k}):
//   q = h_T * xq,  k = h_H * xk,  v = h_K * xv      short explicit featurizers
//   y = q . (h_G * (k . v))                          inner filter h_G
// (xq, xk, xv are the outputs of the dense projections, which are not part of
// this operator).
//   - SE / MR (explicit inner filter of up to kMaxLG taps): one fused kernel,
//     each CTA one (b, c) row and one time tile, inputs staged with their
//     causal halo in shared memory, the inner sum in a register sliding window.
//   - LI (long implicit inner filter): the featurizer kernel writes q and
//     u = k . v, and y = q . (h_G * u) is an order-1 forward on the FFT path.
// Plus the LI filter h_t = sum_n R_n lambda_n^t (section 3, Hyena-LI; the
// pages' 1-based t - 1 is the 0-based lag t).
#include "fft_engine.cuh"
#include "kernels.cuh"
#include "mbar.cuh"

namespace hyena {

namespace {

constexpr int kStThreads = 256;
constexpr int kStTile = 2048;        // outputs per CTA
constexpr int kStPer = kStTile / kStThreads;   // consecutive outputs per thread (8)
// The bulk kernel zero-fills the halo of a row's first tile only (t0 < halo);
// every later tile must start at least one full halo into the row.
static_assert(kStTile >= ((kMaxStripedLG - 1 + kMaxStripedLF - 1 + 7) / 8) * 8,
              "a tile must be at least as long as the longest staged halo");

template <typename T>
__device__ __forceinline__ float ld1(const T* p);
template <>
__device__ __forceinline__ float ld1<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }

template <typename T>
__device__ __forceinline__ void st1(T* p, float v);
template <>
__device__ __forceinline__ void st1<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void st1<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Staged row: s[P + t - t0] = x[row + t] as float for t in [t0 - halo, t0 + n),
// zero outside [0, L). P = padded halo (a multiple of 4), so the main part
// starts on a 16-byte boundary; it is filled with 16-byte loads when the row
// is suitably aligned (vec), else element by element.
template <typename T>
__device__ __forceinline__ void stage_row(float* s, const T* __restrict__ x, size_t row, int t0, int halo, int P,
                                          int n, int L, bool vec, int tid) {
  for (int i = tid; i < halo; i += kStThreads) {
    const int t = t0 - halo + i;
    s[P - halo + i] = (t >= 0) ? ld1<T>(x + row + t) : 0.f;
  }
  constexpr int V = 16 / (int)sizeof(T);   // elements per 16-byte load
  const int nv = vec ? n / V : 0;
  for (int g = tid; g < nv; g += kStThreads) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + row + t0) + g);
    float* d = s + P + g * V;
    if constexpr (V == 8) {
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        d[2 * k] = __uint_as_float(w[k] << 16);
        d[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
      }
    } else {
      *reinterpret_cast<float4*>(d) = make_float4(__uint_as_float(u.x), __uint_as_float(u.y),
                                                  __uint_as_float(u.z), __uint_as_float(u.w));
    }
  }
  for (int i = nv * V + tid; i < n; i += kStThreads) s[P + i] = ld1<T>(x + row + t0 + i);
}

__device__ __forceinline__ int pad4(int h) { return (h + 3) & ~3; }

// acc[p] = sum_{j < len} f[j] s[P + base + p - j], p < kStPer, as a sliding
// window over the staged row (positions below P - halo hold zeros or halo)
__device__ __forceinline__ void fir8(const float* f, int len, const float* s, int pos, float (&acc)[kStPer]) {
  float win[kStPer];
#pragma unroll
  for (int p = 0; p < kStPer; ++p) {
    win[p] = s[pos + p];
    acc[p] = 0.f;
  }
  for (int j = 0; j < len; ++j) {
    const float g = f[j];
#pragma unroll
    for (int p = 0; p < kStPer; ++p) acc[p] = fmaf(g, win[p], acc[p]);
#pragma unroll
    for (int p = kStPer - 1; p > 0; --p) win[p] = win[p - 1];
    if (j + 1 < len) win[0] = s[pos - j - 1];
  }
}

template <typename T>
__device__ __forceinline__ void store8(T* dst, const float (&v)[kStPer]);
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* dst, const float (&v)[kStPer]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
    w[k] = *reinterpret_cast<const uint32_t*>(&b);
  }
  *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}
template <>
__device__ __forceinline__ void store8<float>(float* dst, const float (&v)[kStPer]) {
  reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// FUSED: y = q . (hG * u); otherwise q and u = k . v are written.
template <typename T, bool FUSED>
__global__ void __launch_bounds__(kStThreads)
striped_kernel(const T* __restrict__ xq, const T* __restrict__ xk, const T* __restrict__ xv,
               const float* __restrict__ hT, const float* __restrict__ hH, const float* __restrict__ hK, int lf,
               const float* __restrict__ hG, int lg, int D, int L, T* __restrict__ y, T* __restrict__ qout,
               T* __restrict__ uout) {
  extern __shared__ __align__(16) float st[];
  const int tid = threadIdx.x;
  const int tiles = (L + kStTile - 1) / kStTile;
  const long long rowi = blockIdx.x / tiles;
  const int c = (int)(rowi % D);
  const size_t row = (size_t)rowi * L;
  const int t0 = (int)(blockIdx.x % tiles) * kStTile;
  const int n_out = min(kStTile, L - t0);
  const int hg = FUSED ? lg - 1 : 0;     // u halo for the inner filter
  const int hf = lf - 1;                  // featurizer halo
  const int Hx = hg + hf, Px = pad4(Hx);  // k, v rows
  const int Pq = pad4(hf);                // q row
  const int Pu = pad4(hg);                // u row
  const int S = pad4(kStTile + lg + 24);  // capacity of each staged row (16-byte multiple)
  float* fT = st;                         // [16]
  float* fH = fT + 16;
  float* fK = fH + 16;
  float* fG = fK + 16;                    // [pad4(lg)]
  float* sk = fG + (FUSED ? pad4(lg) : 0);
  float* sv = sk + S;
  float* su = sv + S;
  float* sq = su + S;
  for (int i = tid; i < lf; i += kStThreads) {
    fT[i] = hT[(size_t)c * lf + i];
    fH[i] = hH[(size_t)c * lf + i];
    fK[i] = hK[(size_t)c * lf + i];
  }
  if (FUSED)
    for (int i = tid; i < lg; i += kStThreads) fG[i] = hG[(size_t)c * lg + i];
  // rows of 16-byte multiples start 16-byte aligned: vector loads and stores
  const bool vec = ((L * (int)sizeof(T)) & 15) == 0;
  stage_row<T>(sk, xk, row, t0, Hx, Px, n_out, L, vec, tid);
  stage_row<T>(sv, xv, row, t0, Hx, Px, n_out, L, vec, tid);
  stage_row<T>(sq, xq, row, t0, hf, Pq, n_out, L, vec, tid);
  __syncthreads();
  const int base = tid * kStPer;
  const bool full = base + kStPer <= n_out;
  // u at t = t0 + base + p from the sliding windows; the halo t in [t0 - hg, t0) below
  if (base < n_out) {
    float a[kStPer], b[kStPer];
    fir8(fH, lf, sk, Px + base, a);
    fir8(fK, lf, sv, Px + base, b);
#pragma unroll
    for (int p = 0; p < kStPer; ++p) su[Pu + base + p] = a[p] * b[p];
  }
  for (int i = tid; i < hg; i += kStThreads) {
    const int t = t0 - hg + i;
    float a = 0.f, b = 0.f;
    for (int j = 0; j < lf; ++j) {
      a = fmaf(fH[j], sk[Px - hg + i - j], a);
      b = fmaf(fK[j], sv[Px - hg + i - j], b);
    }
    su[Pu - hg + i] = t >= 0 ? a * b : 0.f;
  }
  __syncthreads();
  if (base >= n_out) return;
  float q[kStPer];
  fir8(fT, lf, sq, Pq + base, q);
  float out[kStPer], u8[kStPer];
  if (FUSED) {
    fir8(fG, lg, su, Pu + base, out);
#pragma unroll
    for (int p = 0; p < kStPer; ++p) out[p] *= q[p];
  } else {
#pragma unroll
    for (int p = 0; p < kStPer; ++p) u8[p] = su[Pu + base + p];
  }
  if (vec && full) {
    if (FUSED) {
      store8<T>(y + row + t0 + base, out);
    } else {
      store8<T>(qout + row + t0 + base, q);
      store8<T>(uout + row + t0 + base, u8);
    }
  } else {
#pragma unroll
    for (int p = 0; p < kStPer; ++p) {
      if (base + p >= n_out) break;
      if (FUSED) {
        st1<T>(y + row + t0 + base + p, out[p]);
      } else {
        st1<T>(qout + row + t0 + base + p, q[p]);
        st1<T>(uout + row + t0 + base + p, u8[p]);
      }
    }
  }
}

// ---- persistent, bulk-copy-fed variant (rows of 16-byte multiples) ----------
//
// Work item = (row, tile of kStTile outputs). Each CTA walks items with a grid
// stride; the three input windows [t0 - H, t0 + n) of item i + 1 are fetched
// by one thread with cp.async.bulk (completion counted in bytes on the
// stage's mbarrier) while item i is computed from the other stage. Inputs
// stay in their storage type in shared memory; H is the causal halo rounded
// up to 16 bytes (zeros are written there by the threads for t0 = 0).

__device__ int g_striped_timeout;

template <typename T>
__device__ __forceinline__ float ldsT(const T* p);
template <>
__device__ __forceinline__ float ldsT<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ldsT<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// acc[p] = sum_{j < len} f[j] x[pos + p - j] over a staged row in storage type T
template <typename T>
__device__ __forceinline__ void fir8T(const float* f, int len, const T* x, int pos, float (&acc)[kStPer]) {
  float win[kStPer];
#pragma unroll
  for (int p = 0; p < kStPer; ++p) {
    win[p] = ldsT<T>(x + pos + p);
    acc[p] = 0.f;
  }
  for (int j = 0; j < len; ++j) {
    const float g = f[j];
#pragma unroll
    for (int p = 0; p < kStPer; ++p) acc[p] = fmaf(g, win[p], acc[p]);
#pragma unroll
    for (int p = kStPer - 1; p > 0; --p) win[p] = win[p - 1];
    if (j + 1 < len) win[0] = ldsT<T>(x + pos - j - 1);
  }
}

// Eight consecutive staged elements as floats, from one 16-byte (bf16) or two
// (float) aligned shared-memory loads.
template <typename T>
__device__ __forceinline__ void load8f(const T* p, float* w);
template <>
__device__ __forceinline__ void load8f<__nv_bfloat16>(const __nv_bfloat16* p, float* w) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t v[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    w[2 * k] = __uint_as_float(v[k] << 16);
    w[2 * k + 1] = __uint_as_float(v[k] & 0xffff0000u);
  }
}
template <>
__device__ __forceinline__ void load8f<float>(const float* p, float* w) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
}

// acc[p] = sum_{j < LEN} f[j] x[pos + p - j] for a compile-time LEN <= 9:
// the 16 points pos-8 .. pos+7 come from two aligned vector loads and every
// tap is unrolled (pos a multiple of 8 elements, 16-byte aligned).
template <typename T, int LEN>
__device__ __forceinline__ void fir8v(const float* f, const T* x, int pos, float (&acc)[kStPer]) {
  static_assert(LEN >= 1 && LEN <= 9, "fir8v covers up to 9 taps");
  float w[16];
  load8f<T>(x + pos - 8, w);
  load8f<T>(x + pos, w + 8);
  float g[LEN];
#pragma unroll
  for (int j = 0; j < LEN; ++j) g[j] = f[j];
#pragma unroll
  for (int p = 0; p < kStPer; ++p) {
    float a = 0.f;
#pragma unroll
    for (int j = 0; j < LEN; ++j) a = fmaf(g[j], w[8 + p - j], a);
    acc[p] = a;
  }
}

// LFC, LGC > 0: filter lengths fixed at compile time (the Hyena-SE sizes),
// taps unrolled over vector-loaded windows; 0: any length (sliding windows).
template <typename T, int LFC, int LGC>
__global__ void __launch_bounds__(kStThreads)
striped_bulk_kernel(const T* __restrict__ xq, const T* __restrict__ xk, const T* __restrict__ xv,
                    const float* __restrict__ hT, const float* __restrict__ hH, const float* __restrict__ hK, int lf,
                    const float* __restrict__ hG, int lg, int D, int L, long long items, T* __restrict__ y) {
  extern __shared__ __align__(128) unsigned char sraw[];
  constexpr int E = (int)sizeof(T), V = 16 / E;
  const int tid = threadIdx.x;
  const int tiles = (L + kStTile - 1) / kStTile;
  const int hg = lg - 1, hf = lf - 1, Hx = hg + hf;
  const int HP = ((Hx + V - 1) / V) * V;           // halo slots, 16-byte multiple
  const int W = HP + kStTile;                       // elements per staged window
  // u row offset; the vector windows of fir8v read 8 slots before each output
  const int Pu = LGC > 0 ? max(pad4(hg), 8) : pad4(hg);
  const int S = pad4(kStTile + lg + 24);
  const size_t winb = ((size_t)W * E + 127) & ~(size_t)127;
  // [stage][xq, xk, xv] windows, then su (float), filters, mbarriers
  float* su = reinterpret_cast<float*>(sraw + 6 * winb);
  float* fT = su + S;
  float* fH = fT + 16;
  float* fK = fH + 16;
  float* fG = fK + 16;
  uint64_t* bars = reinterpret_cast<uint64_t*>(fG + pad4(lg) + 4);
  auto win = [&](int stage, int a) { return reinterpret_cast<T*>(sraw + (size_t)(3 * stage + a) * winb); };
  const T* srcs[3] = {xq, xk, xv};

  if (tid == 0) {
    for (int k = 0; k < 2; ++k) mbar_init(smem_u32(&bars[k]), 1);
    mbar_init_fence();
  }
  __syncthreads();

  // one thread: expected bytes, then the three window copies of item it into stage
  auto issue = [&](long long it, int stage) {
    const long long rowi = it / tiles;
    const int t0 = (int)(it % tiles) * kStTile;
    const int n = min(kStTile, L - t0);
    const int h = t0 >= HP ? HP : 0;               // first tile: halo zero-filled by the threads
    const uint32_t bytes = (uint32_t)((h + n) * E);
    const uint32_t bar = smem_u32(&bars[stage]);
    mbar_arrive_expect_tx(bar, 3 * bytes);
    for (int a = 0; a < 3; ++a)
      bulk_g2s(smem_u32(win(stage, a) + (HP - h)), srcs[a] + (size_t)rowi * L + t0 - h, bytes, bar);
  };

  uint32_t phase[2] = {0, 0};
  bool pending[2] = {false, false};   // thread 0: a copy issued into the stage and not yet waited for
  long long it = blockIdx.x;
  if (tid == 0 && it < items) {
    issue(it, 0);
    pending[0] = true;
  }
  int stage = 0;
  bool ok = true;
  for (; it < items; it += gridDim.x, stage ^= 1) {
    const long long rowi = it / tiles;
    const int c = (int)(rowi % D);
    const int t0 = (int)(it % tiles) * kStTile;
    const int n_out = min(kStTile, L - t0);
    // the other stage was released by the barrier that ended the last item
    if (tid == 0 && it + gridDim.x < items) {
      issue(it + gridDim.x, stage ^ 1);
      pending[stage ^ 1] = true;
    }
    const bool done = mbar_wait(smem_u32(&bars[stage]), phase[stage]);
    if (done) {
      phase[stage] ^= 1;
      pending[stage] = false;
    } else if (tid == 0) {
      atomicExch(&g_striped_timeout, 1);
    }
    const T* wq = win(stage, 0);
    const T* wk = win(stage, 1);
    const T* wv = win(stage, 2);
    if (t0 < HP)
      for (int i = tid; i < 3 * HP; i += kStThreads) win(stage, i / HP)[i % HP] = T(0.f);
    for (int i = tid; i < lf; i += kStThreads) {
      fT[i] = hT[(size_t)c * lf + i];
      fH[i] = hH[(size_t)c * lf + i];
      fK[i] = hK[(size_t)c * lf + i];
    }
    for (int i = tid; i < lg; i += kStThreads) fG[i] = hG[(size_t)c * lg + i];
    ok = __syncthreads_and(done) != 0;
    if (!ok) break;
    // u = (hH * xk)(hK * xv) at t = t0 + base + p, and the halo t in [t0 - hg, t0)
    const int base = tid * kStPer;
    if (base < n_out) {
      float a[kStPer], b[kStPer];
      if constexpr (LFC > 0) {
        fir8v<T, LFC>(fH, wk, HP + base, a);
        fir8v<T, LFC>(fK, wv, HP + base, b);
        float4* su4 = reinterpret_cast<float4*>(su + Pu + base);
        su4[0] = make_float4(a[0] * b[0], a[1] * b[1], a[2] * b[2], a[3] * b[3]);
        su4[1] = make_float4(a[4] * b[4], a[5] * b[5], a[6] * b[6], a[7] * b[7]);
      } else {
        fir8T<T>(fH, lf, wk, HP + base, a);
        fir8T<T>(fK, lf, wv, HP + base, b);
#pragma unroll
        for (int p = 0; p < kStPer; ++p) su[Pu + base + p] = a[p] * b[p];
      }
    }
    for (int i = tid; i < hg; i += kStThreads) {
      const int t = t0 - hg + i;
      float a = 0.f, b = 0.f;
      for (int j = 0; j < lf; ++j) {
        a = fmaf(fH[j], ldsT<T>(wk + HP - hg + i - j), a);
        b = fmaf(fK[j], ldsT<T>(wv + HP - hg + i - j), b);
      }
      su[Pu - hg + i] = t >= 0 ? a * b : 0.f;
    }
    __syncthreads();
    if (base < n_out) {
      float q[kStPer], out[kStPer];
      if constexpr (LFC > 0) {
        fir8v<T, LFC>(fT, wq, HP + base, q);
        fir8v<float, LGC>(fG, su, Pu + base, out);
      } else {
        fir8T<T>(fT, lf, wq, HP + base, q);
        fir8(fG, lg, su, Pu + base, out);
      }
#pragma unroll
      for (int p = 0; p < kStPer; ++p) out[p] *= q[p];
      T* dst = y + (size_t)rowi * L + t0 + base;
      if (base + kStPer <= n_out) {
        store8<T>(dst, out);
      } else {
        for (int p = 0; p < kStPer && base + p < n_out; ++p) st1<T>(dst + p, out[p]);
      }
    }
    // generic-proxy writes to this stage (halo zeros) before its next bulk copy
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
  }
  // after a timeout: wait (bounded, 1 s each) for the copies still in flight
  // into this CTA's shared memory before it exits (normal exits leave none)
  if (tid == 0)
    for (int k = 0; k < 2; ++k)
      if (pending[k]) mbar_wait(smem_u32(&bars[k]), phase[k], 1000000000ull);
  __syncthreads();
}

// h[c][t] = sum_n R[c][n] lambda[c][n]^t
__global__ void exp_sum_filter_kernel(const float* __restrict__ R, const float* __restrict__ lam, int d, int D, int L,
                                      float* __restrict__ h) {
  const size_t n = (size_t)D * L;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int c = (int)(i / L), t = (int)(i % L);
    float acc = 0.f;
    for (int k = 0; k < d; ++k) acc = fmaf(R[(size_t)c * d + k], powf(lam[(size_t)c * d + k], (float)t), acc);
    h[i] = acc;
  }
}

size_t striped_smem(bool fused, int lg) {
  return sizeof(float) * (size_t)(16 * 3 + (fused ? ((lg + 3) & ~3) : 0) + 4 * ((kStTile + lg + 24 + 3) & ~3));
}

size_t striped_bulk_smem(int E, int lf, int lg) {
  const int V = 16 / E, Hx = lg - 1 + lf - 1;
  const size_t HP = (size_t)((Hx + V - 1) / V) * V;
  const size_t winb = ((HP + kStTile) * E + 127) & ~(size_t)127;
  const size_t S = (size_t)((kStTile + lg + 24 + 3) & ~3);   // u row: offset (<= max(pad4(lg-1), 8)) + tile
  return 6 * winb + sizeof(float) * (S + 48 + (size_t)((lg + 3) & ~3) + 4) + 2 * sizeof(uint64_t);
}

template <typename T>
cudaError_t launch_striped_bulk(const void* xq, const void* xk, const void* xv, const float* hT, const float* hH,
                                const float* hK, int lf, const float* hG, int lg, int B, int D, int L, void* y,
                                cudaStream_t s) {
  // the Hyena-SE sizes (featurizers of 4 taps, inner filter of 7) take the unrolled kernel
  auto k = (lf == 4 && lg == 7) ? striped_bulk_kernel<T, 4, 7> : striped_bulk_kernel<T, 0, 0>;
  const size_t smem = striped_bulk_smem((int)sizeof(T), lf, lg);
  int grid = 0;
  cudaError_t e = persistent_grid((const void*)k, kStThreads, smem, &grid);
  if (e != cudaSuccess) return e;
  const long long items = (long long)((L + kStTile - 1) / kStTile) * B * D;
  if ((long long)grid > items) grid = (int)items;
  k<<<grid, kStThreads, smem, s>>>(reinterpret_cast<const T*>(xq), reinterpret_cast<const T*>(xk),
                                   reinterpret_cast<const T*>(xv), hT, hH, hK, lf, hG, lg, D, L, items,
                                   reinterpret_cast<T*>(y));
  return cudaGetLastError();
}

template <typename T, bool FUSED>
cudaError_t launch_striped_t(const void* xq, const void* xk, const void* xv, const float* hT, const float* hH,
                             const float* hK, int lf, const float* hG, int lg, int B, int D, int L, void* y, void* q,
                             void* u, cudaStream_t s) {
  auto k = striped_kernel<T, FUSED>;
  const size_t smem = striped_smem(FUSED, lg);
  cudaError_t e = cudaFuncSetAttribute((const void*)k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long blocks = (long long)((L + kStTile - 1) / kStTile) * B * D;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  k<<<(unsigned)blocks, kStThreads, smem, s>>>(reinterpret_cast<const T*>(xq), reinterpret_cast<const T*>(xk),
                                   reinterpret_cast<const T*>(xv), hT, hH, hK, lf, hG, lg, D, L,
                                   reinterpret_cast<T*>(y), reinterpret_cast<T*>(q), reinterpret_cast<T*>(u));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_striped(const void* xq, const void* xk, const void* xv, const float* hT, const float* hH,
                           const float* hK, int lf, const float* hG, int lg, int B, int D, int L, bool bf16, void* y,
                           void* q, void* u, cudaStream_t s) {
  const bool fused = (hG != nullptr);
  // rows of 16-byte multiples: persistent kernel fed by bulk copies
  if (fused && ((long long)L * (bf16 ? 2 : 4)) % 16 == 0)
    return bf16 ? launch_striped_bulk<__nv_bfloat16>(xq, xk, xv, hT, hH, hK, lf, hG, lg, B, D, L, y, s)
                : launch_striped_bulk<float>(xq, xk, xv, hT, hH, hK, lf, hG, lg, B, D, L, y, s);
  if (bf16)
    return fused ? launch_striped_t<__nv_bfloat16, true>(xq, xk, xv, hT, hH, hK, lf, hG, lg, B, D, L, y, q, u, s)
                 : launch_striped_t<__nv_bfloat16, false>(xq, xk, xv, hT, hH, hK, lf, hG, lg, B, D, L, y, q, u, s);
  return fused ? launch_striped_t<float, true>(xq, xk, xv, hT, hH, hK, lf, hG, lg, B, D, L, y, q, u, s)
               : launch_striped_t<float, false>(xq, xk, xv, hT, hH, hK, lf, hG, lg, B, D, L, y, q, u, s);
}

int striped_read_and_clear_timeout() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_striped_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (v) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_striped_timeout, &zero, sizeof(int));
  }
  return v;
}

cudaError_t launch_exp_sum_filter(const float* R, const float* lam, int d, int D, int L, float* h, cudaStream_t s) {
  const size_t n = (size_t)D * L;
  size_t blocks = (n + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  exp_sum_filter_kernel<<<(int)blocks, 256, 0, s>>>(R, lam, d, D, L, h);
  return cudaGetLastError();
}

}  // namespace hyena

using namespace hyena;

namespace {
bool st_aligned16(const void* q) { return q && ((reinterpret_cast<uintptr_t>(q) & 15u) == 0); }

hyena_status striped_check(const void* xq, const void* xk, const void* xv, const float* hT, const float* hH,
                           const float* hK, int lf, int B, int D, int L, hyena_dtype dtype) {
  if (B < 1 || D < 1 || L < 1 || lf < 1 || lf > kMaxStripedLF) return HYENA_ERR_INVALID_ARG;
  if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
  if (!st_aligned16(xq) || !st_aligned16(xk) || !st_aligned16(xv) || !st_aligned16(hT) || !st_aligned16(hH) ||
      !st_aligned16(hK))
    return HYENA_ERR_INVALID_ARG;
  if ((long long)B * D > (1LL << 40) / L) return HYENA_ERR_INVALID_ARG;
  return HYENA_OK;
}
}  // namespace

extern "C" {

hyena_status hyena_striped_forward(const void* xq, const void* xk, const void* xv, const float* hT, const float* hH,
                                   const float* hK, int lf, const float* hG, int lg, int B, int D, int L,
                                   hyena_dtype dtype, void* y, hyena_stream stream) {
  hyena_status st = striped_check(xq, xk, xv, hT, hH, hK, lf, B, D, L, dtype);
  if (st != HYENA_OK) return st;
  if (!st_aligned16(hG) || !st_aligned16(y) || lg < 1 || lg > kMaxStripedLG) return HYENA_ERR_INVALID_ARG;
  const cudaError_t e = launch_striped(xq, xk, xv, hT, hH, hK, lf, hG, lg, B, D, L, dtype == HYENA_BF16, y, nullptr,
                                       nullptr, (cudaStream_t)stream);
  return e == cudaSuccess ? HYENA_OK : report_cuda_error(e);
}

hyena_status hyena_striped_featurize(const void* xq, const void* xk, const void* xv, const float* hT,
                                     const float* hH, const float* hK, int lf, int B, int D, int L,
                                     hyena_dtype dtype, void* q, void* u, hyena_stream stream) {
  hyena_status st = striped_check(xq, xk, xv, hT, hH, hK, lf, B, D, L, dtype);
  if (st != HYENA_OK) return st;
  if (!st_aligned16(q) || !st_aligned16(u)) return HYENA_ERR_INVALID_ARG;
  const cudaError_t e = launch_striped(xq, xk, xv, hT, hH, hK, lf, nullptr, 0, B, D, L, dtype == HYENA_BF16, nullptr,
                                       q, u, (cudaStream_t)stream);
  return e == cudaSuccess ? HYENA_OK : report_cuda_error(e);
}

hyena_status hyena_filter_exponential(const float* R, const float* lambda, int d, int D, int L, float* h,
                                      hyena_stream stream) {
  if (!st_aligned16(R) || !st_aligned16(lambda) || !st_aligned16(h) || d < 1 || d > 64 || D < 1 || L < 1)
    return HYENA_ERR_INVALID_ARG;
  if ((long long)D * L > (1LL << 40)) return HYENA_ERR_INVALID_ARG;
  const cudaError_t e = launch_exp_sum_filter(R, lambda, d, D, L, h, (cudaStream_t)stream);
  return e == cudaSuccess ? HYENA_OK : report_cuda_error(e);
}

}  // extern "C"
