// backward.cu -- gradients of a scalar loss through the order-N operator and
// through the implicit-filter FFN.
//
// The pages print no backward formulas (they mention training at 1M tokens:
// glossary "Hyena（ハイエナ）", section 超長系列タスクでの優位性); this is the chain rule through
// the forward definitions (order-N recurrence, "Hyena Hierarchy" digest,
// 방법 / 프레임워크 개요; causal FIR sum, "02. 3つの Hyena 演算子", section 4):
//   u_n = h_n * z_n,  z_{n+1} = x_n . u_n,  g_{N+1} = dy,  r_n = g_{n+1} . x_n
//   dx_n = g_{n+1} . u_n
//   g_n[s]  = sum_{t>=s} h_n[t-s] r_n[t]
//   dh_n[j] = sum_b sum_{t>=j} r_n[t] z_n[t-j]
//   dv = g_1.
// With rev(a)[t] = a[L-1-t] both correlations are causal convolutions:
//   g_n  = rev(h_n * rev(r_n))
//   dh_n = rev(sum_b z_n * rev(r_n))
// so every long correlation runs on the forward's 2L-grid FFT kernels (fused
// or four-step, float32 I/O): h_n * rev(r_n) is an order-1 forward with unit
// gates on the cached spectrum of h_n, and sum_b z_n * rev(r_n) is an order-1
// forward of a unit impulse on the spectrum sum_b Z_b R_b, formed pointwise
// from the spectra of the z and rev(r) rows.
#include "fft_engine.cuh"
#include "kernels.cuh"

namespace hyena {

namespace {

constexpr int kPwThreads = 256;

int pw_blocks(size_t n) {
  size_t b = (n + kPwThreads - 1) / kPwThreads;
  if (b > 148 * 16) b = 148 * 16;
  return b < 1 ? 1 : (int)b;
}

__device__ __forceinline__ float2 ldf2(const float* p) { return __ldg(reinterpret_cast<const float2*>(p)); }
__device__ __forceinline__ void stf2(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }

// z_n as float32: v (n = 1) or x_{n-1} . u_{n-1}
template <typename T>
__global__ void bwd_make_z(const T* __restrict__ v, const T* __restrict__ xp, const float* __restrict__ up,
                           float* __restrict__ z, size_t npairs) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < npairs; i += (size_t)gridDim.x * blockDim.x) {
    float2 r;
    if (xp) {
      const float2 a = IO<T>::load2(xp + 2 * i), b = ldf2(up + 2 * i);
      r = make_float2(a.x * b.x, a.y * b.y);
    } else {
      r = IO<T>::load2(v + 2 * i);
    }
    stf2(z + 2 * i, r);
  }
}

// From g_{n+1} (dy in T, natural order; or float32 stored time-reversed):
//   dx_n = g . u_n  (T),   rrev = rev(g . x_n)  (float32)
template <typename T>
__global__ void bwd_stage_grad(const T* __restrict__ dy, const float* __restrict__ grev, const T* __restrict__ x,
                               const float* __restrict__ u, T* __restrict__ dx, float* __restrict__ rrev, int L,
                               size_t npairs) {
  const int H = L / 2;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < npairs; i += (size_t)gridDim.x * blockDim.x) {
    const size_t row = i / H;
    const int p = (int)(i - row * H);
    const size_t j = row * H + (H - 1 - p);   // pair holding times L-2-2p, L-1-2p
    float2 g;
    if (grev) {
      const float2 q = ldf2(grev + 2 * j);
      g = make_float2(q.y, q.x);
    } else {
      g = IO<T>::load2(dy + 2 * i);
    }
    const float2 xv = IO<T>::load2(x + 2 * i), uv = ldf2(u + 2 * i);
    IO<T>::store2(dx + 2 * i, make_float2(g.x * uv.x, g.y * uv.y));
    stf2(rrev + 2 * j, make_float2(g.y * xv.y, g.x * xv.x));
  }
}

// out[row][t] = in[row][L-1-t]
template <typename T>
__global__ void bwd_reverse_rows(const float* __restrict__ in, T* __restrict__ out, int L, size_t npairs) {
  const int H = L / 2;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < npairs; i += (size_t)gridDim.x * blockDim.x) {
    const size_t row = i / H;
    const int p = (int)(i - row * H);
    const float2 q = ldf2(in + 2 * (row * H + (H - 1 - p)));
    IO<T>::store2(out + 2 * i, make_float2(q.y, q.x));
  }
}

// S[c][k] = scale * sum_b Zs[b D + c][k] Rs[b D + c][k] over the library-order
// spectrum rows; index 0 packs the real DC and Nyquist bins (multiplied
// componentwise).
__global__ void bwd_spec_product(const float2* __restrict__ zs, const float2* __restrict__ rs,
                                 float2* __restrict__ S, int B, int D, int M, float scale) {
  const size_t n = (size_t)D * M;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int k = (int)(i % M);
    float2 acc = make_float2(0.f, 0.f);
    for (int b = 0; b < B; ++b) {
      const size_t o = (size_t)b * D * M + i;
      const float2 a = __ldg(zs + o), r = __ldg(rs + o);
      if (k == 0) {
        acc.x = fmaf(a.x, r.x, acc.x);
        acc.y = fmaf(a.y, r.y, acc.y);
      } else {
        acc = cadd(acc, cmul(a, r));
      }
    }
    S[i] = make_float2(acc.x * scale, acc.y * scale);
  }
}

// ones[i] = 1 for i < n_ones; delta rows [D][L] with delta[c][0] = 1
__global__ void bwd_fill(float* __restrict__ ones, size_t n_ones, float* __restrict__ delta, int D, int L) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_ones; i += stride) ones[i] = 1.f;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < (size_t)D * L; i += stride)
    delta[i] = (i % L) == 0 ? 1.f : 0.f;
}

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

struct BwdPlan {
  size_t U, ZR, G, ONES, DELTA, Q, SPEC2, SBLK, FWS, total;
  size_t fws_bytes;
};

bool plan_backward(int B, int D, int N, const Layout& ly, BwdPlan* p) {
  const size_t BDL = (size_t)B * D * ly.L, DL = (size_t)D * ly.L;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += align256(bytes);
    return at;
  };
  p->U = take(sizeof(float) * N * BDL);
  p->ZR = take(sizeof(float) * 2 * BDL);
  p->G = take(sizeof(float) * BDL);
  p->ONES = take(sizeof(float) * BDL);
  p->DELTA = take(sizeof(float) * DL);
  p->Q = take(sizeof(float) * DL);
  if ((long long)2 * B * D > (1LL << 31) - 1) return false;
  p->SPEC2 = take(sizeof(float2) * spectrum_block_floats2(ly, 2 * B * D));
  p->SBLK = take(sizeof(float2) * spectrum_block_floats2(ly, D));
  p->fws_bytes = ly.fourstep ? fourstep_wave_bytes((long long)B * D, ly, WaveRule::kBackward) : 0;
  p->FWS = take(p->fws_bytes);
  p->total = o;
  return true;
}

template <typename T>
cudaError_t run_backward(const void* v, const void* const* x, const void* const* hhat, const void* dy, int B, int D,
                         const Layout& ly, int N, void* dv, void* const* dx, float* const* dh, char* ws,
                         const BwdPlan& pl, cudaStream_t s) {
  const int L = ly.L;
  const size_t BDL = (size_t)B * D * L, DL = (size_t)D * L;
  float* U = reinterpret_cast<float*>(ws + pl.U);
  float* Z = reinterpret_cast<float*>(ws + pl.ZR);
  float* R = Z + BDL;
  float* G = reinterpret_cast<float*>(ws + pl.G);
  float* ones = reinterpret_cast<float*>(ws + pl.ONES);
  float* delta = reinterpret_cast<float*>(ws + pl.DELTA);
  float* Q = reinterpret_cast<float*>(ws + pl.Q);
  float2* spec2 = reinterpret_cast<float2*>(ws + pl.SPEC2);
  float2* sblk = reinterpret_cast<float2*>(ws + pl.SBLK);
  void* fws = pl.fws_bytes ? reinterpret_cast<void*>(ws + pl.FWS) : nullptr;
  const T* vt = reinterpret_cast<const T*>(v);
  const int gp = pw_blocks(BDL / 2);
  const void* gate1[1] = {ones};
  cudaError_t e;

  bwd_fill<<<pw_blocks(BDL), kPwThreads, 0, s>>>(ones, BDL, delta, D, L);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_fill_tables(sblk + tables_offset(ly, D), ly, s)) != cudaSuccess) return e;

  // forward again, keeping u_n = h_n * z_n
  for (int n = 0; n < N; ++n) {
    const T* xp = n ? reinterpret_cast<const T*>(x[n - 1]) : nullptr;
    bwd_make_z<T><<<gp, kPwThreads, 0, s>>>(vt, xp, n ? U + (n - 1) * BDL : nullptr, Z, BDL / 2);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const void* hh1[1] = {hhat[n]};
    e = forward_dispatch(Z, gate1, hh1, B, D, ly, 1, false, U + n * BDL, fws, pl.fws_bytes, false, s);
    if (e != cudaSuccess) return e;
  }
  // reverse sweep; G holds rev(g_{n+1}) after the first step
  const size_t M = (size_t)ly.M;
  for (int n = N - 1; n >= 0; --n) {
    bwd_stage_grad<T><<<gp, kPwThreads, 0, s>>>(reinterpret_cast<const T*>(dy), n == N - 1 ? nullptr : G,
                                                reinterpret_cast<const T*>(x[n]), U + n * BDL,
                                                reinterpret_cast<T*>(dx[n]), R, L, BDL / 2);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const T* xp = n ? reinterpret_cast<const T*>(x[n - 1]) : nullptr;
    bwd_make_z<T><<<gp, kPwThreads, 0, s>>>(vt, xp, n ? U + (n - 1) * BDL : nullptr, Z, BDL / 2);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // dh_n = rev(sum_b z * rev(r)): spectra of the z and rev(r) rows, their
    // product summed over the batch (x 4M: each stored spectrum carries 1/4M),
    // then the inverse through an order-1 forward of a unit impulse
    if ((e = spectrum_dispatch(Z, spec2, 2 * B * D, ly, false, s)) != cudaSuccess) return e;
    bwd_spec_product<<<pw_blocks(DL), kPwThreads, 0, s>>>(spec2, spec2 + (size_t)B * D * M, sblk, B, D, (int)M,
                                                          4.f * (float)M);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const void* sb[1] = {sblk};
    e = forward_dispatch(delta, gate1, sb, 1, D, ly, 1, false, Q, fws, pl.fws_bytes, false, s);
    if (e != cudaSuccess) return e;
    bwd_reverse_rows<float><<<pw_blocks(DL / 2), kPwThreads, 0, s>>>(Q, dh[n], L, DL / 2);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // rev(g_n) = h_n * rev(r_n)
    const void* hh1[1] = {hhat[n]};
    e = forward_dispatch(R, gate1, hh1, B, D, ly, 1, false, G, fws, pl.fws_bytes, false, s);
    if (e != cudaSuccess) return e;
  }
  bwd_reverse_rows<T><<<gp, kPwThreads, 0, s>>>(G, reinterpret_cast<T*>(dv), L, BDL / 2);
  return cudaGetLastError();
}

// ------------------------------------------------ filter-weight gradients --

constexpr int kFbTile = 32;
constexpr int kFbThreads = 256;
constexpr int kFbMinChunk = 256;   // taps per partial sum (at least)
constexpr int kFbMaxChunks = 64;

// Per tap t: E[t] = e(t), P1 = W1 e + b1, S1 = sin P1, P2 = W2 S1 + b2, S2 = sin P2.
__global__ void fb_activations(const float* __restrict__ W1, const float* __restrict__ b1,
                               const float* __restrict__ W2, const float* __restrict__ b2, int K, int H, int L,
                               float* __restrict__ E, float* __restrict__ P1, float* __restrict__ S1,
                               float* __restrict__ P2, float* __restrict__ S2) {
  extern __shared__ float fs[];
  const int Ed = 1 + 2 * K;
  float* e = fs;                    // [32][Ed]
  float* s1 = e + kFbTile * Ed;     // [32][H]
  const int t0 = blockIdx.x * kFbTile, tid = threadIdx.x;
  for (int idx = tid; idx < kFbTile * Ed; idx += blockDim.x) {
    const int tt = idx / Ed, i = idx % Ed, t = t0 + tt;
    float val = 0.f;
    if (t < L) {
      if (i == 0) {
        val = (float)t / (float)L;
      } else {
        const int k = (i <= K) ? i : i - K;
        const long long num = (2LL * k * t) % (2LL * L);
        float sn, cs;
        sincospif((float)num / (float)L, &sn, &cs);
        val = (i <= K) ? sn : cs;
      }
      E[(size_t)t * Ed + i] = val;
    }
    e[idx] = val;
  }
  __syncthreads();
  for (int idx = tid; idx < kFbTile * H; idx += blockDim.x) {
    const int tt = idx / H, o = idx % H, t = t0 + tt;
    float acc = __ldg(&b1[o]);
    for (int i = 0; i < Ed; ++i) acc = fmaf(__ldg(&W1[o * Ed + i]), e[tt * Ed + i], acc);
    const float sv = sinf(acc);
    s1[idx] = sv;
    if (t < L) {
      P1[(size_t)t * H + o] = acc;
      S1[(size_t)t * H + o] = sv;
    }
  }
  __syncthreads();
  for (int idx = tid; idx < kFbTile * H; idx += blockDim.x) {
    const int tt = idx / H, o = idx % H, t = t0 + tt;
    float acc = __ldg(&b2[o]);
    for (int i = 0; i < H; ++i) acc = fmaf(__ldg(&W2[o * H + i]), s1[tt * H + i], acc);
    if (t < L) {
      P2[(size_t)t * H + o] = acc;
      S2[(size_t)t * H + o] = sinf(acc);
    }
  }
}

// A(t, p) for the tap-contraction kernels: row-major [L][P], or the filter
// gradient dO(t, j) = dh[j][t] exp(-alpha_{j mod D} t / L) read from [P][L].
struct AOperand {
  const float* p;
  int P;
  bool dh_window;   // read as dh [P][L] times the window
  int D;
  float alpha_lo, alpha_hi;
  __device__ __forceinline__ float at(int t, int j, int L) const {
    if (!dh_window) return __ldg(p + (size_t)t * P + j);
    const int c = j % D;
    const float alpha = (D > 1) ? alpha_lo + (alpha_hi - alpha_lo) * (float)c / (float)(D - 1) : alpha_lo;
    return __ldg(p + (size_t)j * L + t) * expf(-alpha * ((float)t / (float)L));
  }
};

// Partial sums over one chunk of taps: part[chunk][p][q] = sum_t A(t,p) B[t][q]
// and bias[chunk][p] = sum_t A(t,p). Tiles of 32 p x 32 q x 32 t.
__global__ void __launch_bounds__(kFbThreads)
fb_tap_contract(AOperand A, const float* __restrict__ Bm, int Q, int L, int chunk_len, float* __restrict__ part,
                float* __restrict__ bias) {
  __shared__ float As[kFbTile][kFbTile + 1];
  __shared__ float Bs[kFbTile][kFbTile + 1];
  const int tid = threadIdx.x, pl = tid & 31, qb = (tid >> 5) * 4;
  const int p0 = blockIdx.x * kFbTile, q0 = blockIdx.y * kFbTile, chunk = blockIdx.z;
  const int tb = chunk * chunk_len, te = min(L, tb + chunk_len);
  float acc[4] = {0.f, 0.f, 0.f, 0.f}, bacc = 0.f;
  for (int t0 = tb; t0 < te; t0 += kFbTile) {
    for (int idx = tid; idx < kFbTile * kFbTile; idx += blockDim.x) {
      int tt, pp;
      if (A.dh_window) { pp = idx / kFbTile; tt = idx % kFbTile; }   // consecutive threads along t
      else { tt = idx / kFbTile; pp = idx % kFbTile; }
      const int t = t0 + tt, p = p0 + pp;
      As[tt][pp] = (t < te && p < A.P) ? A.at(t, p, L) : 0.f;
      const int q = q0 + (idx % kFbTile), tq = idx / kFbTile;
      Bs[tq][idx % kFbTile] = (t0 + tq < te && q < Q) ? __ldg(Bm + (size_t)(t0 + tq) * Q + q) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int tt = 0; tt < kFbTile; ++tt) {
      const float a = As[tt][pl];
      bacc += a;
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(a, Bs[tt][qb + i], acc[i]);
    }
    __syncthreads();
  }
  const int p = p0 + pl;
  if (p < A.P) {
    float* out = part + ((size_t)chunk * A.P + p) * Q;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (q0 + qb + i < Q) out[q0 + qb + i] = acc[i];
    if (blockIdx.y == 0 && qb == 0) bias[(size_t)chunk * A.P + p] = bacc;
  }
}

// out[i] = sum over chunks of part[chunk][i]
__global__ void fb_reduce(const float* __restrict__ part, size_t n, int chunks, float* __restrict__ out) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int c = 0; c < chunks; ++c) acc += part[(size_t)c * n + i];
    out[i] = acc;
  }
}

// out[t][q] = cos(Pre[t][q]) * sum_p A(t,p) W[p][q]   (W row-major [P][Q])
__global__ void __launch_bounds__(kFbThreads)
fb_back_layer(AOperand A, const float* __restrict__ W, int Q, int L, const float* __restrict__ Pre,
              float* __restrict__ out) {
  __shared__ float As[kFbTile][kFbTile + 1];   // [t][p]
  __shared__ float Ws[kFbTile][kFbTile + 1];   // [p][q]
  const int tid = threadIdx.x, ql = tid & 31, tb = (tid >> 5) * 4;
  const int t0 = blockIdx.x * kFbTile, q0 = blockIdx.y * kFbTile;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int p0 = 0; p0 < A.P; p0 += kFbTile) {
    for (int idx = tid; idx < kFbTile * kFbTile; idx += blockDim.x) {
      int tt, pp;
      if (A.dh_window) { pp = idx / kFbTile; tt = idx % kFbTile; }
      else { tt = idx / kFbTile; pp = idx % kFbTile; }
      const int t = t0 + tt, p = p0 + pp;
      As[tt][pp] = (t < L && p < A.P) ? A.at(t, p, L) : 0.f;
      const int pw = idx / kFbTile, qw = idx % kFbTile;
      Ws[pw][qw] = (p0 + pw < A.P && q0 + qw < Q) ? __ldg(W + (size_t)(p0 + pw) * Q + q0 + qw) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int pp = 0; pp < kFbTile; ++pp) {
      const float w = Ws[pp][ql];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(As[tb + i][pp], w, acc[i]);
    }
    __syncthreads();
  }
  const int q = q0 + ql;
  if (q < Q) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + tb + i;
      if (t < L) out[(size_t)t * Q + q] = acc[i] * cosf(__ldg(Pre + (size_t)t * Q + q));
    }
  }
}

struct FbPlan {
  size_t E, P1, S1, P2, S2, DP2, DP1, PART, BIAS, total;
  int chunks, chunk_len;
};

FbPlan plan_filter_backward(int N, int D, int L, int K, int H) {
  FbPlan p{};
  const int Ed = 1 + 2 * K;
  const size_t O = (size_t)N * D;
  p.chunk_len = kFbMinChunk;
  while ((L + p.chunk_len - 1) / p.chunk_len > kFbMaxChunks) p.chunk_len *= 2;
  p.chunks = (L + p.chunk_len - 1) / p.chunk_len;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += align256(bytes);
    return at;
  };
  p.E = take(sizeof(float) * (size_t)L * Ed);
  p.P1 = take(sizeof(float) * (size_t)L * H);
  p.S1 = take(sizeof(float) * (size_t)L * H);
  p.P2 = take(sizeof(float) * (size_t)L * H);
  p.S2 = take(sizeof(float) * (size_t)L * H);
  p.DP2 = take(sizeof(float) * (size_t)L * H);
  p.DP1 = take(sizeof(float) * (size_t)L * H);
  size_t pq = O * H;
  if ((size_t)H * H > pq) pq = (size_t)H * H;
  if ((size_t)H * Ed > pq) pq = (size_t)H * Ed;
  size_t pb = O > (size_t)H ? O : (size_t)H;
  p.PART = take(sizeof(float) * pq * p.chunks);
  p.BIAS = take(sizeof(float) * pb * p.chunks);
  p.total = o;
  return p;
}

}  // namespace

}  // namespace hyena

using namespace hyena;

namespace {
bool aligned16(const void* q) { return q && ((reinterpret_cast<uintptr_t>(q) & 15u) == 0); }
}  // namespace

extern "C" {

size_t hyena_backward_workspace_bytes(int B, int D, int L, int N, hyena_dtype dtype) {
  Layout ly;
  if (B < 1 || D < 1 || N < 1 || N > kMaxOrder || (dtype != HYENA_F32 && dtype != HYENA_BF16)) return 0;
  if (!make_layout(L, &ly)) return 0;
  if ((long long)B * D > (1LL << 40) / L) return 0;
  BwdPlan p;
  if (!plan_backward(B, D, N, ly, &p)) return 0;
  return p.total;
}

hyena_status hyena_backward(const void* v, const void* const* x, const void* const* hhat, const void* dy, int B,
                            int D, int L, int N, hyena_dtype dtype, void* dv, void* const* dx, float* const* dh,
                            void* workspace, size_t workspace_bytes, hyena_stream stream) {
  if (N < 1 || N > kMaxOrder || B < 1 || D < 1) return HYENA_ERR_INVALID_ARG;
  if (dtype != HYENA_F32 && dtype != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
  if (!x || !hhat || !dx || !dh || !aligned16(v) || !aligned16(dy) || !aligned16(dv)) return HYENA_ERR_INVALID_ARG;
  for (int n = 0; n < N; ++n)
    if (!aligned16(x[n]) || !aligned16(hhat[n]) || !aligned16(dx[n]) || !aligned16(dh[n]))
      return HYENA_ERR_INVALID_ARG;
  Layout ly;
  if (!make_layout(L, &ly)) return HYENA_ERR_UNSUPPORTED;
  if ((long long)B * D > (1LL << 40) / L) return HYENA_ERR_INVALID_ARG;
  BwdPlan pl;
  if (!plan_backward(B, D, N, ly, &pl)) return HYENA_ERR_INVALID_ARG;
  if (!aligned16(workspace) || workspace_bytes < pl.total) return HYENA_ERR_WORKSPACE;
  char* ws = reinterpret_cast<char*>(workspace);
  cudaStream_t s = (cudaStream_t)stream;
  const cudaError_t e =
      dtype == HYENA_BF16
          ? run_backward<__nv_bfloat16>(v, x, hhat, dy, B, D, ly, N, dv, dx, dh, ws, pl, s)
          : run_backward<float>(v, x, hhat, dy, B, D, ly, N, dv, dx, dh, ws, pl, s);
  return e == cudaSuccess ? HYENA_OK : report_cuda_error(e);
}

size_t hyena_filter_backward_workspace_bytes(int N, int D, int L, int n_bands, int width) {
  Layout ly;
  if (N < 1 || N > kMaxOrder || D < 1 || n_bands < 1 || n_bands > 32 || width < 1 || width > 128) return 0;
  if (!make_layout(L, &ly)) return 0;
  return plan_filter_backward(N, D, L, n_bands, width).total;
}

hyena_status hyena_filter_backward(const hyena_filter_params* p, int N, int D, int L, float alpha_lo,
                                   float alpha_hi, const float* dh, const hyena_filter_grads* g, void* workspace,
                                   size_t workspace_bytes, hyena_stream stream) {
  if (!p || !g || N < 1 || N > kMaxOrder || D < 1) return HYENA_ERR_INVALID_ARG;
  if (!p->W1 || !p->b1 || !p->W2 || !p->b2 || !p->W3 || !p->b3) return HYENA_ERR_INVALID_ARG;
  if (!g->W1 || !g->b1 || !g->W2 || !g->b2 || !g->W3 || !g->b3) return HYENA_ERR_INVALID_ARG;
  if (p->n_bands < 1 || p->n_bands > 32 || p->width < 1 || p->width > 128) return HYENA_ERR_INVALID_ARG;
  if (!aligned16(dh)) return HYENA_ERR_INVALID_ARG;
  if ((long long)N * D > (1LL << 24)) return HYENA_ERR_INVALID_ARG;
  Layout ly;
  if (!make_layout(L, &ly)) return HYENA_ERR_UNSUPPORTED;
  const int K = p->n_bands, H = p->width, Ed = 1 + 2 * K, O = N * D;
  const FbPlan pl = plan_filter_backward(N, D, L, K, H);
  if (!aligned16(workspace) || workspace_bytes < pl.total) return HYENA_ERR_WORKSPACE;
  char* ws = reinterpret_cast<char*>(workspace);
  float *E = reinterpret_cast<float*>(ws + pl.E), *P1 = reinterpret_cast<float*>(ws + pl.P1),
        *S1 = reinterpret_cast<float*>(ws + pl.S1), *P2 = reinterpret_cast<float*>(ws + pl.P2),
        *S2 = reinterpret_cast<float*>(ws + pl.S2), *DP2 = reinterpret_cast<float*>(ws + pl.DP2),
        *DP1 = reinterpret_cast<float*>(ws + pl.DP1), *part = reinterpret_cast<float*>(ws + pl.PART),
        *bias = reinterpret_cast<float*>(ws + pl.BIAS);
  cudaStream_t s = (cudaStream_t)stream;
  const int ct = (L + kFbTile - 1) / kFbTile;
  cudaError_t e;
  {
    const size_t smem = sizeof(float) * kFbTile * (Ed + H);
    fb_activations<<<ct, kFbThreads, smem, s>>>(p->W1, p->b1, p->W2, p->b2, K, H, L, E, P1, S1, P2, S2);
    if ((e = cudaGetLastError()) != cudaSuccess) return report_cuda_error(e);
  }
  auto contract = [&](AOperand A, const float* Bm, int Q, float* gW, float* gb) -> cudaError_t {
    dim3 grid((A.P + kFbTile - 1) / kFbTile, (Q + kFbTile - 1) / kFbTile, pl.chunks);
    fb_tap_contract<<<grid, kFbThreads, 0, s>>>(A, Bm, Q, L, pl.chunk_len, part, bias);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const size_t n = (size_t)A.P * Q;
    fb_reduce<<<pw_blocks(n), kPwThreads, 0, s>>>(part, n, pl.chunks, gW);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    fb_reduce<<<pw_blocks(A.P), kPwThreads, 0, s>>>(bias, (size_t)A.P, pl.chunks, gb);
    return cudaGetLastError();
  };
  const AOperand dO{dh, O, true, D, alpha_lo, alpha_hi};
  // last layer: dW3 = sum_t dO s2^T, db3 = sum_t dO
  if ((e = contract(dO, S2, H, g->W3, g->b3)) != cudaSuccess) return report_cuda_error(e);
  // dp2 = cos(P2) . (W3^T dO)
  {
    dim3 grid(ct, (H + kFbTile - 1) / kFbTile);
    fb_back_layer<<<grid, kFbThreads, 0, s>>>(dO, p->W3, H, L, P2, DP2);
    if ((e = cudaGetLastError()) != cudaSuccess) return report_cuda_error(e);
  }
  const AOperand dp2{DP2, H, false, 1, 0.f, 0.f};
  if ((e = contract(dp2, S1, H, g->W2, g->b2)) != cudaSuccess) return report_cuda_error(e);
  // dp1 = cos(P1) . (W2^T dp2)
  {
    dim3 grid(ct, (H + kFbTile - 1) / kFbTile);
    fb_back_layer<<<grid, kFbThreads, 0, s>>>(dp2, p->W2, H, L, P1, DP1);
    if ((e = cudaGetLastError()) != cudaSuccess) return report_cuda_error(e);
  }
  const AOperand dp1{DP1, H, false, 1, 0.f, 0.f};
  if ((e = contract(dp1, E, Ed, g->W1, g->b1)) != cudaSuccess) return report_cuda_error(e);
  return HYENA_OK;
}

}  // extern "C"
