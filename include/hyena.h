/*
 * hyena.h -- C ABI of the B200 (sm_100a) Hyena order-N forward/backward library.
 *
 * The operator (order-N recurrence; "Hyena Hierarchy - Towards Larger
 * Convolutional Language Models" digest, section 방법 (Method) / 프레임워크
 * 개요, and the explainer "Hyena Hierarchy: Towards Larger Convolutional
 * Language Models", section Hyena 演算子の形):
 *
 *     z_1 = v,   z_{n+1} = x_n (.) (h_n * z_n),   y = z_{N+1},   n = 1..N
 *
 * where (.) is the elementwise product and * the causal long convolution
 * (h * z)_t = sum_{s=0..t} h_{t-s} z_s ("02. 3つの Hyena 演算子", section 4,
 * the FIR sum), evaluated by FFT on a 2L zero-padded grid (glossary
 * "Hyena（ハイエナ）", section 計算効率; "Native Multi-Dimensional Subquadratic
 * Operators via Input Dependent Long Convolutions", section 境界の処理).
 * The filters are implicit (glossary "Hyena（ハイエナ）", section
 * 暗黙的畳み込みフィルタ: h(t) = Window(t) FFN(t/L, sin, cos)).
 *
 * Conventions for every call:
 *  - Every pointer named "device" is CUDA device memory of the current
 *    device, 16-byte aligned; the caller owns it. The library never
 *    allocates device memory and keeps no state between calls, apart from
 *    the static scratch of hyena_forward_static_workspace and the sticky
 *    timeout flag that hyena_device_timeouts reads and clears.
 *  - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream). Inputs must stay valid until the work on
 *    the stream has finished.
 *  - Arguments are checked on the host before anything is launched; a
 *    rejected call launches nothing. HYENA_ERR_CUDA reports a launch error
 *    (see hyena_last_cuda_error()).
 *  - Activations v, x_n, y are row-major [B][D][L] (time fastest) in the
 *    storage type `dtype`; bf16 results are rounded to nearest even. The
 *    arithmetic is float32, except that hyena_forward with bf16 I/O and B
 *    even runs its transforms on the tensor cores with f16 operands (scaled
 *    by exact powers of two) and float32 accumulation for L in {1024, 2048}
 *    and, up to order N = 3, for L = 8192; that adds an error of the order of
 *    the bf16 output rounding (relative L2 within the bf16 tolerance of 8e-3).
 *  - For the 1-D FFT calls L must be a power of two with 16 <= L <= 2^20
 *    (HYENA_ERR_UNSUPPORTED otherwise); 1 <= N <= 8; B, D >= 1. The
 *    StripedHyena calls take any L >= 1 and the HyenaND calls state their
 *    own grid rules.
 *  - All entry points may be called from several host threads at once, with
 *    one exception: calls of hyena_forward_static_workspace share one device
 *    scratch array, so two of them whose GPU work overlaps race (see there).
 */
#ifndef HYENA_B200_H
#define HYENA_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HYENA_ABI_VERSION 2

typedef enum {
  HYENA_OK = 0,
  HYENA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad count or dtype */
  HYENA_ERR_UNSUPPORTED = 2,   /* shape outside what the call supports (e.g. L not a power of two in [16, 2^20]) */
  HYENA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
  HYENA_ERR_CUDA = 4,          /* a CUDA launch or attribute call failed */
  HYENA_ERR_TIMEOUT = 5        /* a bounded device-side wait ran out (see hyena_device_timeouts) */
} hyena_status;

typedef enum { HYENA_F32 = 0, HYENA_BF16 = 1 } hyena_dtype;

typedef void *hyena_stream; /* cudaStream_t */

/*
 * Weights of the implicit-filter FFN, device float32, row-major [out][in]:
 *   W1 [width][1 + 2 n_bands], b1 [width]
 *   W2 [width][width],          b2 [width]
 *   W3 [N*D][width],            b3 [N*D]
 * n_bands in [1, 32], width in [1, 128].
 */
typedef struct {
  const float *W1, *b1, *W2, *b2, *W3, *b3;
  int n_bands;
  int width;
} hyena_filter_params;

/*
 * hyena_filter_generate -- implicit filters h_1..h_N.
 * Glossary "Hyena（ハイエナ）", section 暗黙的畳み込みフィルタ; the workload
 * recipe fixes the details:
 *   e(t) = [t/L, sin(2 pi k t/L) for k = 1..K, cos(2 pi k t/L) for k = 1..K]
 *   s1 = sin(W1 e + b1), s2 = sin(W2 s1 + b2), o = W3 s2 + b3
 *   h[n][c][t] = o[n*D + c] * exp(-alpha_c t / L),
 *   alpha_c = alpha_lo + (alpha_hi - alpha_lo) c / (D - 1)   (alpha_lo if D = 1)
 * Output h: device float32 [N][D][L]. Returns HYENA_ERR_UNSUPPORTED for an
 * unsupported L.
 */
hyena_status hyena_filter_generate(const hyena_filter_params *p, int N, int D, int L, float alpha_lo,
                                   float alpha_hi, float *h, hyena_stream stream);

/*
 * Bytes of one filter's spectrum block for D channels and length L: the
 * spectrum in library order plus the FFT tables the forward reads, and the
 * kernel-specific copies of the tensor-core paths (L = 1024, 2048, 8192: a
 * copy in the kernel's bin order; L = 2^19 and 2^20: each channel's largest
 * spectrum component, [D] float padded to 16 bytes, then an f16 copy of the
 * spectrum, [D][L] __half2 at the end of the block). 0 when L is unsupported
 * or D < 1.
 */
size_t hyena_filter_spectrum_bytes(int D, int L);

/*
 * hyena_filter_rfft -- cache the spectrum of ONE filter (D channels):
 *   H_c[k] = sum_{t<L} h_c[t] exp(-2 pi i k t / 2L) / (4 M),  k = 0..M,
 * with M = max(L, 128) (rfft of the filter zero-padded to the 2L grid; the
 * 1/(4M) folds the inverse transform's scale). Input h: device float32
 * [D][L] (for example h + n*D*L from hyena_filter_generate). Output hhat:
 * device block of hyena_filter_spectrum_bytes(D, L) bytes, library order
 * (see hyena_spectrum_layout). Call once per filter n; reuse for every
 * forward with the same weights.
 */
hyena_status hyena_filter_rfft(const float *h, int D, int L, void *hhat, hyena_stream stream);

/*
 * Describe the library order of a spectrum block (for inspection and tests):
 * *M = points per channel, bin k < M of channel c sits at float2 index
 * c*M + (k mod M1)*MV + (k / M1); bin 0 holds (Re H[0], Re H[M]). Returns
 * HYENA_ERR_UNSUPPORTED for an unsupported L.
 */
hyena_status hyena_spectrum_layout(int L, int *M, int *M1, int *MV);

/*
 * Workspace bytes hyena_forward wants for this shape: 0 for L <= 16384 (the
 * fused kernel keeps everything on chip); for longer L, 8*L bytes per
 * channel (8*L + 8 when L is 2^19 or 2^20) for a wave of channels: sized to
 * stay resident in L2 (5/8 of the current device's L2 capacity) where the
 * row pass runs on the tensor cores (bf16, N <= 3, L = 2^19 or 2^20), else
 * all channels up to 1 GiB (the SIMT row kernels are faster in fewer, larger
 * waves). Any workspace of at least one channel's bytes works (smaller
 * waves); 0 when the shape is invalid.
 */
size_t hyena_forward_workspace_bytes(int B, int D, int L, int N, hyena_dtype dtype);

/*
 * hyena_forward -- y = z_{N+1} of the order-N recurrence.
 *   v:    device [B][D][L] dtype
 *   x:    host array of N device pointers, x[n] = gate x_{n+1}, [B][D][L] dtype
 *   hhat: host array of N device pointers to spectrum blocks from
 *         hyena_filter_rfft (D channels, the same L)
 *   y:    device [B][D][L] dtype; may alias v or any x[n] (each element is
 *         read before the same thread block writes it)
 *   workspace: device scratch of workspace_bytes (>= 8*L when L > 16384;
 *         ignored otherwise, may be NULL)
 */
hyena_status hyena_forward(const void *v, const void *const *x, const void *const *hhat, int B, int D, int L,
                           int N, hyena_dtype dtype, void *y, void *workspace, size_t workspace_bytes,
                           hyena_stream stream);

/*
 * hyena_forward_static_workspace -- hyena_forward for callers that cannot
 * allocate device memory (no counterpart on the pages: it is a deployment
 * convenience, not part of the method).
 *
 * Some callers may not call cudaMalloc at run time: runtimes that own the
 * whole device through their own pool allocator and forbid allocations
 * behind its back, fixed-budget deployments, and latency-critical paths that
 * cannot afford cudaMalloc's implicit device synchronisation. This entry point
 * needs no workspace argument: the four-step scratch lives in a file-scope
 * device array of HYENA_STATIC_WORKSPACE_BYTES inside the library. It
 * allocates nothing and calls no allocating routine itself; the array is
 * reserved when the library module that holds it is loaded into a CUDA
 * context -- with CUDA's default lazy module loading, that is the first call
 * of this entry point in the context (make one warm-up call outside any
 * phase that must not reserve memory) -- and held until the process exits.
 * A call rejected by the host-side checks loads nothing.
 *
 *  - Only for 16384 < L <= 2^20 (the lengths whose forward needs scratch);
 *    shorter L returns HYENA_ERR_UNSUPPORTED: use hyena_forward with a NULL
 *    workspace there, which already allocates nothing.
 *  - Channels are processed in waves of HYENA_STATIC_WORKSPACE_BYTES / (8 L);
 *    a length whose single channel would not fit is rejected with
 *    HYENA_ERR_WORKSPACE (never the case for supported L).
 *  - The first call in a CUDA context looks up the array's device address
 *    (cudaGetSymbolAddress) with that context current and caches it under
 *    the context's unique id; make that first call before any stream capture
 *    in the context. A context destroyed and re-created (cudaDeviceReset, or
 *    a different context made current) is looked up afresh.
 *  - Every call on a device shares the one array and leaves its last
 *    contents there (nothing needs clearing: every element is written before
 *    it is read). Calls whose GPU work overlaps -- on different streams, or
 *    from different threads -- race on the array: order them on one stream
 *    or otherwise serialise them.
 * Other arguments, layouts and errors are those of hyena_forward.
 */
#define HYENA_STATIC_WORKSPACE_BYTES ((size_t)16 << 20)
hyena_status hyena_forward_static_workspace(const void *v, const void *const *x, const void *const *hhat, int B,
                                            int D, int L, int N, hyena_dtype dtype, void *y, hyena_stream stream);

/*
 * Reduced-precision filter spectra (no counterpart on the pages, which fix
 * no precision for the cached spectrum: page "Hyena Hierarchy: Towards
 * Larger Convolutional Language Models", section 計算方法, only states that
 * the long convolution runs through the FFT). The forward reads the spectrum of every
 * filter once per channel, and at D*L of that size the float32 spectrum is
 * the largest stream of a step; the f16 block halves it.
 *
 * Block of hyena_filter_spectrum_bytes_f16(D, L) bytes (0 when L is
 * unsupported or D < 1):
 *   [0, 4*D*M)            bins of the float32 block, same library order, as
 *                         f16 pairs (re, im) scaled by s_c
 *   [4*D*M, 4*D*M + 4*D)  1/s_c per channel, float32
 *   (rounded up to 16 bytes) the float32 block's FFT tables, copied
 * s_c is the power of two that brings every component of channel c below
 * 2^15 in magnitude (1 for an all-zero channel), so scaling adds no error:
 * each bin carries f16 rounding only (relative 2^-11 of the channel's
 * largest component, or f16 subnormal spacing for bins more than 2^-24
 * below it).
 */
size_t hyena_filter_spectrum_bytes_f16(int D, int L);

/*
 * hyena_filter_spectrum_to_f16 -- convert one float32 spectrum block
 * (from hyena_filter_rfft, D channels, length L) into an f16 block.
 *   hhat:   device, hyena_filter_spectrum_bytes(D, L) bytes, 16-byte aligned
 *   hhat16: device, hyena_filter_spectrum_bytes_f16(D, L) bytes, 16-byte
 *           aligned, must not overlap hhat
 * Errors: HYENA_ERR_INVALID_ARG (alignment, D < 1), HYENA_ERR_UNSUPPORTED (L),
 * HYENA_ERR_CUDA (launch). Asynchronous on stream.
 */
hyena_status hyena_filter_spectrum_to_f16(const void *hhat, int D, int L, void *hhat16, hyena_stream stream);

/*
 * hyena_forward_f16_spectra -- hyena_forward whose hhat[n] are f16 blocks
 * from hyena_filter_spectrum_to_f16, for bf16 I/O only: dtype HYENA_F32
 * returns HYENA_ERR_UNSUPPORTED, because the f16 rounding of the spectra
 * (relative L2 up to 2^-11 per stage) is far above the float32 accuracy
 * that f32 I/O stands for, while it stays below the bf16 output rounding
 * (2^-9). Other arguments, layouts, aliasing, workspace and errors are those
 * of hyena_forward. It always runs the SIMT kernels (the tensor-core
 * forward reads a float32 copy of its own).
 */
hyena_status hyena_forward_f16_spectra(const void *v, const void *const *x, const void *const *hhat16, int B, int D,
                                       int L, int N, hyena_dtype dtype, void *y, void *workspace,
                                       size_t workspace_bytes, hyena_stream stream);

/*
 * Gradients (no counterpart printed on the pages, which only mention training
 * at 1M tokens: glossary "Hyena（ハイエナ）", section 超長系列タスクでの優位性). They are the chain
 * rule through the definitions above:
 *   u_n = h_n * z_n,  z_{n+1} = x_n (.) u_n,  g_{N+1} = dy,  r_n = g_{n+1} (.) x_n
 *   dx_n       = g_{n+1} (.) u_n
 *   g_n[s]     = sum_{t>=s} h_n[t-s] r_n[t]             (transpose of the causal sum)
 *   dh_n[c][j] = sum_b sum_{t>=j} r_n[b][c][t] z_n[b][c][t-j]
 *   dv         = g_1
 * Both correlations are causal convolutions of time-reversed rows and run on
 * the forward's 2L-grid FFT kernels in float32.
 */

/* Workspace bytes hyena_backward needs for this shape (0 when invalid):
 * about (N + 5) * 4 * B*D*L + 24 * B*D*L + 8 * D*L bytes. */
size_t hyena_backward_workspace_bytes(int B, int D, int L, int N, hyena_dtype dtype);

/*
 * hyena_backward -- dv, dx_n and dh_n for the loss gradient dy = dL/dy of
 * y = hyena_forward(v, x, hhat).
 *   v, x, hhat, B, D, L, N, dtype: exactly as given to hyena_forward
 *   dy:  device [B][D][L] dtype
 *   dv:  device [B][D][L] dtype
 *   dx:  host array of N device pointers, dx[n] = dL/dx_{n+1}, [B][D][L] dtype
 *   dh:  host array of N device pointers, dh[n] = dL/dh_{n+1}, float32 [D][L]
 *        (time-domain filter gradient, summed over the batch; the layout of
 *        hyena_filter_generate's output, so dh[n] may point at h_grad + n*D*L)
 *   workspace: device scratch of at least hyena_backward_workspace_bytes()
 *        (HYENA_ERR_WORKSPACE otherwise). Outputs must not alias inputs or
 *        the workspace.
 */
hyena_status hyena_backward(const void *v, const void *const *x, const void *const *hhat, const void *dy, int B,
                            int D, int L, int N, hyena_dtype dtype, void *dv, void *const *dx, float *const *dh,
                            void *workspace, size_t workspace_bytes, hyena_stream stream);

/* Gradients of the implicit-filter weights: device float32 arrays shaped
 * like the fields of hyena_filter_params; every element is overwritten. */
typedef struct {
  float *W1, *b1, *W2, *b2, *W3, *b3;
} hyena_filter_grads;

/* Workspace bytes hyena_filter_backward needs (0 when invalid). */
size_t hyena_filter_backward_workspace_bytes(int N, int D, int L, int n_bands, int width);

/*
 * hyena_filter_backward -- gradients of sum_{n,c,t} dh[n][c][t] h[n][c][t]
 * with respect to the FFN weights of hyena_filter_generate, by the chain rule
 * through h = window (W3 s2 + b3), s2 = sin(W2 s1 + b2), s1 = sin(W1 e + b1):
 *   dO = dh * window;  dW3 = sum_t dO s2^T,  db3 = sum_t dO
 *   dp2 = cos(W2 s1 + b2) (.) W3^T dO;  dW2 = sum_t dp2 s1^T,  db2 = sum_t dp2
 *   dp1 = cos(W1 e + b1) (.) W2^T dp2;  dW1 = sum_t dp1 e^T,   db1 = sum_t dp1
 * dh: device float32 [N][D][L] (e.g. hyena_backward's dh outputs laid end to
 * end). Sums over taps run in float32 in fixed chunks (deterministic).
 */
hyena_status hyena_filter_backward(const hyena_filter_params *p, int N, int D, int L, float alpha_lo,
                                   float alpha_hi, const float *dh, const hyena_filter_grads *g, void *workspace,
                                   size_t workspace_bytes, hyena_stream stream);

/* Static description of a status code. */
const char *hyena_status_string(hyena_status s);

/* Text of the last CUDA error seen by this thread inside the library ("" if none). */
const char *hyena_last_cuda_error(void);

/*
 * StripedHyena-form operator ("02. 3つの Hyena 演算子", section 2, the operator
 * structure; section 3, the SE / MR / LI variants; section 4, the FIR sum
 * y_t = sum_{k < l_h} h_k x_{t-k}):
 *   q = hT * xq,  k = hH * xk,  v = hK * xv     (short explicit featurizers)
 *   y = q (.) (hG * (k (.) v))
 * where * is the causal FIR sum (zero before t = 0). xq, xk, xv are the
 * outputs of the operator's dense input projections (not part of this call).
 *   xq, xk, xv, y: device [B][D][L] dtype, y not aliasing an input
 *   hT, hH, hK:    device float32 [D][lf], 1 <= lf <= 16
 *   hG:            device float32 [D][lg], 1 <= lg <= 1024 (SE: a few taps;
 *                  MR: hundreds, e.g. an explicit filter times a decay)
 * Any L >= 1. Arithmetic in float32; bf16 results rounded to nearest even.
 * Every pointer must be 16-byte aligned. Errors: HYENA_ERR_INVALID_ARG
 * (alignment, lf, lg, B, D or L out of range, B*D*L above 2^40),
 * HYENA_ERR_CUDA (launch). Asynchronous on stream.
 */
hyena_status hyena_striped_forward(const void *xq, const void *xk, const void *xv, const float *hT, const float *hH,
                                   const float *hK, int lf, const float *hG, int lg, int B, int D, int L,
                                   hyena_dtype dtype, void *y, hyena_stream stream);

/*
 * The featurizer half of the operator for a long implicit inner filter
 * (Hyena-LI): q = hT * xq and u = (hH * xk) (.) (hK * xv), device [B][D][L]
 * dtype. The operator is then y = hyena_forward(u, {q}, {hyena_filter_rfft(hG)},
 * N = 1). Arguments, alignment and errors as in hyena_striped_forward; q and u
 * must not alias the inputs.
 */
hyena_status hyena_striped_featurize(const void *xq, const void *xk, const void *xv, const float *hT,
                                     const float *hH, const float *hK, int lf, int B, int D, int L,
                                     hyena_dtype dtype, void *q, void *u, hyena_stream stream);

/*
 * Hyena-LI filter ("02. 3つの Hyena 演算子", section 3): a sum of real
 * exponentials, h[c][t] = sum_{n < d} R[c][n] lambda[c][n]^t for t < L (the
 * page's exponent t - 1 with 1-based t). R, lambda: device float32 [D][d],
 * 1 <= d <= 64; h: device float32 [D][L]. Pointers 16-byte aligned.
 * Errors: HYENA_ERR_INVALID_ARG (alignment, d, D, L), HYENA_ERR_CUDA.
 */
hyena_status hyena_filter_exponential(const float *R, const float *lambda, int d, int D, int L, float *h,
                                      hyena_stream stream);

/*
 * Kernels that wait on mbarriers for asynchronous copies or tensor-core
 * completions (the striped bulk-copy kernel of hyena_striped_forward, taken
 * when a row's byte length is a multiple of 16; in hyena_forward the tcgen05
 * kernel for bf16, B even, L = 8192, N <= 3, and the four-step row passes,
 * whose spectrum rows arrive by bulk copies: rows of 1024 points, and the
 * tcgen05 rows of 4096 points for bf16, N <= 3, L = 2^19 and 2^20) bound every
 * wait in time: a wait gives up 0.2 s of GPU global time after it started
 * (each polling step suspends for at most 20 us). A wait that runs out sets a
 * sticky flag on the current device and the outputs of that launch are then
 * invalid; the block waits at most 1 s more for the copies or tensor-core
 * work it still has in flight, then stops early (the striped and tcgen05
 * kernels) or finishes its item (the rows of 1024) and exits.
 * This call synchronises with the device, reads and clears the flag:
 * HYENA_OK if no wait ran out since the last call, HYENA_ERR_TIMEOUT
 * otherwise (HYENA_ERR_CUDA if it cannot be read).
 */
hyena_status hyena_device_timeouts(void);

/*
 * HyenaND (page "Native Multi-Dimensional Subquadratic Operators via Input
 * Dependent Long Convolutions", section 手法: a global convolution evaluated on
 * the L_1 x ... x L_nd grid through an nd-dimensional FFT; circular for
 * periodic data, or with the input zero-padded to twice the grid so that
 * nothing leaks across the boundary). The order-N recurrence of
 * hyena_forward with the causal 1-D sum replaced by
 *   boundary HYENA_ND_CIRCULAR: (K conv z)[p] = sum_q K[(p - q) mod dims] z[q]
 *   boundary HYENA_ND_ZERO:     (K conv z)[p] = sum_{0 <= q <= p} K[p - q] z[q]
 *                               (componentwise q <= p: the linear convolution
 *                               of the two grid signals, kept on the grid)
 * K_n are given as values on the grid (offset 0 at index 0); how they are
 * generated (the summary's SIREN/FiLM kernel and Gaussian window) is up to
 * the caller.
 *
 * Shapes: nd in 1..3, dims[a] powers of two (host array of nd ints, row-major
 * grid, axis nd-1 contiguous); padded axis P_a = 2 dims[a] (zero) or dims[a]
 * (circular) at most 1024, and P = prod P_a at most 16384. Others return
 * HYENA_ERR_UNSUPPORTED (0 bytes from hyena_nd_spectrum_bytes).
 */
#define HYENA_ND_ZERO 0
#define HYENA_ND_CIRCULAR 1

/* Bytes of one filter's spectrum block: [D][P] float2 then a twiddle table. */
size_t hyena_nd_spectrum_bytes(int D, int nd, const int *dims, int boundary);

/*
 * hyena_nd_filter_spectrum -- cache the spectrum of ONE filter:
 *   K:    device float32 [D][grid] (16-byte aligned)
 *   khat: device block of hyena_nd_spectrum_bytes(D, nd, dims, boundary)
 *         bytes (16-byte aligned): the padded-grid DFT of K_c times 1/P in
 *         the library's transform order (each axis index bit-reversed), then
 *         the twiddle table the forward reads.
 * Errors: HYENA_ERR_INVALID_ARG (pointers, D), HYENA_ERR_UNSUPPORTED (shape),
 * HYENA_ERR_CUDA (launch). Asynchronous on stream.
 */
hyena_status hyena_nd_filter_spectrum(const float *K, int D, int nd, const int *dims, int boundary, void *khat,
                                      hyena_stream stream);

/*
 * hyena_nd_forward -- y = z_{N+1} of the recurrence above.
 *   v, x[n], y: device [B][D][grid] in dtype (16-byte aligned); x is a host
 *         array of N device pointers; y may alias v or any x[n]
 *   khat: host array of N device pointers to blocks from
 *         hyena_nd_filter_spectrum (same D, nd, dims, boundary)
 * No workspace: every stage stays on chip. Errors as hyena_forward.
 */
hyena_status hyena_nd_forward(const void *v, const void *const *x, const void *const *khat, int B, int D, int nd,
                              const int *dims, int boundary, int N, hyena_dtype dtype, void *y, hyena_stream stream);

/* HYENA_ABI_VERSION of the loaded library. */
int hyena_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HYENA_B200_H */
