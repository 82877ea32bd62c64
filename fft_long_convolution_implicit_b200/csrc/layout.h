// layout.h -- how a problem of length L is split, and where the library keeps
// its filter spectrum and FFT tables. Shared by host dispatch and kernels.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace hyena {

// Lengths up to this run the fused per-channel kernel (whole channel in shared
// memory); longer ones run the four-step decomposition through a workspace.
constexpr int kFusedMaxL = 16384;
constexpr int kMinM = 128;          // smallest internal transform (zero-extended below)
constexpr int kMaxL = 1 << 20;
constexpr int kFourStepMaxMV = 4096;
constexpr int kFourStepRowMV = 1024;   // preferred row length (measured fastest at L = 2^17)
constexpr int kFourStepMinM1 = 16;
constexpr int kFourStepMaxM1 = 256;    // columns: radix 16 x (M1 / 16) with M1 / 16 <= 16

struct Layout {
  int L;        // caller's length
  int M;        // packed complex points per channel (real length of the causal problem)
  int M1;       // four-step column length (1 for the fused path)
  int MV;       // row length, M = M1 * MV
  int logMV;
  int mb;       // M1 / 16 for the four-step path (radix of the second column pass)
  bool fourstep;
  // table region (float2 offsets from its start)
  int tw_v;     // MV-point plan twiddles (MV entries)
  int w_v;      // w_{2 MV}^k, k < MV
  int tw_1;     // M1-point column plan twiddles (M1 entries, four-step only)
  // tensor-core paths (bf16, pairs of batch items): mma.sync kernel with
  // 2L = R0 * 256 (tc), or tcgen05 GEMM levels 2L = 16 * 32 * 32 (tcg)
  bool tc;
  bool tcg;
  int R0;
  int tc_otw;   // outer twiddles w_{2L}^{m k0}, [k0 = 1..R0-1][m < 256] (R0 * 256 entries)
  int table_len;
};

// Lengths with a tensor-core forward (outer radix R0 = L / 128 in {8, 16}).
constexpr int kTcMinL = 1024;
constexpr int kTcMaxL = 2048;
// Length of the tcgen05 GEMM-level forward, and the highest order it serves:
// its f16 operands add an error that compounds through the gates, within the
// bf16 tolerance up to order 3 (float64 model of its scalings: 3.1e-3 at order
// 3, 6.1e-3 at order 4 and 1.3e-2 at order 8 on seeded N(0,1) gates).
constexpr int kTcgL = 8192;
constexpr int kTcgMaxOrder = 3;

inline int ilog2_exact(int v) {
  int l = 0;
  while ((1 << l) < v) ++l;
  return ((1 << l) == v) ? l : -1;
}

// Returns false when L is not supported (not a power of two in [16, 2^20]).
inline bool make_layout(int L, Layout* out) {
  if (L < 16 || L > kMaxL) return false;
  if (ilog2_exact(L) < 0) return false;
  Layout y{};
  y.L = L;
  if (L <= kFusedMaxL) {
    y.M = L < kMinM ? kMinM : L;
    y.M1 = 1;
    y.MV = y.M;
    y.fourstep = false;
    y.mb = 0;
  } else {
    y.M = L;
    // rows of 1024 points while the columns stay within 256 points; longer
    // transforms use rows of 4096 points
    y.M1 = L / kFourStepRowMV;
    if (y.M1 > kFourStepMaxM1) y.M1 = L / kFourStepMaxMV;
    if (y.M1 < kFourStepMinM1) y.M1 = kFourStepMinM1;
    y.MV = L / y.M1;
    y.fourstep = true;
    y.mb = y.M1 / 16;
  }
  y.logMV = ilog2_exact(y.MV);
  y.tw_v = 0;
  y.w_v = y.MV;
  y.tw_1 = 2 * y.MV;
  y.table_len = 2 * y.MV + (y.fourstep ? y.M1 : 0);
  y.tc = (L >= kTcMinL && L <= kTcMaxL);
  y.tcg = (L == kTcgL);
  y.R0 = y.tc ? L / 128 : 0;
  y.tc_otw = y.table_len;
  if (y.tc) y.table_len += y.R0 * 256;
  y.table_len = (y.table_len + 1) & ~1;   // keep the block a multiple of 16 bytes
  *out = y;
  return true;
}

// One filter's spectrum block: [D][M] float2 spectrum (library order); for
// tensor-core lengths a second copy [D][L + 2] float2 in the kernel's order;
// then the table region.
// tensor-core copy rows: L float2 bins (mma.sync kernel) or 2L f16x2 bins
// (tcgen05 kernel), then the channel's 1 / f_c and padding (16 bytes)
inline int tc_row(const Layout& y) { return y.L + 2; }
inline bool has_tc_copy(const Layout& y) { return y.tc || y.tcg; }
inline size_t tc_spectrum_offset(const Layout& y, int D) { return (size_t)D * y.M; }
inline size_t tables_offset(const Layout& y, int D) {
  return (size_t)D * y.M + (has_tc_copy(y) ? (size_t)D * tc_row(y) : 0);
}
// Four-step layouts with rows of 4096 points may run their row pass on the
// tensor cores; their spectrum block ends with each channel's largest
// spectrum component ([D] float, padded to 16 bytes) and an f16 copy of the
// spectrum ([D][M] __half2 in the same bin order, channel c times the power
// of two f_c that puts its largest component in [2^14, 2^15)), whose rows the
// row pass stages in shared memory. Their workspace holds two words per
// channel beside the scratch (the column pass's per-channel maxima).
inline bool tcr_layout(const Layout& y) { return y.fourstep && y.logMV == 12; }
inline size_t hmax_offset(const Layout& y, int D) { return tables_offset(y, D) + y.table_len; }
inline size_t tcr_half_offset(const Layout& y, int D) { return hmax_offset(y, D) + ((size_t)D + 3) / 4 * 2; }
inline size_t spectrum_block_floats2(const Layout& y, int D) {
  return tcr_layout(y) ? tcr_half_offset(y, D) + (size_t)D * y.M / 2 : hmax_offset(y, D);
}
constexpr size_t kTcrChannelExtraBytes = 8;

// Reduced-precision spectrum block: [D][M] __half2 bins (same order, each
// channel scaled by a power of two), [D] float 1 / scale (padded to 16 bytes),
// then the same table region as the float32 block.
inline size_t spec16_scales_offset_bytes(const Layout& y, int D) { return (size_t)4 * D * y.M; }
inline size_t spec16_tables_offset_bytes(const Layout& y, int D) {
  return ((size_t)4 * D * y.M + (size_t)4 * D + 15) & ~(size_t)15;
}
inline size_t spec16_block_bytes(const Layout& y, int D) { return spec16_tables_offset_bytes(y, D) + 8 * (size_t)y.table_len; }

}  // namespace hyena
