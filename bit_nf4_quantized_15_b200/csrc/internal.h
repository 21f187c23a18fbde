// Internal declarations shared by the kernels and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace qnf4 {

// NF4 codebook and decision thresholds as the kernels use them.
//   q[i] : the 16 levels (fp32), ascending, q[7] = 0 exactly.
//   t[i] : RD32 of the exact midpoint (q[i] + q[i+1]) / 2; for an fp32 x,
//          x > midpoint  <=>  x > t[i].
struct Nf4Tables {
  float q[16];
  float t[15];
  // Code search used by the quantiser: a degree-5 polynomial f(x) with
  // f(t[i]) in [i + 0.1, i + 0.9], f(-1) >= 0.1, f(1) <= 14.9 and f increasing
  // on [-1, 1], so that k = round(f(x) - 1/2) is the code of x or one less and
  // code = k + (x > t[k]).  poly[0] already includes the -1/2.
  float poly[6];
  bool poly_ok;  // the conditions above were verified when the tables were built
};

// Derived once per process on the host, from the normal quantiles.
const Nf4Tables& nf4_tables();

// Code formats (QLORA_FMT_*): NF4, and the two formats the method is
// compared with, FP4 (E2M1 / 6) and Int4 (k / 7), each with a pad level
// below -1 that is never produced.  Same table layout; only NF4 has a
// code-search polynomial (poly_ok is false for the others, whose quantiser
// searches the thresholds).
constexpr int kNumFormats = 3;
const Nf4Tables& code_tables(int format);  // format in [0, kNumFormats)

// Process-wide count of kernels launched through the library.
void count_launches(uint64_t n);
uint64_t launches_so_far();

// ------------------------------------------------------------------ engine
// Where the UMMA A operand of the main segment comes from.
enum AMode : int {
  A_TMA = 0,     // TMA tile (K- or MN-major per args)
  A_DEQ_K = 1,   // NF4 dequantised on chip, K-major  (A = W^, rows = n, k along K)
  A_DEQ_MN = 2,  // NF4 dequantised on chip, MN-major (A = W^T, rows = k, reduction over n)
};

// Final store of an accumulator element (row, col) of the output tile:
//   out [row*rs  + col*cs ] = alpha  * v   (fp32 or bf16)
//   out2[row*rs2 + col*cs2] = alpha2 * v   (bf16, optional)
struct EpiArgs {
  void* out;
  int out_bf16;
  float alpha;
  int64_t rs, cs;
  void* out2;
  float alpha2;
  int64_t rs2, cs2;
};

struct EngineArgs {
  CUtensorMap tmA;   // main A (A_TMA) or the NF4 code tensor (A_DEQ_*)
  CUtensorMap tmB;   // main B
  CUtensorMap tmAx;  // extension A (LoRA term)
  CUtensorMap tmBx;  // extension B
  const uint8_t* codes;  // NF4 codes [wN][wK/2] (read directly by the pair forward)
  const uint8_t* c2;
  int c2_e5m2;           // c2 holds E5M2 codes instead of E4M3
  int c1_mean;           // mean-centred codec: c1 holds [c1, mean] per group
  const float* c1;
  int64_t wN, wK;    // quantised weight shape (for scale indexing)
  int rows, cols;    // output extent: UMMA-M side, UMMA-N side
  int kb_main;       // 64-wide reduction blocks of the main segment
  int kb_ext;        // 64-wide reduction blocks of the extension (0: none)
  int splits;        // split of the main reduction across grid.z
  int a_mn_main, b_mn_main, a_mn_ext, b_mn_ext;
  float* partial;    // [splits][cols][rows] fp32 when splits > 1
  EpiArgs epi;
  int* status;
  uint64_t wait_ns;  // bound of every internal wait (0: the default, 4 s)
  int stall;         // failure-detection hook: the producer issues no loads
  float q[16];
};

struct GemmPlan {
  int BN;
  int m_tiles, n_tiles, splits;
  size_t partial_bytes;
};

GemmPlan plan_gemm(int rows, int cols, int kb_main, int num_sms);
size_t engine_smem_bytes(int BN, int amode);
cudaError_t launch_engine(const EngineArgs& a, int amode, const GemmPlan& p, cudaStream_t st);
cudaError_t launch_split_reduce(const float* partial, int splits, int rows, int cols, const EpiArgs& e,
                                cudaStream_t st);

// Forward dequant-GEMM on CTA pairs (cta_group::2, 256 x 256 output tile per
// pair).  Same EngineArgs as A_DEQ_K with these tensor maps: tmA codes (box
// 32 x 128 bytes), tmB X (K-major, box 64 x 128), tmAx L2 (MN-major, 64 x 64),
// tmBx RNbf16(s.T) (K-major, box 64 x 128); bf16 output, no split.
bool pair_fwd_supported(int rows, int cols, int kb_ext);
size_t pair_fwd_smem_bytes();
cudaError_t launch_pair_fwd(const EngineArgs& a, cudaStream_t st);

// ------------------------------------------------------------ small-M GEMV
// Forward for M <= kGemvMaxM tokens: Y = X.W^T + s.(X.L1).L2 with the weight
// streamed once from HBM.  Three kernels:
//   (1) T partials: Tp[p][m][j] = sum_{k in slice p} X[m,k] L1[k,j]
//   (2) stream-K dequant-GEMV: the units (128-row tile, 256-wide k range) of
//       W split in equal runs over three workers per SM; every maximal run
//       inside one row tile (a segment) leaves a 128 x 16 fp32 partial tile;
//       one warp per CTA also sums its share of the T partials (T saved,
//       RNbf16(s.T) for (3));
//   (3) finish: Y = RNbf16(sum of a row tile's partials in worker order
//       + RNbf16(s.T).L2).
constexpr int kGemvMaxM = 16;
constexpr int kGemvTSlices = 128;  // max T partial slices

struct GemvPlan {
  int m_tiles, kbt;   // 128-row tiles of W, 64-wide k blocks per row
  int upr;            // units per row tile (256-wide k ranges)
  int64_t units;      // m_tiles * upr
  int grid, workers;  // CTAs (<= SMs), stream-K workers (3 per CTA)
  int maxc;           // max workers covering one row tile
  int t_slices, bps;  // T partial slices, k blocks per slice
  size_t part_bytes;  // segment partials [m_tiles * maxc][16][128] fp32
  size_t tp_bytes;    // T partials [t_slices][16][128] fp32
  size_t stw_bytes;   // RNbf16(s.T) as fp32 [16][128]
};

struct GemvArgs {
  CUtensorMap tmCodes;  // uint8 [N][K/2], box 128 x 128, 128-byte swizzle
  CUtensorMap tmX;      // bf16 [M][K] as 3-D (64, M, K/64), box 64 x 16 x 4, 128-byte swizzle
  const uint8_t* c2;
  int c2_e5m2;          // c2 holds E5M2 codes instead of E4M3
  int c1_mean;          // mean-centred codec: c1 holds [c1, mean] per group
  const float* c1;
  int64_t N, K;
  int M;
  int kbt, upr, m_tiles, maxc;
  int64_t units;
  float* part;
  // LoRA: T partials in, T (saved) and RNbf16(s.T) out
  const float* tp;
  int t_slices, r;
  float s;
  float* T_save;
  float* sTw;
  int* status;
  uint32_t smem_bytes;
  float q[16];
};

GemvPlan plan_gemv(int64_t M, int64_t N, int64_t K, int num_sms);
cudaError_t launch_gemv(const GemvArgs& a, const GemvPlan& p, const uint16_t* X, const uint16_t* L1,
                        const uint16_t* L2, uint16_t* Y, cudaStream_t st);

// ------------------------------------------------- small-M backward (GEMV)
// Backward for M <= kGemvMaxM tokens with the weight streamed once:
//   (1) lora_bwd_n_kernel: over N slices, dL2 = s.T^T.dY and the slices'
//       partials of dT = dY.L2^T; zeroes the k-range arrival counters;
//   (2) nf4_gemv_t_kernel: dX = dY.W^ by stream-K over units (128-row tile
//       of W, 256-wide k range) ordered by k range; the last worker of a k
//       range adds s.dT.L1^T, rounds dX and forms dL1 = s.X^T.dT there.
struct GemvTPlan {
  int n_tiles, kbt, k_ranges;  // 128-row tiles of W, 64-wide k blocks, 256-wide k ranges
  int64_t units;               // n_tiles * k_ranges
  int grid, workers, maxc;     // CTAs, stream-K workers (3 per CTA), max workers per k range
  int slice, t_slices;         // dT slices over N
  size_t part_bytes;           // [k_ranges][maxc][16][256] fp32
  size_t tp_bytes;             // [t_slices][16][128] fp32
  size_t cnt_bytes;            // [k_ranges] int
};

struct GemvTArgs {
  CUtensorMap tmCodes;  // uint8 [N][K/2], box 128 x 128, 128-byte swizzle
  CUtensorMap tmDY;     // bf16 [M][N], box 64 x 16, 128-byte swizzle
  const uint8_t* c2;
  int c2_e5m2, c1_mean;
  const float* c1;
  int64_t N, K;
  int M, r, kbt, n_tiles, maxc, t_slices;
  int64_t units;
  float s;
  float* part;
  const float* tp;
  int* cnt;
  const uint16_t* L1;
  const uint16_t* X;
  uint16_t* dX;   // may be null
  float* dL1;     // may be null
  int* status;
  uint32_t smem_bytes;
  float q[16];
};

GemvTPlan plan_gemv_t(int64_t M, int64_t N, int64_t K, int num_sms);
cudaError_t launch_gemv_t(const GemvTArgs& a, const GemvTPlan& p, const uint16_t* dY, const uint16_t* L2,
                          const float* T, float* dL2, cudaStream_t st);

// --------------------------------------------------------- quantise kernels
cudaError_t launch_quantize(const uint16_t* W, int64_t n_weights, uint8_t* codes, uint8_t* c2, float* c1,
                            int* status, int format, int scale_codec, cudaStream_t st);
cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* c2, const float* c1, int64_t n_weights,
                           uint16_t* out, int format, int scale_codec, cudaStream_t st);
cudaError_t launch_scale_to_bf16(const float* in, int64_t n, float s, uint16_t* out, cudaStream_t st);

// ------------------------------------------------------- adapter kernels
// W_merged = RNbf16(W^ + s (L1 L2)^T), one CTA per 128 x 128 output tile.
size_t merge_smem_bytes(int r);
cudaError_t launch_adapter_merge(const uint8_t* codes, const uint8_t* c2, const float* c1, int format, int scale_codec,
                                 int64_t N, int64_t K, const uint16_t* L1, const uint16_t* L2, int r, float s,
                                 uint16_t* out, cudaStream_t st);
// AdamW step; sc = lr, b1, 1-b1, b2, 1-b2, eps, wd, 1-b1^t, 1-b2^t (fp32).
cudaError_t launch_adamw(float* p, uint16_t* pb, const float* g, float* m, float* v, int64_t n, const float* sc,
                         cudaStream_t st);

}  // namespace qnf4
