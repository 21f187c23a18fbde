// The C ABI (include/qlora_nf4.h): argument checks, TMA tensor maps, the
// launch plan of each call and the launches themselves.  No allocation, no
// synchronisation: all work is queued on the caller's stream.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/qlora_nf4.h"
#include "internal.h"

using namespace qnf4;

namespace {

// --------------------------------------------------------------- device info
struct DevInfo {
  int ok = 0;
  int sms = 148;
};

int current_device_info(DevInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  static DevInfo cache[64];
  static std::mutex mu;
  std::lock_guard<std::mutex> g(mu);
  if (dev < 0 || dev >= 64) return QLORA_ERR_DEVICE;
  if (!cache[dev].ok) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return QLORA_ERR_CUDA;
    if (major != 10 || minor != 0) return QLORA_ERR_DEVICE;
    cache[dev].sms = sms;
    cache[dev].ok = 1;
  }
  *out = cache[dev];
  return QLORA_OK;
}

// ----------------------------------------------------------------- TMA maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D map over a row-major matrix [outer][inner] of `esize`-byte elements.
int make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t inner, uint64_t outer,
             uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return QLORA_ERR_CUDA;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * (uint64_t)esize};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QLORA_OK : QLORA_ERR_CUDA;
}

// 3-D map over a row-major matrix [rows][cols] of bf16 viewed as
// (64, rows, cols / 64): element (x, y, z) is [y][64 z + x]; box 64 x
// box_rows x box_blocks, 128-byte swizzle.  One load brings box_blocks
// consecutive 64-wide column blocks of box_rows rows.
int map_blocks3d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                 uint32_t box_blocks) {
  auto fn = encode_fn();
  if (!fn) return QLORA_ERR_CUDA;
  const cuuint64_t dims[3] = {64, rows, cols / 64};
  const cuuint64_t strides[2] = {cols * 2, 128};
  const cuuint32_t box[3] = {64, box_rows, box_blocks};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QLORA_OK : QLORA_ERR_CUDA;
}

// bf16 operand of the engine.  K-major: matrix [mn][k] (k contiguous), box
// 64 k x `rows` mn.  MN-major: matrix [k][mn] (mn contiguous), box 64 x 64.
int map_operand(CUtensorMap* m, const void* base, int mn_major, uint64_t mn_extent, uint64_t k_extent, int rows) {
  if (!mn_major)
    return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k_extent, mn_extent, 64, (uint32_t)rows,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, mn_extent, k_extent, 64, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

int map_codes(CUtensorMap* m, const uint8_t* codes, int64_t N, int64_t K, int mn_mode) {
  // codes viewed as uint8 [N][K/2]
  // Swizzled so that the dequant threads' 16-byte reads are bank-conflict free.
  if (!mn_mode)
    return make_map(m, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K / 2, (uint64_t)N, 32, 128,
                    CU_TENSOR_MAP_SWIZZLE_32B);
  return make_map(m, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K / 2, (uint64_t)N, 64, 64,
                  CU_TENSOR_MAP_SWIZZLE_64B);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

EpiArgs epi_none() {
  EpiArgs e;
  std::memset(&e, 0, sizeof(e));
  e.alpha = 1.0f;
  e.alpha2 = 1.0f;
  return e;
}

bool format_ok(const qlora_nf4_weight* w) {
  return w->format >= 0 && w->format < kNumFormats &&
         (w->scale_codec == QLORA_SCALE_E4M3 || w->scale_codec == QLORA_SCALE_E5M2 ||
          w->scale_codec == QLORA_SCALE_E4M3_MEAN);
}

// The mean-centred codec reads [c1, mean] pairs as 8-byte loads.
bool c1_aligned(const qlora_nf4_weight* w) {
  return w->scale_codec != QLORA_SCALE_E4M3_MEAN || (reinterpret_cast<uintptr_t>(w->c1) & 7u) == 0;
}

void fill_common(EngineArgs* a, int* status, int format, int scale_codec) {
  std::memset(a, 0, sizeof(*a));
  a->status = status;
  a->c2_e5m2 = scale_codec == QLORA_SCALE_E5M2;
  a->c1_mean = scale_codec == QLORA_SCALE_E4M3_MEAN;
  const Nf4Tables& t = code_tables(format);
  for (int i = 0; i < 16; ++i) a->q[i] = t.q[i];
}

// The forward dequant-GEMM on CTA pairs (launch_pair_fwd): used, for plans
// with full 256-token tiles and no split, when QLORA_NF4_PAIR=1 is set in
// the environment.  It computes the same result as the single-CTA engine
// and measured slower on the LLaMA-7B linears, so the single-CTA engine is
// the default.
constexpr int A_PAIR_K = 3;

bool use_pair_fwd(const GemmPlan& p, int rows, int cols, int kb_ext) {
  if (p.BN != 256 || p.splits != 1 || !pair_fwd_supported(rows, cols, kb_ext)) return false;
  const char* env = std::getenv("QLORA_NF4_PAIR");
  return env && env[0] == '1';
}

// Launch the engine and, for a split reduction, the fixed-order sum.
int run(EngineArgs& a, int amode, const GemmPlan& p, float* partial, cudaStream_t st) {
  a.splits = p.splits;
  a.partial = p.splits > 1 ? partial : nullptr;
  if (amode == A_PAIR_K) return launch_pair_fwd(a, st) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
  if (launch_engine(a, amode, p, st) != cudaSuccess) return QLORA_ERR_CUDA;
  if (p.splits > 1 && launch_split_reduce(partial, p.splits, a.rows, a.cols, a.epi, st) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Diagnostic events around the fused dequant-GEMM (qlora_set_gemm_events).
cudaEvent_t g_ev_start = nullptr, g_ev_end = nullptr;
// Failure-detection hook (qlora_debug_stall_next_gemm): wait bound of the
// next fused dequant-GEMM launch, whose producer then issues no loads.
uint64_t g_stall_ns = 0;

int run_timed(EngineArgs& a, int amode, const GemmPlan& p, float* partial, cudaStream_t st) {
  cudaEvent_t e0 = g_ev_start, e1 = g_ev_end;
  g_ev_start = g_ev_end = nullptr;
  const uint64_t stall_ns = g_stall_ns;
  g_stall_ns = 0;
  if (stall_ns && amode != A_PAIR_K) {
    a.stall = 1;
    a.wait_ns = stall_ns;
  }
  if (e0 && cudaEventRecord(e0, st) != cudaSuccess) return QLORA_ERR_CUDA;
  const int rc = run(a, amode, p, partial, st);
  if (rc == QLORA_OK && e1 && cudaEventRecord(e1, st) != cudaSuccess) return QLORA_ERR_CUDA;
  return rc;
}

bool valid_rank(int r) { return r >= 8 && r <= 128 && r % 8 == 0; }

// Workspace layout shared by the forward and the backward:
//   [0]             bf16 s.T   [M][r]
//   [ofs_sdT]       bf16 s.dT  [M][r]
//   [ofs_partial]   fp32 split partials of the largest split GEMM
struct WsLayout {
  size_t ofs_sdT, ofs_partial, total;
  GemmPlan t_fwd, y_fwd, dt, dx, dl1, dl2;
  GemvPlan gemv;    // M <= kGemvMaxM only
  GemvTPlan gemvt;  // M <= kGemvMaxM only
};

WsLayout ws_layout(int64_t M, int64_t N, int64_t K, int r, int sms) {
  WsLayout w{};
  const size_t mr = align256((size_t)M * r * 2);
  w.ofs_sdT = mr;
  w.ofs_partial = 2 * mr;
  const int kbK = (int)(K / 64), kbN = (int)((N + 63) / 64), kbM = (int)((M + 63) / 64);
  w.t_fwd = plan_gemm((int)M, r, kbK, sms);
  w.y_fwd = plan_gemm((int)N, (int)M, kbK, sms);
  w.dt = plan_gemm((int)M, r, kbN, sms);
  w.dx = plan_gemm((int)K, (int)M, kbN, sms);
  w.dl1 = plan_gemm((int)K, r, kbM, sms);
  w.dl2 = plan_gemm((int)N, r, kbM, sms);
  size_t part = 0;
  for (const GemmPlan* p : {&w.t_fwd, &w.y_fwd, &w.dt, &w.dx, &w.dl1, &w.dl2})
    part = p->partial_bytes > part ? p->partial_bytes : part;
  if (M <= kGemvMaxM) {  // few tokens: stream-K partials + T / dT slices (+ arrival counters)
    w.gemv = plan_gemv(M, N, K, sms);
    const size_t g = align256(w.gemv.part_bytes) + align256(w.gemv.tp_bytes) + w.gemv.stw_bytes;
    part = g > part ? g : part;
    w.gemvt = plan_gemv_t(M, N, K, sms);
    const size_t gt = align256(w.gemvt.part_bytes) + align256(w.gemvt.tp_bytes) + w.gemvt.cnt_bytes;
    part = gt > part ? gt : part;
  }
  w.total = w.ofs_partial + align256(part);
  return w;
}

bool shape_ok(int64_t M, int64_t N, int64_t K) {
  return M >= 1 && N >= 8 && K >= 64 && K % 64 == 0 && N % 8 == 0 && M <= (1 << 24) && N <= (1 << 24) &&
         K <= (1 << 24);
}

}  // namespace

extern "C" {

const char* qlora_status_string(int code) {
  switch (code) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_NULL: return "a required pointer is NULL";
    case QLORA_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case QLORA_ERR_SHAPE: return "invalid shape (need K % 64 == 0, N % 8 == 0, sizes >= 1)";
    case QLORA_ERR_RANK: return "unsupported LoRA rank (need r % 8 == 0, 8 <= r <= 128)";
    case QLORA_ERR_WORKSPACE: return "workspace too small";
    case QLORA_ERR_CUDA: return "CUDA runtime or driver call failed";
    case QLORA_ERR_NONFINITE: return "weight holds an Inf or NaN";
    case QLORA_ERR_TIMEOUT: return "an internal GPU wait expired";
    case QLORA_ERR_DEVICE: return "current device is not an sm_100 GPU";
    case QLORA_ERR_FORMAT: return "unknown code format (QLORA_FMT_*) or scale codec (QLORA_SCALE_*)";
    case QLORA_ERR_SCRATCH_LIMIT: return "problem needs more workspace than the library's 8 MiB static scratch";
  }
  return "unknown status";
}

int qlora_weight_storage_bytes(int64_t N, int64_t K, int scale_codec, size_t* codes_bytes, size_t* c2_bytes,
                               size_t* c1_bytes) {
  if (N < 1 || K < 64 || K % 64) return QLORA_ERR_SHAPE;
  if (scale_codec != QLORA_SCALE_E4M3 && scale_codec != QLORA_SCALE_E5M2 && scale_codec != QLORA_SCALE_E4M3_MEAN)
    return QLORA_ERR_FORMAT;
  const int64_t n = N * K, nb = n / 64;
  if (codes_bytes) *codes_bytes = (size_t)(n / 2);
  if (c2_bytes) *c2_bytes = (size_t)nb;
  if (c1_bytes) *c1_bytes = (size_t)((nb + 255) / 256) * (scale_codec == QLORA_SCALE_E4M3_MEAN ? 8 : 4);
  return QLORA_OK;
}

int qlora_nf4_storage_bytes(int64_t N, int64_t K, size_t* codes_bytes, size_t* c2_bytes, size_t* c1_bytes) {
  return qlora_weight_storage_bytes(N, K, QLORA_SCALE_E4M3, codes_bytes, c2_bytes, c1_bytes);
}

uint64_t qlora_kernel_launches(void) { return launches_so_far(); }

int qlora_debug_stall_next_gemm(uint64_t wait_ns) {
  g_stall_ns = wait_ns;
  return QLORA_OK;
}

int qlora_set_gemm_events(void* ev_start, void* ev_end) {
  g_ev_start = (ev_start && ev_end) ? reinterpret_cast<cudaEvent_t>(ev_start) : nullptr;
  g_ev_end = (ev_start && ev_end) ? reinterpret_cast<cudaEvent_t>(ev_end) : nullptr;
  return QLORA_OK;
}

int qlora_nf4_codebook(float levels[16]) {
  if (!levels) return QLORA_ERR_NULL;
  const Nf4Tables& t = nf4_tables();
  for (int i = 0; i < 16; ++i) levels[i] = t.q[i];
  return QLORA_OK;
}

int qlora_code_levels(int format, float levels[16]) {
  if (!levels) return QLORA_ERR_NULL;
  if (format < 0 || format >= kNumFormats) return QLORA_ERR_FORMAT;
  const Nf4Tables& t = code_tables(format);
  for (int i = 0; i < 16; ++i) levels[i] = t.q[i];
  return QLORA_OK;
}

int qlora_nf4_quantize(const uint16_t* W, int64_t N, int64_t K, const qlora_nf4_weight* out, int* status_dev,
                       qlora_stream_t stream) {
  if (!W || !out || !out->codes || !out->c2 || !out->c1) return QLORA_ERR_NULL;
  if (N < 1 || K < 64 || K % 64) return QLORA_ERR_SHAPE;
  if (!format_ok(out)) return QLORA_ERR_FORMAT;
  if (!c1_aligned(out)) return QLORA_ERR_ALIGN;
  if (!aligned16(W) || !aligned16(out->codes)) return QLORA_ERR_ALIGN;
  DevInfo di;
  if (int rc = current_device_info(&di)) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return launch_quantize(W, N * K, out->codes, out->c2, out->c1, status_dev, out->format, out->scale_codec, st) ==
                 cudaSuccess
             ? QLORA_OK
             : QLORA_ERR_CUDA;
}

int qlora_nf4_dequant(const qlora_nf4_weight* w, uint16_t* W_out, int* status_dev, qlora_stream_t stream) {
  (void)status_dev;
  if (!w || !W_out || !w->codes || !w->c2 || !w->c1) return QLORA_ERR_NULL;
  if (w->n_rows < 1 || w->n_cols < 64 || w->n_cols % 64) return QLORA_ERR_SHAPE;
  if (!format_ok(w)) return QLORA_ERR_FORMAT;
  if (!c1_aligned(w)) return QLORA_ERR_ALIGN;
  if (!aligned16(W_out) || !aligned16(w->codes)) return QLORA_ERR_ALIGN;
  DevInfo di;
  if (int rc = current_device_info(&di)) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return launch_dequant(w->codes, w->c2, w->c1, w->n_rows * w->n_cols, W_out, w->format, w->scale_codec, st) ==
                 cudaSuccess
             ? QLORA_OK
             : QLORA_ERR_CUDA;
}

size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
  if (!shape_ok(M, N, K) || !valid_rank(r)) return 0;
  DevInfo di;
  if (current_device_info(&di)) di.sms = 148;
  return ws_layout(M, N, K, r, di.sms).total;
}

int qlora_linear_fwd(const uint16_t* X, int64_t M, const qlora_nf4_weight* w, const uint16_t* L1,
                     const uint16_t* L2, int r, float s, uint16_t* Y, float* T_save, void* ws, size_t ws_bytes,
                     int* status_dev, qlora_stream_t stream) {
  if (!X || !w || !w->codes || !w->c2 || !w->c1 || !L1 || !L2 || !Y || !T_save || !ws) return QLORA_ERR_NULL;
  const int64_t N = w->n_rows, K = w->n_cols;
  if (!shape_ok(M, N, K)) return QLORA_ERR_SHAPE;
  if (!format_ok(w)) return QLORA_ERR_FORMAT;
  if (!c1_aligned(w)) return QLORA_ERR_ALIGN;
  if (!valid_rank(r)) return QLORA_ERR_RANK;
  for (const void* p : {(const void*)X, (const void*)w->codes, (const void*)L1, (const void*)L2, (const void*)Y,
                        (const void*)T_save, (const void*)ws})
    if (!aligned16(p)) return QLORA_ERR_ALIGN;
  DevInfo di;
  if (int rc = current_device_info(&di)) return rc;
  const WsLayout lay = ws_layout(M, N, K, r, di.sms);
  if (ws_bytes < lay.total) return QLORA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint16_t* sT = reinterpret_cast<uint16_t*>(wsb);
  float* partial = reinterpret_cast<float*>(wsb + lay.ofs_partial);

  if (M <= kGemvMaxM) {
    // Few tokens: weight-streaming dequant-GEMV (stream-K over all SMs).
    const GemvPlan& gp = lay.gemv;
    GemvArgs ga;
    std::memset(&ga, 0, sizeof(ga));
    if (make_map(&ga.tmCodes, w->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K / 2, (uint64_t)N, 128, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
        map_blocks3d(&ga.tmX, X, (uint64_t)M, (uint64_t)K, 16, 4))
      return QLORA_ERR_CUDA;
    ga.c2 = w->c2;
    ga.c1 = w->c1;
    ga.N = N;
    ga.K = K;
    ga.M = (int)M;
    ga.kbt = gp.kbt;
    ga.upr = gp.upr;
    ga.m_tiles = gp.m_tiles;
    ga.maxc = gp.maxc;
    ga.units = gp.units;
    ga.part = partial;
    uint8_t* gws = wsb + lay.ofs_partial + align256(gp.part_bytes);
    ga.tp = reinterpret_cast<float*>(gws);
    ga.sTw = reinterpret_cast<float*>(gws + align256(gp.tp_bytes));
    ga.r = r;
    ga.s = s;
    ga.T_save = T_save;
    ga.status = status_dev;
    const Nf4Tables& tb = code_tables(w->format);
    ga.c2_e5m2 = w->scale_codec == QLORA_SCALE_E5M2;
    ga.c1_mean = w->scale_codec == QLORA_SCALE_E4M3_MEAN;
    for (int i = 0; i < 16; ++i) ga.q[i] = tb.q[i];
    cudaEvent_t e0 = g_ev_start, e1 = g_ev_end;
    g_ev_start = g_ev_end = nullptr;
    if (e0 && cudaEventRecord(e0, st) != cudaSuccess) return QLORA_ERR_CUDA;
    if (launch_gemv(ga, gp, X, L1, L2, Y, st) != cudaSuccess) return QLORA_ERR_CUDA;
    if (e1 && cudaEventRecord(e1, st) != cudaSuccess) return QLORA_ERR_CUDA;
    return QLORA_OK;
  }

  // (1) T = X.L1 (fp32, saved) and s.T in bf16 for the LoRA extension.
  {
    EngineArgs a;
    fill_common(&a, status_dev, w->format, w->scale_codec);
    const GemmPlan& p = lay.t_fwd;
    if (map_operand(&a.tmA, X, 0, M, K, 128) || map_operand(&a.tmB, L1, 1, r, K, p.BN)) return QLORA_ERR_CUDA;
    a.rows = (int)M;
    a.cols = r;
    a.kb_main = (int)(K / 64);
    a.b_mn_main = 1;
    a.epi = epi_none();
    a.epi.out = T_save;
    a.epi.rs = r;
    a.epi.cs = 1;
    a.epi.out2 = sT;
    a.epi.alpha2 = s;
    a.epi.rs2 = r;
    a.epi.cs2 = 1;
    if (int rc = run(a, A_TMA, p, partial, st)) return rc;
  }
  // (2) Y^T = W^.X^T + L2^T.(s.T)^T, W^ dequantised on chip.
  {
    EngineArgs a;
    fill_common(&a, status_dev, w->format, w->scale_codec);
    const GemmPlan& p = lay.y_fwd;
    const int kb_ext = (r + 63) / 64;
    const bool pair = use_pair_fwd(p, (int)N, (int)M, kb_ext);
    const int brows = pair ? 128 : p.BN;  // a pair CTA holds half of the 256 tokens
    if (map_codes(&a.tmA, w->codes, N, K, 0) || map_operand(&a.tmB, X, 0, M, K, brows) ||
        map_operand(&a.tmAx, L2, 1, N, r, 128) || map_operand(&a.tmBx, sT, 0, M, r, brows))
      return QLORA_ERR_CUDA;
    a.codes = w->codes;
    a.c2 = w->c2;
    a.c1 = w->c1;
    a.wN = N;
    a.wK = K;
    a.rows = (int)N;
    a.cols = (int)M;
    a.kb_main = (int)(K / 64);
    a.kb_ext = kb_ext;
    a.a_mn_ext = 1;
    a.epi = epi_none();
    a.epi.out = Y;
    a.epi.out_bf16 = 1;
    a.epi.rs = 1;
    a.epi.cs = N;
    if (int rc = run_timed(a, pair ? A_PAIR_K : A_DEQ_K, p, partial, st)) return rc;
  }
  return QLORA_OK;
}

int qlora_adapter_merge(const qlora_nf4_weight* w, const uint16_t* L1, const uint16_t* L2, int r, float s,
                        uint16_t* W_out, int* status_dev, qlora_stream_t stream) {
  (void)status_dev;
  if (!w || !w->codes || !w->c2 || !w->c1 || !L1 || !L2 || !W_out) return QLORA_ERR_NULL;
  const int64_t N = w->n_rows, K = w->n_cols;
  if (!shape_ok(1, N, K)) return QLORA_ERR_SHAPE;
  if (!format_ok(w)) return QLORA_ERR_FORMAT;
  if (!c1_aligned(w)) return QLORA_ERR_ALIGN;
  if (!valid_rank(r)) return QLORA_ERR_RANK;
  for (const void* p : {(const void*)w->codes, (const void*)L1, (const void*)L2, (const void*)W_out})
    if (!aligned16(p)) return QLORA_ERR_ALIGN;
  DevInfo di;
  if (int rc = current_device_info(&di)) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return launch_adapter_merge(w->codes, w->c2, w->c1, w->format, w->scale_codec, N, K, L1, L2, r, s, W_out, st) ==
                 cudaSuccess
             ? QLORA_OK
             : QLORA_ERR_CUDA;
}

int qlora_adamw_step(float* p, uint16_t* p_bf16, const float* g, float* m, float* v, int64_t n,
                     const qlora_adamw_config* cfg, qlora_stream_t stream) {
  if (!p || !g || !m || !v || !cfg) return QLORA_ERR_NULL;
  if (n < 0 || cfg->step < 1) return QLORA_ERR_SHAPE;
  for (const void* q : {(const void*)p, (const void*)g, (const void*)m, (const void*)v})
    if (!aligned16(q)) return QLORA_ERR_ALIGN;
  if (p_bf16 && (reinterpret_cast<uintptr_t>(p_bf16) & 7u)) return QLORA_ERR_ALIGN;
  if (n == 0) return QLORA_OK;
  DevInfo di;
  if (int rc = current_device_info(&di)) return rc;
  // every constant computed in double and rounded once to float
  const double t = (double)cfg->step;
  const float sc[9] = {(float)cfg->lr, (float)cfg->beta1, (float)(1.0 - cfg->beta1), (float)cfg->beta2,
                       (float)(1.0 - cfg->beta2), (float)cfg->eps, (float)cfg->weight_decay,
                       (float)(1.0 - std::pow(cfg->beta1, t)), (float)(1.0 - std::pow(cfg->beta2, t))};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return launch_adamw(p, p_bf16, g, m, v, n, sc, st) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

int qlora_paged_alloc(size_t bytes, void** out) {
  if (!out) return QLORA_ERR_NULL;
  *out = nullptr;
  if (bytes == 0) return QLORA_ERR_SHAPE;
  return cudaMallocManaged(out, bytes, cudaMemAttachGlobal) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

int qlora_paged_free(void* p) {
  if (!p) return QLORA_OK;
  return cudaFree(p) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

int qlora_paged_prefetch(const void* p, size_t bytes, int device, qlora_stream_t stream) {
  if (!p) return QLORA_ERR_NULL;
  if (bytes == 0) return QLORA_OK;
  const int dst = device < 0 ? cudaCpuDeviceId : device;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return cudaMemPrefetchAsync(p, bytes, dst, st) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

int qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, int64_t M, const float* T_saved,
                     const qlora_nf4_weight* w, const uint16_t* L1, const uint16_t* L2, int r, float s, uint16_t* dX,
                     float* dL1, float* dL2, void* ws, size_t ws_bytes, int* status_dev, qlora_stream_t stream) {
  if (!dY || !X || !T_saved || !w || !w->codes || !w->c2 || !w->c1 || !L1 || !L2 || !ws) return QLORA_ERR_NULL;
  const int64_t N = w->n_rows, K = w->n_cols;
  if (!shape_ok(M, N, K)) return QLORA_ERR_SHAPE;
  if (!format_ok(w)) return QLORA_ERR_FORMAT;
  if (!c1_aligned(w)) return QLORA_ERR_ALIGN;
  if (!valid_rank(r)) return QLORA_ERR_RANK;
  for (const void* p : {(const void*)dY, (const void*)X, (const void*)T_saved, (const void*)w->codes,
                        (const void*)L1, (const void*)L2, (const void*)ws})
    if (!aligned16(p)) return QLORA_ERR_ALIGN;
  for (const void* p : {(const void*)dX, (const void*)dL1, (const void*)dL2})
    if (p && !aligned16(p)) return QLORA_ERR_ALIGN;
  DevInfo di;
  if (int rc = current_device_info(&di)) return rc;
  const WsLayout lay = ws_layout(M, N, K, r, di.sms);
  if (ws_bytes < lay.total) return QLORA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint16_t* sT = reinterpret_cast<uint16_t*>(wsb);
  uint16_t* sdT = reinterpret_cast<uint16_t*>(wsb + lay.ofs_sdT);
  float* partial = reinterpret_cast<float*>(wsb + lay.ofs_partial);

  if (M <= kGemvMaxM) {
    // Few tokens: weight-streaming backward (dT and dL2 over N slices, then
    // dX and dL1 by stream-K over the weight).
    const GemvTPlan& gp = lay.gemvt;
    GemvTArgs ga;
    std::memset(&ga, 0, sizeof(ga));
    if (make_map(&ga.tmCodes, w->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K / 2, (uint64_t)N, 128, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
        make_map(&ga.tmDY, dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)N, (uint64_t)M, 64, 16,
                 CU_TENSOR_MAP_SWIZZLE_128B))
      return QLORA_ERR_CUDA;
    ga.c2 = w->c2;
    ga.c1 = w->c1;
    ga.c2_e5m2 = w->scale_codec == QLORA_SCALE_E5M2;
    ga.c1_mean = w->scale_codec == QLORA_SCALE_E4M3_MEAN;
    ga.N = N;
    ga.K = K;
    ga.M = (int)M;
    ga.r = r;
    ga.kbt = gp.kbt;
    ga.n_tiles = gp.n_tiles;
    ga.maxc = gp.maxc;
    ga.t_slices = gp.t_slices;
    ga.units = gp.units;
    ga.s = s;
    uint8_t* g0 = wsb + lay.ofs_partial;
    ga.part = reinterpret_cast<float*>(g0);
    ga.tp = reinterpret_cast<float*>(g0 + align256(gp.part_bytes));
    ga.cnt = reinterpret_cast<int*>(g0 + align256(gp.part_bytes) + align256(gp.tp_bytes));
    ga.L1 = L1;
    ga.X = X;
    ga.dX = dX;
    ga.dL1 = dL1;
    ga.status = status_dev;
    const Nf4Tables& tb = code_tables(w->format);
    for (int i = 0; i < 16; ++i) ga.q[i] = tb.q[i];
    cudaEvent_t e0 = g_ev_start, e1 = g_ev_end;
    g_ev_start = g_ev_end = nullptr;
    g_stall_ns = 0;
    if (e0 && cudaEventRecord(e0, st) != cudaSuccess) return QLORA_ERR_CUDA;
    if (launch_gemv_t(ga, gp, dY, L2, T_saved, dL2, st) != cudaSuccess) return QLORA_ERR_CUDA;
    if (e1 && cudaEventRecord(e1, st) != cudaSuccess) return QLORA_ERR_CUDA;
    return QLORA_OK;
  }

  // (0) s.T in bf16, the operand of dL2.
  if (dL2 && launch_scale_to_bf16(T_saved, M * r, s, sT, st) != cudaSuccess) return QLORA_ERR_CUDA;
  // (1) dT = dY.L2^T, kept as s.dT in bf16.
  {
    EngineArgs a;
    fill_common(&a, status_dev, w->format, w->scale_codec);
    const GemmPlan& p = lay.dt;
    if (map_operand(&a.tmA, dY, 0, M, N, 128) || map_operand(&a.tmB, L2, 0, r, N, p.BN)) return QLORA_ERR_CUDA;
    a.rows = (int)M;
    a.cols = r;
    a.kb_main = (int)((N + 63) / 64);
    a.epi = epi_none();
    a.epi.out2 = sdT;
    a.epi.alpha2 = s;
    a.epi.rs2 = r;
    a.epi.cs2 = 1;
    if (int rc = run(a, A_TMA, p, partial, st)) return rc;
  }
  // (2) dX^T = W^T.dY^T + L1.(s.dT)^T, W^ dequantised on chip (MN-major).
  if (dX) {
    EngineArgs a;
    fill_common(&a, status_dev, w->format, w->scale_codec);
    const GemmPlan& p = lay.dx;
    if (map_codes(&a.tmA, w->codes, N, K, 1) || map_operand(&a.tmB, dY, 0, M, N, p.BN) ||
        map_operand(&a.tmAx, L1, 0, K, r, 128) || map_operand(&a.tmBx, sdT, 0, M, r, p.BN))
      return QLORA_ERR_CUDA;
    a.c2 = w->c2;
    a.c1 = w->c1;
    a.wN = N;
    a.wK = K;
    a.rows = (int)K;
    a.cols = (int)M;
    a.kb_main = (int)((N + 63) / 64);
    a.kb_ext = (r + 63) / 64;
    a.epi = epi_none();
    a.epi.out = dX;
    a.epi.out_bf16 = 1;
    a.epi.rs = 1;
    a.epi.cs = K;
    if (int rc = run_timed(a, A_DEQ_MN, p, partial, st)) return rc;
  }
  // (3) dL1 = X^T.(s.dT): rows k, reduction over tokens.
  if (dL1) {
    EngineArgs a;
    fill_common(&a, status_dev, w->format, w->scale_codec);
    const GemmPlan& p = lay.dl1;
    if (map_operand(&a.tmA, X, 1, K, M, 128) || map_operand(&a.tmB, sdT, 1, r, M, p.BN)) return QLORA_ERR_CUDA;
    a.rows = (int)K;
    a.cols = r;
    a.kb_main = (int)((M + 63) / 64);
    a.a_mn_main = 1;
    a.b_mn_main = 1;
    a.epi = epi_none();
    a.epi.out = dL1;
    a.epi.rs = r;
    a.epi.cs = 1;
    if (int rc = run(a, A_TMA, p, partial, st)) return rc;
  }
  // (4) dL2^T = dY^T.(s.T): rows n, reduction over tokens, stored as dL2[r][N].
  if (dL2) {
    EngineArgs a;
    fill_common(&a, status_dev, w->format, w->scale_codec);
    const GemmPlan& p = lay.dl2;
    if (map_operand(&a.tmA, dY, 1, N, M, 128) || map_operand(&a.tmB, sT, 1, r, M, p.BN)) return QLORA_ERR_CUDA;
    a.rows = (int)N;
    a.cols = r;
    a.kb_main = (int)((M + 63) / 64);
    a.a_mn_main = 1;
    a.b_mn_main = 1;
    a.epi = epi_none();
    a.epi.out = dL2;
    a.epi.rs = 1;
    a.epi.cs = N;
    if (int rc = run(a, A_TMA, p, partial, st)) return rc;
  }
  return QLORA_OK;
}

}  // extern "C"
