/*
 * qlora_nf4.h -- C ABI of the QLoRA NF4 quantized linear layer for NVIDIA
 * B200 (sm_100a).  Library: libqlora_nf4.so.
 *
 * The operation (nlp-lineage "QLoRA" milestone page, section "The idea",
 * notation paragraph):
 *
 *     Y = X . doubleDequant(c1, c2, W_NF4) + s . X . L1 . L2
 *
 * with W frozen in 4 bits and only L1, L2 receiving weight gradients.  The
 * weight is the nn.Linear weight W[N][K] (out x in); the pages' "X . W" uses
 * its transpose.  s = alpha / r is the usual LoRA scale (the pages' formula
 * has s = 1).
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers, owned and allocated by the
 *     caller.  The library never allocates, frees or synchronises (except
 *     the paged-state helpers qlora_paged_alloc / qlora_paged_free, whose job
 *     is to allocate); every call is asynchronous on `stream` (a
 *     cudaStream_t, 0 = legacy default).
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Tensors are dense row-major.  Every pointer must be 16-byte aligned.
 *   - Return value: QLORA_OK, or a negative QLORA_ERR_* from the host-side
 *     checks (nothing is launched then) or from the launch itself.
 *   - `status_dev` is a device int the kernels write on conditions found on
 *     the GPU (non-finite weights, an expired internal wait).  Kernels only
 *     ever store a nonzero QLORA_ERR_* value there; the caller zeroes it and
 *     reads it after synchronising.  It may be NULL to ignore such reports.
 *   - Output buffers are overwritten, never accumulated into.
 *   - Calls that overlap on the GPU must not share a workspace.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

typedef void* qlora_stream_t; /* a cudaStream_t */

enum {
  QLORA_OK = 0,
  QLORA_ERR_NULL = -1,        /* a required pointer is NULL */
  QLORA_ERR_ALIGN = -2,       /* a pointer is not 16-byte aligned */
  QLORA_ERR_SHAPE = -3,       /* K % 64 != 0, N % 8 != 0, a size < 1 or too large */
  QLORA_ERR_RANK = -4,        /* r not a multiple of 8 in [8, 128] */
  QLORA_ERR_WORKSPACE = -5,   /* ws too small (see qlora_workspace_bytes) */
  QLORA_ERR_CUDA = -6,        /* a CUDA runtime / driver call failed */
  QLORA_ERR_NONFINITE = -7,   /* device status: W holds an Inf or NaN */
  QLORA_ERR_TIMEOUT = -8,     /* device status: an internal wait expired */
  QLORA_ERR_DEVICE = -9,      /* current device is not sm_100 */
  QLORA_ERR_SCRATCH_LIMIT = -10, /* problem needs more than the library's static scratch */
  QLORA_ERR_FORMAT = -11        /* unknown code format or scale codec */
};

/*
 * 4-bit code formats.  NF4 is the method's own; FP4 and Int4 are the two
 * formats the pages compare it with (nlp-lineage "QLoRA", section "What it
 * showed", third bullet: "a standard 4-bit float" and "4-bit integers"),
 * read as OCP E2M1 divided by 6 and as symmetric integers k/7.  All three
 * use the same blocks, absmax scales and E4M3 double quantisation; a code is
 * an index into the format's 16 ascending levels (qlora_code_levels), the
 * nearest level to RN32(w / c_b), ties to the lower code.  FP4 and Int4 have
 * 15 reachable levels; their lowest entry (-2 and -8/7) lies below -1 and is
 * never produced.
 */
enum {
  QLORA_FMT_NF4 = 0,
  QLORA_FMT_FP4 = 1,
  QLORA_FMT_INT4 = 2
};

/*
 * Codec of the 8-bit block scales c2.  The pages say only that the scales
 * become 8-bit floats; E4M3 (max 448) is the reading taken, E5M2 (max 57344:
 * two more exponent bits, one fewer mantissa bit) the compared alternative.
 * With E5M2, c1_g = RN32(max c_b / 57344) and c2_b = E5M2_RNE_satfinite(
 * RN32(c_b / c1_g)); the dequantiser decodes accordingly.  Codes and storage
 * are unchanged.
 */
enum {
  QLORA_SCALE_E4M3 = 0,
  QLORA_SCALE_E5M2 = 1,
  QLORA_SCALE_E4M3_MEAN = 2
};

/*
 * QLORA_SCALE_E4M3_MEAN: mean-centred double quantisation.  The block scales
 * are all non-negative, so each group of 256 is centred on its mean first and
 * the signed residuals take the sign bit of E4M3:
 *   mu_g = RN32(S_g / n_g), S_g the fp32 sum of the group's c_b as a pairwise
 *          tree over 256 slots (adjacent pairs first; empty slots of a partial
 *          group are zeros), n_g its number of blocks
 *   d_b  = RN32(c_b - mu_g);  c1_g = RN32(max |d_b| / 448)
 *   c2_b = E4M3_RNE_satfinite(RN32(d_b / c1_g)) (signed), 0 when c1_g = 0
 *   c^_b = RN32(RN32(dec(c2_b) * c1_g) + mu_g)
 * The c1 array then holds two floats per group, c1_g then mu_g (8-byte
 * aligned): 4 + 8/64 + 64/16384 bits per weight.  Codes are unchanged.
 */

/*
 * The quantized weight (nlp-lineage "QLoRA", section "The idea": blocks of
 * 64 weights, 4-bit NormalFloat codes, 8-bit block scales c2 and 32-bit
 * second-level scales c1; inferensys glossary "QLoRA": the scales become
 * 8-bit floats).
 *   codes : uint8[N*K/2]   two 4-bit codes per byte, flat row-major order,
 *                          element 2j in the low nibble, 2j+1 in the high.
 *   c2    : uint8[N*K/64]  OCP FP8 E4M3 code of each 64-weight block scale.
 *   c1    : float[ceil(N*K/16384)]  one fp32 scale per 256 consecutive blocks.
 * Storage: 4 + 8/64 + 32/16384 = 4.127 bits per weight.
 */
typedef struct qlora_nf4_weight {
  uint8_t* codes;
  uint8_t* c2;
  float* c1;
  int64_t n_rows; /* N: output features, >= 1 */
  int64_t n_cols; /* K: input features, a multiple of 64 */
  int32_t format;      /* QLORA_FMT_*: the levels the codes index (0 = NF4) */
  int32_t scale_codec; /* QLORA_SCALE_*: the 8-bit float of c2 (0 = E4M3) */
} qlora_nf4_weight;

/* Bytes of codes, c2 and c1 for an N x K weight (sizes for the caller's
 * allocations) with E4M3 or E5M2 block scales.  Returns QLORA_ERR_SHAPE for
 * an invalid shape. */
QLORA_API int qlora_nf4_storage_bytes(int64_t N, int64_t K, size_t* codes_bytes, size_t* c2_bytes,
                            size_t* c1_bytes);

/* The same for any scale codec (QLORA_SCALE_*): the mean-centred codec
 * stores two floats per group in c1.  QLORA_ERR_FORMAT for an unknown codec. */
QLORA_API int qlora_weight_storage_bytes(int64_t N, int64_t K, int scale_codec, size_t* codes_bytes,
                                         size_t* c2_bytes, size_t* c1_bytes);

/* The 16 NF4 levels the kernels use (ascending, -1 ... 0 ... 1), copied to a
 * host array.  The library derives them at load from the normal quantiles:
 * 8 positive and 7 negative levels at equally spaced probabilities between
 * 1/2 and 1 - (1/32 + 1/30)/2, plus an exact zero, scaled to +-1
 * (nlp-lineage "QLoRA", section "The idea", NF4 bullet). */
QLORA_API int qlora_nf4_codebook(float levels[16]);

/* The 16 levels of a code format (QLORA_FMT_*), ascending, as the kernels
 * use them.  Returns QLORA_ERR_FORMAT for an unknown format. */
QLORA_API int qlora_code_levels(int format, float levels[16]);

/*
 * NF4 double quantisation of a bf16 weight W[N][K] (section "The idea",
 * NF4 and double-quantisation bullets).
 *   c_b   = max |w| over each block of 64 (fp32, exact)
 *   code  = nearest NF4 level to RN32(w / c_b), ties to the lower level
 *           (all-zero block: the code of the exact zero, 7 for NF4 and 8
 *           for FP4 and Int4)
 *   c1_g  = RN32(max_{b in g} c_b / 448)      (groups of 256 blocks)
 *   c2_b  = E4M3_RNE_satfinite(RN32(c_b / c1_g)), 0 when c1_g = 0
 * W: device bf16[N*K].  out: descriptor whose buffers receive the result
 * (out->n_rows/n_cols are ignored and N, K used; out->format selects the
 * levels, see QLORA_FMT_*, and out->scale_codec the c2 codec, QLORA_SCALE_*).  A non-finite weight sets
 * *status_dev = QLORA_ERR_NONFINITE (the outputs are then unspecified).
 */
QLORA_API int qlora_nf4_quantize(const uint16_t* W, int64_t N, int64_t K, const qlora_nf4_weight* out,
                       int* status_dev, qlora_stream_t stream);

/*
 * doubleDequant(c1, c2, W_NF4) to bf16 (section "The idea", notation
 * paragraph; inferensys glossary: NF4 dequantised to BFloat16):
 *   c^_b = RN32(dec_E4M3(c2_b) * c1_g);  w^ = RNbf16(RN32(q[code] * c^_b))
 * W_out: device bf16[N*K].
 */
QLORA_API int qlora_nf4_dequant(const qlora_nf4_weight* w, uint16_t* W_out, int* status_dev,
                      qlora_stream_t stream);

/* Workspace bytes needed by qlora_linear_fwd and qlora_linear_bwd for M
 * tokens, an N x K weight and rank r (the maximum over both calls).
 * Returns 0 for an invalid shape. */
QLORA_API size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);

/*
 * Forward of the quantized linear layer:
 *   T = X . L1                       (fp32, saved for the backward)
 *   Y = RNbf16( X . W^T + s . T . L2 )
 * W^ is the doubleDequant weight, produced tile by tile on chip and never
 * written to memory (examadda "QLoRA", "The Core Idea": dequantised on the
 * fly; inferensys: decompressed in shared memory and fed to the tensor cores).
 *   X   : bf16[M][K]     L1 : bf16[K][r]     L2 : bf16[r][N]
 *   Y   : bf16[M][N]     T_save : float[M][r]
 *   ws  : device workspace of ws_bytes >= qlora_workspace_bytes(M, N, K, r)
 * Requires K % 64 == 0, N % 8 == 0, r % 8 == 0 and 8 <= r <= 128.
 * With QLORA_NF4_PAIR=1 in the environment (read at each call), grids of at
 * least one 128 x 256 tile per SM run on the CTA-pair kernel (cta_group::2)
 * instead of the single-CTA one: same result within the same tolerance.
 */
QLORA_API int qlora_linear_fwd(const uint16_t* X, int64_t M, const qlora_nf4_weight* w,
                     const uint16_t* L1, const uint16_t* L2, int r, float s, uint16_t* Y,
                     float* T_save, void* ws, size_t ws_bytes, int* status_dev,
                     qlora_stream_t stream);

/*
 * Backward of the same layer for an upstream gradient dY (gradients flow
 * through the frozen 4-bit weight into the adapters; W gets none: section
 * "The idea"; examadda "The Flow"):
 *   dT  = dY . L2^T
 *   dX  = RNbf16( dY . W^ + s . dT . L1^T )
 *   dL1 = s . X^T . dT        (fp32)
 *   dL2 = s . T^T . dY        (fp32)
 *   dY : bf16[M][N]   X : bf16[M][K]   T_saved : float[M][r] (from the forward)
 *   dX : bf16[M][K]   dL1 : float[K][r]   dL2 : float[r][N]
 * dX, dL1 or dL2 may be NULL to skip that output.  Same shape rules as the
 * forward.
 */
QLORA_API int qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, int64_t M, const float* T_saved,
                     const qlora_nf4_weight* w, const uint16_t* L1, const uint16_t* L2, int r,
                     float s, uint16_t* dX, float* dL1, float* dL2, void* ws, size_t ws_bytes,
                     int* status_dev, qlora_stream_t stream);

/*
 * Adapter merge (examadda "QLoRA", "Practical Notes", third bullet: merging
 * an adapter back into a 4-bit base is lossy, so dequantise first):
 *   W_out = RNbf16( W^ + s . (L1 . L2)^T ),   W^ = doubleDequant(c1, c2, W_NF4)
 * computed as RN32(W^ + s . acc) with acc the rank-r product accumulated in
 * fp32 on the tensor cores (summation order unspecified), then rounded once
 * to bf16.  W_out: device bf16[N][K] (the nn.Linear layout of W).  L1, L2 as
 * in qlora_linear_fwd; same rank rules.  Quantising W_out again
 * (qlora_nf4_quantize) is a separate, lossy step.
 */
QLORA_API int qlora_adapter_merge(const qlora_nf4_weight* w, const uint16_t* L1, const uint16_t* L2, int r,
                                  float s, uint16_t* W_out, int* status_dev, qlora_stream_t stream);

/*
 * One AdamW step on the adapters (the optimizer whose state the paged
 * optimizers keep in memory that moves between GPU and host: nlp-lineage
 * "QLoRA", section "The idea", paged-optimizers bullet; inferensys glossary,
 * paged-optimizers paragraph).  Decoupled weight decay, each operation
 * rounded to fp32 in this order (t = step, constants computed in double and
 * rounded once to float):
 *   m = b1 m + (1 - b1) g;   v = b2 v + ((1 - b2) g) g
 *   p = p - lr ( (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps) + wd p )
 * p, g, m, v: float[n], 16-byte aligned, device or managed memory (see
 * qlora_paged_alloc); p_bf16 (optional, 8-byte aligned) receives RNbf16(p),
 * the copy the layer multiplies with.  Updates p, m, v in place.
 */
typedef struct qlora_adamw_config {
  double lr, beta1, beta2, eps, weight_decay;
  int64_t step; /* 1 for the first step */
} qlora_adamw_config;

QLORA_API int qlora_adamw_step(float* p, uint16_t* p_bf16, const float* g, float* m, float* v, int64_t n,
                               const qlora_adamw_config* cfg, qlora_stream_t stream);

/*
 * Paged optimizer state: memory that the driver pages between the GPU and
 * host memory on demand (CUDA managed memory), so optimizer state can exceed
 * the GPU's free memory for a moment without failing.  These are the only
 * calls of the library that allocate or free.  qlora_paged_prefetch moves a
 * range ahead of use: device >= 0 to that GPU, -1 to host memory; it is
 * asynchronous on `stream`.
 */
QLORA_API int qlora_paged_alloc(size_t bytes, void** out);
QLORA_API int qlora_paged_free(void* p);
QLORA_API int qlora_paged_prefetch(const void* p, size_t bytes, int device, qlora_stream_t stream);

/*
 * Forward without a caller workspace, for callers that cannot allocate
 * device memory (no counterpart on the pages: this is an interface for
 * embedding the layer, not part of the method).  Such callers include
 * plugins and custom operators run by a host framework that owns the device
 * memory pool and forbids allocation inside its execute callback, and
 * serving loops whose policy forbids cudaMalloc after start-up.  Same
 * arguments and results as qlora_linear_fwd minus ws / ws_bytes: the
 * workspace is a static device array inside the library, 8 MiB on every GPU
 * that loads it, held until exit.  A problem whose qlora_workspace_bytes()
 * exceeds 8 MiB is rejected with QLORA_ERR_SCRATCH_LIMIT before anything is
 * launched.  The first call on a device looks up the array's device address
 * (once per device, that device current; again after the device's context
 * has been re-created, e.g. by cudaDeviceReset); make that first call before
 * any stream capture.  All calls share the one array: calls that overlap on the
 * GPU race and must be serialised by the caller.  Allocates nothing.
 */
QLORA_API int qlora_linear_fwd_noalloc(const uint16_t* X, int64_t M, const qlora_nf4_weight* w,
                                       const uint16_t* L1, const uint16_t* L2, int r, float s,
                                       uint16_t* Y, float* T_save, int* status_dev,
                                       qlora_stream_t stream);

/* Diagnostic timing hook.  When both are non-NULL (cudaEvent_t handles),
 * the next qlora_linear_fwd / qlora_linear_bwd records `ev_start` on its
 * stream just before the fused dequant-GEMM launch (Y, resp. dX) and `ev_end`
 * just after it (and after its split reduction, if any); the hook is then
 * cleared.  Process-wide, not thread-safe; NULL, NULL clears it. */
QLORA_API int qlora_set_gemm_events(void* ev_start, void* ev_end);

/* Failure-detection test hook (diagnostic; the method has no counterpart).
 * The next fused dequant-GEMM launch of qlora_linear_fwd or qlora_linear_bwd
 * (the Y launch of a forward with more than 16 tokens, resp. the dX launch
 * of a backward; not the opt-in CTA-pair forward) runs with its TMA producer
 * issuing no loads and every internal wait bounded by wait_ns nanoseconds
 * instead of 4 s.  Its waits then expire: the kernel writes
 * QLORA_ERR_TIMEOUT to *status_dev, frees its tensor memory and returns
 * with nothing in flight, so the context stays usable; that call's outputs
 * are unspecified.  One-shot and process-wide, not thread-safe; 0 cancels a
 * pending request. */
QLORA_API int qlora_debug_stall_next_gemm(uint64_t wait_ns);

/* Number of kernels this process has launched through the library so far
 * (all devices, all calls).  A diagnostic for counting launches. */
QLORA_API uint64_t qlora_kernel_launches(void);

/* Human-readable text for a QLORA_* code.  Never NULL. */
QLORA_API const char* qlora_status_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
