// NF4 double quantisation (bf16 -> codes, c2, c1) and dequantisation
// (codes, c2, c1 -> bf16): the two HBM-bound passes.  The same kernels serve
// the two compared 4-bit formats (FP4, Int4), which swap only the levels.
//
// nlp-lineage "QLoRA" milestone page, section "The idea": blocks of 64
// weights with an absmax scale, the scales themselves quantised to 8 bits
// (E4M3 here) with one fp32 second-level scale per 256 blocks.
#include "common.cuh"
#include "internal.h"

namespace qnf4 {
namespace {

constexpr int kGroupBlocks = 256;                 // first-level blocks per c1 scale
constexpr int kQuantThreads = 256;

struct QuantParams {
  float t[15];    // decision thresholds, RD32 of the level midpoints
  float poly[6];  // code-search polynomial (see Nf4Tables)
};

constexpr uint32_t kMagicBits = 0x4B400000u;  // bits of 1.5 * 2^23: adding it rounds to an integer

// x = RN32(w / c) for a pair of weights against one block scale c.  For c in
// [2^-90, 2^100) a correctly rounded reciprocal, one product and one fused
// correction step give the IEEE quotient's NF4 code for every bf16 pair
// (checked exhaustively on the host); the other scales take the IEEE division.
// A zero or non-finite scale gives x = 0 (a non-finite block is reported
// through the status word).
QDEV float2 ratio_fast(float2 w, float2 c, float2 rc) {
  const float2 q0 = __fmul2_rn(w, rc);
  const float2 e = __ffma2_rn(q0, make_float2(-c.x, -c.y), w);
  return __ffma2_rn(e, rc, q0);
}
QDEV float ratio_slow(float w, float c) {
  return (c > 0.0f && c <= 3.402823466e38f) ? __fdiv_rn(w, c) : 0.0f;
}

QDEV float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

// NF4 codes of four pairs x[0..3] (|x| <= 1), packed as 8 nibbles (pair j
// -> nibbles 2j, 2j+1).  k = round(f(x) - 1/2) is the code or one less (f:
// the code-search polynomial) and code = k + (x > t[k]).  Adding 1.5 * 2^23
// leaves k in the low bits of the float, so the nibbles are accumulated
// straight from those bits and the constant part is removed once at the end.
// The table address is masked to the 16-entry table whatever the input.
QDEV uint32_t nf4_codes8(const float2 (&x)[4], const float2 (&P)[6], uint32_t t_addr) {
  uint32_t acc = 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float2 f = __ffma2_rn(P[5], x[j], P[4]);
    f = __ffma2_rn(f, x[j], P[3]);
    f = __ffma2_rn(f, x[j], P[2]);
    f = __ffma2_rn(f, x[j], P[1]);
    f = __ffma2_rn(f, x[j], P[0]);
    const float2 y = __fadd2_rn(f, make_float2(12582912.0f, 12582912.0f));
    const uint32_t ba = __float_as_uint(y.x), bb = __float_as_uint(y.y);
    acc += ba * (1u << (8 * j)) + bb * (1u << (8 * j + 4));
    const float ta = lds_f32(t_addr + ((ba << 2) & 0x3Cu));
    const float tb = lds_f32(t_addr + ((bb << 2) & 0x3Cu));
    if (x[j].x > ta) acc += 1u << (8 * j);
    if (x[j].y > tb) acc += 1u << (8 * j + 4);
  }
  return acc - kMagicBits * 0x11111111u;  // remove sum_i magic * 16^i (mod 2^32)
}

// Codes of four pairs x[0..3] for any 16-level table: a branch-free binary
// search over the 15 thresholds (code = number of thresholds below x), the
// thresholds read from shared memory (16 words in 16 banks: no conflicts).
// Used for the compared formats, whose levels have no fitted polynomial.
QDEV uint32_t search_codes8(const float2 (&x)[4], uint32_t t_addr) {
  uint32_t acc = 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float v = h ? x[j].y : x[j].x;
      uint32_t c = v > lds_f32(t_addr + 7u * 4u) ? 8u : 0u;
      c += v > lds_f32(t_addr + (c + 3u) * 4u) ? 4u : 0u;
      c += v > lds_f32(t_addr + (c + 1u) * 4u) ? 2u : 0u;
      c += v > lds_f32(t_addr + c * 4u) ? 1u : 0u;
      acc |= c << (8 * j + 4 * h);
    }
  }
  return acc;
}

// One CTA per 16384-weight group (256 blocks = one c1 scale), 256 threads;
// 4 threads share a 64-weight block, 16 weights (32 bytes) each, 4 rounds.
// kPoly: NF4's polynomial code search; otherwise the threshold search.
template <bool kPoly>
__global__ void __launch_bounds__(kQuantThreads) nf4_quantize_kernel(const uint16_t* __restrict__ W,
                                                                      int64_t n_blocks,
                                                                      uint2* __restrict__ codes,
                                                                      uint8_t* __restrict__ c2,
                                                                      float* __restrict__ c1, int* status,
                                                                      QuantParams qp, int codec) {
  __shared__ float s_t[16];
  __shared__ float s_absmax[kGroupBlocks];
  __shared__ float s_wmax[kQuantThreads / 32];
  __shared__ float s_wsum[kQuantThreads / 32];
  const bool e5m2 = codec == QLORA_SCALE_E5M2, mean = codec == QLORA_SCALE_E4M3_MEAN;
  const int t = threadIdx.x;
  if (t < 16) s_t[t] = t < 15 ? qp.t[t] : 2.0f;
  float2 P[6];
#pragma unroll
  for (int k = 0; k < 6; ++k) P[k] = make_float2(qp.poly[k], qp.poly[k]);
  const uint32_t t_addr = smem_u32(s_t);
  __syncthreads();

  const int64_t n_groups = (n_blocks + kGroupBlocks - 1) / kGroupBlocks;
  for (int64_t g = blockIdx.x; g < n_groups; g += gridDim.x) {
    const int64_t blk0 = g * kGroupBlocks;
    const int nblk = (int)min((int64_t)kGroupBlocks, n_blocks - blk0);
    // round i: unit u = i*256 + t holds 16 weights of block u/4 (part u%4)
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int u = i * kQuantThreads + t;
      if ((u >> 2) < nblk) {
        const uint4* p = reinterpret_cast<const uint4*>(W + (blk0 * 64 + (int64_t)u * 16));
        v[2 * i] = __ldg(p);
        v[2 * i + 1] = __ldg(p + 1);
      } else {
        v[2 * i] = v[2 * i + 1] = make_uint4(0, 0, 0, 0);
      }
    }
    uint32_t bad = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int u = i * kQuantThreads + t;
      const uint32_t w8[8] = {v[2 * i].x, v[2 * i].y, v[2 * i].z, v[2 * i].w,
                              v[2 * i + 1].x, v[2 * i + 1].y, v[2 * i + 1].z, v[2 * i + 1].w};
      // |w| max with NaN propagation (bf16x2), then over the 4 threads of the block
      __nv_bfloat162 m2 = __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w8[0]));
#pragma unroll
      for (int k = 1; k < 8; ++k) m2 = __hmax2_nan(m2, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w8[k])));
      const uint32_t mb = *reinterpret_cast<uint32_t*>(&m2);
      uint32_t m = max(mb & 0xFFFFu, mb >> 16);  // sign-cleared bits: integer order = magnitude, NaN highest
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      bad |= (m >= 0x7F80u) ? 1u : 0u;  // Inf or NaN in the block
      const float c = bf16_bits_to_float(m);
      if ((t & 3) == 0 && (u >> 2) < nblk) s_absmax[u >> 2] = c;
      const bool fast = c >= 0x1p-90f && c < 0x1p100f;
      uint32_t out[2];
      float2 x[2][4];
      if (__all_sync(0xFFFFFFFFu, fast)) {
        const float rc = __frcp_rn(c);
        const float2 rc2 = make_float2(rc, rc), cc = make_float2(c, c);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          x[k >> 2][k & 3] = ratio_fast(make_float2(__uint_as_float(w8[k] << 16), __uint_as_float(w8[k] & 0xFFFF0000u)),
                                        cc, rc2);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          x[k >> 2][k & 3] = make_float2(ratio_slow(__uint_as_float(w8[k] << 16), c),
                                         ratio_slow(__uint_as_float(w8[k] & 0xFFFF0000u), c));
      }
      if (kPoly) {
        out[0] = nf4_codes8(x[0], P, t_addr);
        out[1] = nf4_codes8(x[1], P, t_addr);
      } else {
        out[0] = search_codes8(x[0], t_addr);
        out[1] = search_codes8(x[1], t_addr);
      }
      if ((u >> 2) < nblk) codes[blk0 * 4 + u] = make_uint2(out[0], out[1]);
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (t & 31) == 0) report(status, QLORA_ERR_NONFINITE);
    __syncthreads();
    // second level: c1 = RN32(max c_b / 448), c2_b = E4M3(RN32(c_b / c1));
    // for E5M2 scale codes 57344 and E5M2.  Mean-centred: the group mean mu
    // (fp32 pairwise tree over the 256 slots, empty slots zero: the butterfly
    // of lane sums, then the eight warp sums pairwise), d_b = RN32(c_b - mu),
    // c1 = RN32(max |d_b| / 448), signed E4M3 codes of RN32(d_b / c1).
    const float cb = t < nblk ? s_absmax[t] : 0.0f;
    float d = cb, mu = 0.0f;
    if (mean) {
      float sum = cb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xFFFFFFFFu, sum, o));
      if ((t & 31) == 0) s_wsum[t >> 5] = sum;
      __syncthreads();
      const float s01 = __fadd_rn(s_wsum[0], s_wsum[1]), s23 = __fadd_rn(s_wsum[2], s_wsum[3]);
      const float s45 = __fadd_rn(s_wsum[4], s_wsum[5]), s67 = __fadd_rn(s_wsum[6], s_wsum[7]);
      const float total = __fadd_rn(__fadd_rn(s01, s23), __fadd_rn(s45, s67));
      mu = __fdiv_rn(total, (float)nblk);
      d = t < nblk ? __fsub_rn(cb, mu) : 0.0f;
    }
    float wm = fabsf(d);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xFFFFFFFFu, wm, o));
    if ((t & 31) == 0) s_wmax[t >> 5] = wm;
    __syncthreads();
    float gmax = s_wmax[0];
#pragma unroll
    for (int k = 1; k < kQuantThreads / 32; ++k) gmax = fmaxf(gmax, s_wmax[k]);
    const float c1v = __fdiv_rn(gmax, e5m2 ? 57344.0f : 448.0f);
    if (t == 0) {
      if (mean) reinterpret_cast<float2*>(c1)[g] = make_float2(c1v, mu);
      else c1[g] = c1v;
    }
    if (t < nblk) {
      uint8_t code = 0;
      if (c1v > 0.0f)
        code = (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(d, c1v), __NV_SATFINITE, e5m2 ? __NV_E5M2 : __NV_E4M3);
      c2[blk0 + t] = code;
    }
    __syncthreads();
  }
}

// doubleDequant: w^ = RNbf16(RN32(q[code] * RN32(dec(c2) * c1))).
// A thread turns 8 weights (one 32-bit code word) into one 16-byte bf16
// store per step; consecutive threads take consecutive words (coalesced), and
// 8 steps per loop trip keep 8 loads in flight per thread.
constexpr int kDeqSteps = 8;

__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint32_t* __restrict__ codes,
                                                          const uint8_t* __restrict__ c2,
                                                          const float* __restrict__ c1, int64_t n_chunks,
                                                          uint4* __restrict__ out, Nf4Tables tab, int codec) {
  const bool e5m2 = codec == QLORA_SCALE_E5M2, mean = codec == QLORA_SCALE_E4M3_MEAN;
  __shared__ float lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = tab.q[threadIdx.x];
  __syncthreads();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t c0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c0 < n_chunks; c0 += kDeqSteps * stride) {
    uint32_t cw[kDeqSteps];
    uint32_t s2[kDeqSteps];
    GroupScale s1[kDeqSteps];
#pragma unroll
    for (int u = 0; u < kDeqSteps; ++u) {
      const int64_t ci = c0 + u * stride;
      if (ci < n_chunks) {
        cw[u] = __ldcs(codes + ci);
        const int64_t blk = ci >> 3;
        s2[u] = __ldg(c2 + blk);
        s1[u] = load_group_scale(c1, blk >> 8, mean);
      }
    }
#pragma unroll
    for (int u = 0; u < kDeqSteps; ++u) {
      const int64_t ci = c0 + u * stride;
      if (ci < n_chunks) {
        const float chat = decode_scale(s2[u], s1[u], e5m2, mean);
        const float2 cc = make_float2(chat, chat);
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t b = cw[u] >> (8 * k);
          const float2 pr = __fmul2_rn(make_float2(lut[b & 15u], lut[(b >> 4) & 15u]), cc);
          o[k] = pack_bf16x2(pr.x, pr.y);
        }
        __stcs(out + ci, make_uint4(o[0], o[1], o[2], o[3]));
      }
    }
  }
}

__global__ void scale_to_bf16_kernel(const float* __restrict__ in, int64_t n, float s,
                                     __nv_bfloat16* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = __float2bfloat16_rn(__fmul_rn(in[i], s));
}

int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace

cudaError_t launch_quantize(const uint16_t* W, int64_t n_weights, uint8_t* codes, uint8_t* c2, float* c1,
                            int* status, int format, int scale_codec, cudaStream_t st) {
  const int64_t n_blocks = n_weights / 64;
  const int64_t n_groups = (n_blocks + kGroupBlocks - 1) / kGroupBlocks;
  QuantParams qp;
  const Nf4Tables& tab = code_tables(format);
  const bool poly = format == 0;
  if (poly && !tab.poly_ok) return cudaErrorNotSupported;
  for (int i = 0; i < 15; ++i) qp.t[i] = tab.t[i];
  for (int k = 0; k < 6; ++k) qp.poly[k] = poly ? tab.poly[k] : 0.0f;
  const int64_t grid = n_groups < (int64_t)num_sms() * 16 ? n_groups : (int64_t)num_sms() * 16;
  if (poly)
    nf4_quantize_kernel<true><<<(unsigned)grid, kQuantThreads, 0, st>>>(W, n_blocks, reinterpret_cast<uint2*>(codes),
                                                                         c2, c1, status, qp, scale_codec);
  else
    nf4_quantize_kernel<false><<<(unsigned)grid, kQuantThreads, 0, st>>>(W, n_blocks, reinterpret_cast<uint2*>(codes),
                                                                          c2, c1, status, qp, scale_codec);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* c2, const float* c1, int64_t n_weights,
                           uint16_t* out, int format, int scale_codec, cudaStream_t st) {
  const int64_t n_chunks = n_weights / 8;
  const int64_t want = (n_chunks + 256 * kDeqSteps - 1) / (256 * kDeqSteps);
  const int64_t cap = (int64_t)num_sms() * 8;
  const int64_t grid = want < cap ? (want > 0 ? want : 1) : cap;
  nf4_dequant_kernel<<<(unsigned)grid, 256, 0, st>>>(reinterpret_cast<const uint32_t*>(codes), c2, c1, n_chunks,
                                                     reinterpret_cast<uint4*>(out), code_tables(format), scale_codec);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_scale_to_bf16(const float* in, int64_t n, float s, uint16_t* out, cudaStream_t st) {
  const int64_t want = (n + 255) / 256;
  const int64_t grid = want < 4096 ? (want > 0 ? want : 1) : 4096;
  scale_to_bf16_kernel<<<(unsigned)grid, 256, 0, st>>>(in, n, s, reinterpret_cast<__nv_bfloat16*>(out));
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qnf4
