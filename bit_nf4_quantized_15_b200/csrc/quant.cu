// NF4 double quantisation (bf16 -> codes, c2, c1) and dequantisation
// (codes, c2, c1 -> bf16): the two HBM-bound passes.
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
  float t[15];  // decision thresholds, RD32 of the level midpoints
};

QDEV uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// x = RN32(w / c) for |w| <= c.  For c in [2^-90, 2^100) a correctly rounded
// reciprocal, one product and one fused correction step give the IEEE
// quotient's NF4 code for every bf16 pair (checked exhaustively); other
// finite scales use the IEEE division directly.  A zero or non-finite scale
// gives x = 0 (a non-finite block is reported through the status word).
QDEV float ratio(float w, float c, float rc, bool fast) {
  if (fast) {
    const float q0 = __fmul_rn(w, rc);
    const float e = __fmaf_rn(-q0, c, w);
    return __fmaf_rn(e, rc, q0);
  }
  return (c > 0.0f && c <= 3.402823466e38f) ? __fdiv_rn(w, c) : 0.0f;
}

// Code of x via a 129-entry bucket table: bucket j = RN(64 x) + 64 covers the
// closed interval [(j - 64.5)/64, (j - 63.5)/64], which holds at most one
// threshold (thresholds are >= 0.079 apart).  Entry: (that threshold or +2,
// number of thresholds below the bucket).
QDEV uint32_t nf4_code(float x, const float2* bucket) {
  const float y = __fmaf_rn(x, 64.0f, 12582976.0f);  // 1.5 * 2^23 + 64
  const int j = __float_as_int(y) - 0x4B400000;       // bits of 1.5 * 2^23
  const float2 b = bucket[min((unsigned)j, 128u)];     // |x| <= 1 keeps j in [0, 128]
  return (uint32_t)__float_as_int(b.y) + (x > b.x ? 1u : 0u);
}

__global__ void __launch_bounds__(kQuantThreads) nf4_quantize_kernel(const uint16_t* __restrict__ W,
                                                                      int64_t n_blocks,
                                                                      uint32_t* __restrict__ codes,
                                                                      uint8_t* __restrict__ c2,
                                                                      float* __restrict__ c1, int* status,
                                                                      QuantParams qp) {
  __shared__ float2 s_bucket[129];
  __shared__ float s_absmax[kGroupBlocks];
  __shared__ float s_wmax[kQuantThreads / 32];
  const int t = threadIdx.x;
  if (t < 129) {
    const float lo = ((float)t - 64.5f) * 0.015625f;
    const float hi = ((float)t - 63.5f) * 0.015625f;
    int base = 0;
    float th = 2.0f;
    for (int i = 0; i < 15; ++i) {
      if (qp.t[i] < lo) ++base;
      else if (qp.t[i] <= hi) th = qp.t[i];
    }
    s_bucket[t] = make_float2(th, __int_as_float(base));
  }
  __syncthreads();

  const int64_t n_groups = (n_blocks + kGroupBlocks - 1) / kGroupBlocks;
  for (int64_t g = blockIdx.x; g < n_groups; g += gridDim.x) {
    const int64_t blk0 = g * kGroupBlocks;
    const int nblk = (int)min((int64_t)kGroupBlocks, n_blocks - blk0);
    // 8 rounds; in round i thread t owns 8 consecutive weights of block
    // i*32 + t/8 (16-byte chunk i*256 + t of the group).
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ci = i * kQuantThreads + t;
      if ((ci >> 3) < nblk) v[i] = ld_stream_v4(W + (blk0 * 64 + (int64_t)ci * 8));
      else v[i] = make_uint4(0, 0, 0, 0);
    }
    uint32_t bad = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ci = i * kQuantThreads + t;
      const uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      uint32_t m2 = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t a = w4[k] & 0x7FFF7FFFu;  // |w| as sign-magnitude bits
        bad |= ((a & 0x7F800000u) == 0x7F800000u) | ((a & 0x7F80u) == 0x7F80u);
        m2 = __vmaxu2(m2, a);
      }
      uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
      const float c = bf16_bits_to_float(m);
      if ((t & 7) == 0 && (ci >> 3) < nblk) s_absmax[ci >> 3] = c;
      const bool fast = c >= 0x1p-90f && c < 0x1p100f;
      const float rc = fast ? __frcp_rn(c) : 0.0f;
      uint32_t packed = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float w0 = bf16_bits_to_float(w4[k] & 0xFFFFu);
        const float w1 = bf16_bits_to_float(w4[k] >> 16);
        const uint32_t q0 = nf4_code(ratio(w0, c, rc, fast), s_bucket);
        const uint32_t q1 = nf4_code(ratio(w1, c, rc, fast), s_bucket);
        packed |= (q0 | (q1 << 4)) << (8 * k);
      }
      if ((ci >> 3) < nblk) codes[blk0 * 8 + ci] = packed;
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (t & 31) == 0) report(status, QLORA_ERR_NONFINITE);
    __syncthreads();
    // second level: c1 = RN32(max c_b / 448), c2_b = E4M3(RN32(c_b / c1))
    float cb = t < nblk ? s_absmax[t] : 0.0f;
    float wm = cb;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xFFFFFFFFu, wm, o));
    if ((t & 31) == 0) s_wmax[t >> 5] = wm;
    __syncthreads();
    float gmax = s_wmax[0];
#pragma unroll
    for (int k = 1; k < kQuantThreads / 32; ++k) gmax = fmaxf(gmax, s_wmax[k]);
    const float c1v = __fdiv_rn(gmax, 448.0f);
    if (t == 0) c1[g] = c1v;
    if (t < nblk) {
      uint8_t code = 0;
      if (c1v > 0.0f) code = (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(cb, c1v), __NV_SATFINITE, __NV_E4M3);
      c2[blk0 + t] = code;
    }
    __syncthreads();
  }
}

// doubleDequant: w^ = RNbf16(RN32(q[code] * RN32(dec(c2) * c1))).
// Thread handles 8 weights (one 32-bit code word, one 16-byte output) per
// step, 4 steps per loop trip for memory-level parallelism.
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint32_t* __restrict__ codes,
                                                          const uint8_t* __restrict__ c2,
                                                          const float* __restrict__ c1, int64_t n_chunks,
                                                          uint4* __restrict__ out, Nf4Tables tab) {
  __shared__ float lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = tab.q[threadIdx.x];
  __syncthreads();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t c0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c0 < n_chunks; c0 += 4 * stride) {
    uint32_t cw[4];
    float chat[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t ci = c0 + u * stride;
      if (ci < n_chunks) {
        cw[u] = __ldcs(codes + ci);
        const int64_t blk = ci >> 3;
        chat[u] = decode_scale(__ldg(c2 + blk), __ldg(c1 + (blk >> 8)));
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t ci = c0 + u * stride;
      if (ci < n_chunks) {
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t b = cw[u] >> (8 * k);
          o[k] = pack_bf16x2(__fmul_rn(lut[b & 15u], chat[u]), __fmul_rn(lut[(b >> 4) & 15u], chat[u]));
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
                            int* status, cudaStream_t st) {
  const int64_t n_blocks = n_weights / 64;
  const int64_t n_groups = (n_blocks + kGroupBlocks - 1) / kGroupBlocks;
  QuantParams qp;
  const Nf4Tables& tab = nf4_tables();
  for (int i = 0; i < 15; ++i) qp.t[i] = tab.t[i];
  const int64_t grid = n_groups < (int64_t)num_sms() * 16 ? n_groups : (int64_t)num_sms() * 16;
  nf4_quantize_kernel<<<(unsigned)grid, kQuantThreads, 0, st>>>(W, n_blocks, reinterpret_cast<uint32_t*>(codes),
                                                                 c2, c1, status, qp);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* c2, const float* c1, int64_t n_weights,
                           uint16_t* out, cudaStream_t st) {
  const int64_t n_chunks = n_weights / 8;
  const int64_t want = (n_chunks + 1023) / 1024;
  const int64_t cap = (int64_t)num_sms() * 8;
  const int64_t grid = want < cap ? (want > 0 ? want : 1) : cap;
  nf4_dequant_kernel<<<(unsigned)grid, 256, 0, st>>>(reinterpret_cast<const uint32_t*>(codes), c2, c1, n_chunks,
                                                     reinterpret_cast<uint4*>(out), nf4_tables());
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
