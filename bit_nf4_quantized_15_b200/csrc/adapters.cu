// Adapter-side kernels around the QLoRA layer.
//
// * adapter_merge_kernel: W_merged = RNbf16(W^ + s (L1 L2)^T).  examadda
//   "QLoRA", "Practical Notes", third bullet: merging an adapter back into a
//   4-bit base is lossy, so the merge goes into the dequantised 16-bit weight
//   (re-quantising the result is a separate qlora_nf4_quantize call).  One
//   CTA per 128 x 128 tile of the [N, K] output: the rank-r product on
//   warp-level tensor-core MMAs (bf16 in, fp32 accumulate), the dequantised
//   weight W^ = RNbf16(RN32(q[code] . c^)) formed in the epilogue from the
//   tile's codes and block scales, one fused multiply-add
//   RN32(W^ + s . acc), one rounding to bf16, coalesced 16-byte stores
//   through shared memory.  The HBM traffic is the codes (0.5 B per weight)
//   and the output (2 B per weight); L1 and L2 tiles come from L2.
// * adamw_kernel: the optimizer step on the adapters whose state the paged
//   optimizer keeps in managed memory (nlp-lineage "QLoRA", section "The
//   idea", paged-optimizers bullet).  AdamW with decoupled weight decay,
//   every operation rounded to fp32 in a fixed order (no contraction into
//   fused multiply-adds), so the result is bit-for-bit reproducible.
#include "common.cuh"
#include "internal.h"

namespace qnf4 {
namespace {

constexpr int kMT = 128;       // tile rows (n) and columns (k)
constexpr int kOutRow = kMT * 2 + 16;  // output tile row (bytes), padded: rows fall in different banks
constexpr int kMThreads = 256;  // 8 warps: 2 (n) x 4 (k), 64 x 32 outputs each

struct MergeSmem {
  // byte offsets inside the dynamic window
  int a, b, codes, chat, out, total;
};

constexpr int kARow = kMT * 2 + 16;  // L2 tile row (128 n of one j, bytes), padded for ldmatrix

__host__ __device__ inline MergeSmem merge_smem(int rp) {
  MergeSmem s;
  const int brow = (rp + 8) * 2;         // padded L1 row (bytes)
  s.a = 0;                               // L2 tile  [rp j][128 n] bf16, as stored in L2
  s.b = s.a + rp * kARow;                // L1 tile  [128 k][rp] bf16
  s.codes = s.b + kMT * brow;            // [128 n][64] code bytes
  s.chat = s.codes + kMT * 64;           // c^ [128 n][2 blocks] fp32
  s.out = 0;                             // [128 n][128 k] bf16 (padded rows), reuses the window after the MMAs
  s.total = s.chat + kMT * 2 * 4;
  const int out_bytes = kMT * kOutRow;
  if (s.total < out_bytes) s.total = out_bytes;
  return s;
}

QDEV void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16-byte asynchronous copy global -> shared; src_bytes = 0 fills zeros.
QDEV void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
QDEV void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Four 8x8 bf16 matrices, transposed on the way: with the row addresses of
// matrix t/8 in threads 8(t/8) .. 8(t/8)+7, register i of thread t holds
// elements (2(t%4), t/4) and (2(t%4)+1, t/4) of matrix i as stored.
QDEV void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

__global__ void __launch_bounds__(kMThreads) adapter_merge_kernel(const uint8_t* __restrict__ codes,
                                                                   const uint8_t* __restrict__ c2,
                                                                   const float* __restrict__ c1, int codec,
                                                                   int64_t N, int64_t K,
                                                                   const uint16_t* __restrict__ L1,
                                                                   const uint16_t* __restrict__ L2, int r, float s,
                                                                   uint16_t* __restrict__ out, Nf4Tables tab) {
  extern __shared__ __align__(16) uint8_t msm[];
  const int rp = (r + 15) & ~15;  // rank padded to whole 16-wide MMA steps (zeros beyond r)
  const int brow = (rp + 8) * 2;
  const MergeSmem L = merge_smem(rp);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n0 = (int64_t)blockIdx.y * kMT, k0 = (int64_t)blockIdx.x * kMT;
  const int nv = (int)min((int64_t)kMT, N - n0), kv = (int)min((int64_t)kMT, K - k0);
  const uint32_t sbase = smem_u32(msm);
  __shared__ float q[16];
  if (tid < 16) q[tid] = tab.q[tid];

  // ---- stage with 16-byte asynchronous copies (zero-filled outside the
  // weight and beyond r): the L2 tile as stored ([j][n], 8 n per piece; N %
  // 8 == 0 keeps every piece inside or outside the weight), the L1 rows, the
  // code bytes; then one block scale per thread.
  for (int i = tid; i < rp * (kMT / 8); i += kMThreads) {
    const int j = i / (kMT / 8), c = i % (kMT / 8);
    const bool ok = j < r && c * 8 < nv;
    cp_async16(sbase + L.a + j * kARow + c * 16, ok ? (const void*)(L2 + (int64_t)j * N + n0 + c * 8) : (const void*)L2,
               ok ? 16u : 0u);
  }
  const int vpr = rp / 8;  // 16-byte pieces per padded L1 row
  for (int i = tid; i < kMT * vpr; i += kMThreads) {
    const int k = i / vpr, c = i % vpr;
    const bool ok = k < kv && c * 8 < r;
    cp_async16(sbase + L.b + k * brow + c * 16, ok ? (const void*)(L1 + (k0 + k) * r + c * 8) : (const void*)L1,
               ok ? 16u : 0u);
  }
  for (int i = tid; i < kMT * 4; i += kMThreads) {  // 64 code bytes per row: four 16-byte pieces
    const int n = i >> 2, c = i & 3;
    const bool ok = n < nv && c * 32 < kv;
    cp_async16(sbase + L.codes + n * 64 + c * 16, ok ? (const void*)(codes + ((n0 + n) * K + k0) / 2 + c * 16)
                                                     : (const void*)codes,
               ok ? 16u : 0u);
  }
  {
    const int n = tid >> 1, b = tid & 1;  // 256 threads: one (row, block) scale each
    float ch = 0.0f;
    if (n < nv && b * 64 < kv) {
      const int64_t f = ((n0 + n) * K + k0) / 64 + b;
      ch = decode_scale(__ldg(c2 + f), load_group_scale(c1, f >> 8, codec == QLORA_SCALE_E4M3_MEAN),
                        codec == QLORA_SCALE_E5M2, codec == QLORA_SCALE_E4M3_MEAN);
    }
    reinterpret_cast<float*>(msm + L.chat)[tid] = ch;
  }
  cp_async_wait_all();
  __syncthreads();

  // ---- MMAs: warp (wn, wk) owns rows 64 wn .. +63 and columns 32 wk .. +31
  const int wn = warp >> 2, wk = warp & 3;
  const int gr = lane >> 2, cq = lane & 3;
  float acc[4][4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[a][b][e] = 0.0f;
  // A = L2^T (rows n, reduction j) by transposing loads of the [j][n] tile:
  // matrix mq of a 16 x 16 step = rows n + 8 (mq & 1), reduction j + 8 (mq >> 1).
  const int mq = lane >> 3, mr = lane & 7;
  const uint32_t a_lane = sbase + L.a + (uint32_t)(((mq >> 1) * 8 + mr) * kARow + (64 * wn + (mq & 1) * 8) * 2);
  const uint8_t* Bs = msm + L.b + (32 * wk) * brow;
  for (int j0 = 0; j0 < rp; j0 += 16) {
    uint32_t af[4][4], bfr[4][2];
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
      ldmatrix_x4_trans(a_lane + (uint32_t)(j0 * kARow + mi * 32), af[mi][0], af[mi][1], af[mi][2], af[mi][3]);
#pragma unroll
    for (int ni = 0; ni < 4; ++ni) {
      const uint8_t* p = Bs + (8 * ni + gr) * brow + (j0 + 2 * cq) * 2;
      bfr[ni][0] = *reinterpret_cast<const uint32_t*>(p);
      bfr[ni][1] = *reinterpret_cast<const uint32_t*>(p + 16);
    }
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
      for (int ni = 0; ni < 4; ++ni)
        mma_16816(acc[mi][ni], af[mi][0], af[mi][1], af[mi][2], af[mi][3], bfr[ni][0], bfr[ni][1]);
  }

  // ---- epilogue: W^ from the codes, RN32(W^ + s acc), RNbf16, into the output tile.
  // The output tile may overlap the codes and scales (small ranks), so each
  // thread reads its code bytes and scales into registers before the barrier
  // after which the tile is written.
  uint32_t cb[4][2][4];  // code bytes: [mi][row half][ni]
  float chs[4][2];
#pragma unroll
  for (int mi = 0; mi < 4; ++mi)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = 64 * wn + 16 * mi + gr + 8 * h;
      chs[mi][h] = reinterpret_cast<const float*>(msm + L.chat)[n * 2 + (32 * wk) / 64];
#pragma unroll
      for (int ni = 0; ni < 4; ++ni) cb[mi][h][ni] = msm[L.codes + n * 64 + (32 * wk + 8 * ni + 2 * cq) / 2];
    }
  __syncthreads();
#pragma unroll
  for (int mi = 0; mi < 4; ++mi)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = 64 * wn + 16 * mi + gr + 8 * h;
#pragma unroll
      for (int ni = 0; ni < 4; ++ni) {
        const int k = 32 * wk + 8 * ni + 2 * cq;
        const uint32_t c = cb[mi][h][ni];
        const float w0 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(q[c & 15u], chs[mi][h])));
        const float w1 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(q[c >> 4], chs[mi][h])));
        const float v0 = __fmaf_rn(s, acc[mi][ni][2 * h], w0);
        const float v1 = __fmaf_rn(s, acc[mi][ni][2 * h + 1], w1);
        *reinterpret_cast<uint32_t*>(msm + L.out + n * kOutRow + k * 2) = pack_bf16x2(v0, v1);
      }
    }
  __syncthreads();
  for (int i = tid; i < kMT * (kMT / 8); i += kMThreads) {  // 16-byte pieces, row-major
    const int n = i / (kMT / 8), c = i % (kMT / 8);
    if (n < nv && c * 8 < kv)
      *reinterpret_cast<uint4*>(out + (n0 + n) * K + k0 + c * 8) =
          *reinterpret_cast<const uint4*>(msm + L.out + n * kOutRow + c * 16);
  }
}

struct AdamScalars {
  float lr, b1, omb1, b2, omb2, eps, wd, bc1, bc2;
};

QDEV float adam_one(float& p, float g, float& m, float& v, const AdamScalars& c) {
  m = __fadd_rn(__fmul_rn(c.b1, m), __fmul_rn(c.omb1, g));
  v = __fadd_rn(__fmul_rn(c.b2, v), __fmul_rn(__fmul_rn(c.omb2, g), g));
  const float mhat = __fdiv_rn(m, c.bc1);
  const float vhat = __fdiv_rn(v, c.bc2);
  const float denom = __fadd_rn(__fsqrt_rn(vhat), c.eps);
  const float upd = __fadd_rn(__fdiv_rn(mhat, denom), __fmul_rn(c.wd, p));
  p = __fsub_rn(p, __fmul_rn(c.lr, upd));
  return p;
}

// Four parameters per thread and step (16-byte accesses); the tail of n % 4
// elements by thread 0 of the grid's first block.
__global__ void __launch_bounds__(256) adamw_kernel(float* __restrict__ p, uint16_t* __restrict__ pb,
                                                    const float* __restrict__ g, float* __restrict__ m,
                                                    float* __restrict__ v, int64_t n, AdamScalars c) {
  const int64_t n4 = n / 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 P = reinterpret_cast<float4*>(p)[i];
    const float4 G = __ldg(reinterpret_cast<const float4*>(g) + i);
    float4 Mv = reinterpret_cast<float4*>(m)[i];
    float4 Vv = reinterpret_cast<float4*>(v)[i];
    adam_one(P.x, G.x, Mv.x, Vv.x, c);
    adam_one(P.y, G.y, Mv.y, Vv.y, c);
    adam_one(P.z, G.z, Mv.z, Vv.z, c);
    adam_one(P.w, G.w, Mv.w, Vv.w, c);
    reinterpret_cast<float4*>(p)[i] = P;
    reinterpret_cast<float4*>(m)[i] = Mv;
    reinterpret_cast<float4*>(v)[i] = Vv;
    if (pb) reinterpret_cast<uint2*>(pb)[i] = make_uint2(pack_bf16x2(P.x, P.y), pack_bf16x2(P.z, P.w));
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (int64_t i = n4 * 4; i < n; ++i) {
      float P = p[i], Mv = m[i], Vv = v[i];
      adam_one(P, g[i], Mv, Vv, c);
      p[i] = P;
      m[i] = Mv;
      v[i] = Vv;
      if (pb) pb[i] = (uint16_t)(pack_bf16x2(P, 0.0f) & 0xFFFFu);
    }
  }
}

int num_sms_now() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace

size_t merge_smem_bytes(int r) { return (size_t)merge_smem((r + 15) & ~15).total; }

cudaError_t launch_adapter_merge(const uint8_t* codes, const uint8_t* c2, const float* c1, int format, int scale_codec,
                                 int64_t N, int64_t K, const uint16_t* L1, const uint16_t* L2, int r, float s,
                                 uint16_t* out, cudaStream_t st) {
  const int smem = (int)merge_smem_bytes(r);
  cudaError_t err = cudaFuncSetAttribute(adapter_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  dim3 grid((unsigned)((K + kMT - 1) / kMT), (unsigned)((N + kMT - 1) / kMT));
  adapter_merge_kernel<<<grid, kMThreads, smem, st>>>(codes, c2, c1, scale_codec, N, K, L1, L2, r, s, out,
                                                       code_tables(format));
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_adamw(float* p, uint16_t* pb, const float* g, float* m, float* v, int64_t n, const float* sc,
                         cudaStream_t st) {
  AdamScalars c{sc[0], sc[1], sc[2], sc[3], sc[4], sc[5], sc[6], sc[7], sc[8]};
  const int64_t want = (n / 4 + 255) / 256;
  const int64_t cap = (int64_t)num_sms_now() * 8;
  const int64_t grid = want < 1 ? 1 : (want < cap ? want : cap);
  adamw_kernel<<<(unsigned)grid, 256, 0, st>>>(p, pb, g, m, v, n, c);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qnf4
