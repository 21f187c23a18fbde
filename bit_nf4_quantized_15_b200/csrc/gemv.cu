// Few-token forward (M <= 16): the dequant-GEMV regime, where the time is the
// stream of 4-bit weights from HBM (0.516 byte per weight) and the tensor
// cores have almost nothing to do.
//
//   Y = RNbf16( X . W^T  +  RNbf16(s.T) . L2 ),   T = X . L1
//
// nlp-lineage "QLoRA" milestone page, section "The idea": the layer equation
// (the 4-bit weight is dequantised to bf16 and multiplied, the adapters stay
// bf16).  Three kernels, chained with programmatic dependent launch so each
// one's launch overlaps the previous one's run:
//
// * lora_t_partial_kernel: T = X.L1 in K slices on CUDA cores (fp32).
// * nf4_gemv_kernel: one CTA per SM holding three independent stream-K
//   workers.  The work is the list of units (128-row tile of W, 256-wide k
//   range) in row-tile-major order, cut into equal contiguous runs, one per
//   worker, so every SM streams the same number of weight bytes whatever the
//   shape.  A worker is four warps with a two-stage TMA ring (16 KB code tile
//   of 128-byte rows + 8 KB X tile of 16 tokens, rows beyond M zero-filled).
//   Each warp owns 32 rows of the tile and multiplies them with warp-level
//   tensor-core MMAs (m16n8k16, bf16 in, fp32 accumulate in registers):
//   the dequantised weights are produced directly as A fragments, so they
//   never go through shared or tensor memory, and a segment's partial (a
//   maximal run inside one row tile) is written straight from registers.
//   Single-thread tcgen05 MMAs were measured to be the bottleneck here: with
//   N = 16 each UMMA carries 128 x 16 weights and costs about as much to
//   issue as a 128 x 256 one.
//   The k order inside each 64-wide block is permuted identically in A and
//   B (a sum is order-free up to rounding, and both operands see the same
//   permutation): thread (g, c) of the warp takes code bytes 8c .. 8c+7 of
//   its rows, i.e. k = 16c .. 16c+15, handing k-step s the pairs 2s (A
//   columns 2c, 2c+1) and 2s+1 (columns 2c+8, 2c+9), and reads the matching
//   X values k = 16c+4s .. 16c+4s+3 as one 8-byte load.
//   The block scale is applied after the product: a weight row's 64-wide
//   block contributes c^ . sum_k x[k] q[code_k] (one fp32 multiply-add per
//   accumulator element after the block's four MMAs, which start from zero),
//   the same sum as sum_k x[k] (q[code_k] c^) up to rounding, within the
//   layer's stated tolerance.  So the A operand is the level itself, and a
//   32 KB shared-memory table of code pairs serves the whole kernel: entry e
//   (one code byte: element 2j in the low nibble, 2j+1 in the high one) holds
//   the bf16 pair (RNbf16(q[e & 15]), RNbf16(q[e >> 4])), one copy per lane at
//   a 4-byte offset so a warp's loads fall in 32 different banks.  Per code
//   byte: one byte permute forms the address and one 4-byte load fetches the
//   A-fragment register for both weights.
//   Warp 0: lanes 0..2 are the three TMA producers; the last warp sums this
//   CTA's share of the T partials.
// * gemv_finish_kernel: per row, the row tile's segment partials in worker
//   order (deterministic) plus the LoRA term, rounded to bf16.
#include "common.cuh"
#include "internal.h"

namespace qnf4 {
namespace {

constexpr int kWG = 3;                     // stream-K workers per CTA
constexpr int kWS = 2;                     // ring stages per worker
constexpr int kNS = kWG * kWS;             // stages per CTA
constexpr int kUnitKB = 4;                 // 64-wide k blocks per unit
constexpr int kCodeBytes = 16384;          // 128 rows x 128 bytes (256 codes)
constexpr int kXBytes = 8192;              // 16 tokens x 256 bf16: one 3-D box of 4 x (16 x 64)
constexpr int kStageBytes = kCodeBytes + kXBytes;
// A worker's warps each own kRG 16-row groups of the 128-row tile.
constexpr int kRG = 1;
constexpr int kWW = 8 / kRG;                  // warps per worker
// Warps: 0 producers, 1 .. kWW*kWG workers, last: T reduction.
constexpr int kWarpT = 1 + kWW * kWG;
constexpr int kGThreads = 32 * (kWarpT + 1);
constexpr int kTabBytes = 65536;           // 256 pairs x 256-byte lines (32 lanes x 4 bytes used)
constexpr int kBarBytes = 1024;
// Shared window: two stages and the barriers, then (at the next 64 KB
// boundary, so the table's address bits 16.. come from one register in the
// byte permute) the pair table, then the other four stages.
constexpr int kFrontStages = 2;
constexpr uint32_t kFrontBytes = kFrontStages * kStageBytes + kBarBytes;
// With the dynamic window starting below 15 KB (it starts at 0 or 1 KB), the
// layout ends at 64 KB + 64 KB + 4 stages = 224 KB; the kernel checks the fit.
constexpr uint32_t kGemvSmemMin = 65536 + kTabBytes + (kNS - kFrontStages) * kStageBytes;
static_assert(kFrontBytes <= 65536 - 15360, "front region must fit below the table");

struct GemvSmem {
  uint32_t base;  // stages 0 .. kFrontStages-1 (codes, then X)
  uint8_t* raw;
  uint32_t raw_addr;
  uint64_t* bars;
  volatile int* abort_flag;
  uint32_t tab;
  bool fits;
};

QDEV GemvSmem carve(uint8_t* raw_ptr, uint32_t smem_bytes) {
  GemvSmem g;
  const uint32_t raw = smem_u32(raw_ptr);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t bars = base + kFrontStages * kStageBytes;
  const uint32_t tab = (bars + kBarBytes + 0xFFFFu) & ~0xFFFFu;
  g.base = base;
  const uint32_t end = tab + kTabBytes + (kNS - kFrontStages) * kStageBytes;
  g.fits = end - raw <= smem_bytes && tab <= 0x00FF0000u;
  g.raw = raw_ptr;
  g.raw_addr = raw;
  g.bars = reinterpret_cast<uint64_t*>(raw_ptr + (bars - raw));
  g.abort_flag = reinterpret_cast<volatile int*>(g.bars + 64);
  g.tab = tab;
  return g;
}

// Barriers of worker g: full[kWS] (TMA bytes), empty[kWS] (one arrival per warp).
QDEV uint64_t* bar_full(const GemvSmem& s, int g, int j) { return s.bars + g * 2 * kWS + j; }
QDEV uint64_t* bar_empty(const GemvSmem& s, int g, int j) { return s.bars + g * 2 * kWS + kWS + j; }
// Shared-window address of ring stage st (0 .. kNS-1).
QDEV uint32_t stage_addr(const GemvSmem& s, int st) {
  return st < kFrontStages ? s.base + (uint32_t)(st * kStageBytes)
                           : s.tab + kTabBytes + (uint32_t)((st - kFrontStages) * kStageBytes);
}

// The worker whose run holds unit u (runs: [w*U/W, (w+1)*U/W)).
__host__ __device__ __forceinline__ int worker_of(int64_t u, int64_t U, int W) {
  return (int)(((u + 1) * (int64_t)W - 1) / U);
}

QDEV uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// bf16x2 of code byte k (0..3) of word w: RNbf16(q[lo]) low half,
// RNbf16(q[hi]) high half.  lanereg = table address bits 16..23 in byte 2,
// lane * 4 in byte 0; the code byte becomes address byte 1.
QDEV uint32_t pair_lookup(uint32_t w, int k, uint32_t lanereg) {
  const uint32_t addr = __byte_perm(w, lanereg, 0x7604u | ((uint32_t)k << 4));
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

QDEV void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

QDEV bool warp_wait_g(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status, int lane) {
  int ok = 1;
  if (lane == 0) ok = mbar_wait(bar, parity, abort_flag, status) ? 1 : 0;
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  if (ok) mbar_test_wait(smem_u32(bar), parity);
  return ok != 0;
}

QDEV void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
QDEV void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Block scales of unit (rt, un) for one weight row of the tile: the four
// E4M3 codes packed in one word, and the c1 of the first and the last k
// block (four consecutive blocks cross at most one 256-block group).
struct RowScales {
  uint32_t c2;
  GroupScale ga, gb;  // groups of the unit's first and last block
};
// Issued one unit ahead of use.  The four codes come as one 32-bit load
// when they are 4-byte aligned (K a multiple of 256 makes every row's unit
// aligned), so no instruction consumes the loaded values before the next
// unit: packing bytes right after their loads would stall the warp for the
// whole memory latency at the prefetch.
QDEV RowScales load_row_scales(const GemvArgs& a, int rt, int un, int rl) {
  RowScales s{0u, GroupScale{0.0f, 0.0f}, GroupScale{0.0f, 0.0f}};
  const int64_t n = (int64_t)rt * 128 + rl;
  if (n >= a.N) return s;
  const int kb0 = un * kUnitKB;
  const int64_t f0 = n * a.kbt + kb0;
  const int nkb = min(kUnitKB, a.kbt - kb0);
  if (nkb == kUnitKB && (f0 & 3) == 0) {
    s.c2 = __ldg(reinterpret_cast<const uint32_t*>(a.c2 + f0));
  } else {
#pragma unroll
    for (int q = 0; q < kUnitKB; ++q)
      if (q < nkb) s.c2 |= (uint32_t)__ldg(a.c2 + f0 + q) << (8 * q);
  }
  s.ga = load_group_scale(a.c1, f0 >> 8, a.c1_mean != 0);
  s.gb = load_group_scale(a.c1, (f0 + nkb - 1) >> 8, a.c1_mean != 0);
  return s;
}
// c^ = RN32(dec(c2) . c1) of the unit's four k blocks for one row, whose
// first block has flat index f0 (block q lies in the next c1 group when
// (f0 mod 256) + q >= 256).  Two codes per conversion: an E4M3 pair through
// the hardware fp8x2 -> f16x2 conversion, an E5M2 byte as the high byte of
// an fp16; both exact.
QDEV void row_chats(const RowScales& s, int64_t f0, bool e5m2, bool mean, float (&out)[kUnitKB]) {
  float2 v01, v23;
  if (e5m2) {
    const uint32_t b01 = __byte_perm(s.c2, 0u, 0x1404u), b23 = __byte_perm(s.c2, 0u, 0x3424u);
    v01 = __half22float2(*reinterpret_cast<const __half2*>(&b01));
    v23 = __half22float2(*reinterpret_cast<const __half2*>(&b23));
  } else {
    const __half2_raw h01 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(s.c2 & 0xFFFFu), __NV_E4M3);
    const __half2_raw h23 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(s.c2 >> 16), __NV_E4M3);
    v01 = __half22float2(__half2(h01));
    v23 = __half22float2(__half2(h23));
  }
  const int g0 = (int)(f0 & 255);
  const float v[kUnitKB] = {v01.x, v01.y, v23.x, v23.y};
#pragma unroll
  for (int q = 0; q < kUnitKB; ++q) {
    const GroupScale& gs = g0 + q < 256 ? s.ga : s.gb;
    const float p = __fmul_rn(v[q], gs.c1);
    out[q] = mean ? __fadd_rn(p, gs.mu) : p;  // mean-centred codec: + group mean, rounded again
  }
}

// NT = 8-token column tiles (1 for M <= 8, 2 for M <= 16).
template <int NT>
__global__ void __launch_bounds__(kGThreads, 1) nf4_gemv_kernel(const __grid_constant__ GemvArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const GemvSmem S = carve(smem_raw, args.smem_bytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (!S.fits) {  // shared-window layout not as planned: refuse, uniformly
    if (tid == 0) report(args.status, QLORA_ERR_CUDA);
    return;
  }
  const int G = gridDim.x, c = blockIdx.x;
  const int W = G * kWG;
  const int64_t U = args.units;
  const int upr = args.upr;

  if (tid == 0) {
    for (int g = 0; g < kWG; ++g)
      for (int j = 0; j < kWS; ++j) {
        mbar_init(bar_full(S, g, j), 1);
        mbar_init(bar_empty(S, g, j), kWW);
      }
    *S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&args.tmCodes);
    tma_prefetch_desc(&args.tmX);
  }
  // Pair table: entry e, lane l at tab + e*256 + l*4.
  for (int idx = tid; idx < 256 * 32; idx += kGThreads) {
    const int e = idx >> 5, l = idx & 31;
    const uint32_t v = pack_bf16x2(args.q[e & 15], args.q[e >> 4]);
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(S.tab + (uint32_t)(e * 256 + l * 4)), "r"(v) : "memory");
  }
  __syncthreads();
  // The finish kernel may be launched now: it reads this kernel's results
  // only after griddepcontrol.wait, and its launch latency overlaps the GEMV.
  grid_dep_launch();

  if (warp == 0) {
    // ------------------------------------ producers: one lane per ring stage
    // (lane 2g + j fills stage j of worker g; they poll with a short sleep,
    // so their turns in the warp cost nothing measurable here)
    if (lane < kWG * kWS) {
      const int g = lane / kWS, wk = c * kWG + g;
      const int64_t u0 = (int64_t)wk * U / W, u1 = (int64_t)(wk + 1) * U / W;
      const int nu = (int)(u1 - u0);
      int issued = 0;
      for (int i = lane % kWS; i < nu; i += kWS) {
        const int j = i % kWS;
        if (!mbar_wait_backoff(bar_empty(S, g, j), ((uint32_t)(i / kWS) & 1u) ^ 1u, S.abort_flag, args.status, 128))
          break;
        const int64_t u = u0 + i;
        const int rt = (int)(u / upr), un = (int)(u % upr);
        const uint32_t st = stage_addr(S, kWS * g + j);
        uint8_t* sp = S.raw + (st - S.raw_addr);
        mbar_arrive_expect_tx(bar_full(S, g, j), kCodeBytes + kXBytes);
        tma_load_2d(sp, &args.tmCodes, bar_full(S, g, j), un * 128, rt * 128);
        // the unit's four 64-wide X blocks in one box (blocks beyond K read as zeros)
        tma_load_3d(sp + kCodeBytes, &args.tmX, bar_full(S, g, j), 0, 0, un * kUnitKB);
        issued = i + 1;
      }
      if (*S.abort_flag && issued > 0) {  // let this lane's last load land before exit
        const int i = issued - 1;
        mbar_wait_drain(bar_full(S, g, i % kWS), (uint32_t)(i / kWS) & 1u, 10000000ull);
      }
    }
  } else if (warp == kWarpT) {
    // ------------------------------------------------------ T reduction
    // This CTA's share of T = sum_p Tp[p] (fixed order): T saved for the
    // backward, RNbf16(s.T) for the finish kernel.  The T partials come from
    // the previous kernel of the stream.
    grid_dep_wait();
    const int E = args.M * args.r, P = args.t_slices;
    const int e_hi = (int)((int64_t)(c + 1) * E / G);
    for (int e = (int)((int64_t)c * E / G) + lane; e < e_hi; e += 32) {
      const int m = e / args.r, jj = e % args.r;
      const float* src = args.tp + (int64_t)m * 128 + jj;
      float T = 0.0f;
      for (int p0 = 0; p0 < P; p0 += 8) {  // eight loads in flight, sum in slice order
        float v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = p0 + k < P ? __ldg(src + (int64_t)(p0 + k) * 16 * 128) : 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (p0 + k < P) T += v[k];
      }
      args.T_save[e] = T;
      args.sTw[m * 128 + jj] = __bfloat162float(__float2bfloat16_rn(__fmul_rn(args.s, T)));
    }
  } else {
    // ------------------------------------------------- worker warps
    const int g = (warp - 1) / kWW, wk = c * kWG + g, wq = (warp - 1) % kWW;
    const int gr = lane >> 2, cq = lane & 3;  // fragment row / column quad
    // tile rows of this thread: kRG 16-row groups, rows gr and gr + 8 of each
    int rows[2 * kRG];
#pragma unroll
    for (int i = 0; i < 2 * kRG; ++i) rows[i] = wq * 16 * kRG + (i >> 1) * 16 + (i & 1) * 8 + gr;
    const uint32_t lanereg = (S.tab & 0x00FF0000u) | (uint32_t)(lane * 4);
    const int64_t u0 = (int64_t)wk * U / W, u1 = (int64_t)(wk + 1) * U / W;
    const int nu = (int)(u1 - u0);
    float acc[kRG][NT][4];
#pragma unroll
    for (int a = 0; a < kRG; ++a)
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[a][t][e] = 0.0f;
    RowScales sc[2 * kRG];
    if (nu > 0) {
#pragma unroll
      for (int i = 0; i < 2 * kRG; ++i) sc[i] = load_row_scales(args, (int)(u0 / upr), (int)(u0 % upr), rows[i]);
    }
    bool aborted = false;
    for (int i = 0; i < nu; ++i) {
      const int64_t u = u0 + i;
      const int rt = (int)(u / upr), un = (int)(u % upr);
      const bool seg_end = i == nu - 1 || un == upr - 1;
      float chs[2 * kRG][kUnitKB];  // c^ of this unit's blocks, per thread row
#pragma unroll
      for (int r = 0; r < 2 * kRG; ++r)
        row_chats(sc[r], ((int64_t)rt * 128 + rows[r]) * args.kbt + (int64_t)un * kUnitKB, args.c2_e5m2 != 0,
                  args.c1_mean != 0, chs[r]);
      if (i + 1 < nu) {
#pragma unroll
        for (int r = 0; r < 2 * kRG; ++r) sc[r] = load_row_scales(args, (int)((u + 1) / upr), (int)((u + 1) % upr), rows[r]);
      }
      const int j = i % kWS;
      if (!aborted && !warp_wait_g(bar_full(S, g, j), (uint32_t)(i / kWS) & 1u, S.abort_flag, args.status, lane))
        aborted = true;
      if (!aborted) {
        const uint32_t st = stage_addr(S, kWS * g + j);
#pragma unroll
        for (int q = 0; q < kUnitKB; ++q) {
          // (blocks beyond K in the last unit of a row: zero codes and X from
          // the TMA fill, zero scales, so they add nothing; no branch keeps
          // the four blocks unrolled and interleaved)
          // X fragments of the four k-steps: token n = 8t + gr, k = 16cq + 4s .. +3
          uint2 xb[NT][4];
          const uint32_t xt = st + kCodeBytes + (uint32_t)q * 2048;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const int n = 8 * t + gr;
#pragma unroll
            for (int s = 0; s < 4; ++s)
              xb[t][s] = lds64(xt + (uint32_t)n * 128 + ((((uint32_t)(2 * cq + (s >> 1))) ^ (uint32_t)(n & 7)) << 4) +
                               8u * (uint32_t)(s & 1));
          }
#pragma unroll
          for (int h = 0; h < kRG; ++h) {  // 16-row group h: rows[2h] (gr) and rows[2h+1] (gr + 8)
            uint2 cw[2];
            float ch[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int rl = rows[2 * h + e];
              cw[e] = lds64(st + (uint32_t)rl * 128 +
                            ((((uint32_t)(2 * q + (cq >> 1))) ^ (uint32_t)(rl & 7)) << 4) + 8u * (uint32_t)(cq & 1));
              ch[e] = chs[2 * h + e][q];
            }
            float blk[NT][4];
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
              for (int e = 0; e < 4; ++e) blk[t][e] = 0.0f;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
              // code bytes 2s and 2s+1 of the thread's 8: word s >> 1, bytes 2(s&1), 2(s&1)+1
              const uint32_t w0 = (s < 2) ? cw[0].x : cw[0].y;
              const uint32_t w1 = (s < 2) ? cw[1].x : cw[1].y;
              const int k0 = 2 * (s & 1);
              const uint32_t a0 = pair_lookup(w0, k0, lanereg);
              const uint32_t a1 = pair_lookup(w1, k0, lanereg);
              const uint32_t a2 = pair_lookup(w0, k0 + 1, lanereg);
              const uint32_t a3 = pair_lookup(w1, k0 + 1, lanereg);
#pragma unroll
              for (int t = 0; t < NT; ++t) mma_bf16_16816(blk[t], a0, a1, a2, a3, xb[t][s].x, xb[t][s].y);
            }
            // the block's scale: accumulator elements 0, 1 are row gr, 2, 3 row gr + 8
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[h][t][e] = __fmaf_rn(blk[t][e], ch[e >> 1], acc[h][t][e]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty(S, g, j));  // this warp is done with the stage
      if (seg_end) {
        if (!aborted) {
          const int jw = wk - worker_of((int64_t)rt * upr, U, W);
          if (jw < 0 || jw >= args.maxc) {
            if (lane == 0) report(args.status, QLORA_ERR_CUDA);
          } else {
            float* base = args.part + ((int64_t)rt * args.maxc + jw) * (16 * 128);
#pragma unroll
            for (int h = 0; h < kRG; ++h)
#pragma unroll
              for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int m = 8 * t + 2 * cq + (e & 1);
                  const int rl = rows[2 * h + (e >> 1)];
                  if (m < args.M) base[m * 128 + rl] = acc[h][t][e];
                }
          }
        }
#pragma unroll
        for (int a = 0; a < kRG; ++a)
#pragma unroll
          for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[a][t][e] = 0.0f;
      }
    }
  }

}

// T partials: Tp[p][m][j] = sum over the k of slice p of X[m,k] L1[k,j], fp32,
// fixed order, m < MB (M <= MB).  Slice p = k blocks [p*bps, (p+1)*bps),
// walked in chunks of 256 rows staged in shared memory with every 16-byte
// load of a chunk issued before the first use.  Thread t: column pair
// jp = t % (r/2) and k lane kl = t / (r/2) (rows kl, kl + nkl, ...); the k
// lanes' sums are added in lane order at the end.
constexpr int kTChunk = 256;  // rows of L1 per staged chunk
template <int MB>
__global__ void __launch_bounds__(256) lora_t_partial_kernel(const uint16_t* __restrict__ X,
                                                             const uint16_t* __restrict__ L1, int M, int64_t K,
                                                             int r, int bps, float* __restrict__ tp) {
  extern __shared__ __align__(16) uint8_t tsm[];
  uint16_t* sL = reinterpret_cast<uint16_t*>(tsm);                    // [kTChunk][r]
  uint16_t* sX = reinterpret_cast<uint16_t*>(tsm + kTChunk * r * 2);  // [16][kTChunk]
  float* red = reinterpret_cast<float*>(tsm);                          // reused after the last chunk
  grid_dep_launch();  // the GEMV kernel may start at once: it reads Tp only later
  const int p = blockIdx.x, t = threadIdx.x;
  const int64_t k_lo = (int64_t)p * bps * 64;
  const int64_t k_hi = min((int64_t)(p + 1) * bps * 64, K);
  const int r2 = r / 2, nkl = 256 / r2;
  const int jp = t % r2, kl = t / r2;
  float acc[MB][2];
#pragma unroll
  for (int i = 0; i < MB; ++i) acc[i][0] = acc[i][1] = 0.0f;
  for (int64_t k0 = k_lo; k0 < k_hi; k0 += kTChunk) {
    const int rows = (int)min((int64_t)kTChunk, k_hi - k0);  // a multiple of 64
    const int nL = rows * r / 8, nX = M * rows / 8;            // 16-byte pieces
    const uint4* gL = reinterpret_cast<const uint4*>(L1 + k0 * r);
    for (int i = t; i < nL; i += 256) reinterpret_cast<uint4*>(sL)[i] = __ldg(gL + i);
    for (int i = t; i < nX; i += 256) {
      const int m = i / (rows / 8), cc = i % (rows / 8);
      reinterpret_cast<uint4*>(sX + m * kTChunk)[cc] =
          __ldg(reinterpret_cast<const uint4*>(X + (int64_t)m * K + k0) + cc);
    }
    __syncthreads();
    if (kl < nkl) {
      for (int k = kl; k < rows; k += nkl) {
        const uint32_t lw = reinterpret_cast<const uint32_t*>(sL + k * r)[jp];
        const float l0 = bf16_bits_to_float(lw & 0xFFFFu), l1 = bf16_bits_to_float(lw >> 16);
#pragma unroll
        for (int m = 0; m < MB; ++m) {
          if (m < M) {
            const float x = bf16_bits_to_float(sX[m * kTChunk + k]);
            acc[m][0] = __fmaf_rn(x, l0, acc[m][0]);
            acc[m][1] = __fmaf_rn(x, l1, acc[m][1]);
          }
        }
      }
    }
    __syncthreads();
  }
  // red[kl][m][j] (at most 256 x 32 floats: nkl * MB * r <= 256/r2 * 16 * 2 r2)
  if (kl < nkl) {
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      red[(kl * MB + m) * r + 2 * jp] = acc[m][0];
      red[(kl * MB + m) * r + 2 * jp + 1] = acc[m][1];
    }
  }
  __syncthreads();
  for (int idx = t; idx < M * r; idx += 256) {
    const int m = idx / r, j = idx % r;
    float sum = 0.0f;
    for (int q = 0; q < nkl; ++q) sum += red[(q * MB + m) * r + j];
    tp[((int64_t)p * 16 + m) * 128 + j] = sum;
  }
}

// Y for 32 weight rows per CTA (512 threads), tokens m < MB (M <= MB).
// Warp w sums the row tile's partials of contributors j = w, w + 16, ...
// (all of a warp's loads in flight together) and the LoRA products of
// adapter columns j = w, w + 16, ...; the sixteen warps' sums are then added
// in warp order (fixed, so the result is repeatable).
constexpr int kFinWarps = 16;
template <int MB>
__global__ void __launch_bounds__(32 * kFinWarps) gemv_finish_kernel(const float* __restrict__ part,
                                                                    const float* __restrict__ sTw,
                                                                    const uint16_t* __restrict__ L2, int M,
                                                                    int64_t N, int r, int upr, int64_t U, int W,
                                                                    int maxc, uint16_t* __restrict__ Y) {
  __shared__ __align__(16) float sT[16 * 128];
  __shared__ float red[kFinWarps][MB][32];
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int64_t n0 = (int64_t)blockIdx.x * 32, n = n0 + lane;
  const int rt = (int)(n0 / 128), rl = (int)(n % 128);
  const bool valid = n < N;
  // L2 first: it does not depend on the previous kernels (r <= 128: at most 8 columns per warp)
  float l2v[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int j = w + kFinWarps * q;
    l2v[q] = (valid && j < r) ? bf16_bits_to_float(__ldg(L2 + (int64_t)j * N + n)) : 0.0f;
  }
  grid_dep_wait();
  for (int idx = t * 4; idx < M * 128; idx += 32 * kFinWarps * 4)  // 16-byte pieces
    *reinterpret_cast<float4*>(sT + idx) = __ldcg(reinterpret_cast<const float4*>(sTw + idx));
  const int c_lo = worker_of((int64_t)rt * upr, U, W);
  const int cnt = min(worker_of((int64_t)(rt + 1) * upr - 1, U, W) - c_lo + 1, maxc);
  float acc[MB];
#pragma unroll
  for (int m = 0; m < MB; ++m) acc[m] = 0.0f;
  for (int j = w; j < cnt; j += kFinWarps) {
    const float* src = part + ((int64_t)rt * maxc + j) * (16 * 128) + rl;
    float v[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) v[m] = m < M ? __ldcg(src + m * 128) : 0.0f;
#pragma unroll
    for (int m = 0; m < MB; ++m) acc[m] += v[m];
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int j = w + kFinWarps * q;
    if (j < r) {
#pragma unroll
      for (int m = 0; m < MB; ++m)
        if (m < M) acc[m] = __fmaf_rn(sT[m * 128 + j], l2v[q], acc[m]);
    }
  }
#pragma unroll
  for (int m = 0; m < MB; ++m) red[w][m][lane] = acc[m];
  __syncthreads();
  if (w == 0 && valid) {
#pragma unroll
    for (int m = 0; m < MB; ++m)
      if (m < M) {
        float y = red[0][m][lane];
#pragma unroll
        for (int q = 1; q < kFinWarps; ++q) y += red[q][m][lane];
        reinterpret_cast<__nv_bfloat16*>(Y)[(int64_t)m * N + n] = __float2bfloat16_rn(y);
      }
  }
}

// Launch with programmatic stream serialisation: the kernel may start while
// the previous kernel of the stream still runs; it synchronises with
// griddepcontrol.wait where it needs that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace

GemvPlan plan_gemv(int64_t M, int64_t N, int64_t K, int num_sms) {
  (void)M;
  GemvPlan p{};
  p.m_tiles = (int)((N + 127) / 128);
  p.kbt = (int)(K / 64);
  p.upr = (p.kbt + kUnitKB - 1) / kUnitKB;
  p.units = (int64_t)p.m_tiles * p.upr;
  const int64_t want = (p.units + kWG - 1) / kWG;
  p.grid = (int)(want < num_sms ? want : num_sms);
  p.workers = p.grid * kWG;
  const int64_t min_run = p.units / p.workers;  // 0 when some workers get nothing
  p.maxc = min_run > 0 ? (int)((p.upr + min_run - 1) / min_run + 1) : p.workers;
  if (p.maxc > p.workers) p.maxc = p.workers;
  if (p.m_tiles <= 4096) {  // the exact count: the most workers any range is split over
    int mx = 1;
    for (int64_t q = 0; q < p.m_tiles; ++q) {
      const int lo = worker_of(q * p.upr, p.units, p.workers);
      const int hi = worker_of(q * p.upr + p.upr - 1, p.units, p.workers);
      mx = hi - lo + 1 > mx ? hi - lo + 1 : mx;
    }
    p.maxc = mx;
  }
  // T slices: at most kGemvTSlices, a whole number of k blocks each
  p.bps = (p.kbt + kGemvTSlices - 1) / kGemvTSlices;
  p.t_slices = (p.kbt + p.bps - 1) / p.bps;
  p.part_bytes = (size_t)p.m_tiles * p.maxc * 16 * 128 * sizeof(float);
  p.tp_bytes = (size_t)p.t_slices * 16 * 128 * sizeof(float);
  p.stw_bytes = (size_t)16 * 128 * sizeof(float);
  return p;
}

namespace {

template <int MB>
cudaError_t launch_gemv_mb(const GemvArgs& a, const GemvPlan& p, const uint16_t* X, const uint16_t* L1,
                           const uint16_t* L2, uint16_t* Y, uint32_t smem, cudaStream_t st) {
  // T kernel: staged chunk (L1 rows + X rows), reused for the k-lane sums
  const int stage = kTChunk * a.r * 2 + 16 * kTChunk * 2;
  const int tsmem = stage > 2048 * MB ? stage : 2048 * MB;
  cudaError_t err = cudaFuncSetAttribute(lora_t_partial_kernel<MB>, cudaFuncAttributeMaxDynamicSharedMemorySize, tsmem);
  if (err != cudaSuccess) return err;
  GemvArgs args = a;
  args.smem_bytes = smem;
  args.t_slices = p.t_slices;
  args.upr = p.upr;
  lora_t_partial_kernel<MB><<<p.t_slices, 256, tsmem, st>>>(X, L1, a.M, a.K, a.r, p.bps, const_cast<float*>(a.tp));
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  if (a.M <= 8) err = launch_pdl(nf4_gemv_kernel<1>, dim3(p.grid), dim3(kGThreads), smem, st, args);
  else err = launch_pdl(nf4_gemv_kernel<2>, dim3(p.grid), dim3(kGThreads), smem, st, args);
  if (err != cudaSuccess) return err;
  err = launch_pdl(gemv_finish_kernel<MB>, dim3((unsigned)((a.N + 31) / 32)), dim3(32 * kFinWarps), 0, st, a.part, a.sTw, L2,
                   a.M, a.N, a.r, p.upr, p.units, p.workers, p.maxc, Y);
  count_launches(3);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemv(const GemvArgs& a, const GemvPlan& p, const uint16_t* X, const uint16_t* L1,
                        const uint16_t* L2, uint16_t* Y, cudaStream_t st) {
  int dev = 0, optin = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err == cudaSuccess) err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (err != cudaSuccess) return err;
  if ((uint32_t)optin < kGemvSmemMin) return cudaErrorInvalidConfiguration;
  const uint32_t smem = (uint32_t)optin;  // everything the block may have; the kernel checks its layout fits
  err = cudaFuncSetAttribute(nf4_gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(nf4_gemv_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  if (a.M <= 1) return launch_gemv_mb<1>(a, p, X, L1, L2, Y, smem, st);
  if (a.M <= 4) return launch_gemv_mb<4>(a, p, X, L1, L2, Y, smem, st);
  return launch_gemv_mb<16>(a, p, X, L1, L2, Y, smem, st);
}

}  // namespace qnf4
