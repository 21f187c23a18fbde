// Few-token backward (M <= 16 tokens): the weight-streaming regime of the
// backward pass, where the time is the 4-bit weight read once from HBM.
//
//   dT  = dY . L2^T                       dL2 = s . T^T . dY
//   dX  = RNbf16( dY . W^ + s . dT . L1^T )   dL1 = s . X^T . dT
//
// nlp-lineage "QLoRA" milestone page, section "The idea": gradients flow
// through the frozen 4-bit weight into the adapters only.  Two kernels,
// chained with programmatic dependent launch:
//
// * lora_bwd_n_kernel: one pass over N in slices: dL2 for the slice (T is
//   saved by the forward) and the slice's partial of dT; it also zeroes the
//   arrival counters of the next kernel (it is launched without overlap, so
//   no earlier kernel still uses them).
// * nf4_gemv_t_kernel: dX = dY . W^ streams W once as units (128-row tile of
//   W x 256-wide k range) ordered by k range, cut into equal contiguous runs
//   over three workers per SM (stream-K, as the forward GEMV).  The
//   reduction runs over the rows n of W, so the warp-level MMA (m16n8k16)
//   takes A = W^T (16 k x 16 n) and B = dY^T (16 n x 8 tokens):
//     - A pairs two weights of one k from rows n and n + 1.  Thread (g, c)
//       reads a 32-bit word (8 codes = bytes 4g .. 4g+3 of its warp's
//       64-wide k block) from rows 2c, 2c+1, 2c+8, 2c+9 of each 16-row step
//       and recombines the nibbles of two rows with four logic operations
//       into pair indices: byte h of lo(w0, w1) indexes the pair
//       (code of row 2c, code of row 2c+1) at even k 8g + 2h, hi(w0, w1) at
//       the odd k next to it.  A 32 KB shared-memory table of pairs
//       (RNbf16(q[i]), RNbf16(q[j])), one copy per lane, turns an index into
//       the A-fragment register: one byte permute and one 4-byte load.
//     - The block scale c^ varies along this reduction (one per row n and
//       64-wide k block), so it goes into B: B = RNbf16(c^_n . dY[m, n]).
//       The product equals dY . W^ up to the roundings, within the layer's
//       stated tolerance.
//   Each maximal run inside one k range (a segment) leaves an fp32 partial
//   [tokens][256] tile.  The worker that completes a k range last (an
//   arrival counter) sums its partials in worker order (deterministic), adds
//   s . dT . L1^T, rounds dX to bf16, and forms dL1 = s . X^T . dT for those
//   256 rows of L1; dT is the sum of the first kernel's slice partials, in
//   slice order.
#include "common.cuh"
#include "internal.h"

namespace qnf4 {
namespace {

constexpr int kTG = 3;                  // stream-K workers per CTA
constexpr int kTS = 2;                  // ring stages per worker
constexpr int kTW = 4;                  // warps per worker: one 64-wide k block of the unit each
constexpr int kTCode = 16384;           // 128 rows x 128 bytes (256 k)
constexpr int kTdY = 4096;              // 16 tokens x 128 n bf16, two boxes of 16 x 64
constexpr int kTStage = kTCode + kTdY;
constexpr int kTWarps = 1 + kTG * kTW;  // producer warp + workers
constexpr int kTThreads = 32 * kTWarps;
constexpr int kTTab = 65536;            // 256 pairs x 256-byte lines (32 lanes x 4 bytes used)
constexpr int kTFront = 3;              // stages below the table
constexpr int kTMisc = 1024;            // barriers, abort flag, fixup flags
constexpr int kTScale = 512;            // per warp: c^ of the unit's 128 rows
constexpr int kTFix = 16 * 128 * 4;     // per worker: dT [16][128] fp32 for the fixup
constexpr uint32_t kGemvTSmemMin =
    65536 + kTTab + (kTG * kTS - kTFront) * kTStage + (kTG * kTW) * kTScale + kTG * kTFix;
static_assert(kTFront * kTStage + kTMisc <= 65536 - 3072, "front region must fit below the table");

struct TSmem {
  uint32_t base;
  uint8_t* raw;
  uint32_t raw_addr;
  uint64_t* bars;
  volatile int* abort_flag;
  volatile int* fix_flag;  // [kTG]
  uint32_t tab;
  uint32_t scales;  // [warps][128] fp32
  uint32_t fix;     // [kTG][16][128] fp32
  bool fits;
};

QDEV TSmem carve_t(uint8_t* raw_ptr, uint32_t smem_bytes) {
  TSmem g;
  const uint32_t raw = smem_u32(raw_ptr);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t misc = base + kTFront * kTStage;
  const uint32_t tab = (misc + kTMisc + 0xFFFFu) & ~0xFFFFu;
  g.base = base;
  g.tab = tab;
  g.scales = tab + kTTab + (kTG * kTS - kTFront) * kTStage;
  g.fix = g.scales + (kTG * kTW) * kTScale;
  const uint32_t end = g.fix + kTG * kTFix;
  g.fits = end - raw <= smem_bytes && tab <= 0x00FF0000u;
  g.raw = raw_ptr;
  g.raw_addr = raw;
  g.bars = reinterpret_cast<uint64_t*>(raw_ptr + (misc - raw));
  g.abort_flag = reinterpret_cast<volatile int*>(g.bars + 32);
  g.fix_flag = g.abort_flag + 1;
  return g;
}
QDEV uint8_t* sptr(const TSmem& s, uint32_t a) { return s.raw + (a - s.raw_addr); }
QDEV uint64_t* tfull(const TSmem& s, int g, int j) { return s.bars + g * 2 * kTS + j; }
QDEV uint64_t* tempty(const TSmem& s, int g, int j) { return s.bars + g * 2 * kTS + kTS + j; }
QDEV uint32_t tstage(const TSmem& s, int st) {
  return st < kTFront ? s.base + (uint32_t)(st * kTStage) : s.tab + kTTab + (uint32_t)((st - kTFront) * kTStage);
}

__host__ __device__ __forceinline__ int t_worker_of(int64_t u, int64_t U, int W) {
  return (int)(((u + 1) * (int64_t)W - 1) / U);
}

QDEV uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
QDEV float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
QDEV void sts_f32(uint32_t addr, float v) { asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory"); }

QDEV uint32_t pair_lookup_t(uint32_t w, int k, uint32_t lanereg) {
  const uint32_t addr = __byte_perm(w, lanereg, 0x7604u | ((uint32_t)k << 4));
  return lds32(addr);
}

QDEV void mma_t(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

QDEV void t_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
QDEV void t_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
QDEV void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

QDEV bool warp_wait_t(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status, int lane) {
  int ok = 1;
  if (lane == 0) ok = mbar_wait(bar, parity, abort_flag, status) ? 1 : 0;
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  if (ok) mbar_test_wait(smem_u32(bar), parity);
  return ok != 0;
}

// Scale codes of one row for the warp's k block of a unit, loaded one unit
// ahead (nothing consumes them until the next unit).
struct RowScaleRaw {
  uint32_t c2;
  GroupScale gs;
};

// ------------------------------------------------------------- kernel 1
// Slice p of N: columns [p*S, min((p+1)*S, N)), in chunks of 256 staged in
// shared memory: dY [16][256] and L2^T [256][r] (transposed while staging so
// that threads of consecutive adapter columns read consecutive banks).
constexpr int kBChunk = 256;
template <int MB>
__global__ void __launch_bounds__(256) lora_bwd_n_kernel(const uint16_t* __restrict__ dY,
                                                         const uint16_t* __restrict__ L2,
                                                         const float* __restrict__ T, int M, int64_t N, int r,
                                                         float s, int S, float* __restrict__ dL2,
                                                         float* __restrict__ tp, int* __restrict__ cnt, int n_cnt) {
  extern __shared__ __align__(16) uint8_t bsm[];
  uint16_t* sY = reinterpret_cast<uint16_t*>(bsm);                          // [MB][256]
  uint16_t* sL = reinterpret_cast<uint16_t*>(bsm + MB * kBChunk * 2);       // [256][r]
  float* sT = reinterpret_cast<float*>(bsm + MB * kBChunk * 2 + kBChunk * r * 2);  // [MB][r]
  const int p = blockIdx.x, t = threadIdx.x;
  if (p == 0)
    for (int i = t; i < n_cnt; i += 256) cnt[i] = 0;
  t_dep_launch();  // the dX kernel may start: it reads what this kernel writes only after griddepcontrol.wait
  const int64_t n_lo = (int64_t)p * S, n_hi = min(N, n_lo + S);
  for (int i = t; i < M * r; i += 256) sT[i] = T[i];
  constexpr int kMaxOut = MB * 128 / 256;  // dT outputs per thread (M*r <= MB*128)
  float acc[kMaxOut > 0 ? kMaxOut : 1];
#pragma unroll
  for (int q = 0; q < (kMaxOut > 0 ? kMaxOut : 1); ++q) acc[q] = 0.0f;
  for (int64_t n0 = n_lo; n0 < n_hi; n0 += kBChunk) {
    const int cw = (int)min((int64_t)kBChunk, n_hi - n0);  // a multiple of 8
    __syncthreads();                                      // previous chunk done
    for (int i = t; i < M * (cw / 8); i += 256) {         // dY rows: 16-byte pieces
      const int m = i / (cw / 8), c = i % (cw / 8);
      *reinterpret_cast<uint4*>(sY + m * kBChunk + c * 8) =
          __ldg(reinterpret_cast<const uint4*>(dY + (int64_t)m * N + n0) + c);
    }
#pragma unroll 4
    for (int i = t; i < r * (cw / 8); i += 256) {         // L2 [j][n] -> sL [n][j], 16-byte loads
      const int j = i / (cw / 8), c = i % (cw / 8);
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(L2 + (int64_t)j * N + n0) + c);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        sL[(c * 8 + 2 * e) * r + j] = (uint16_t)(w4[e] & 0xFFFFu);
        sL[(c * 8 + 2 * e + 1) * r + j] = (uint16_t)(w4[e] >> 16);
      }
    }
    __syncthreads();
    if (dL2) {                                            // dL2[j][n] = s . sum_m T[m][j] dY[m][n]
      for (int nn = t; nn < cw; nn += 256) {
        float dy[MB];
#pragma unroll
        for (int m = 0; m < MB; ++m) dy[m] = m < M ? bf16_bits_to_float(sY[m * kBChunk + nn]) : 0.0f;
        for (int j = 0; j < r; ++j) {
          float a = 0.0f;
#pragma unroll
          for (int m = 0; m < MB; ++m)
            if (m < M) a = __fmaf_rn(sT[m * r + j], dy[m], a);
          dL2[(int64_t)j * N + n0 + nn] = __fmul_rn(s, a);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < (kMaxOut > 0 ? kMaxOut : 1); ++q) {  // dT partial: output e = t + 256 q
      const int e = t + 256 * q;
      if (e < M * r) {
        const int m = e / r, j = e % r;
        float a = acc[q];
        for (int nn = 0; nn < cw; ++nn) a = __fmaf_rn(bf16_bits_to_float(sY[m * kBChunk + nn]),
                                                      bf16_bits_to_float(sL[nn * r + j]), a);
        acc[q] = a;
      }
    }
  }
#pragma unroll
  for (int q = 0; q < (kMaxOut > 0 ? kMaxOut : 1); ++q) {
    const int e = t + 256 * q;
    if (e < M * r) tp[((int64_t)p * 16 + e / r) * 128 + e % r] = acc[q];
  }
}

// ------------------------------------------------------------- kernel 2
template <int NT>
__global__ void __launch_bounds__(kTThreads, 1) nf4_gemv_t_kernel(const __grid_constant__ GemvTArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const TSmem S = carve_t(smem_raw, args.smem_bytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (!S.fits) {
    if (tid == 0) report(args.status, QLORA_ERR_CUDA);
    return;
  }
  const int G = gridDim.x, c = blockIdx.x;
  const int W = G * kTG;
  const int64_t U = args.units;
  const int ntl = args.n_tiles;

  if (tid == 0) {
    for (int g = 0; g < kTG; ++g)
      for (int j = 0; j < kTS; ++j) {
        mbar_init(tfull(S, g, j), 1);
        mbar_init(tempty(S, g, j), kTW);
      }
    *S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&args.tmCodes);
    tma_prefetch_desc(&args.tmDY);
  }
  for (int idx = tid; idx < 256 * 32; idx += kTThreads) {  // pair table: entry e, lane l at tab + e*256 + l*4
    const int e = idx >> 5, l = idx & 31;
    const uint32_t v = pack_bf16x2(args.q[e & 15], args.q[e >> 4]);
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(S.tab + (uint32_t)(e * 256 + l * 4)), "r"(v) : "memory");
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------ producers: one lane per ring stage
    if (lane < kTG * kTS) {
      const int g = lane / kTS, wk = c * kTG + g;
      const int64_t u0 = (int64_t)wk * U / W, u1 = (int64_t)(wk + 1) * U / W;
      const int nu = (int)(u1 - u0);
      int issued = 0;
      for (int i = lane % kTS; i < nu; i += kTS) {
        const int j = i % kTS;
        if (!mbar_wait_backoff(tempty(S, g, j), ((uint32_t)(i / kTS) & 1u) ^ 1u, S.abort_flag, args.status, 64))
          break;
        const int64_t u = u0 + i;
        const int kr = (int)(u / ntl), nt = (int)(u % ntl);
        uint8_t* sp = sptr(S, tstage(S, kTS * g + j));
        mbar_arrive_expect_tx(tfull(S, g, j), kTStage);
        tma_load_2d(sp, &args.tmCodes, tfull(S, g, j), kr * 128, nt * 128);
        tma_load_2d(sp + kTCode, &args.tmDY, tfull(S, g, j), nt * 128, 0);
        tma_load_2d(sp + kTCode + 2048, &args.tmDY, tfull(S, g, j), nt * 128 + 64, 0);
        issued = i + 1;
      }
      if (*S.abort_flag && issued > 0) {
        const int i = issued - 1;
        mbar_wait_drain(tfull(S, g, i % kTS), (uint32_t)(i / kTS) & 1u, 10000000ull);
      }
    }
    return;  // no barrier below involves warp 0
  }

  // ------------------------------------------------------- worker warps
  const int wv = warp - 1, g = wv / kTW, wq = wv % kTW;
  const int wk = c * kTG + g;
  const int gr = lane >> 2, cq = lane & 3;
  const int tw = wq * 32 + lane;  // thread index inside the worker (0..127)
  const uint32_t lanereg = (S.tab & 0x00FF0000u) | (uint32_t)(lane * 4);
  const uint32_t my_scales = S.scales + (uint32_t)(wv * kTScale);
  const bool e5m2 = args.c2_e5m2 != 0, mean = args.c1_mean != 0;
  const int64_t u0 = (int64_t)wk * U / W, u1 = (int64_t)(wk + 1) * U / W;
  const int nu = (int)(u1 - u0);
  float acc[4][NT][4];
#pragma unroll
  for (int h = 0; h < 4; ++h)
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[h][t][e] = 0.0f;

  // c^ of rows (nt*128 + lane + 32i) for k block (kr*4 + wq), loaded one unit ahead
  RowScaleRaw sr[4];
  auto load_scales = [&](int64_t u) {
    const int kr = (int)(u / ntl), nt = (int)(u % ntl);
    const int blk = kr * 4 + wq;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t n = (int64_t)nt * 128 + lane + 32 * i;
      sr[i].c2 = 0;
      sr[i].gs = GroupScale{0.0f, 0.0f};
      if (n < args.N && blk < args.kbt) {
        const int64_t f = n * args.kbt + blk;
        sr[i].c2 = __ldg(args.c2 + f);
        sr[i].gs = load_group_scale(args.c1, f >> 8, mean);
      }
    }
  };
  if (nu > 0) load_scales(u0);
  bool aborted = false;
  for (int i = 0; i < nu; ++i) {
    const int64_t u = u0 + i;
    const int kr = (int)(u / ntl), nt = (int)(u % ntl);
    const bool seg_end = i == nu - 1 || nt == ntl - 1;
#pragma unroll
    for (int q = 0; q < 4; ++q)  // this unit's scales into the warp's table
      sts_f32(my_scales + (uint32_t)((lane + 32 * q) * 4), decode_scale(sr[q].c2, sr[q].gs, e5m2, mean));
    if (i + 1 < nu) load_scales(u + 1);
    __syncwarp();
    const int j = i % kTS;
    if (!aborted && !warp_wait_t(tfull(S, g, j), (uint32_t)(i / kTS) & 1u, S.abort_flag, args.status, lane))
      aborted = true;
    if (!aborted) {
      const uint32_t st = tstage(S, kTS * g + j);
      const uint32_t bo = (uint32_t)(32 * wq + 4 * gr);  // byte of the row: 4 consecutive bytes = 8 k
#pragma unroll 2
      for (int step = 0; step < 8; ++step) {
        const int r0 = 16 * step + 2 * cq;
        uint32_t w[4];
        const int rows[4] = {r0, r0 + 1, r0 + 8, r0 + 9};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w[e] = lds32(st + (uint32_t)rows[e] * 128u + ((((bo >> 4) ^ (uint32_t)(rows[e] & 7))) << 4) + (bo & 15u));
        const uint32_t lo01 = (w[0] & 0x0F0F0F0Fu) | ((w[1] & 0x0F0F0F0Fu) << 4);
        const uint32_t hi01 = ((w[0] >> 4) & 0x0F0F0F0Fu) | (w[1] & 0xF0F0F0F0u);
        const uint32_t lo23 = (w[2] & 0x0F0F0F0Fu) | ((w[3] & 0x0F0F0F0Fu) << 4);
        const uint32_t hi23 = ((w[2] >> 4) & 0x0F0F0F0Fu) | (w[3] & 0xF0F0F0F0u);
        const float s0 = lds_f32(my_scales + (uint32_t)(r0 * 4)), s1 = lds_f32(my_scales + (uint32_t)((r0 + 1) * 4));
        const float s2 = lds_f32(my_scales + (uint32_t)((r0 + 8) * 4)), s3 = lds_f32(my_scales + (uint32_t)((r0 + 9) * 4));
        uint32_t b0[NT], b1[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          // dY tile: box (16 n-step / 64), token m, n pair (2c, 2c+1) and (2c+8, 2c+9) of the step
          const int m = 8 * t + gr;
          const uint32_t bx = st + kTCode + (uint32_t)((step >> 2) * 2048 + m * 128);
          const uint32_t nb = (uint32_t)(((16 * step) & 63) + 2 * cq) * 2u;  // byte of the pair in the 128-byte row
          const uint32_t y01 = lds32(bx + ((((nb >> 4) ^ (uint32_t)(m & 7))) << 4) + (nb & 15u));
          const uint32_t y23 = lds32(bx + (((((nb + 16u) >> 4) ^ (uint32_t)(m & 7))) << 4) + (nb & 15u));
          b0[t] = pack_bf16x2(__fmul_rn(bf16_bits_to_float(y01 & 0xFFFFu), s0), __fmul_rn(bf16_bits_to_float(y01 >> 16), s1));
          b1[t] = pack_bf16x2(__fmul_rn(bf16_bits_to_float(y23 & 0xFFFFu), s2), __fmul_rn(bf16_bits_to_float(y23 >> 16), s3));
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const uint32_t a0 = pair_lookup_t(lo01, h, lanereg);
          const uint32_t a1 = pair_lookup_t(hi01, h, lanereg);
          const uint32_t a2 = pair_lookup_t(lo23, h, lanereg);
          const uint32_t a3 = pair_lookup_t(hi23, h, lanereg);
#pragma unroll
          for (int t = 0; t < NT; ++t) mma_t(acc[h][t], a0, a1, a2, a3, b0[t], b1[t]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(tempty(S, g, j));
    if (!seg_end) continue;
    // ---- segment end: partial tile, arrival on the k range, fixup by the last arriver
    const int jw = wk - t_worker_of((int64_t)kr * ntl, U, W);
    const bool part_ok = !aborted && jw >= 0 && jw < args.maxc;
    if (!aborted && !part_ok && lane == 0) report(args.status, QLORA_ERR_CUDA);
    if (part_ok) {
      float* base = args.part + ((int64_t)kr * args.maxc + jw) * (16 * 256);
#pragma unroll
      for (int h = 0; h < 4; ++h)
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int m = 8 * t + 2 * cq + (e & 1);
            const int kl = 64 * wq + 8 * gr + 2 * h + (e >> 1);
            if (m < args.M) base[m * 256 + kl] = acc[h][t][e];
          }
    }
#pragma unroll
    for (int h = 0; h < 4; ++h)
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[h][t][e] = 0.0f;
    __threadfence();
    named_sync(1 + g, 32 * kTW);
    if (tw == 0) {
      int last = 0;
      if (!*S.abort_flag) {
        t_dep_wait();  // the counters were zeroed by the previous kernel
        const int c_lo = t_worker_of((int64_t)kr * ntl, U, W);
        const int need = t_worker_of((int64_t)kr * ntl + ntl - 1, U, W) - c_lo + 1;
        last = atomicAdd(args.cnt + kr, 1) == need - 1;
      }
      S.fix_flag[g] = last;
    }
    named_sync(1 + g, 32 * kTW);
    if (!S.fix_flag[g]) continue;
    __threadfence();
    t_dep_wait();  // the dT slice partials
    // dT = sum of the slice partials (slice order) into this worker's region,
    // eight loads in flight per element
    const uint32_t fix = S.fix + (uint32_t)(g * kTFix);
    for (int e = tw; e < args.M * args.r; e += 32 * kTW) {
      const int m = e / args.r, jj = e % args.r;
      const float* src = args.tp + (int64_t)m * 128 + jj;
      float a = 0.0f;
      for (int p0 = 0; p0 < args.t_slices; p0 += 8) {
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = p0 + q < args.t_slices ? __ldcg(src + (int64_t)(p0 + q) * 16 * 128) : 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (p0 + q < args.t_slices) a += v[q];
      }
      sts_f32(fix + (uint32_t)((m * 128 + jj) * 4), a);
    }
    named_sync(1 + g, 32 * kTW);
    const int c_lo = t_worker_of((int64_t)kr * ntl, U, W);
    const int cnt_c = min(t_worker_of((int64_t)kr * ntl + ntl - 1, U, W) - c_lo + 1, args.maxc);
    const int kl = 2 * tw;  // this thread: columns k, k + 1 of the k range
    const int64_t k = (int64_t)kr * 256 + kl;
    if (k < args.K) {       // K % 64 == 0: k + 1 < K as well
      if (args.dX) {
        // the segment partials of every token, in worker order, two workers at a time
        float2 acc2[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) acc2[m] = make_float2(0.0f, 0.0f);
        const float* pbase = args.part + (int64_t)kr * args.maxc * (16 * 256) + kl;
        for (int jc = 0; jc < cnt_c; jc += 2) {
          float2 v0[16], v1[16];
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            v0[m] = m < args.M ? __ldcg(reinterpret_cast<const float2*>(pbase + ((int64_t)jc * 16 + m) * 256))
                               : make_float2(0.0f, 0.0f);
            v1[m] = (m < args.M && jc + 1 < cnt_c)
                        ? __ldcg(reinterpret_cast<const float2*>(pbase + ((int64_t)(jc + 1) * 16 + m) * 256))
                        : make_float2(0.0f, 0.0f);
          }
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            acc2[m].x += v0[m].x;
            acc2[m].y += v0[m].y;
            if (jc + 1 < cnt_c) {
              acc2[m].x += v1[m].x;
              acc2[m].y += v1[m].y;
            }
          }
        }
        // + s . dT . L1^T for the two columns, L1 rows read eight adapter columns at a time
        float2 l2[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) l2[m] = make_float2(0.0f, 0.0f);
        for (int j0 = 0; j0 < args.r; j0 += 8) {
          const uint4 la = __ldg(reinterpret_cast<const uint4*>(args.L1 + k * args.r + j0));
          const uint4 lb = __ldg(reinterpret_cast<const uint4*>(args.L1 + (k + 1) * args.r + j0));
          const uint32_t wa[4] = {la.x, la.y, la.z, la.w}, wb[4] = {lb.x, lb.y, lb.z, lb.w};
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float fa = bf16_bits_to_float((wa[q >> 1] >> (16 * (q & 1))) & 0xFFFFu);
            const float fb = bf16_bits_to_float((wb[q >> 1] >> (16 * (q & 1))) & 0xFFFFu);
#pragma unroll
            for (int m = 0; m < 16; ++m) {
              if (m < args.M) {
                const float tv = lds_f32(fix + (uint32_t)((m * 128 + j0 + q) * 4));
                l2[m].x = __fmaf_rn(tv, fa, l2[m].x);
                l2[m].y = __fmaf_rn(tv, fb, l2[m].y);
              }
            }
          }
        }
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m < args.M)
            *reinterpret_cast<uint32_t*>(args.dX + (int64_t)m * args.K + k) =
                pack_bf16x2(__fmaf_rn(args.s, l2[m].x, acc2[m].x), __fmaf_rn(args.s, l2[m].y, acc2[m].y));
      }
      if (args.dL1) {
        float xa[16], xb[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const uint32_t xv = m < args.M ? __ldg(reinterpret_cast<const uint32_t*>(args.X + (int64_t)m * args.K + k)) : 0u;
          xa[m] = bf16_bits_to_float(xv & 0xFFFFu);
          xb[m] = bf16_bits_to_float(xv >> 16);
        }
        for (int jj = 0; jj < args.r; ++jj) {
          float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            if (m < args.M) {
              const float tv = lds_f32(fix + (uint32_t)((m * 128 + jj) * 4));
              a0 = __fmaf_rn(xa[m], tv, a0);
              a1 = __fmaf_rn(xb[m], tv, a1);
            }
          }
          args.dL1[k * args.r + jj] = __fmul_rn(args.s, a0);
          args.dL1[(k + 1) * args.r + jj] = __fmul_rn(args.s, a1);
        }
      }
    }
    named_sync(1 + g, 32 * kTW);  // the region is reused by this worker's next fixup
  }
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_t(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
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

GemvTPlan plan_gemv_t(int64_t M, int64_t N, int64_t K, int num_sms) {
  (void)M;
  GemvTPlan p{};
  p.n_tiles = (int)((N + 127) / 128);
  p.kbt = (int)(K / 64);
  p.k_ranges = (int)((K + 255) / 256);
  p.units = (int64_t)p.n_tiles * p.k_ranges;
  // at least 2 units per worker (fewer partial tiles to sum), at most one CTA per SM
  const int64_t want = (p.units + kTG * 2 - 1) / (kTG * 2);
  p.grid = (int)(want < num_sms ? (want > 0 ? want : 1) : num_sms);
  p.workers = p.grid * kTG;
  const int64_t min_run = p.units / p.workers;
  p.maxc = min_run > 0 ? (int)((p.n_tiles + min_run - 1) / min_run + 1) : p.workers;
  if (p.maxc > p.workers) p.maxc = p.workers;
  if (p.k_ranges <= 4096) {  // the exact count: the most workers any range is split over
    int mx = 1;
    for (int64_t q = 0; q < p.k_ranges; ++q) {
      const int lo = t_worker_of(q * p.n_tiles, p.units, p.workers);
      const int hi = t_worker_of(q * p.n_tiles + p.n_tiles - 1, p.units, p.workers);
      mx = hi - lo + 1 > mx ? hi - lo + 1 : mx;
    }
    p.maxc = mx;
  }
  // dT slices over N: at most 32, whole multiples of 8 columns
  int P = (int)((N + 255) / 256);
  if (P > 32) P = 32;
  if (P < 1) P = 1;
  int64_t Sl = (N + P - 1) / P;
  Sl = (Sl + 7) / 8 * 8;
  p.slice = (int)Sl;
  p.t_slices = (int)((N + Sl - 1) / Sl);
  p.part_bytes = (size_t)p.k_ranges * p.maxc * 16 * 256 * sizeof(float);
  p.tp_bytes = (size_t)p.t_slices * 16 * 128 * sizeof(float);
  p.cnt_bytes = (size_t)p.k_ranges * sizeof(int);
  return p;
}

cudaError_t launch_gemv_t(const GemvTArgs& a, const GemvTPlan& p, const uint16_t* dY, const uint16_t* L2,
                          const float* T, float* dL2, cudaStream_t st) {
  int dev = 0, optin = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err == cudaSuccess) err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (err != cudaSuccess) return err;
  if ((uint32_t)optin < kGemvTSmemMin) return cudaErrorInvalidConfiguration;
  const uint32_t smem = (uint32_t)optin;
  err = cudaFuncSetAttribute(nf4_gemv_t_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(nf4_gemv_t_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int bsmem = 16 * kBChunk * 2 + kBChunk * a.r * 2 + 16 * a.r * 4;
  auto k1 = a.M <= 1 ? lora_bwd_n_kernel<1> : a.M <= 4 ? lora_bwd_n_kernel<4> : lora_bwd_n_kernel<16>;
  err = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, bsmem);
  if (err != cudaSuccess) return err;
  k1<<<p.t_slices, 256, bsmem, st>>>(dY, L2, T, a.M, a.N, a.r, a.s, p.slice, dL2, const_cast<float*>(a.tp), a.cnt,
                                     p.k_ranges);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  GemvTArgs args = a;
  args.smem_bytes = smem;
  if (a.M <= 8) err = launch_pdl_t(nf4_gemv_t_kernel<1>, dim3(p.grid), dim3(kTThreads), smem, st, args);
  else err = launch_pdl_t(nf4_gemv_t_kernel<2>, dim3(p.grid), dim3(kTThreads), smem, st, args);
  count_launches(2);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace qnf4
