// The tcgen05 GEMM engine behind every contraction of the layer.
//
//   D[rows x cols] (fp32, in TMEM) = sum_k A[row, k] * B[col, k]
//
// Persistent: one CTA per SM walks a static round-robin list of 128 x BN
// output tiles (cta_group::1 UMMA, M = 128).  The reduction of every tile
// runs in 64-wide blocks through one 4-stage shared-memory ring that keeps
// flowing from tile to tile:
//   * warp 0, one lane: TMA producer (B tiles, A tiles or NF4 code tiles);
//   * warp 1, one lane: UMMA issuer, 4 x (128 x BN x 16) MMAs per stage,
//     tcgen05.commit frees the stage and, after a tile's last stage, hands
//     the accumulator to the epilogue;
//   * warps 2..17, four groups of four: when A is the NF4 weight, group g
//     turns the code tile of ring stage g into bf16 (one NF4 block per thread)
//     -- into tensor memory for X.W^T, into the 128-byte-swizzled MN-major
//     shared-memory layout for dY.W;
//   * warps 18..21: epilogue (TMEM -> registers -> global).  With two
//     accumulators in TMEM the epilogue of one tile overlaps the MMAs of the
//     next.
// An optional extension segment appends more reduction blocks from other
// operands into the same accumulator: this is how the LoRA term s.T.L2
// (forward) and s.dT.L1^T (backward) is added to the dequantised product.
// A split of the main reduction writes fp32 partial tiles that a second
// kernel sums in a fixed order (deterministic).
//
// inferensys glossary "QLoRA", kernel paragraph: 4-bit weights are loaded,
// decompressed on chip and fed to the tensor cores as BFloat16.
#include <cstdlib>

#include "common.cuh"
#include "internal.h"

namespace qnf4 {
namespace {

constexpr int kStages = 4;
constexpr int kDeqWarps = 16;  // warps 2..17: four groups, group g fills ring stage g
constexpr int kGroupWarps = 4;
constexpr int kEpiWarps = 4;   // warps 18..21
constexpr int kEpiWarp0 = 2 + kDeqWarps;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kA = 16384;  // 128 rows x 64 bf16

constexpr uint32_t pow2_cols(uint32_t n) { return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512; }

// Tensor-memory columns: n_acc fp32 accumulators of max(BN, 32) columns and,
// for the forward fused GEMM, the dequantised A tile of every ring stage
// (128 lanes x 32 columns: 64 bf16 per lane).
template <int BN, int AMODE>
struct Tmem {
  static constexpr uint32_t acc = BN < 32 ? 32 : BN;
  static constexpr uint32_t a_cols = AMODE == A_DEQ_K ? kStages * 32 : 0;
  static constexpr int n_acc = (2 * acc + a_cols <= 512) ? 2 : 1;
  static constexpr uint32_t a_col = n_acc * acc;
  static constexpr uint32_t cols = pow2_cols(a_col + a_cols);
};

template <int BN, int AMODE>
struct Layout {
  static constexpr int B = BN * 128 > 8192 ? BN * 128 : 8192;
  static constexpr int C = AMODE == A_TMA ? 0 : 4096;
  static constexpr int STAGE = kA + B + C;
  static constexpr int BAR = kStages * STAGE;
  static constexpr int TOTAL = BAR + 256 + 1024;  // barriers etc. + alignment slack
};

QDEV uint32_t tx_bytes(int mn_major, int extent) {
  return mn_major ? (uint32_t)((extent + 63) / 64) * 8192u : (uint32_t)extent * 128u;
}

// Load one operand tile (extent rows of UMMA M/N, 64 of the reduction).
QDEV void load_operand(uint8_t* dst, const CUtensorMap* m, uint64_t* bar, int mn_major, int mn0, int k0,
                       int extent) {
  if (!mn_major) {
    tma_load_2d(dst, m, bar, k0, mn0);
  } else {
    for (int j = 0; j < (extent + 63) / 64; ++j) tma_load_2d(dst + j * 8192, m, bar, mn0 + 64 * j, k0);
  }
}

QDEV uint64_t operand_desc(const uint8_t* base, int mn_major, int kk) {
  const uint32_t a = smem_u32(base);
  return mn_major ? sdesc_sw128(a + kk * 2048, 8192, 1024) : sdesc_sw128(a + kk * 32, 16, 1024);
}

QDEV void epi_store(const EpiArgs& e, int64_t row, int64_t col, float v) {
  if (e.out) {
    const int64_t i = row * e.rs + col * e.cs;
    if (e.out_bf16) reinterpret_cast<__nv_bfloat16*>(e.out)[i] = __float2bfloat16_rn(__fmul_rn(v, e.alpha));
    else reinterpret_cast<float*>(e.out)[i] = __fmul_rn(v, e.alpha);
  }
  if (e.out2) {
    const int64_t i = row * e.rs2 + col * e.cs2;
    reinterpret_cast<__nv_bfloat16*>(e.out2)[i] = __float2bfloat16_rn(__fmul_rn(v, e.alpha2));
  }
}

// Warp-wide wait: lane 0 polls (bounded), then every lane takes one
// acquiring look at the completed phase.
QDEV bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status, int lane) {
  int ok = 1;
  if (lane == 0) ok = mbar_wait(bar, parity, abort_flag, status) ? 1 : 0;
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  if (ok) mbar_try_wait(smem_u32(bar), parity);
  return ok != 0;
}

// The tile list all roles walk in the same order: tile t = blockIdx.x + i *
// gridDim.x; the weight-row tile varies fastest, then the token tile, then
// the split of the reduction.  `it` indexes the reduction blocks of a tile
// (main blocks first, then the extension blocks of split 0).
struct TileIter {
  int t, it;
  int row0, col0, z, kb_lo, my_kb, n_iters;
  bool valid;

  QDEV void load(const EngineArgs& a, int BN) {
    const int mt = t % a.m_tiles;
    const int r = t / a.m_tiles;
    const int nt = r % a.n_tiles;
    z = r / a.n_tiles;
    row0 = mt * 128;
    col0 = nt * BN;
    kb_lo = (int)((int64_t)z * a.kb_main / a.splits);
    my_kb = (int)((int64_t)(z + 1) * a.kb_main / a.splits) - kb_lo;
    n_iters = my_kb + (z == 0 ? a.kb_ext : 0);
  }
  QDEV void begin(const EngineArgs& a, int BN) {
    t = blockIdx.x;
    it = 0;
    valid = t < a.total_tiles;
    if (valid) load(a, BN);
  }
  QDEV void next(const EngineArgs& a, int BN) {
    if (++it >= n_iters) {
      t += gridDim.x;
      it = 0;
      valid = t < a.total_tiles;
      if (valid) load(a, BN);
    }
  }
};

template <int BN, int AMODE>
__global__ void __launch_bounds__(kThreads, 1) umma_engine_kernel(const __grid_constant__ EngineArgs args) {
  using L = Layout<BN, AMODE>;
  using TM = Tmem<BN, AMODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR);
  uint64_t* afull = full + kStages;
  uint64_t* empty = afull + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(afull + s, kGroupWarps);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&args.tmA);
    tma_prefetch_desc(&args.tmB);
    if (args.kb_ext) {
      tma_prefetch_desc(&args.tmAx);
      tma_prefetch_desc(&args.tmBx);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TM::cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      TileIter ti;
      uint32_t G = 0;
      for (ti.begin(args, BN); ti.valid; ti.next(args, BN), ++G) {
        const int s = (int)(G % kStages);
        const uint32_t ph = (G / kStages) & 1u;
        if (!mbar_wait(empty + s, ph ^ 1u, abort_flag, args.status)) break;
        uint8_t* sa = smem + s * L::STAGE;
        uint8_t* sb = sa + kA;
        uint8_t* sc = sb + L::B;
        if (ti.it < ti.my_kb) {
          const int kb = ti.kb_lo + ti.it;
          uint32_t bytes = tx_bytes(args.b_mn_main, BN);
          bytes += AMODE == A_TMA ? tx_bytes(args.a_mn_main, 128) : 4096u;
          mbar_arrive_expect_tx(full + s, bytes);
          if (AMODE == A_DEQ_K) tma_load_2d(sc, &args.tmA, full + s, kb * 32, ti.row0);
          else if (AMODE == A_DEQ_MN) tma_load_2d(sc, &args.tmA, full + s, ti.row0 / 2, kb * 64);
          else load_operand(sa, &args.tmA, full + s, args.a_mn_main, ti.row0, kb * 64, 128);
          load_operand(sb, &args.tmB, full + s, args.b_mn_main, ti.col0, kb * 64, BN);
        } else {
          const int kb = ti.it - ti.my_kb;
          mbar_arrive_expect_tx(full + s, tx_bytes(args.a_mn_ext, 128) + tx_bytes(args.b_mn_ext, BN));
          load_operand(sa, &args.tmAx, full + s, args.a_mn_ext, ti.row0, kb * 64, 128);
          load_operand(sb, &args.tmBx, full + s, args.b_mn_ext, ti.col0, kb * 64, BN);
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- UMMA
    if (lane == 0) {
      const int a_mn_main = AMODE == A_DEQ_MN ? 1 : (AMODE == A_DEQ_K ? 0 : args.a_mn_main);
      const uint32_t id_main = idesc_bf16(128, BN, a_mn_main, args.b_mn_main);
      const uint32_t id_ext = idesc_bf16(128, BN, args.a_mn_ext, args.b_mn_ext);
      TileIter ti;
      uint32_t G = 0, tile_no = 0, acc_addr = tmem_d;
      uint32_t aphase = 0;  // afull completes only for main-segment stages: own parity bit per stage
      bool ok = true;
      for (ti.begin(args, BN); ti.valid && ok; ti.next(args, BN), ++G) {
        if (ti.it == 0) {  // new tile: wait until the epilogue has drained this accumulator
          const uint32_t b = tile_no % TM::n_acc, use = tile_no / TM::n_acc;
          if (!mbar_wait(acc_empty + b, (use & 1u) ^ 1u, abort_flag, args.status)) break;
          tc_fence_after();
          acc_addr = tmem_d + b * TM::acc;
        }
        const int s = (int)(G % kStages);
        const uint32_t ph = (G / kStages) & 1u;
        const bool ext = ti.it >= ti.my_kb;
        ok = mbar_wait(full + s, ph, abort_flag, args.status);
        if (ok && AMODE != A_TMA && !ext) {
          ok = mbar_wait(afull + s, (aphase >> s) & 1u, abort_flag, args.status);
          aphase ^= 1u << s;
        }
        if (!ok) break;
        tc_fence_after();
        const uint8_t* sa = smem + s * L::STAGE;
        const uint8_t* sb = sa + kA;
        if (AMODE == A_DEQ_K && !ext) {
          // A: dequantised weight tile in tensor memory, 8 columns per K = 16
          const uint32_t a_tmem = tmem_d + TM::a_col + (uint32_t)(s * 32);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_tmem_a(acc_addr, a_tmem + kk * 8, operand_desc(sb, args.b_mn_main, kk), id_main,
                             (ti.it | kk) != 0);
        } else {
          const int amn = ext ? args.a_mn_ext : a_mn_main;
          const int bmn = ext ? args.b_mn_ext : args.b_mn_main;
          const uint32_t id = ext ? id_ext : id_main;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(acc_addr, operand_desc(sa, amn, kk), operand_desc(sb, bmn, kk), id, (ti.it | kk) != 0);
        }
        umma_commit(empty + s);
        if (ti.it == ti.n_iters - 1) {  // tile complete: hand the accumulator over
          umma_commit(acc_full + (tile_no % TM::n_acc));
          ++tile_no;
        }
      }
    }
    __syncwarp();
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------------------------- dequant
    if (AMODE != A_TMA) {
      const int grp = (warp - 2) >> 2;  // this group fills ring stage grp
      const int q4 = warp & 3;          // TMEM lane quarter this warp may access
      const int u = q4 * 32 + lane;     // thread index within the group
      const int64_t bpr = args.wK / 64; // NF4 blocks per weight row
      float q[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) q[i] = args.q[i];
      // Walk the global stage sequence G = grp, grp + 4, ...; dequantise the
      // main-segment blocks among them.
      TileIter ti;
      ti.begin(args, BN);
      uint32_t G = 0;
      for (; G < (uint32_t)grp && ti.valid; ++G) ti.next(args, BN);
      for (; ti.valid;) {
        const uint32_t ph = (G / kStages) & 1u;
        if (ti.it >= ti.my_kb) {
          // Extension stage: A arrives by TMA.  Still pass through this stage's
          // phases so that no later wait of the group is two phases ahead of a
          // barrier (a parity wait cannot tell those apart).
          if (!warp_wait(empty + grp, ph ^ 1u, abort_flag, args.status, lane)) break;
          if (!warp_wait(full + grp, ph, abort_flag, args.status, lane)) break;
        } else {
          const int kb = ti.kb_lo + ti.it;
          if (AMODE == A_DEQ_K) {
            // thread u = tile row (= TMEM lane), k = 0..63 of the stage
            const int64_t n = ti.row0 + u;
            float chat = 0.0f;
            if (n < args.wN) {
              const int64_t f = n * bpr + kb;
              chat = decode_scale(__ldg(args.c2 + f), __ldg(args.c1 + (f >> 8)));
            }
            const Nf4BlockTable tab = nf4_block_table(q, chat);
            if (!warp_wait(empty + grp, ph ^ 1u, abort_flag, args.status, lane)) break;
            tc_fence_after();
            if (!warp_wait(full + grp, ph, abort_flag, args.status, lane)) break;
            const uint8_t* ctile = smem + grp * L::STAGE + kA + L::B + u * 32;
            const int sw = (u >> 2) & 1;  // 32-byte swizzle of the code tile
            const uint4 c0 = *reinterpret_cast<const uint4*>(ctile + (sw << 4));
            const uint4 c1 = *reinterpret_cast<const uint4*>(ctile + ((sw ^ 1) << 4));
            const uint32_t taddr = tmem_d + ((uint32_t)(q4 * 32) << 16) + TM::a_col + (uint32_t)(grp * 32);
            uint32_t o[16];
            nf4_lookup8(c0.x, tab, o + 0);
            nf4_lookup8(c0.y, tab, o + 4);
            nf4_lookup8(c0.z, tab, o + 8);
            nf4_lookup8(c0.w, tab, o + 12);
            tmem_st16(taddr, o);
            nf4_lookup8(c1.x, tab, o + 0);
            nf4_lookup8(c1.y, tab, o + 4);
            nf4_lookup8(c1.z, tab, o + 8);
            nf4_lookup8(c1.w, tab, o + 12);
            tmem_st16(taddr + 16, o);
            tmem_wait_st();
            tc_fence_before();
          } else {
            // A = W^T in shared memory, MN-major: thread u = (W row n0 + nl,
            // NF4 block mb of the 128 tile rows), 64 weights.
            const int nl = u & 63, mb = u >> 6;
            const int64_t kblk = (int64_t)(ti.row0 >> 6) + mb;
            const int64_t nn = (int64_t)kb * 64 + nl;
            float chat = 0.0f;
            if (kblk < bpr && nn < args.wN) {
              const int64_t f = nn * bpr + kblk;
              chat = decode_scale(__ldg(args.c2 + f), __ldg(args.c1 + (f >> 8)));
            }
            const Nf4BlockTable tab = nf4_block_table(q, chat);
            if (!warp_wait(empty + grp, ph ^ 1u, abort_flag, args.status, lane)) break;
            if (!warp_wait(full + grp, ph, abort_flag, args.status, lane)) break;
            uint8_t* sa = smem + grp * L::STAGE;
            const uint8_t* ctile = sa + kA + L::B + nl * 64;
            const int swz = (nl >> 1) & 3;  // 64-byte swizzle of the code tile
            const int r8 = nl & 7;
            uint8_t* atile = sa + mb * 8192 + (nl >> 3) * 1024 + r8 * 128;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint4 cw = *reinterpret_cast<const uint4*>(ctile + (((2 * mb + h) ^ swz) << 4));
              const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint32_t o[4];
                nf4_lookup8(words[j], tab, o);
                const uint32_t c = (uint32_t)(4 * h + j);
                *reinterpret_cast<uint4*>(atile + ((c ^ (uint32_t)r8) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
              }
            }
            fence_proxy_async_smem();
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(afull + grp);
        }
        for (int k = 0; k < kStages && ti.valid; ++k, ++G) ti.next(args, BN);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;
    uint32_t tile_no = 0;
    for (int t = blockIdx.x; t < args.total_tiles; t += gridDim.x, ++tile_no) {
      TileIter ti;
      ti.t = t;
      ti.load(args, BN);
      const uint32_t b = tile_no % TM::n_acc, use = tile_no / TM::n_acc;
      const bool ok = warp_wait(acc_full + b, use & 1u, abort_flag, args.status, lane);
      if (!ok) break;
      tc_fence_after();
      const int64_t row = ti.row0 + q4 * 32 + lane;
      const bool row_ok = row < args.rows;
      const uint32_t tbase = tmem_d + b * TM::acc + ((uint32_t)(q4 * 32) << 16);
      for (int c = 0; c < BN; c += 16) {
        uint32_t v[16];
        tmem_ld16(tbase + (uint32_t)c, v);
        tmem_wait_ld();
        if (!row_ok) continue;
        const int ncol = min(16, args.cols - (ti.col0 + c));
        if (args.splits > 1) {
          float* dst = args.partial + ((int64_t)ti.z * args.cols + ti.col0 + c) * args.rows + row;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < ncol) dst[(int64_t)j * args.rows] = __uint_as_float(v[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < ncol) epi_store(args.epi, row, ti.col0 + c + j, __uint_as_float(v[j]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + b);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*abort_flag && lane == 0) {  // let in-flight copies and MMAs land before freeing TMEM
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 2000000ull) {
      }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_d, TM::cols);
  }
}

__global__ void split_reduce_kernel(const float* __restrict__ partial, int splits, int rows, int cols, EpiArgs e) {
  const int64_t total = (int64_t)rows * cols;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i % rows, col = i / rows;
    float acc = 0.0f;
    for (int z = 0; z < splits; ++z) acc += partial[((int64_t)z * cols + col) * rows + row];
    epi_store(e, row, col, acc);
  }
}

template <int BN, int AMODE>
cudaError_t launch_t(const EngineArgs& a, const GemmPlan& p, cudaStream_t st) {
  using L = Layout<BN, AMODE>;
  auto kern = umma_engine_kernel<BN, AMODE>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::TOTAL);
  if (err != cudaSuccess) return err;
  const int grid = a.total_tiles < p.num_sms ? a.total_tiles : p.num_sms;
  kern<<<grid, kThreads, L::TOTAL, st>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

template <int AMODE>
cudaError_t launch_mode(const EngineArgs& a, const GemmPlan& p, cudaStream_t st) {
  switch (p.BN) {
    case 16: return launch_t<16, AMODE>(a, p, st);
    case 32: return launch_t<32, AMODE>(a, p, st);
    case 64: return launch_t<64, AMODE>(a, p, st);
    case 128: return launch_t<128, AMODE>(a, p, st);
    case 192: return launch_t<192, AMODE>(a, p, st);
    case 256: return launch_t<256, AMODE>(a, p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

// Widest token tile: 256, or 192 where a second accumulator then fits in
// tensor memory next to the forward's dequantised A stages
// (QLORA_NF4_WIDE_BN=256|192 overrides the default for that case).
int wide_bn(int amode) {
  if (amode != A_DEQ_K) return 256;
  static int v = [] {
    const char* e = std::getenv("QLORA_NF4_WIDE_BN");
    const int x = e ? std::atoi(e) : 0;
    return (x == 192 || x == 256) ? x : 256;
  }();
  return v;
}

int bn_for_cols(int cols, int amode) {
  return cols <= 16 ? 16 : cols <= 32 ? 32 : cols <= 64 ? 64 : cols <= 128 ? 128 : wide_bn(amode);
}

GemmPlan plan_gemm(int rows, int cols, int kb_main, int num_sms, int amode) {
  GemmPlan p{};
  p.num_sms = num_sms;
  p.BN = bn_for_cols(cols, amode);
  p.m_tiles = (rows + 127) / 128;
  p.n_tiles = (cols + p.BN - 1) / p.BN;
  const int tiles = p.m_tiles * p.n_tiles;
  const int target = num_sms * (p.BN <= 64 ? 2 : 1);
  int splits = 1;
  if (tiles < target) {
    splits = (target + tiles - 1) / tiles;
    const int cap = kb_main / 4 > 1 ? kb_main / 4 : 1;
    if (splits > cap) splits = cap;
    if (splits > 64) splits = 64;
  }
  p.splits = splits;
  p.partial_bytes = splits > 1 ? (size_t)splits * rows * cols * sizeof(float) : 0;
  return p;
}

size_t engine_smem_bytes(int BN, int amode) {
  const int b = BN * 128 > 8192 ? BN * 128 : 8192;
  const int c = amode == A_TMA ? 0 : 4096;
  return (size_t)kStages * (kA + b + c) + 256 + 1024;
}

cudaError_t launch_engine(const EngineArgs& a, int amode, const GemmPlan& p, cudaStream_t st) {
  switch (amode) {
    case A_TMA: return launch_mode<A_TMA>(a, p, st);
    case A_DEQ_K: return launch_mode<A_DEQ_K>(a, p, st);
    case A_DEQ_MN: return launch_mode<A_DEQ_MN>(a, p, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_split_reduce(const float* partial, int splits, int rows, int cols, const EpiArgs& e,
                                cudaStream_t st) {
  const int64_t total = (int64_t)rows * cols;
  const int64_t want = (total + 255) / 256;
  const int grid = (int)(want < 4096 ? (want > 0 ? want : 1) : 4096);
  split_reduce_kernel<<<grid, 256, 0, st>>>(partial, splits, rows, cols, e);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qnf4
