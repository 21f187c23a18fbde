// The tcgen05 GEMM engine behind every contraction of the layer.
//
//   D[rows x cols] (fp32, in TMEM) = sum_k A[row, k] * B[col, k]
//
// One CTA computes a 128 x BN output tile with cta_group::1 UMMA (M = 128).
// The reduction runs in 64-wide blocks through a shared-memory ring (see
// Ring for its depth per mode):
//   * warp 0, one lane: TMA producer (B tiles, A tiles or NF4 code tiles),
//     stages in order; for dX a second producer warp fills a separate ring
//     of code tiles;
//   * warp 1, one lane: UMMA issuer, 4 x (128 x BN x 16) MMAs per stage,
//     tcgen05.commit frees the stage;
//   * dequant groups of 4 warps (128 threads): when A is the NF4 weight,
//     they turn the code tile into a bf16 tile, in tensor memory for X.W^T
//     or in the 128-byte-swizzled MN-major shared-memory layout for dY.W,
//     then all groups run the epilogue (TMEM -> registers -> global, one
//     accumulator row per thread).
// An optional extension segment appends more reduction blocks from other
// operands into the same accumulator: this is how the LoRA term s.T.L2
// (forward) and s.dT.L1^T (backward) is added to the dequantised product.
// A split of the main reduction over grid.z writes fp32 partial tiles that
// a second kernel sums in a fixed order (deterministic).
//
// inferensys glossary "QLoRA", kernel paragraph: 4-bit weights are loaded,
// decompressed in shared memory and fed to the tensor cores as BFloat16.
#include "engine_util.cuh"

namespace qnf4 {
namespace {

constexpr int kGroupWarps = 4;  // a dequant group: 4 warps, one per TMEM lane quarter
constexpr int kRasterGroup = 4;  // column tiles per raster group (see the kernel's tile mapping)

// Ring shape per A source.  The forward keeps its dequantised A tile in
// TMEM, so its stages hold only B and the codes (36 KB) and six of them fit
// (measured: the TMA bytes land and the stage is dequantised well before the
// UMMA thread reaches it; 4 or 5 stages were a few percent slower).  Three
// dequant groups (stage s always served by group s % 3).  dX and the plain GEMMs keep A in shared memory: four stages of
// A + B (48 KB at BN = 256), four groups (dX: group g owns stage g).
//
// dX keeps its code tiles in a ring of their own (CS stages of 4 KB, filled by
// a second producer warp): a dequant group frees a code stage as soon as it
// has read it, so the codes of the group's next stage are already there when
// the MMAs free its A buffer, instead of being fetched only then (measured:
// the group waited ~0.7 us per stage for them).
template <int AMODE>
struct Ring {
  static constexpr int S = AMODE == A_DEQ_K ? 6 : 4;     // stages
  static constexpr int G = AMODE == A_DEQ_K ? 3 : 4;     // dequant (and epilogue) groups
  static constexpr int KA = AMODE == A_DEQ_K ? 0 : 16384;  // A tile in shared memory (128 x 64 bf16)
  static constexpr int CS = AMODE == A_DEQ_MN ? 8 : 0;     // dX code-ring stages (a multiple of S)
  static constexpr int CODE_WARP = 2 + kGroupWarps * G;    // dX: the code producer's warp
  // producer warp + UMMA warp + dequant groups (+ the dX code producer warp)
  static constexpr int THREADS = 64 + 32 * kGroupWarps * G + (CS ? 32 : 0);
};

// Tensor-memory columns: the fp32 accumulator (BN columns, at least 32) and,
// for the forward fused GEMM, the dequantised A tile of every stage
// (128 lanes x 32 columns: 64 bf16 per lane).
template <int BN, int AMODE>
struct Tmem {
  static constexpr uint32_t acc = BN < 32 ? 32 : BN;
  static constexpr uint32_t a_col = acc;
  static constexpr uint32_t need = acc + (AMODE == A_DEQ_K ? Ring<AMODE>::S * 32 : 0);
  static constexpr uint32_t cols = need <= 32 ? 32 : need <= 64 ? 64 : need <= 128 ? 128 : need <= 256 ? 256 : 512;
};

// Stage = [A (KA)] [B] [codes (forward)]; then dX's code ring.  In the
// forward the B slot also carries the LoRA extension's A tiles (L2^T, 16 KB
// per 64-wide block, up to two), so it is at least 32 KB there.
template <int BN, int AMODE>
struct Layout {
  static constexpr int BMIN = AMODE == A_DEQ_K ? 32768 : 8192;
  static constexpr int B = BN * 128 > BMIN ? BN * 128 : BMIN;
  static constexpr int C = AMODE == A_DEQ_K ? 4096 : 0;
  static constexpr int STAGE = Ring<AMODE>::KA + B + C;
  static constexpr int CODE = Ring<AMODE>::S * STAGE;  // dX code ring (1024-aligned: STAGE is)
  static constexpr int BAR = CODE + Ring<AMODE>::CS * 4096;
  static constexpr int TOTAL = BAR + 512 + 1024;  // barriers etc. + alignment slack
};

template <int BN, int AMODE>
__global__ void __launch_bounds__(Ring<AMODE>::THREADS, 1) umma_engine_kernel(const __grid_constant__ EngineArgs args) {
  using L = Layout<BN, AMODE>;
  using TM = Tmem<BN, AMODE>;
  using R = Ring<AMODE>;
  constexpr int kStages = R::S;
  constexpr int kA = R::KA;
  constexpr int kCS = R::CS;
  constexpr int kCSd = kCS ? kCS : 1;  // divisor for the code-ring index (dX only)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR);
  uint64_t* afull = full + kStages;
  uint64_t* empty = afull + kStages;
  uint64_t* cfull = empty + kStages;  // dX code ring
  uint64_t* cempty = cfull + kCS;
  uint64_t* accum = cempty + kCS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Grouped raster over the linear block index: consecutive CTAs take up to
  // kRasterGroup column tiles (tokens) of one row tile (weight), then the
  // next row tile.  The CTAs resident at a time then share a few activation
  // tiles (kept in L2) and each weight tile's codes are read from HBM once
  // per group of column tiles instead of once per column tile.
  int row_tile, col_tile;
  {
    const int m_tiles = (args.rows + 127) / 128, n_tiles = (args.cols + BN - 1) / BN;
    const int id = blockIdx.x;
    const int per_group = kRasterGroup * m_tiles;
    const int gid = id / per_group, local = id % per_group;
    const int gsize = min(kRasterGroup, n_tiles - gid * kRasterGroup);
    col_tile = gid * kRasterGroup + local % gsize;
    row_tile = local / gsize;
  }
  const int row0 = row_tile * 128, col0 = col_tile * BN, z = blockIdx.z;
  const int kb_lo = (int)((int64_t)z * args.kb_main / args.splits);
  const int kb_hi = (int)((int64_t)(z + 1) * args.kb_main / args.splits);
  const int my_kb = kb_hi - kb_lo;
  // The LoRA extension: forward = one stage with the L2^T tiles (A) then one
  // stage per 64-wide block with the s.T tile (B); otherwise one stage per
  // block holding both.
  const int ext_iters = z == 0 && args.kb_ext ? (AMODE == A_DEQ_K ? 1 + args.kb_ext : args.kb_ext) : 0;
  const int n_iters = my_kb + ext_iters;
  const uint64_t lim = args.wait_ns ? args.wait_ns : QNF4_WAIT_NS;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(afull + s, kGroupWarps);
      mbar_init(empty + s, 1);
    }
    for (int c = 0; c < kCS; ++c) {
      mbar_init(cfull + c, 1);
      mbar_init(cempty + c, kGroupWarps);
    }
    mbar_init(accum, 1);
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
  bool committed_accum = false;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // One thread issues every stage in order.  (Spreading the stages over
    // several lanes of this warp, each spinning on its own barrier, was
    // measured slower: divergent spinning lanes of one warp take turns, so a
    // lane whose stage is free can wait behind another's spin loop.)
    if (lane == 0 && !args.stall) {
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        if (!mbar_wait(empty + s, ph ^ 1u, abort_flag, args.status, lim)) break;
        uint8_t* sa = smem + s * L::STAGE;
        uint8_t* sb = sa + kA;
        uint8_t* sc = sb + L::B;
        if (it < my_kb) {
          const int kb = kb_lo + it;
          uint32_t bytes = tx_bytes(args.b_mn_main, BN);
          bytes += AMODE == A_TMA ? tx_bytes(args.a_mn_main, 128) : AMODE == A_DEQ_K ? 4096u : 0u;
          mbar_arrive_expect_tx(full + s, bytes);
          if (AMODE == A_DEQ_K) tma_load_2d(sc, &args.tmA, full + s, kb * 32, row0);
          else if (AMODE == A_TMA) load_operand(sa, &args.tmA, full + s, args.a_mn_main, row0, kb * 64, 128);
          load_operand(sb, &args.tmB, full + s, args.b_mn_main, col0, kb * 64, BN);
        } else if (AMODE == A_DEQ_K) {
          if (it == my_kb) {  // all extension A tiles into this stage's B slot
            mbar_arrive_expect_tx(full + s, (uint32_t)args.kb_ext * tx_bytes(args.a_mn_ext, 128));
            for (int kb = 0; kb < args.kb_ext; ++kb)
              load_operand(sb + kb * 16384, &args.tmAx, full + s, args.a_mn_ext, row0, kb * 64, 128);
          } else {            // the s.T tile of extension block it - my_kb - 1
            const int kb = it - my_kb - 1;
            mbar_arrive_expect_tx(full + s, tx_bytes(args.b_mn_ext, BN));
            load_operand(sb, &args.tmBx, full + s, args.b_mn_ext, col0, kb * 64, BN);
          }
        } else {
          const int kb = it - my_kb;
          mbar_arrive_expect_tx(full + s, tx_bytes(args.a_mn_ext, 128) + tx_bytes(args.b_mn_ext, BN));
          load_operand(sa, &args.tmAx, full + s, args.a_mn_ext, row0, kb * 64, 128);
          load_operand(sb, &args.tmBx, full + s, args.b_mn_ext, col0, kb * 64, BN);
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- UMMA
    if (lane == 0) {
      const int a_mn_main = AMODE == A_DEQ_MN ? 1 : (AMODE == A_DEQ_K ? 0 : args.a_mn_main);
      const uint32_t id_main = idesc_bf16(128, BN, a_mn_main, args.b_mn_main);
      const uint32_t id_ext = idesc_bf16(128, BN, args.a_mn_ext, args.b_mn_ext);
      int s_ext_a = -1;  // forward: stage holding the extension's A tiles
      // The barrier that says iteration i may be issued.  A dequantised
      // stage is waited on through afull alone: its group arrives there only
      // after it has seen the stage's TMA bytes land (full, acquire), so the
      // B tile is complete too.
      auto ready_bar = [&](int i) { return (AMODE != A_TMA && i < my_kb ? afull : full) + i % kStages; };
      bool next_ready = false;
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        const bool ext = it >= my_kb;
        const bool ok = next_ready || mbar_wait(ready_bar(it), ph, abort_flag, args.status, lim);
        if (!ok) break;
        tc_fence_after();
        // Look at the next iteration's barrier now, before this stage's
        // MMAs and commit go out, so that a stage found ready needs no
        // barrier read between one stage's commit and the next stage's MMAs
        // (measured: 3-5 % faster forward).
        next_ready = it + 1 < n_iters &&
                     mbar_test_wait(smem_u32(ready_bar(it + 1)), (uint32_t)((it + 1) / kStages) & 1u);
        const uint8_t* sa = smem + s * L::STAGE;
        const uint8_t* sb = sa + kA;
        if (AMODE == A_DEQ_K && !ext) {
          // A: dequantised weight tile in tensor memory, 8 columns per K = 16
          const uint32_t a_tmem = tmem_d + TM::a_col + (uint32_t)(s * 32);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_tmem_a(tmem_d, a_tmem + kk * 8, operand_desc(sb, args.b_mn_main, kk), id_main,
                             (it | kk) != 0);
          umma_commit(empty + s);
        } else if (AMODE == A_DEQ_K) {
          if (it == my_kb) {  // the A tiles: keep the stage until the last extension block
            s_ext_a = s;
            continue;
          }
          const int kb = it - my_kb - 1;
          const uint8_t* ea = smem + s_ext_a * L::STAGE + kA + kb * 16384;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem_d, operand_desc(ea, args.a_mn_ext, kk), operand_desc(sb, args.b_mn_ext, kk), id_ext,
                      (it | kk) != 0);
          umma_commit(empty + s);
          if (kb == args.kb_ext - 1) umma_commit(empty + s_ext_a);
        } else {
          const int amn = ext ? args.a_mn_ext : a_mn_main;
          const int bmn = ext ? args.b_mn_ext : args.b_mn_main;
          const uint32_t id = ext ? id_ext : id_main;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem_d, operand_desc(sa, amn, kk), operand_desc(sb, bmn, kk), id, (it | kk) != 0);
          umma_commit(empty + s);
        }
      }
      umma_commit(accum);
      committed_accum = true;
    }
    __syncwarp();
  } else if (kCS && warp == R::CODE_WARP) {
    // ----------------------------------------------- dX code-ring producer
    if (lane == 0 && !args.stall) {
      for (int it = 0; it < my_kb; ++it) {
        const int c = it % kCSd;
        if (!mbar_wait(cempty + c, ((uint32_t)(it / kCSd) & 1u) ^ 1u, abort_flag, args.status, lim)) break;
        mbar_arrive_expect_tx(cfull + c, 4096u);
        tma_load_2d(smem + L::CODE + c * 4096, &args.tmA, cfull + c, row0 / 2, (kb_lo + it) * 64);
      }
    }
  } else {
    const int dw = warp - 2;           // dequant warp 0 .. 4G-1
    const int q4 = warp & 3;           // TMEM lane quarter this warp may access
    const int grp = dw >> 2;           // group: iterations grp, grp + G, ...
    const int64_t bpr = args.wK / 64;  // NF4 blocks per weight row
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = args.q[i];
    // ------------------------------------------------------------- dequant
    // Group grp handles the iterations it = grp, grp + G, ... (ring stages
    // it % S, always this group's since G divides S); each thread turns one
    // whole NF4 block (64 weights, one scale) into bf16 per iteration.
    if (AMODE == A_DEQ_K) {
      // Thread: tile row rl (= TMEM lane), k = 0..63 of the stage.
      const int rl = q4 * 32 + lane;
      const int64_t n = row0 + rl;
      const bool valid = n < args.wN;
      const uint32_t tlane = tmem_d + ((uint32_t)(q4 * 32) << 16) + TM::a_col;
      const int sw = (rl >> 2) & 1;  // 32-byte swizzle of the code tile
      uint32_t c2raw = 0;
      GroupScale gsc{0.0f, 0.0f};
      if (valid && grp < my_kb) {
        const int64_t f = n * bpr + kb_lo + grp;
        c2raw = __ldg(args.c2 + f);
        gsc = load_group_scale(args.c1, f >> 8, args.c1_mean != 0);
      }
      for (int it = grp; it < my_kb; it += R::G) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        const uint32_t taddr = tlane + (uint32_t)(s * 32);
        const uint8_t* ctile = smem + s * L::STAGE + kA + L::B + rl * 32;
        const float chat = valid ? decode_scale(c2raw, gsc, args.c2_e5m2 != 0, args.c1_mean != 0) : 0.0f;
        if (valid && it + R::G < my_kb) {  // this group's next scale, one round ahead
          const int64_t f = n * bpr + kb_lo + it + R::G;
          c2raw = __ldg(args.c2 + f);
          gsc = load_group_scale(args.c1, f >> 8, args.c1_mean != 0);
        }
        const Nf4BlockTable tab = nf4_block_table(q, chat);
        if (!warp_wait(empty + s, ph ^ 1u, abort_flag, args.status, lane, lim)) break;
        tc_fence_after();
        if (!warp_wait(full + s, ph, abort_flag, args.status, lane, lim)) break;
        const uint4 c0 = *reinterpret_cast<const uint4*>(ctile + (sw << 4));
        const uint4 c1 = *reinterpret_cast<const uint4*>(ctile + ((sw ^ 1) << 4));
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
        __syncwarp();
        if (lane == 0) mbar_arrive(afull + s);
      }
    } else if (AMODE == A_DEQ_MN) {
      // A = W^T in shared memory, MN-major: rows are k (W columns), the
      // reduction runs over n (W rows).  Thread u of the group: W row
      // n0 + nl and the 64 k of NF4 block mb (k_local = 64*mb ..).
      const int u = q4 * 32 + lane;
      const int nl = u & 63, mb = u >> 6;
      const int64_t kblk = (int64_t)(row0 >> 6) + mb;
      const bool kvalid = kblk < bpr;
      const int r8 = nl & 7;
      const int swz = (nl >> 1) & 3;  // 64-byte swizzle of the code tile
      uint8_t* sa = smem + grp * L::STAGE;
      uint8_t* atile = sa + mb * 8192 + (nl >> 3) * 1024 + r8 * 128;
      uint32_t c2raw = 0;
      GroupScale gsc{0.0f, 0.0f};
      {
        const int64_t nn = (int64_t)(kb_lo + grp) * 64 + nl;
        if (kvalid && nn < args.wN && grp < my_kb) {
          const int64_t f = nn * bpr + kblk;
          c2raw = __ldg(args.c2 + f);
          gsc = load_group_scale(args.c1, f >> 8, args.c1_mean != 0);
        }
      }
      for (int it = grp; it < my_kb; it += kStages) {
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        const int64_t nn = (int64_t)(kb_lo + it) * 64 + nl;
        const bool valid = kvalid && nn < args.wN;
        const float chat = valid ? decode_scale(c2raw, gsc, args.c2_e5m2 != 0, args.c1_mean != 0) : 0.0f;
        if (it + kStages < my_kb) {
          const int64_t nx = nn + 64 * kStages;
          c2raw = 0;
          gsc = GroupScale{0.0f, 0.0f};
          if (kvalid && nx < args.wN) {
            const int64_t f = nx * bpr + kblk;
            c2raw = __ldg(args.c2 + f);
            gsc = load_group_scale(args.c1, f >> 8, args.c1_mean != 0);
          }
        }
        const Nf4BlockTable tab = nf4_block_table(q, chat);
        // the codes first (their ring stage is freed once read), then the A buffer
        const int c = it % kCSd;
        if (!warp_wait(cfull + c, (uint32_t)(it / kCSd) & 1u, abort_flag, args.status, lane, lim)) break;
        const uint8_t* ctile = smem + L::CODE + c * 4096 + nl * 64;
        uint4 cws[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) cws[h] = *reinterpret_cast<const uint4*>(ctile + (((2 * mb + h) ^ swz) << 4));
        // these generic-proxy reads must be ordered before the TMA (async
        // proxy) that refills the stage once it is freed
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(cempty + c);
        if (!warp_wait(empty + grp, ph ^ 1u, abort_flag, args.status, lane, lim)) break;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint4 cw = cws[h];
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
        // the B tile of this stage has landed (usually long since): the UMMA
        // thread waits on afull alone
        if (!warp_wait(full + grp, ph, abort_flag, args.status, lane, lim)) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(afull + grp);
      }
    }
    // ------------------------------------------------------------ epilogue
    // G warps per lane quarter: group grp stores the 16-column chunks
    // grp, grp + G, ... of the tile.
    const bool ok = warp_wait(accum, 0, abort_flag, args.status, lane, lim);
    tc_fence_after();
    const int64_t row = row0 + q4 * 32 + lane;
    const EpiArgs& e = args.epi;
    for (int c = grp * 16; c < BN; c += R::G * 16) {
      uint32_t v[16];
      tmem_ld16(tmem_d + ((uint32_t)(q4 * 32) << 16) + (uint32_t)c, v);
      tmem_wait_ld();
      if (!ok || *abort_flag || row >= args.rows) continue;
      const int64_t col = col0 + c;
      const int ncol = min(16, args.cols - (int)col);
      if (args.splits > 1) {
        float* dst = args.partial + ((int64_t)z * args.cols + col) * args.rows + row;
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (j < ncol) dst[(int64_t)j * args.rows] = __uint_as_float(v[j]);
      } else {
        if (e.out) {
          if (e.out_bf16) {
            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(e.out) + row * e.rs + col * e.cs;
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (j < ncol) dst[j * e.cs] = __float2bfloat16_rn(__fmul_rn(__uint_as_float(v[j]), e.alpha));
          } else {
            float* dst = reinterpret_cast<float*>(e.out) + row * e.rs + col * e.cs;
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (j < ncol) dst[j * e.cs] = __fmul_rn(__uint_as_float(v[j]), e.alpha);
          }
        }
        if (e.out2) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(e.out2) + row * e.rs2 + col * e.cs2;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < ncol) dst[j * e.cs2] = __float2bfloat16_rn(__fmul_rn(__uint_as_float(v[j]), e.alpha2));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*abort_flag && lane == 0 && committed_accum) mbar_wait_drain(accum, 0, 10000000ull);
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
  dim3 grid(p.m_tiles * p.n_tiles, 1, p.splits);
  kern<<<grid, Ring<AMODE>::THREADS, L::TOTAL, st>>>(a);
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
    case 256: return launch_t<256, AMODE>(a, p, st);
  }
  return cudaErrorInvalidValue;
}

template <int AMODE>
size_t smem_for(int BN) {
  switch (BN) {
    case 16: return Layout<16, AMODE>::TOTAL;
    case 32: return Layout<32, AMODE>::TOTAL;
    case 64: return Layout<64, AMODE>::TOTAL;
    case 128: return Layout<128, AMODE>::TOTAL;
    default: return Layout<256, AMODE>::TOTAL;
  }
}

}  // namespace

int bn_for_cols(int cols) { return cols <= 16 ? 16 : cols <= 32 ? 32 : cols <= 64 ? 64 : cols <= 128 ? 128 : 256; }

GemmPlan plan_gemm(int rows, int cols, int kb_main, int num_sms) {
  GemmPlan p{};
  p.BN = bn_for_cols(cols);
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
  switch (amode) {
    case A_DEQ_K: return smem_for<A_DEQ_K>(BN);
    case A_DEQ_MN: return smem_for<A_DEQ_MN>(BN);
    default: return smem_for<A_TMA>(BN);
  }
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
