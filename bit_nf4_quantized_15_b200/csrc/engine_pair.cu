// Forward fused dequant-GEMM on a CTA pair (tcgen05 cta_group::2).
//
//   Y^T[n, m] = RNbf16( sum_k W^[n, k] X[m, k] + sum_j L2^T[n, j] RNbf16(s.T)[m, j] )
//
// nlp-lineage "QLoRA" milestone page, section "The idea": the layer equation
// (the 4-bit weight is dequantised to bf16 and multiplied, the adapters stay
// bf16); inferensys glossary "QLoRA", kernel paragraph: the 4-bit weights are
// decompressed on chip and fed to the tensor cores as BFloat16.
//
// The two CTAs of a cluster compute one 256 (weight rows) x 256 (tokens)
// output tile with M = 256 UMMAs.  Each CTA
//   * dequantises its own 128 weight rows into its tensor memory (A operand),
//     as the single-CTA forward does (one 64-weight block per thread and
//     stage, register byte-plane tables, tcgen05.st), but each thread loads
//     its row's 32 code bytes itself, one round ahead, with two 16-byte
//     global loads.  A TMA box of 128 rows x 32 bytes moves at a fraction of
//     the rate of 128-byte rows: a clock trace of this kernel with the codes
//     on the TMA showed the loads queueing (latency growing to the ring's
//     depth, ~3.5 us) at 42 GB/s per SM, the code tile pacing every block;
//   * loads 128 of the tile's 256 token rows of X (B operand) into its shared
//     memory;
//   * ends with its own 128 x 256 fp32 accumulator in its tensor memory and
//     stores its 128 rows of Y^T.
// The even CTA's MMA thread issues the UMMAs; they read A and B from both
// CTAs.  Per 64-wide reduction block an SM pulls 16 KB of activations + 4 KB
// of codes from L2 instead of 32 + 4 KB for the same tensor work.
//
// Measured on the 4096-token LLaMA-7B linears this kernel is correct but not
// faster than the single-CTA forward (gate 11008 x 4096: 443 against 398 us):
// the block time stays at ~0.49 us whatever the activation bytes per SM, the
// ring depth (8, 10, 12 activation stages: 443, 458, 459 us) or the code
// path, so it is selected only on request (QLORA_NF4_PAIR=1).
//
// Barriers (same offsets in both CTAs):
//   full[b]   even CTA: both CTAs' activation tiles of stage b (each CTA's TMA
//             load completes its bytes on the even CTA's barrier);
//   bempty[b] each CTA: the UMMAs that read activation stage b have finished
//             (one commit, delivered to both CTAs);
//   afull[a]  even CTA: 8 arrivals, the four dequant warps of each CTA that
//             wrote their TMEM A buffer a;
//   aempty[a] each CTA: the UMMAs that read A buffer a have finished;
//   xfull    even CTA: the LoRA extension's A tiles (L2^T rows) of both CTAs;
//   accum    each CTA: the accumulator is final.
// Every wait is bounded (QNF4_WAIT_NS); a CTA that gives up flags the status
// word, and the pair meets at a cluster barrier before it frees its tensor
// memory, so neither CTA leaves while the other may still touch its memory.
#include "engine_util.cuh"

namespace qnf4 {
namespace {

#ifndef QNF4_PAIR_BSTAGES
#define QNF4_PAIR_BSTAGES 8
#endif
#ifndef QNF4_PAIR_GROUPS
#define QNF4_PAIR_GROUPS 4
#endif
// Two rings: activation tiles in shared memory (kPBS deep) and dequantised A
// tiles in tensor memory (kPA deep, all the columns the accumulator leaves).
constexpr int kPBS = QNF4_PAIR_BSTAGES;    // activation stages
constexpr int kPA = 8;                     // TMEM A buffers
constexpr int kPG = QNF4_PAIR_GROUPS;      // dequant / epilogue groups (kPA % kPG == 0)
constexpr int kPThreads = 64 + 32 * 4 * kPG;
constexpr int kPB = 16384;                 // activation tile: 128 token rows x 64 k, bf16, 128-byte swizzle
constexpr int kPStage = kPB;
constexpr int kPXA = 2 * 16384;            // extension A: up to two 64-wide blocks of L2^T, 128 rows each
constexpr int kPXOfs = kPBS * kPStage;
constexpr int kPBar = kPXOfs + kPXA;
constexpr int kPTotal = kPBar + 512 + 1024;  // barriers + alignment slack
constexpr uint32_t kPAcc = 256;            // accumulator columns; A buffer s at kPAcc + 32 s
constexpr uint32_t kPTmemCols = 512;
static_assert(kPA % kPG == 0, "an A buffer must always be served by the same dequant group");
static_assert(kPAcc + kPA * 32 <= kPTmemCols, "tensor memory");
static_assert(kPTotal <= 232448, "shared memory per CTA");
static_assert(kPStage % 1024 == 0 && kPXOfs % 1024 == 0, "swizzled tiles need 1024-byte alignment");

// ------------------------------------------------------ pair primitives
QDEV uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
QDEV uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
QDEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
QDEV void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
QDEV bool mbar_test_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait with cluster-scope acquire (arrivals from the peer CTA).
QDEV bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test_wait_cluster(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_test_wait_cluster(a, parity)) return true;
    if ((i & 63) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > QNF4_WAIT_NS) {
        *abort_flag = 1;
        report(status, QLORA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}
// 2-D TMA tile load into this CTA's shared memory whose bytes complete on an
// mbarrier of either CTA of the pair (`bar` is a cluster address).
QDEV void tma_load_2d_pair(void* dst, const CUtensorMap* m, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)m), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
QDEV void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
QDEV void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
QDEV void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (+)= A * B^T over the pair: A from tensor memory (each CTA's lanes hold
// its 128 rows), B from shared memory (each CTA holds N/2 rows at the same
// offset).
QDEV void umma_pair_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
QDEV void umma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at this offset in both CTAs of the pair when
// every UMMA issued so far has finished.
QDEV void umma_commit_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)0x3)
      : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPThreads, 1)
    umma_pair_fwd_kernel(const __grid_constant__ EngineArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xa = smem + kPXOfs;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPBar);
  uint64_t* bempty = full + kPBS;
  uint64_t* afull = bempty + kPBS;
  uint64_t* aempty = afull + kPA;
  uint64_t* xfull = aempty + kPA;
  uint64_t* accum = xfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = blockIdx.x * 128;            // this CTA's weight rows
  const int col0 = blockIdx.y * 256;            // the pair's tokens
  const int bcol0 = col0 + (int)rank * 128;     // this CTA's half of them
  const int n_kb = args.kb_main, n_ext = args.kb_ext;
  const int n_iters = n_kb + n_ext;

  if (tid == 0) {
    for (int b = 0; b < kPBS; ++b) {
      mbar_init(full + b, 1);
      mbar_init(bempty + b, 1);
    }
    for (int a = 0; a < kPA; ++a) {
      mbar_init(afull + a, 2 * 4);
      mbar_init(aempty + a, 1);
    }
    mbar_init(xfull, 1);
    mbar_init(accum, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&args.tmB);
    if (n_ext) {
      tma_prefetch_desc(&args.tmAx);
      tma_prefetch_desc(&args.tmBx);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kPTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers and tensor memory exist from here on
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  // The even CTA's barriers, addressed from either CTA.
  const uint32_t full0 = mapa_shared(smem_u32(full), 0);
  const uint32_t afull0 = mapa_shared(smem_u32(afull), 0);
  const uint32_t xfull0 = mapa_shared(smem_u32(xfull), 0);
  bool committed_accum = false;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      if (n_ext) {  // the extension's A tiles (L2^T, MN-major 64 x 64 boxes), once
        if (leader) mbar_arrive_expect_tx(xfull, 2u * (uint32_t)n_ext * 16384u);
        for (int kb = 0; kb < n_ext; ++kb)
          for (int j = 0; j < 2; ++j) tma_load_2d_pair(xa + kb * 16384 + j * 8192, &args.tmAx, xfull0, row0 + 64 * j, kb * 64);
      }
      for (int it = 0; it < n_iters; ++it) {
        const int b = it % kPBS;
        const uint32_t ph = (uint32_t)(it / kPBS) & 1u;
        if (!mbar_wait(bempty + b, ph ^ 1u, abort_flag, args.status)) break;
        uint8_t* sb = smem + b * kPStage;
        if (leader) mbar_arrive_expect_tx(full + b, 2u * kPB);
        if (it < n_kb) {
          tma_load_2d_pair(sb, &args.tmB, full0 + 8u * b, it * 64, bcol0);
        } else {  // RNbf16(s.T) tile of extension block it - n_kb
          tma_load_2d_pair(sb, &args.tmBx, full0 + 8u * b, (it - n_kb) * 64, bcol0);
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------- UMMA (even CTA only)
    if (leader && lane == 0) {
      const uint32_t id_main = idesc_bf16(256, 256, 0, 0);
      const uint32_t id_ext = idesc_bf16(256, 256, 1, 0);
      for (int it = 0; it < n_iters; ++it) {
        const int b = it % kPBS, a = it % kPA;
        const uint32_t phb = (uint32_t)(it / kPBS) & 1u, pha = (uint32_t)(it / kPA) & 1u;
        const bool ext = it >= n_kb;
        bool ok = mbar_wait(full + b, phb, abort_flag, args.status);
        if (ok && !ext) ok = mbar_wait_cluster(afull + a, pha, abort_flag, args.status);
        if (ok && it == n_kb) ok = mbar_wait(xfull, 0, abort_flag, args.status);
        if (!ok) break;
        tc_fence_after();
        const uint8_t* sb = smem + b * kPStage;
        if (!ext) {
          const uint32_t a_tmem = tmem_d + kPAcc + (uint32_t)(a * 32);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_pair_tmem_a(tmem_d, a_tmem + kk * 8, operand_desc(sb, 0, kk), id_main, (it | kk) != 0);
        } else {
          const uint8_t* ea = xa + (it - n_kb) * 16384;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_pair(tmem_d, operand_desc(ea, 1, kk), operand_desc(sb, 0, kk), id_ext, (it | kk) != 0);
        }
        umma_commit_both(bempty + b);
        if (!ext) umma_commit_both(aempty + a);
      }
      umma_commit_both(accum);
      committed_accum = true;
    }
    __syncwarp();
  } else {
    const int dw = warp - 2;  // dequant warp 0 .. 4 kPG - 1
    const int q4 = warp & 3;  // TMEM lane quarter this warp may access
    const int grp = dw >> 2;  // iterations grp, grp + kPG, ... (A buffers a with a % kPG == grp)
    const int64_t bpr = args.wK / 64;
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = args.q[i];
    // ------------------------------------------------------------- dequant
    // Thread: weight row rl of this CTA (= its TMEM lane), the stage's 64 k.
    {
      const int rl = q4 * 32 + lane;
      const int64_t n = row0 + rl;
      const bool valid = n < args.wN;
      const uint32_t tlane = tmem_d + ((uint32_t)(q4 * 32) << 16) + kPAcc;
      const uint4* crow = reinterpret_cast<const uint4*>(args.codes + (valid ? n : 0) * (args.wK / 2));
      uint32_t c2raw = 0;
      GroupScale gsc{0.0f, 0.0f};
      uint4 cn0 = make_uint4(0, 0, 0, 0), cn1 = cn0;  // this group's next code block (k 0..31, 32..63)
      if (valid && grp < n_kb) {
        const int64_t f = n * bpr + grp;
        cn0 = __ldg(crow + 2 * grp);
        cn1 = __ldg(crow + 2 * grp + 1);
        c2raw = __ldg(args.c2 + f);
        gsc = load_group_scale(args.c1, f >> 8, args.c1_mean != 0);
      }
      for (int it = grp; it < n_kb; it += kPG) {
        const int a = it % kPA;
        const uint32_t ph = (uint32_t)(it / kPA) & 1u;
        const uint32_t taddr = tlane + (uint32_t)(a * 32);
        const uint4 c0 = cn0, c1 = cn1;
        const float chat = valid ? decode_scale(c2raw, gsc, args.c2_e5m2 != 0, args.c1_mean != 0) : 0.0f;
        if (valid && it + kPG < n_kb) {  // this group's next codes and scale, one round ahead
          const int64_t f = n * bpr + it + kPG;
          cn0 = __ldg(crow + 2 * (it + kPG));
          cn1 = __ldg(crow + 2 * (it + kPG) + 1);
          c2raw = __ldg(args.c2 + f);
          gsc = load_group_scale(args.c1, f >> 8, args.c1_mean != 0);
        }
        const Nf4BlockTable tab = nf4_block_table(q, chat);
        if (!warp_wait(aempty + a, ph ^ 1u, abort_flag, args.status, lane)) break;
        tc_fence_after();
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
        if (lane == 0) mbar_arrive_cluster(afull0 + 8u * a);
      }
    }
    // ------------------------------------------------------------ epilogue
    // kPG warps per lane quarter: group grp stores the 16-column chunks grp,
    // grp + kPG, ... of this CTA's 128 x 256 accumulator.
    const bool ok = warp_wait(accum, 0, abort_flag, args.status, lane);
    tc_fence_after();
    const int64_t row = row0 + q4 * 32 + lane;
    const EpiArgs& e = args.epi;
    for (int c = grp * 16; c < 256; c += kPG * 16) {
      uint32_t v[16];
      tmem_ld16(tmem_d + ((uint32_t)(q4 * 32) << 16) + (uint32_t)c, v);
      tmem_wait_ld();
      if (!ok || *abort_flag || row >= args.rows) continue;
      const int64_t col = col0 + c;
      const int ncol = min(16, args.cols - (int)col);
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(e.out) + row * e.rs + col * e.cs;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < ncol) dst[j * e.cs] = __float2bfloat16_rn(__fmul_rn(__uint_as_float(v[j]), e.alpha));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // Error path: let the even CTA's UMMAs and any TMA load still in flight
    // finish before the pair meets and frees its tensor memory.
    if (warp == 1 && lane == 0 && committed_accum) mbar_wait_drain(accum, 0, 10000000ull);
    if (tid == 0) {
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 2000000ull) {
      }
    }
    __syncthreads();
  }
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_d, kPTmemCols);
  }
}

}  // namespace

bool pair_fwd_supported(int rows, int cols, int kb_ext) {
  (void)rows;
  return cols > 128 && kb_ext >= 0 && kb_ext * 16384 <= kPXA;
}

size_t pair_fwd_smem_bytes() { return kPTotal; }

cudaError_t launch_pair_fwd(const EngineArgs& a, cudaStream_t st) {
  if (!pair_fwd_supported(a.rows, a.cols, a.kb_ext) || a.splits > 1 || !a.epi.out || !a.epi.out_bf16)
    return cudaErrorInvalidValue;
  auto kern = umma_pair_fwd_kernel;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPTotal);
  if (err != cudaSuccess) return err;
  dim3 grid(2 * ((a.rows + 255) / 256), (a.cols + 255) / 256, 1);
  kern<<<grid, kPThreads, kPTotal, st>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qnf4
