// Device helpers for sm_100a: mbarriers with bounded waits, TMA tile loads,
// tcgen05 (TMEM allocation, UMMA issue/commit, TMEM loads) and the shared
// memory / instruction descriptors that UMMA consumes.
//
// Every wait on an mbarrier is bounded: after QNF4_WAIT_NS of spinning the
// waiting thread records QLORA_ERR_TIMEOUT in the caller's status word, raises
// the CTA's abort flag and returns false, so a wedged pipeline ends the
// kernel instead of hanging the GPU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qlora_nf4.h"

#define QDEV __device__ __forceinline__

#ifndef QNF4_WAIT_NS
#define QNF4_WAIT_NS 4000000000ull  // 4 s: far beyond any legitimate wait
#endif

namespace qnf4 {

QDEV uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

QDEV uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

QDEV void report(int* status, int code) {
  if (status) atomicExch(status, code);
}

// ------------------------------------------------------------------ mbarrier
QDEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
QDEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
QDEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
QDEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// Non-blocking test of a phase (test_wait, with acquire semantics).  The
// waits below poll with it rather than with try_wait: try_wait may suspend
// the thread, and a suspended waiter was measured to resume about 0.5 us
// after the phase completed, which put a floor under every pipeline stage
// (one TMA box per 0.5 us per waiting producer).
QDEV bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Bounded: returns
// false (after flagging the CTA and the caller's status) on timeout or when
// another role of the CTA has already aborted.  Plain polling with test_wait
// (see mbar_test_wait).
// `limit_ns` is the bound (QNF4_WAIT_NS unless a launch asks for less).
QDEV bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                    uint64_t limit_ns = QNF4_WAIT_NS) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_test_wait(a, parity)) return true;
    if ((i & 63) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit_ns) {
        *abort_flag = 1;
        report(status, QLORA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// The same bounded wait for a thread that is not on the critical path (a
// producer refilling a ring that is usually full): it sleeps between polls
// so that its spinning does not take issue slots from the warps that work.
QDEV bool mbar_wait_backoff(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                            uint32_t sleep_ns, uint64_t limit_ns = QNF4_WAIT_NS) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    __nanosleep(sleep_ns);
    if (mbar_test_wait(a, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort_flag = 1;
      report(status, QLORA_ERR_TIMEOUT);
      return false;
    }
  }
}

// Short bounded wait used only while draining after an abort.
QDEV void mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer();
  while (!mbar_test_wait(a, parity)) {
    if (globaltimer() - t0 > ns) return;
  }
}

QDEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ----------------------------------------------------------------------- TMA
QDEV void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)m) : "memory");
}
// 2-D tiled load into this CTA's shared memory, completion counted in bytes
// on `bar`.  x is the innermost coordinate (elements), y the outer one.
QDEV void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)m), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// 3-D tiled load (x innermost, then y, then z), completion on `bar`.
QDEV void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)m), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// ------------------------------------------------------------------- tcgen05
QDEV void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
QDEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
QDEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
QDEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
QDEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulation.
QDEV void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Same with A read from tensor memory (M = 128 lanes, 8 columns per K = 16:
// column j of a lane holds the two bf16 elements 2j (low half) and 2j+1).
QDEV void umma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every previously issued tcgen05.mma has finished.
QDEV void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// 32 lanes x 16 consecutive 32-bit columns: thread i of the warp receives
// lane (taddr.lane + i), columns taddr.col .. +15.
QDEV void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
QDEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// 32 lanes x 16 consecutive 32-bit columns, registers -> tensor memory.
QDEV void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
QDEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for a 128-byte-swizzled canonical layout.
//   K-major : atoms of 8 rows x 128 B; sbo = byte stride between 8-row groups.
//   MN-major: atoms of 8 K-rows x 128 B (64 MN elements); lbo = byte stride
//             between 64-element MN blocks, sbo = stride between 8-row K groups.
QDEV uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | ((uint32_t)a_mn_major << 15)  // A major-ness
         | ((uint32_t)b_mn_major << 16)  // B major-ness
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// ------------------------------------------------------------- small codecs
QDEV float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

// E4M3 code -> fp32 (exact: every E4M3 value is an fp16 value).
QDEV float e4m3_to_float(uint32_t code) {
  __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
  return __half2float(__half(hr));
}

// E5M2 code -> fp32 (exact: an E5M2 byte is the high byte of the fp16 of the
// same value).
QDEV float e5m2_to_float(uint32_t code) { return __half2float(__ushort_as_half((unsigned short)(code << 8))); }

// Second-level scale of a group of 256 blocks: c1 and, for the mean-centred
// codec (QLORA_SCALE_E4M3_MEAN, whose c1 array holds [c1, mean] pairs), the
// group mean of the block scales.
struct GroupScale {
  float c1, mu;
};
QDEV GroupScale load_group_scale(const float* c1, int64_t g, bool mean) {
  if (mean) {
    const float2 v = __ldg(reinterpret_cast<const float2*>(c1) + g);
    return GroupScale{v.x, v.y};
  }
  return GroupScale{__ldg(c1 + g), 0.0f};
}

// Decoded block scale c^ = RN32(dec(c2) * c1); c2 is E4M3, or E5M2 for the
// scale-codec variant; the mean-centred codec adds the group mean with a
// second rounding, RN32(RN32(dec(c2) * c1) + mean) (signed E4M3 residual).
QDEV float decode_scale(uint32_t c2code, GroupScale gs, bool e5m2, bool mean) {
  const float p = __fmul_rn(e5m2 ? e5m2_to_float(c2code) : e4m3_to_float(c2code), gs.c1);
  return mean ? __fadd_rn(p, gs.mu) : p;
}

QDEV uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------- NF4 block table in registers
// For one 64-weight block with decoded scale c^, the 16 possible dequantised
// values T[i] = RNbf16(RN32(q[i] * c^)) are computed once and kept as byte
// planes: L[m] holds the low bytes of T[4m .. 4m+3], H[m] the high bytes.
struct Nf4BlockTable {
  uint32_t L[4], H[4];
};

QDEV Nf4BlockTable nf4_block_table(const float (&q)[16], float chat) {
  uint32_t P[8];
  const float2 cc = make_float2(chat, chat);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 pr = __fmul2_rn(make_float2(q[2 * j], q[2 * j + 1]), cc);  // two RN32 products
    P[j] = pack_bf16x2(pr.x, pr.y);
  }
  Nf4BlockTable t;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    t.L[m] = __byte_perm(P[2 * m], P[2 * m + 1], 0x6420);
    t.H[m] = __byte_perm(P[2 * m], P[2 * m + 1], 0x7531);
  }
  return t;
}

// Four codes -> two bf16x2 words (T[c0] | T[c1] << 16, T[c2] | T[c3] << 16)
// by byte permutes: `sel` holds the codes' low three bits (one per nibble),
// they pick a byte out of an 8-entry plane pair; `hi8` (nibble i = i + 4 when
// code i >= 8) picks the plane pair.  A byte permute reads only the low 16
// bits of its selector.
QDEV void nf4_lookup4(uint32_t sel, uint32_t hi8, const Nf4BlockTable& t, uint32_t& out0, uint32_t& out1) {
  const uint32_t lo = __byte_perm(__byte_perm(t.L[0], t.L[1], sel), __byte_perm(t.L[2], t.L[3], sel), hi8);
  const uint32_t hi = __byte_perm(__byte_perm(t.H[0], t.H[1], sel), __byte_perm(t.H[2], t.H[3], sel), hi8);
  out0 = __byte_perm(lo, hi, 0x5140);
  out1 = __byte_perm(lo, hi, 0x7362);
}

// Eight codes (one 32-bit word, element i in nibble i) -> four bf16x2 words.
QDEV void nf4_lookup8(uint32_t w, const Nf4BlockTable& t, uint32_t* out) {
  const uint32_t sel = w & 0x77777777u;
  const uint32_t hi8 = ((w >> 1) & 0x44444444u) | 0x32103210u;
  nf4_lookup4(sel, hi8, t, out[0], out[1]);
  nf4_lookup4(sel >> 16, hi8 >> 16, t, out[2], out[3]);
}

}  // namespace qnf4
