// Operand helpers shared by the tcgen05 GEMM engines: TMA tile loads of
// bf16 operands, their shared-memory descriptors, the epilogue store and a
// warp-wide bounded mbarrier wait.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace qnf4 {
namespace {

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
QDEV bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status, int lane,
                    uint64_t limit_ns = QNF4_WAIT_NS) {
  int ok = 1;
  if (lane == 0) ok = mbar_wait(bar, parity, abort_flag, status, limit_ns) ? 1 : 0;
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  if (ok) mbar_test_wait(smem_u32(bar), parity);
  return ok != 0;
}

}  // namespace
}  // namespace qnf4
