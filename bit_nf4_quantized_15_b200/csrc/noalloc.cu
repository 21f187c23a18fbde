// qlora_linear_fwd_noalloc: the forward of the quantized linear layer for
// callers that cannot allocate device memory.
//
// Some callers run where allocation is not theirs to do: a plugin or custom
// operator executed by a host framework that owns the whole device memory
// pool and forbids allocations inside its execute callback, or a
// latency-critical serving loop whose policy is "no cudaMalloc after
// start-up" (cudaMalloc can synchronise the device and fragment a pool it
// does not own).  They can still hand over inputs and outputs, but not the
// workspace the regular entry point asks for.  This entry point uses a
// workspace that lives in the library itself: a file-scope device array of
// kScratchBytes, present on every GPU that loads the library until the
// process exits.
//
// The array's name is only a host-side handle; its device address is looked
// up once per device (cudaGetSymbolAddress, with that device current) on the
// first call made on that device, and that address is what the kernels get.
// Make that first call before any stream capture.  The address is cached with
// the CUDA context it belongs to: if the device's context is destroyed and
// re-created (cudaDeviceReset), the next call looks it up again.  Every call shares the one
// array and it keeps whatever the previous call left there; the forward
// writes every workspace element it later reads, so nothing needs clearing.
// Calls that overlap on the GPU (other streams, other threads) race on the
// array: serialise them.
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/qlora_nf4.h"
#include "internal.h"

#define QLORA_NOALLOC_SCRATCH_BYTES (8u << 20)  // 8 MiB

static __device__ __align__(256) unsigned char g_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr size_t kScratchBytes = QLORA_NOALLOC_SCRATCH_BYTES;

std::mutex g_mu;
void* g_scratch_dev[64] = {};
CUcontext g_scratch_ctx[64] = {};

// The driver's cuCtxGetCurrent, reached through the runtime (no link-time
// dependency on the driver library).
PFN_cuCtxGetCurrent_v4000 ctx_get_current() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  return fn;
}

// Device address of g_scratch on the current device: looked up on the first
// call on a device, and again whenever that device's current context is not
// the one the cached address was taken in.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QLORA_ERR_CUDA;
  auto get_ctx = ctx_get_current();
  if (!get_ctx) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> g(g_mu);
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return QLORA_ERR_CUDA;
  if (!g_scratch_dev[dev] || !ctx || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return QLORA_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return QLORA_ERR_CUDA;  // current now, if it was not before
    g_scratch_dev[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_dev[dev];
  return QLORA_OK;
}

}  // namespace

extern "C" {

int qlora_linear_fwd_noalloc(const uint16_t* X, int64_t M, const qlora_nf4_weight* w, const uint16_t* L1,
                             const uint16_t* L2, int r, float s, uint16_t* Y, float* T_save, int* status_dev,
                             qlora_stream_t stream) {
  if (!w) return QLORA_ERR_NULL;
  const size_t need = qlora_workspace_bytes(M, w->n_rows, w->n_cols, r);
  if (need == 0) return (r >= 8 && r <= 128 && r % 8 == 0) ? QLORA_ERR_SHAPE : QLORA_ERR_RANK;
  if (need > kScratchBytes) return QLORA_ERR_SCRATCH_LIMIT;
  void* ws = nullptr;
  if (int rc = scratch_address(&ws)) return rc;
  return qlora_linear_fwd(X, M, w, L1, L2, r, s, Y, T_save, ws, kScratchBytes, status_dev, stream);
}

}  // extern "C"
