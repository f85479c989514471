// moe_layer_forward_static: the layer forward for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code that runs inside a memory budget fixed
// up front (an embedding host that owns every device allocation), code that runs where a
// new allocation would block or fail (under memory pressure, or where allocating would
// synchronise the device), and plain C callers that have no allocator of their own for
// device scratch.  This entry point takes the same inputs and outputs as moe_layer_forward
// but needs no workspace: its scratch is one file-scope device array of fixed size,
// kMoeStaticScratchBytes, which every GPU that loads the library holds until the process
// exits.  Nothing here allocates.
#include "../../include/moe.h"
#include "common.cuh"

#include <mutex>

namespace moe {
moe_status set_error(moe_status s, const char* fmt, ...);
moe_status cuda_fail(cudaError_t e, const char* what);
moe_status check_shape(const moe_shape* s);
}  // namespace moe

using namespace moe;

namespace {

constexpr size_t kMoeStaticScratchBytes = size_t(1) << 20;  // 1 MiB

// The scratch.  In host code this name is only a host-side stand-in for the device array:
// it must never be handed to a kernel.  Host code uses the address cudaGetSymbolAddress
// returns for the current device.
__device__ __align__(256) unsigned char g_moe_static_scratch[kMoeStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};  // the context the cached address belongs to

// cuCtxGetCurrent through the runtime's driver entry point (the library does not link the
// driver library); null if the driver does not offer it.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (CtxGetCurrentFn) nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  return fn;
}

// Device address of the scratch on the current device.  It is looked up once per device and
// context: after a device reset (cudaDeviceReset) the device gets a new primary context, the
// cached address no longer names the array, and the next call looks it up again.
moe_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return set_error(MOE_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
  const CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  const auto current_ctx = [&] {
    CUcontext c = nullptr;
    if (!get_ctx || get_ctx(&c) != CUDA_SUCCESS) c = nullptr;
    return c;
  };
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev] || g_scratch_ctx[dev] != current_ctx()) {
    // the lookup also makes the device's primary context current (creating it if needed)
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_moe_static_scratch);
    if (e != cudaSuccess || !p) return cuda_fail(e, "cudaGetSymbolAddress of the static scratch");
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_ctx();
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_layer_forward_static(const moe_shape* shape, const void* x, int32_t T, const void* w_router,
                                               const float* router_bias, const int32_t* topk_idx_in,
                                               const float* topk_w_in, const uint8_t* pool,
                                               const int32_t* slot_table, int64_t n_slots,
                                               const uint8_t* shared_blob, const void* w_shared_gate,
                                               const void* residual, void* out, int32_t* topk_idx_out,
                                               float* topk_w_out, void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (T < 1 || T > kMaxDecodeT)
    return set_error(MOE_ERR_UNSUPPORTED, "T must be in [1, %d] on the decode path (got %d)", kMaxDecodeT, T);
  const size_t need = make_ws_layout(T, shape->n_experts, shape->top_k, shape->inter, shape->shared_inter).total;
  if (need > kMoeStaticScratchBytes)
    return set_error(MOE_ERR_INVALID,
                     "T=%d, E=%d, k=%d, inter=%d needs %zu bytes of scratch; the static scratch holds %zu "
                     "(use moe_layer_forward with a caller workspace)",
                     T, shape->n_experts, shape->top_k, shape->inter, need, kMoeStaticScratchBytes);
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != MOE_OK) return st;
  // The control block (error word, last-CTA ticket) must start at zero; everything else in
  // the scratch is written before it is read.
  cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(Ctrl), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "clearing the static scratch control block");
  return moe_layer_forward(shape, x, T, w_router, router_bias, topk_idx_in, topk_w_in, pool, slot_table, n_slots,
                           shared_blob, w_shared_gate, residual, out, topk_idx_out, topk_w_out, scratch,
                           kMoeStaticScratchBytes, stream);
}
