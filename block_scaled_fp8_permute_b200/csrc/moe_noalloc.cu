// moe_noalloc.cu -- the allocation-free entry point: plan + forward of one
// MoE layer with the workspace taken from a fixed device array that the
// library itself owns.  It serves callers that cannot call cudaMalloc: a
// serving runtime whose memory manager has reserved the free device memory
// for its own pool, or a plug-in that is handed only its inputs and outputs
// and cannot reach its host framework's allocator.
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB

// The scratch workspace.  Every GPU that loads this library holds one copy
// of it until the process exits.  Its host-side name is only a handle: the
// device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array for the current device; looked up the
// first time a device is used, with that device current.
moe_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" {

moe_status moe_forward_noalloc(const moe_shape* shape, const uint8_t* x, const int32_t* x_sf,
                               const int32_t* topk_idx, const float* topk_w, const void* w1_t,
                               const void* w1_sf_t, const void* w2_t, const void* w2_sf_t,
                               uint16_t* y, moe_stream_t stream) {
  if (!shape) return MOE_ERR_INVALID_ARG;  // as moe_forward
  const size_t need = moe_workspace_bytes(shape);
  if (need == 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (need > moe::kStaticScratchBytes) return MOE_ERR_WORKSPACE;
  void* ws = nullptr;
  moe_status st = moe::scratch_for_current_device(&ws);
  if (st != MOE_OK) return st;
  // moe_plan clears the only part of the workspace that must start at zero
  // (the header with the status word and counters); everything else is
  // written before it is read.
  st = moe_plan(shape, topk_idx, ws, moe::kStaticScratchBytes, stream);
  if (st != MOE_OK) return st;
  return moe_forward(shape, x, x_sf, topk_idx, topk_w, w1_t, w1_sf_t, w2_t, w2_sf_t, y, ws,
                     moe::kStaticScratchBytes, stream);
}

}  // extern "C"
