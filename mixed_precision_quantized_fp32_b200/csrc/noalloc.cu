// moe_layer_forward_noalloc: the layer forward with its workspace in a fixed
// device array owned by this library, for callers that cannot allocate device
// memory (graph-capture regions, allocator callbacks, embedded runtimes).  It
// runs the unchanged moe_layer_forward with that array as the workspace.
#include "moe_common.cuh"

namespace {

// The scratch array.  Host code must not use its name as a device address:
// the device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];  // device address of the array on each device (set-up cache)

// Device address of the scratch array on the current device (looked up on the
// first call per device).  Returns null on failure.
void* scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" moe_status moe_layer_forward_noalloc(const void* x, int32_t T, const float* router_w,
                                                const float* router_b, const moe_weights* w, int32_t k, void* y,
                                                const moe_debug* dbg, cudaStream_t stream) {
  uint64_t need = 0;
  // size query first: validates the shapes and formats and launches nothing
  moe_status st = moe_layer_forward(nullptr, T, nullptr, nullptr, w, k, nullptr, nullptr, 0, &need, nullptr, stream);
  if (st != MOE_OK) return st;
  if (need > MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
  void* ws = scratch_for_current_device();
  if (!ws) return MOE_ERR_CUDA;
  return moe_layer_forward(x, T, router_w, router_b, w, k, y, ws, MOE_NOALLOC_SCRATCH_BYTES, nullptr, dbg, stream);
}
