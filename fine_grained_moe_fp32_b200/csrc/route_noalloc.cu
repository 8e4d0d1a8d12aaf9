// moe_route_noalloc: the router for callers that cannot allocate device
// memory at the time they route.
//
// Who needs it: code that is handed a stream and its input/output buffers but
// no allocator -- for example an inference engine's plugin/enqueue hook, or a
// serving loop that forbids device allocation after warm-up because cudaMalloc
// can synchronise the device and fragments a memory pool owned by someone
// else.  moe_route needs a caller-provided workspace for its split-K partial
// logits; this variant keeps that scratch in a fixed array inside the library.
//
// The scratch is a file-scope __device__ array of kScratchBytes (16 MiB).
// Every GPU that loads the library holds it until the process exits.  Host
// code cannot use the array's name as a device address, so on the first call
// on each device (with that device current) its address is looked up with
// cudaGetSymbolAddress and cached; that first call should therefore come
// before any stream capture.  The cache lives as long as the process: after a
// cudaDeviceReset the cached address is stale, and the library must not be
// called again in that process.  Every call shares the array: the router
// overwrites all of the partials it later reads, so nothing has to start at
// zero, but two calls that overlap on the GPU (different streams, or
// different host threads on one device) race on it.
#include <mutex>

#include "../../include/moe_b200.h"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_route_scratch on the current device (set up once per
// device), or nullptr if the lookup failed.
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace moe

extern "C" int moe_route_noalloc(const moe_dims* dims, const moe_bf16* x, const float* w_gate,
                                 const float* bias, float* probs, int32_t* topk_idx,
                                 float* topk_w, void* stream) {
  if (moe_capacity(dims) <= 0) {
    // invalid or unsupported dims: let moe_route report which
    return moe_route(dims, x, w_gate, bias, probs, topk_idx, topk_w, nullptr, 0, stream);
  }
  if (moe_route_workspace_size(dims) - moe::kGuardBytes > moe::kScratchBytes) return MOE_ERR_WORKSPACE;
  void* scratch = moe::scratch_on_current_device();
  if (scratch == nullptr) return MOE_ERR_CUDA;
  return moe_route(dims, x, w_gate, bias, probs, topk_idx, topk_w, scratch, moe::kScratchBytes,
                   stream);
}
