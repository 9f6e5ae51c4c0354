// route_static.cu -- moe_route_static_scratch: the router entry point for
// callers that cannot allocate device memory. Its scratch space is a
// file-scope device array of fixed size that every GPU loading this library
// holds until the process exits; the caller passes only inputs and outputs.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {
size_t route_scratch_bytes(const moe_config& c, int64_t n);
moe_status route_in_scratch(const moe_config* cfg, int64_t n, const void* x, const moe_weights* weights,
                            int32_t* topk_idx, float* topk_w, int32_t* expert_counts, moe_diag* diag, void* scratch,
                            size_t scratch_bytes, moe_stream_t stream);
}  // namespace moe

namespace {

constexpr size_t kStaticScratchBytes = (size_t)MOE_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Shared by every call on a device. In host code this name is only a host-side
// stand-in: kernels receive the device address looked up below.
static __device__ __align__(256) unsigned char g_route_scratch[kStaticScratchBytes];

std::mutex g_lock;
void* g_scratch_addr[kMaxDevices] = {};

// One-time set-up per device, with that device current: the device address of
// the array. Returns nullptr when the lookup fails (the failed call's error is
// cleared, so that it is not reported by a later, unrelated launch check).
void* scratch_for_device(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> guard(g_lock);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_route_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" moe_status moe_route_static_scratch(const moe_config* cfg, int64_t n, const void* x,
                                               const moe_weights* weights, int32_t* topk_idx, float* topk_w,
                                               int32_t* expert_counts, moe_diag* diag, moe_stream_t stream) {
  if (!cfg || n < 0) return MOE_ERR_INVALID_ARG;
  size_t need = 0;
  const moe_status st = moe_workspace_size(cfg, n, &need);  // validates cfg
  if (st != MOE_OK) return st;
  if (moe::route_scratch_bytes(*cfg, n) > kStaticScratchBytes) return MOE_ERR_WORKSPACE;
  // The array's address belongs to one device: the stream must belong to the current device.
  int dev = -1, stream_dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamGetDevice(reinterpret_cast<cudaStream_t>(stream), &stream_dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_INVALID_ARG;
  }
  if (stream_dev != dev) return MOE_ERR_INVALID_ARG;
  void* scratch = scratch_for_device(dev);
  if (!scratch) return MOE_ERR_CUDA;
  return moe::route_in_scratch(cfg, n, x, weights, topk_idx, topk_w, expert_counts, diag, scratch,
                               kStaticScratchBytes, stream);
}
