// common.cuh -- shared device helpers of the MoE library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "moe.h"

namespace moe {

using bf16 = __nv_bfloat16;

constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 32;
constexpr int kMaxGroups = 32;

// ---- element conversion -------------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }
__device__ __forceinline__ double to_f64(float v) { return (double)v; }
__device__ __forceinline__ double to_f64(bf16 v) { return (double)__bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// ---- device status word ---------------------------------------------------------
// The first 64 bytes of the workspace hold an internal moe_diag; its `status`
// field is the device-side error word read by moe_sync_status().
__device__ __forceinline__ void set_status(moe_diag* d, int code) {
  if (d) atomicCAS(&d->status, 0, code);
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + __expf(-z)); }

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Raises a kernel's dynamic shared-memory limit on the current device, once per device: the
// attribute belongs to the device, so a process using several GPUs sets it on each. `done` holds
// one bit per device (devices 64 and above set it on every call).
inline cudaError_t set_smem_limit(std::atomic<uint64_t>& done, const void* func, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t)1 << dev : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}
__host__ __device__ constexpr int64_t align_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

}  // namespace moe
