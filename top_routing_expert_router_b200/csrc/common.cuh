// common.cuh -- shared device helpers of the MoE library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

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
__host__ __device__ constexpr int64_t align_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

}  // namespace moe
