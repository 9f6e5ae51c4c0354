/*
 * synth_cuda.cu -- device-side fill of synthetic input tensors (test and
 * benchmark infrastructure; holds none of the MoE layer's arithmetic). It
 * evaluates the same per-element definition as synth_host.c, so that large
 * inputs can be created directly in HBM while the CPU oracle regenerates any
 * slice of them on the host.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include "synth.h"

namespace {

__global__ void synth_fill_kernel(void* out, int dtype, int64_t count, uint64_t key, int64_t start,
                                  int kind, double a, double b) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
    if (dtype == 2) {
      static_cast<uint8_t*>(out)[i] = synth_byte(key, (uint64_t)(start + i), kind, (int)a, (int)b);
      continue;
    }
    const float v = (float)synth_value(key, (uint64_t)(start + i), kind, a, b);
    if (dtype == 0)
      static_cast<float*>(out)[i] = v;
    else
      static_cast<uint16_t*>(out)[i] = synth_f32_to_bf16_bits(v);
  }
}

}  // namespace

/* dtype: 0 = binary32, 1 = bf16, 2 = bytes (integer kinds). Returns a cudaError_t value (0 on success). */
extern "C" int synth_cuda_fill(void* out, int dtype, int64_t count, uint64_t seed, uint64_t stream,
                               int64_t start, int kind, double a, double b, void* cuda_stream) {
  if (count <= 0) return 0;
  const uint64_t key = synth_key(seed, stream);
  int64_t blocks = (count + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  synth_fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)cuda_stream>>>(out, dtype, count, key, start,
                                                                          kind, a, b);
  return (int)cudaGetLastError();
}
