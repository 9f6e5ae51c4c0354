/*
 * synth_host.c -- host-side fill of synthetic input tensors (test and benchmark
 * infrastructure; holds none of the MoE layer's arithmetic). Element i of the
 * filled range is element (start + i) of the stream defined in synth.h.
 * Built with -ffp-contract=off so that the values match the CUDA fill bit for bit.
 */
#include <stddef.h>
#include <stdint.h>
#include "synth.h"

void synth_fill_f32(float* out, int64_t count, uint64_t seed, uint64_t stream, int64_t start,
                    int kind, double a, double b) {
  const uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i)
    out[i] = (float)synth_value(key, (uint64_t)(start + i), kind, a, b);
}

void synth_fill_bf16(uint16_t* out, int64_t count, uint64_t seed, uint64_t stream, int64_t start,
                     int kind, double a, double b) {
  const uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i)
    out[i] = synth_f32_to_bf16_bits((float)synth_value(key, (uint64_t)(start + i), kind, a, b));
}

void synth_fill_u8(uint8_t* out, int64_t count, uint64_t seed, uint64_t stream, int64_t start, int kind, double a,
                   double b) {
  const uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) out[i] = synth_byte(key, (uint64_t)(start + i), kind, (int)a, (int)b);
}
