/*
 * synth.h -- seeded, counter-based synthetic input generator.
 *
 * This module is test and benchmark infrastructure. It produces the inputs of
 * the MoE layer (activations, router weights, selection bias, expert weights)
 * and holds none of the layer's arithmetic. Both the CPU oracle side and the
 * CUDA side draw their inputs from it, so that both see identical values.
 *
 * Every element is a pure function of (seed, stream, index):
 *   key    = mix64(mix64(seed) + stream)
 *   word_c = mix64(key ^ c)                      (c = counter)
 * mix64 is the SplitMix64 output function (Steele, Lea and Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014).
 *
 * Normal-like values use the Irwin-Hall construction: the sum of twelve
 * independent U(0,1) variates minus 6 has mean 0 and variance 1 and is the
 * classical "sum of twelve uniforms" approximation of N(0,1) (support
 * [-6, 6]). The twelve uniforms are the twelve 16-bit fields of three words,
 * each taken as (u + 1/2) / 2^16. The sum is an integer, so the value
 * ((sum + 6) / 2^16) - 6 is exact in binary64; it is then scaled by sigma with
 * one correctly rounded multiply, rounded to binary32 (round to nearest even)
 * and, for bf16 tensors, rounded once more from binary32 to bf16 (round to
 * nearest even). Only +, -, * and integer operations appear, so a host
 * compiler and the CUDA compiler produce bit-identical values as long as no
 * multiply-add is contracted (device code uses __dmul_rn/__dadd_rn; host code
 * is built with -ffp-contract=off).
 */
#ifndef SYNTH_H_
#define SYNTH_H_

#include <stdint.h>

#if defined(__CUDACC__)
#define SYNTH_FN static __host__ __device__ __forceinline__
#else
#define SYNTH_FN static inline
#endif

#if defined(__CUDA_ARCH__)
#define SYNTH_DMUL(a, b) __dmul_rn((a), (b))
#define SYNTH_DADD(a, b) __dadd_rn((a), (b))
#else
#define SYNTH_DMUL(a, b) ((a) * (b))
#define SYNTH_DADD(a, b) ((a) + (b))
#endif

/* Stream identifiers: one per input tensor of the layer. */
enum {
  SYNTH_STREAM_X = 1,       /* activations x[n, d]                       */
  SYNTH_STREAM_WR = 2,      /* router weight W_r[E, d]                   */
  SYNTH_STREAM_BIAS = 3,    /* selection bias b[E]                       */
  SYNTH_STREAM_WGATE = 4,   /* W_gate[E, I, d]                           */
  SYNTH_STREAM_WUP = 5,     /* W_up[E, I, d]                             */
  SYNTH_STREAM_WDOWN = 6,   /* W_down[E, d, I]                           */
  SYNTH_STREAM_WSGATE = 7,  /* shared gate [I_s, d]                      */
  SYNTH_STREAM_WSUP = 8,    /* shared up   [I_s, d]                      */
  SYNTH_STREAM_WSDOWN = 9,  /* shared down [d, I_s]                      */
  /* FP8 experts: E4M3 codes and UE8M0 block-scale bytes of each weight */
  SYNTH_STREAM_WGATE_Q = 10, SYNTH_STREAM_WUP_Q = 11, SYNTH_STREAM_WDOWN_Q = 12,
  SYNTH_STREAM_WSGATE_Q = 13, SYNTH_STREAM_WSUP_Q = 14, SYNTH_STREAM_WSDOWN_Q = 15,
  SYNTH_STREAM_WGATE_S = 16, SYNTH_STREAM_WUP_S = 17, SYNTH_STREAM_WDOWN_S = 18,
  SYNTH_STREAM_WSGATE_S = 19, SYNTH_STREAM_WSUP_S = 20, SYNTH_STREAM_WSDOWN_S = 21
};

/* Value kinds. */
enum {
  SYNTH_NORMAL = 0,   /* Irwin-Hall(12) - 6, times sigma                */
  SYNTH_UNIFORM = 1,  /* lo + (hi - lo) * u, u in [0, 1)                */
  SYNTH_TERNARY = 2,  /* one of {-1, 0, +1}, each with probability 1/3  */
  SYNTH_BYTE = 3,     /* integer uniform on [a, b] (0 <= a <= b <= 255)  */
  SYNTH_SIGNED_CODE = 4 /* byte (sign << 7) | m, m uniform on [a, b] <= 127, sign a fair bit */
};

SYNTH_FN uint64_t synth_mix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

SYNTH_FN uint64_t synth_key(uint64_t seed, uint64_t stream) {
  return synth_mix64(synth_mix64(seed) + stream);
}

SYNTH_FN uint64_t synth_word(uint64_t key, uint64_t counter) {
  return synth_mix64(key ^ counter);
}

/* Irwin-Hall(12) - 6 for element i, exact in binary64. */
SYNTH_FN double synth_irwin_hall(uint64_t key, uint64_t i) {
  uint64_t s = 0;
  for (int w = 0; w < 3; ++w) {
    uint64_t v = synth_word(key, 3 * i + (uint64_t)w);
    s += (v & 0xFFFFu) + ((v >> 16) & 0xFFFFu) + ((v >> 32) & 0xFFFFu) + (v >> 48);
  }
  /* (s + 6) < 2^20: the division by 2^16 and the subtraction are exact. */
  return SYNTH_DADD(SYNTH_DMUL((double)(s + 6), 1.0 / 65536.0), -6.0);
}

/* u in [0, 1) with 53 random bits, from one word. */
SYNTH_FN double synth_unit(uint64_t key, uint64_t i) {
  return SYNTH_DMUL((double)(synth_word(key, i) >> 11), 1.0 / 9007199254740992.0);
}

/* Element i of a stream as binary64 before the final narrowing. */
SYNTH_FN double synth_value(uint64_t key, uint64_t i, int kind, double a, double b) {
  if (kind == SYNTH_NORMAL) return SYNTH_DMUL(synth_irwin_hall(key, i), a);
  if (kind == SYNTH_UNIFORM) return SYNTH_DADD(a, SYNTH_DMUL(SYNTH_DADD(b, -a), synth_unit(key, i)));
  return (double)((int)(synth_word(key, i) % 3u) - 1);
}

/* Element i of an integer (byte) stream: integer operations only. */
SYNTH_FN uint8_t synth_byte(uint64_t key, uint64_t i, int kind, int lo, int hi) {
  const uint64_t w = synth_word(key, i);
  const uint32_t span = (uint32_t)(hi - lo + 1);
  const uint32_t v = (uint32_t)lo + (uint32_t)((w >> 8) % span);
  if (kind == SYNTH_SIGNED_CODE) return (uint8_t)(((uint32_t)(w & 1u) << 7) | v);
  return (uint8_t)v;
}

/* binary32 -> bf16 bits, round to nearest even (inputs here are finite). */
SYNTH_FN uint16_t synth_f32_to_bf16_bits(float f) {
  union { float f; uint32_t u; } c;
  c.f = f;
  uint32_t u = c.u;
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

#endif /* SYNTH_H_ */
