/*
 * synth.h — seeded, counter-based synthetic input generator.
 *
 * This header is the ONLY code shared between the CPU oracle and the CUDA
 * path.  It holds no arithmetic of the EdgeRock SWA∥RMA layer: it only turns
 * (seed, stream, index) into reproducible numbers, identically on the host
 * (plain C) and on the device (CUDA), so that both sides can build the same
 * synthetic inputs without copying tens of GiB between them.
 *
 * Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), used counter-style: the
 * n-th output of stream k is the SplitMix64 finaliser applied to
 * key(k) + (n+1)·γ, with γ the golden-ratio increment.
 *
 * Normal variates: Irwin–Hall sum of twelve 16-bit uniforms, centred and
 * scaled in exact integer/power-of-two arithmetic, so host and device produce
 * bit-identical float32 values (no libm call is involved).  The result has
 * mean 0, variance 1 - 2^-32 and support [-6, 6].
 */
#ifndef SYNTH_H
#define SYNTH_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYNTH_FN static __host__ __device__ __forceinline__
#else
#define SYNTH_FN static inline
#endif

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL

/* SplitMix64 output finaliser (the published mix13 variant). */
SYNTH_FN uint64_t synth_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Key of one named stream under one seed. */
SYNTH_FN uint64_t synth_key(uint64_t seed, uint64_t stream) {
  return synth_mix64(seed * SYNTH_GAMMA + synth_mix64(stream + 0x632BE59BD9B4E019ULL));
}

/* n-th 64-bit output of a keyed stream. */
SYNTH_FN uint64_t synth_u64(uint64_t key, uint64_t n) {
  return synth_mix64(key + (n + 1ULL) * SYNTH_GAMMA);
}

/* Standard-normal-like float32 for element `index` of a stream
 * (Irwin–Hall of 12 uniforms on 16 bits; exact in float32). */
SYNTH_FN float synth_normal(uint64_t key, uint64_t index) {
  uint32_t s = 0;
  for (int w = 0; w < 3; ++w) {
    uint64_t r = synth_u64(key, index * 3ULL + (uint64_t)w);
    s += (uint32_t)(r & 0xFFFFu) + (uint32_t)((r >> 16) & 0xFFFFu) +
         (uint32_t)((r >> 32) & 0xFFFFu) + (uint32_t)((r >> 48) & 0xFFFFu);
  }
  /* (s - 12*32767.5) / 65536 == (2s - 786420) / 131072, all exact */
  int32_t c = 2 * (int32_t)s - 786420;
  return (float)c * (1.0f / 131072.0f);
}

/* Uniform integer in [0, n) for element `index` (multiply-shift, exact). */
SYNTH_FN uint32_t synth_uniform(uint64_t key, uint64_t index, uint32_t n) {
  uint64_t r = synth_u64(key, index) >> 32;
  return (uint32_t)((r * (uint64_t)n) >> 32);
}

/* float32 -> bfloat16 bits, round to nearest even (finite inputs). */
SYNTH_FN uint16_t synth_f32_to_bf16(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  uint32_t u = v.u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* Stream identifiers: one per synthetic tensor.  Streams that vary per
 * layer / step add (layer << 32) or (step << 40) so every tensor of every
 * layer and step draws from its own stream. */
enum {
  SYNTH_W_QKV = 1,
  SYNTH_W_O = 2,
  SYNTH_G_Q_SWA = 3,
  SYNTH_G_K_SWA = 4,
  SYNTH_G_Q_RMA = 5,
  SYNTH_G_K_RMA = 6,
  SYNTH_W1 = 7,
  SYNTH_W2 = 8,
  SYNTH_WIN_K = 16,
  SYNTH_WIN_V = 17,
  SYNTH_BANK_K = 18,
  SYNTH_BANK_V = 19,
  SYNTH_BANK_SCORE = 20,
  SYNTH_BANK_POS = 21,
  SYNTH_PEND_K = 22,
  SYNTH_PEND_V = 23,
  SYNTH_PEND_SCORE = 24,
  SYNTH_PEND_FILL = 25,
  SYNTH_X = 32,
  SYNTH_DUP = 40,
  SYNTH_MISC = 48
};

#endif /* SYNTH_H */
