/*
 * synth_host.c — host (plain C) fills for the synthetic input generator.
 * Compiled with -ffp-contract=off so that `normal*scale + offset` is two
 * correctly rounded float32 operations, exactly as on the device.
 */
#include <stdint.h>
#include "synth.h"

static inline float synth_affine(float n, float scale, float offset) {
  volatile float t = n * scale; /* rounded product */
  return t + offset;            /* rounded sum */
}

void synth_fill_normal_f32(float* out, int64_t count, uint64_t seed, uint64_t stream,
                           uint64_t index0, float scale, float offset) {
  uint64_t key = synth_key(seed, stream);
  for (int64_t i = 0; i < count; ++i)
    out[i] = synth_affine(synth_normal(key, index0 + (uint64_t)i), scale, offset);
}

void synth_fill_normal_bf16(uint16_t* out, int64_t count, uint64_t seed, uint64_t stream,
                            uint64_t index0, float scale, float offset) {
  uint64_t key = synth_key(seed, stream);
  for (int64_t i = 0; i < count; ++i)
    out[i] = synth_f32_to_bf16(
        synth_affine(synth_normal(key, index0 + (uint64_t)i), scale, offset));
}

void synth_fill_uniform_i32(int32_t* out, int64_t count, uint64_t seed, uint64_t stream,
                            uint64_t index0, uint32_t n, int32_t add) {
  uint64_t key = synth_key(seed, stream);
  for (int64_t i = 0; i < count; ++i)
    out[i] = add + (int32_t)synth_uniform(key, index0 + (uint64_t)i, n);
}

/* out[i] = ((index0+i) % period) * width + uniform[0,width): distinct values
 * within each period (one per stratum). */
void synth_fill_strata_i32(int32_t* out, int64_t count, uint64_t seed, uint64_t stream,
                           uint64_t index0, uint32_t period, uint32_t width) {
  uint64_t key = synth_key(seed, stream);
  for (int64_t i = 0; i < count; ++i) {
    uint64_t g = index0 + (uint64_t)i;
    out[i] = (int32_t)((g % period) * width + synth_uniform(key, g, width));
  }
}

/* Float32 normals in groups of `group` elements where about one element in
 * `one_in` is replaced by a copy of another element's (undisturbed) value of
 * the same group: this plants exact ties. */
void synth_fill_normal_dup_f32(float* out, int64_t count, uint64_t seed, uint64_t stream,
                               uint64_t index0, uint32_t group, uint32_t one_in) {
  uint64_t key = synth_key(seed, stream);
  uint64_t kpick = synth_key(seed, stream + SYNTH_DUP);
  uint64_t ksrc = synth_key(seed, stream + SYNTH_DUP + 1);
  for (int64_t i = 0; i < count; ++i) {
    uint64_t g = index0 + (uint64_t)i;
    uint64_t src = g;
    if (synth_uniform(kpick, g, one_in) == 0)
      src = (g / group) * group + synth_uniform(ksrc, g, group);
    out[i] = synth_normal(key, src);
  }
}
