/*
 * synth_dev.cu — device fills for the synthetic input generator.
 * Same element-for-element definitions as synth_host.c (bit-identical
 * outputs); the affine step uses __fmul_rn/__fadd_rn so it is never fused.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include "synth.h"

namespace {

__device__ __forceinline__ float synth_affine(float n, float scale, float offset) {
  return __fadd_rn(__fmul_rn(n, scale), offset);
}

__global__ void k_normal_f32(float* out, int64_t count, uint64_t key, uint64_t index0,
                             float scale, float offset) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = synth_affine(synth_normal(key, index0 + (uint64_t)i), scale, offset);
}

__global__ void k_normal_bf16(uint16_t* out, int64_t count, uint64_t key, uint64_t index0,
                              float scale, float offset) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = synth_f32_to_bf16(
        synth_affine(synth_normal(key, index0 + (uint64_t)i), scale, offset));
}

__global__ void k_uniform_i32(int32_t* out, int64_t count, uint64_t key, uint64_t index0,
                              uint32_t n, int32_t add) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = add + (int32_t)synth_uniform(key, index0 + (uint64_t)i, n);
}

__global__ void k_strata_i32(int32_t* out, int64_t count, uint64_t key, uint64_t index0,
                             uint32_t period, uint32_t width) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t g = index0 + (uint64_t)i;
    out[i] = (int32_t)((g % period) * width + synth_uniform(key, g, width));
  }
}

__global__ void k_normal_dup_f32(float* out, int64_t count, uint64_t key, uint64_t kpick,
                                 uint64_t ksrc, uint64_t index0, uint32_t group,
                                 uint32_t one_in) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t g = index0 + (uint64_t)i;
    uint64_t src = g;
    if (synth_uniform(kpick, g, one_in) == 0)
      src = (g / group) * group + synth_uniform(ksrc, g, group);
    out[i] = synth_normal(key, src);
  }
}

unsigned grid_for(int64_t count) {
  int64_t b = (count + 255) / 256;
  if (b > 148 * 64) b = 148 * 64;
  if (b < 1) b = 1;
  return (unsigned)b;
}

}  // namespace

extern "C" {

int synthd_fill_normal_f32(float* out, int64_t count, uint64_t seed, uint64_t stream,
                           uint64_t index0, float scale, float offset, cudaStream_t st) {
  if (count <= 0) return 0;
  k_normal_f32<<<grid_for(count), 256, 0, st>>>(out, count, synth_key(seed, stream), index0,
                                                 scale, offset);
  return (int)cudaGetLastError();
}

int synthd_fill_normal_bf16(uint16_t* out, int64_t count, uint64_t seed, uint64_t stream,
                            uint64_t index0, float scale, float offset, cudaStream_t st) {
  if (count <= 0) return 0;
  k_normal_bf16<<<grid_for(count), 256, 0, st>>>(out, count, synth_key(seed, stream), index0,
                                                  scale, offset);
  return (int)cudaGetLastError();
}

int synthd_fill_uniform_i32(int32_t* out, int64_t count, uint64_t seed, uint64_t stream,
                            uint64_t index0, uint32_t n, int32_t add, cudaStream_t st) {
  if (count <= 0) return 0;
  k_uniform_i32<<<grid_for(count), 256, 0, st>>>(out, count, synth_key(seed, stream), index0,
                                                  n, add);
  return (int)cudaGetLastError();
}

int synthd_fill_strata_i32(int32_t* out, int64_t count, uint64_t seed, uint64_t stream,
                           uint64_t index0, uint32_t period, uint32_t width, cudaStream_t st) {
  if (count <= 0) return 0;
  k_strata_i32<<<grid_for(count), 256, 0, st>>>(out, count, synth_key(seed, stream), index0,
                                                 period, width);
  return (int)cudaGetLastError();
}

int synthd_fill_normal_dup_f32(float* out, int64_t count, uint64_t seed, uint64_t stream,
                               uint64_t index0, uint32_t group, uint32_t one_in,
                               cudaStream_t st) {
  if (count <= 0) return 0;
  k_normal_dup_f32<<<grid_for(count), 256, 0, st>>>(
      out, count, synth_key(seed, stream), synth_key(seed, stream + SYNTH_DUP),
      synth_key(seed, stream + SYNTH_DUP + 1), index0, group, one_in);
  return (int)cudaGetLastError();
}

}  // extern "C"
