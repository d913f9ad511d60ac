// score.cu — a3, the RMA retention scorer.
//
// EdgeRock-4B 开源：72 MiB 固定 KV, §架构：递归、局部窗口与记忆锚点三件套: a small
// independent bias-free network maps the 2560-wide hidden state to 256 and
// then to 4 values in FP32, one retention score per KV group (SiLU between
// the two matmuls is this library's reading).
//
// CUDA cores, FP32 FMA throughout.  A block owns RT tokens and all 256 hidden
// units (thread j = unit j); W1 is streamed through shared memory in 32-wide
// K slices (padded, conflict-free), x in the same slices.  The 256→4 step is
// a block reduction.  W1 (2.6 MB) stays in L2 across blocks.
#include "common.cuh"

namespace er {
namespace {

constexpr int RT = 8;    // tokens per block
constexpr int KS = 32;   // K slice

__global__ void __launch_bounds__(256) k_score(const float* __restrict__ w1,
                                               const float* __restrict__ w2,
                                               const uint16_t* __restrict__ x, int n,
                                               float* __restrict__ s) {
  __shared__ float w1s[KS][SH + 1];
  __shared__ float xs[RT][KS];
  __shared__ float red[8][RT][NG];
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * RT;
  const int nt = min(RT, n - t0);
  float h[RT];
#pragma unroll
  for (int r = 0; r < RT; ++r) h[r] = 0.f;

  for (int k0 = 0; k0 < HID; k0 += KS) {
    // W1[:, k0:k0+32] -> w1s[kk][j]  (coalesced 128-byte row pieces)
#pragma unroll
    for (int i = 0; i < (SH * KS) / 256; ++i) {
      const int idx = i * 256 + tid;
      const int row = idx / KS, kk = idx % KS;
      w1s[kk][row] = w1[(size_t)row * HID + k0 + kk];
    }
    {
      const int r = tid / KS, kk = tid % KS;  // 256 threads = 8 tokens x 32
      xs[r][kk] = (r < nt) ? bf1(x[(size_t)(t0 + r) * HID + k0 + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < KS; ++kk) {
      const float w = w1s[kk][tid];
#pragma unroll
      for (int r = 0; r < RT; ++r) h[r] = fmaf(w, xs[r][kk], h[r]);
    }
    __syncthreads();
  }

  // SiLU, then this unit's contribution to the 4 scores of each token
  float c[RT][NG];
  float w2j[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) w2j[g] = w2[g * SH + tid];
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    const float a = h[r] / (1.0f + expf(-h[r]));
#pragma unroll
    for (int g = 0; g < NG; ++g) c[r][g] = w2j[g] * a;
  }
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int g = 0; g < NG; ++g)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) c[r][g] += __shfl_xor_sync(0xffffffffu, c[r][g], o);
  const int warp = tid >> 5, lane = tid & 31;
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int g = 0; g < NG; ++g) red[warp][r][g] = c[r][g];
  }
  __syncthreads();
  if (tid < RT * NG) {
    const int r = tid / NG, g = tid % NG;
    if (r < nt) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) acc += red[w][r][g];
      s[(size_t)(t0 + r) * NG + g] = acc;
    }
  }
}

}  // namespace

int launch_score(const float* w1, const float* w2, const uint16_t* x, int n, float* s,
                 cudaStream_t st) {
  if (n <= 0) return ER_OK;
  k_score<<<(n + RT - 1) / RT, 256, 0, st>>>(w1, w2, x, n, s);
  count_launches(1);
  return launch_status();
}

}  // namespace er

using namespace er;

extern "C" int er_rma_score(const er_layer_weights* w, const er_bf16* x, int32_t n, float* s,
                            er_stream_t stream) {
  if (!w || n < 0 || (n > 0 && (!w->w1 || !w->w2 || !x || !s))) return ER_EINVAL;
  return launch_score(w->w1, w->w2, x, n, s, (cudaStream_t)stream);
}
