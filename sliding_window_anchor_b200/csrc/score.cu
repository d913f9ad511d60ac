// score.cu — a3, the RMA retention scorer.
//
// EdgeRock-4B 开源：72 MiB 固定 KV, §架构：递归、局部窗口与记忆锚点三件套: a small
// independent bias-free network maps the 2560-wide hidden state to 256 and
// then to 4 values in FP32, one retention score per KV group (SiLU between
// the two matmuls is this library's reading).
//
// CUDA cores, FP32 throughout, deterministic:
//  stage 1 (split-K): block (token tile of 32, K split of 160) computes the
//    partial pre-activations h[split][token][256]; thread tile 4 tokens x 8
//    units, K staged through shared memory in slices of 32 (W1 transposed on
//    the way in, padded against bank conflicts; the next slice is fetched into
//    registers while the current one is multiplied); packed FFMA2 products.
//  stage 2: per token, the splits are summed in a fixed order, SiLU, and the
//    256→4 contraction is a block reduction.
// The partials live in caller-provided workspace (er_score_workspace_bytes).
#include <mutex>

#include "common.cuh"

namespace er {
namespace {

constexpr int TT = 32;               // tokens per stage-1 block
constexpr int KSPLIT = 16;           // K splits
constexpr int KPER = HID / KSPLIT;   // 160
constexpr int KS = 32;               // K slice staged in shared memory
constexpr int NSL = KPER / KS;       // 5 slices per block

__global__ void __launch_bounds__(256) k_score_partial(const float* __restrict__ w1,
                                                       const uint16_t* __restrict__ x, int n,
                                                       float* __restrict__ part) {
  __shared__ __align__(16) float ws[KS][SH + 4];   // W1[j][k] stored at [k][j]
  __shared__ __align__(16) float xs[KS][TT + 4];   // x[t][k] stored at [k][t]
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * TT;
  const int kbase = blockIdx.y * KPER;
  const int tq = tid & 7;          // token quad: tokens 4tq..4tq+3
  const int jo = tid >> 3;         // unit octet: units 8jo..8jo+7
  float2 acc[4][4];                // [token][unit pair]
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = make_float2(0.f, 0.f);

  // register double buffer: slice s+1 is fetched while slice s is multiplied
  float4 wr[(SH * KS) / (256 * 4)];
  uint32_t xr[2];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int i = 0; i < (SH * KS) / (256 * 4); ++i) {
      const int idx = i * 256 + tid;  // float4 index: 256 rows x 8
      const int row = idx / (KS / 4), c4 = idx % (KS / 4);
      wr[i] = *reinterpret_cast<const float4*>(w1 + (size_t)row * HID + k0 + c4 * 4);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int idx = i * 256 + tid;  // BF16 pair index: 32 tokens x 16
      const int t = idx / (KS / 2), kp = idx % (KS / 2);
      xr[i] = (t0 + t < n)
                  ? *reinterpret_cast<const uint32_t*>(x + (size_t)(t0 + t) * HID + k0 + kp * 2)
                  : 0u;
    }
  };
  fetch(kbase);
  for (int sl = 0; sl < NSL; ++sl) {
#pragma unroll
    for (int i = 0; i < (SH * KS) / (256 * 4); ++i) {
      const int idx = i * 256 + tid;
      const int row = idx / (KS / 4), c4 = idx % (KS / 4);
      ws[c4 * 4 + 0][row] = wr[i].x;
      ws[c4 * 4 + 1][row] = wr[i].y;
      ws[c4 * 4 + 2][row] = wr[i].z;
      ws[c4 * 4 + 3][row] = wr[i].w;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int idx = i * 256 + tid;
      const int t = idx / (KS / 2), kp = idx % (KS / 2);
      xs[kp * 2][t] = bf_lo(xr[i]);
      xs[kp * 2 + 1][t] = bf_hi(xr[i]);
    }
    __syncthreads();
    if (sl + 1 < NSL) fetch(kbase + (sl + 1) * KS);
#pragma unroll 4
    for (int kk = 0; kk < KS; ++kk) {
      const float4 xv = *reinterpret_cast<const float4*>(&xs[kk][tq * 4]);
      const float4 wa = *reinterpret_cast<const float4*>(&ws[kk][jo * 8]);
      const float4 wb = *reinterpret_cast<const float4*>(&ws[kk][jo * 8 + 4]);
      const float2 w2[4] = {make_float2(wa.x, wa.y), make_float2(wa.z, wa.w),
                            make_float2(wb.x, wb.y), make_float2(wb.z, wb.w)};
      const float xt[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float2 xx = make_float2(xt[a], xt[a]);
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = __ffma2_rn(xx, w2[b], acc[a][b]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int t = t0 + tq * 4 + a;
    if (t < n) {
      float4* dst = reinterpret_cast<float4*>(part + ((size_t)blockIdx.y * n + t) * SH + jo * 8);
      dst[0] = make_float4(acc[a][0].x, acc[a][0].y, acc[a][1].x, acc[a][1].y);
      dst[1] = make_float4(acc[a][2].x, acc[a][2].y, acc[a][3].x, acc[a][3].y);
    }
  }
}

// One block per token: h_j = sum of the splits (fixed order), SiLU, then s = W2·a.
__global__ void __launch_bounds__(256) k_score_finish(const float* __restrict__ part,
                                                      const float* __restrict__ w2, int n,
                                                      float* __restrict__ s) {
  __shared__ float red[8][NG];
  const int t = blockIdx.x, j = threadIdx.x;
  float h = 0.f;
#pragma unroll
  for (int sp = 0; sp < KSPLIT; ++sp) h += part[((size_t)sp * n + t) * SH + j];
  const float a = h / (1.0f + expf(-h));
  float c[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) c[g] = w2[g * SH + j] * a;
#pragma unroll
  for (int g = 0; g < NG; ++g)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c[g] += __shfl_xor_sync(0xffffffffu, c[g], o);
  const int warp = j >> 5, lane = j & 31;
  if (lane == 0)
#pragma unroll
    for (int g = 0; g < NG; ++g) red[warp][g] = c[g];
  __syncthreads();
  if (j < NG) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) acc += red[w][j];
    s[(size_t)t * NG + j] = acc;
  }
}

}  // namespace

size_t score_part_floats(int n) { return (size_t)KSPLIT * n * SH; }

int launch_score(const float* w1, const float* w2, const uint16_t* x, int n, float* s,
                 float* part, cudaStream_t st) {
  if (n <= 0) return ER_OK;
  k_score_partial<<<dim3((n + TT - 1) / TT, KSPLIT), 256, 0, st>>>(w1, x, n, part);
  k_score_finish<<<n, 256, 0, st>>>(part, w2, n, s);
  count_launches(2);
  return launch_status();
}

}  // namespace er

// ---------------------------------------------------------------------------
// Allocation-free variant.  The split-K partial sums normally live in scratch
// the caller passes in; here they live in this fixed array, which every GPU
// that loads the library keeps for the life of the process (ER_SCORE_NOALLOC_
// MAX_TOKENS x 16 splits x 256 floats = 4 MiB).  Host code must not hand the
// array's name to a kernel: on the host it only stands in for the symbol, so
// its device address is looked up with cudaGetSymbolAddress, once per device.
static __device__ __align__(256) float g_score_noalloc_scratch[(size_t)16 *
                                                               ER_SCORE_NOALLOC_MAX_TOKENS *
                                                               er::SH];

namespace er {
namespace {

static_assert(KSPLIT == 16, "the allocation-free scratch is sized for 16 K splits");

std::mutex g_noalloc_mu;
float* g_noalloc_ptr[64] = {nullptr};

}  // namespace
}  // namespace er

using namespace er;

extern "C" {

int er_rma_score_noalloc(const er_layer_weights* w, const er_bf16* x, int32_t n, float* s,
                         er_stream_t stream) {
  if (!w || n < 0 || (n > 0 && (!w->w1 || !w->w2 || !x || !s))) return ER_EINVAL;
  if (n > ER_SCORE_NOALLOC_MAX_TOKENS) return ER_ECAPACITY;
  if (n == 0) return ER_OK;
  if (!aligned16(w->w1) || ((uintptr_t)x & 3u)) return ER_EINVAL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ER_ECUDA;
  float* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      // first call on this device (which is current): find the array's device address
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_score_noalloc_scratch) != cudaSuccess || !p)
        return ER_ECUDA;
      g_noalloc_ptr[dev] = static_cast<float*>(p);
    }
    scratch = g_noalloc_ptr[dev];
  }
  // every split's partial sums are written before they are read: nothing to clear
  return launch_score(w->w1, w->w2, x, n, s, scratch, (cudaStream_t)stream);
}

size_t er_score_workspace_bytes(int32_t n) {
  if (n < 0) return 0;
  Carver c(nullptr);
  c.take<float>(score_part_floats(n));
  return c.used();
}

int er_rma_score(const er_layer_weights* w, const er_bf16* x, int32_t n, float* s, void* ws,
                 size_t ws_bytes, er_stream_t stream) {
  if (!w || n < 0 || (n > 0 && (!w->w1 || !w->w2 || !x || !s || !ws))) return ER_EINVAL;
  if (n == 0) return ER_OK;
  if (!aligned16(w->w1) || !aligned16(ws) || ((uintptr_t)x & 3u)) return ER_EINVAL;
  if (ws_bytes < er_score_workspace_bytes(n)) return ER_ECAPACITY;
  return launch_score(w->w1, w->w2, x, n, s, reinterpret_cast<float*>(ws),
                      (cudaStream_t)stream);
}

}  // extern "C"
