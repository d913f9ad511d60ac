// gemv.cu — the layer's projections for a few tokens (decode batches of up to
// 32 sequences): a1 (x·W_qkvᵀ, with the prepared weights also the scorer's W1
// terms) and a6 (o·W_oᵀ).  Layer shapes from EdgeRock-4B 开源：72 MiB 固定 KV,
// §架构：递归、局部窗口与记忆锚点三件套.
//
// With T <= 32 tokens each weight element is used at most 32 times, so the
// product is a stream of the weights (67 MB for q/k/v + W1 terms, 21 MB for
// o_proj) that HBM bounds.  A warp owns 16 weight rows and a slice of K; per
// 32-wide step of K every lane loads 16 contiguous bytes of two rows (rows g
// and g+8, columns 8c..8c+7 of the step, g = lane/4, c = lane%4) and 16 bytes
// of x for token g of each 8-token tile, and feeds them unchanged to two
// m16n8k16 tensor-core products: the eight K columns a lane holds are given to
// the MMA as columns (2c, 2c+1, 2c+8, 2c+9) of one product and of the next.
// The same K column then meets the same K column on both operands, and a dot
// product does not depend on the order of its terms, so no data is rearranged.
// BF16 products are exact and accumulate in FP32; the warps of a block (the
// K slices of the same rows) add their partial sums in a fixed order, so the
// same inputs give the same bits.
#include "common.cuh"

namespace er {
namespace {

constexpr int GV_MAXW = 8;  // warps (K slices) per block

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ld_x(const uint16_t* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// D += A·B, m16n8k16, BF16 operands, FP32 accumulators.
__device__ __forceinline__ void mma16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Y[t][f] = Σ_k X[t][k] W[f][k] for t < T <= 8·NT, f < F (F a multiple of 16);
// block b owns rows 16b..16b+15, its warp w the K slice [w·K/S, (w+1)·K/S)
// (K/S a multiple of 32).  Y FP32 or BF16 (round to nearest even), row stride ldy.
template <int NT, int U>
__global__ void __launch_bounds__(32 * GV_MAXW)
    k_gemv(const uint16_t* __restrict__ X, int T, const uint16_t* __restrict__ W, void* Y, int K,
           int ldy, int yf32) {
  __shared__ float red[GV_MAXW][32][4 * NT];
  grid_dep_trigger();  // the kernel after this one may set itself up
  const int S = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int ks_n = K / S / 32;  // 32-wide K steps of this warp
  const int row0 = blockIdx.x * 16;
  const size_t kbeg = (size_t)warp * (K / S) + 8 * c;
  const uint16_t* wa = W + (size_t)(row0 + g) * K + kbeg;
  const uint16_t* wb = wa + (size_t)8 * K;
  const uint16_t* xp[NT];
  bool xv[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    xv[j] = 8 * j + g < T;
    xp[j] = X + (size_t)(xv[j] ? 8 * j + g : 0) * K + kbeg;
  }
  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[j][i] = 0.f;

  const uint4 z = make_uint4(0, 0, 0, 0);
  uint4 a[U], b[U];
  // the weights are never written by the library: the first step's rows are
  // requested before waiting for the kernel that writes x
#pragma unroll
  for (int u = 0; u < U; ++u) {
    a[u] = u < ks_n ? ld_stream(wa + 32 * u) : z;
    b[u] = u < ks_n ? ld_stream(wb + 32 * u) : z;
  }
  grid_dep_wait();
  for (int ks = 0; ks < ks_n; ks += U) {
    uint4 x[NT][U];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int u = 0; u < U; ++u) x[j][u] = (xv[j] && ks + u < ks_n) ? ld_x(xp[j] + 32 * (ks + u)) : z;
#pragma unroll
    for (int u = 0; u < U; ++u) {
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        mma16816(acc[j], a[u].x, b[u].x, a[u].y, b[u].y, x[j][u].x, x[j][u].y);
        mma16816(acc[j], a[u].z, b[u].z, a[u].w, b[u].w, x[j][u].z, x[j][u].w);
      }
    }
    // the next step's rows
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = ks + U + u;
      a[u] = k < ks_n ? ld_stream(wa + 32 * k) : z;
      b[u] = k < ks_n ? ld_stream(wb + 32 * k) : z;
    }
  }
  // acc[j][i]: row g + 8·(i >> 1), token 8j + 2c + (i & 1)
  if (S > 1) {
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp][lane][4 * j + i] = acc[j][i];
    __syncthreads();
    if (warp != 0) return;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float s = red[0][lane][4 * j + i];
        for (int w = 1; w < S; ++w) s += red[w][lane][4 * j + i];
        acc[j][i] = s;
      }
  }
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = 8 * j + 2 * c + (i & 1);
      const int row = row0 + g + 8 * (i >> 1);
      if (t < T) {
        if (yf32)
          static_cast<float*>(Y)[(size_t)t * ldy + row] = acc[j][i];
        else
          static_cast<uint16_t*>(Y)[(size_t)t * ldy + row] = f2bf(acc[j][i]);
      }
    }
}

template <int NT, int U>
int launch_t(const uint16_t* X, int T, const uint16_t* W, void* Y, int F, int K, int ldy,
             bool yf32, cudaStream_t st) {
  // K slices per block: enough warps to keep ~8 per SM streaming, each slice a
  // whole number of 32-wide steps
  const int blocks = F / 16;
  int S = 1;
  while (S < GV_MAXW && blocks * S < 8 * num_sms() && (K / 32) % (2 * S) == 0) S <<= 1;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(32 * S);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k_gemv<NT, U>, X, T, W, Y, K, ldy, yf32 ? 1 : 0) != cudaSuccess)
    return ER_ECUDA;
  count_launches(1);
  return launch_status();
}

}  // namespace

// Y = X · Wᵀ for 1 <= T <= 32 tokens (see the top of this file).  F a multiple
// of 16, K of 32; X [T][K], W [F][K] BF16, 16-byte aligned; Y row stride ldy.
int launch_gemv(const uint16_t* X, int T, const uint16_t* W, int F, int K, void* Y, bool yf32,
                int ldy, cudaStream_t st) {
  if (T <= 0) return ER_OK;
  if (T > kGemvMaxTokensAll || F <= 0 || F % 16 || K <= 0 || K % 32 || ldy < F) return ER_EINVAL;
  if (T <= 8) return launch_t<1, 8>(X, T, W, Y, F, K, ldy, yf32, st);
  if (T <= 16) return launch_t<2, 6>(X, T, W, Y, F, K, ldy, yf32, st);
  return launch_t<4, 4>(X, T, W, Y, F, K, ldy, yf32, st);
}

}  // namespace er
