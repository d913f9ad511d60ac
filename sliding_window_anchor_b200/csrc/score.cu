// score.cu — a3, the RMA retention scorer.
//
// EdgeRock-4B 开源：72 MiB 固定 KV, §架构：递归、局部窗口与记忆锚点三件套: a small
// independent bias-free network maps the 2560-wide hidden state to 256 and
// then to 4 values in FP32, one retention score per KV group (SiLU between
// the two matmuls is this library's reading).
//
// The 2560→256 product is a dense contraction over all tokens of a call, so
// it runs on the 5th-generation tensor cores (tcgen05.mma, accumulator in
// TMEM).  FP32 accuracy without FP32 tensor math: x is BF16 already, and W1
// is split into three BF16 terms W1 ≈ hi + mid + lo (residual below 2^-24 of
// |W1|), so x·W1 is the sum of three exact BF16 products accumulated in FP32.
//   k_w1_split   : W1 (FP32) -> the three BF16 terms, in the scratch buffer;
//   k_score_tc   : block (128 tokens, 32 hidden units): warp 0 streams x and
//                  the W1 terms with TMA (64-wide K slices, 128-byte swizzle,
//                  4-stage mbarrier ring), warp 1 allocates TMEM and issues
//                  the MMAs (M=128, N=32, K=16; 3 per K step), warps 2-5 read
//                  the accumulator from TMEM, apply SiLU and contract with
//                  their 32 columns of W2 into 4 partial scores per token;
//   k_score_sum  : the 8 partial scores of each token summed in a fixed order.
// Deterministic.  Scratch (er_score_workspace_bytes): the W1 terms and the
// partial scores.
#include <mutex>

#include "common.cuh"
#include "tc.cuh"

namespace er {
namespace {

constexpr int TM = 128;            // tokens per block (MMA M)
constexpr int TN = 32;             // hidden units per block (MMA N)
constexpr int NCH = SH / TN;       // 8 hidden chunks
constexpr int KB = 64;             // K slice: one 128-byte swizzled row
constexpr int NKB = HID / KB;      // 40
constexpr int SST = 4;             // pipeline stages
constexpr int NPART = 3;           // BF16 terms of W1
constexpr int A_BYTES = TM * 128;  // 16 KB
constexpr int B_BYTES = TN * 128;  // 4 KB per term

struct __align__(1024) ScoreSmem {
  unsigned char a[SST][A_BYTES];
  unsigned char b[SST][NPART][B_BYTES];
  float w2c[NG][TN];
  uint64_t full[SST], empty[SST], acc_full;
  uint32_t tmem_base;
};

static_assert(sizeof(ScoreSmem) + 1024 <= 232448, "shared memory above the per-block limit");

struct ScoreParams {
  CUtensorMap tmap_x;  // x [n][2560] BF16, box 64 x 128
  CUtensorMap tmap_w;  // W1 terms [3*256][2560] BF16, box 64 x 32
  const float* w2;
  float* part;         // [8][n][4]
  int n;
  int32_t* err;
};

// W1 -> hi + mid + lo, each BF16 (round to nearest), stacked [3][256][2560].
__global__ void k_w1_split(const float* __restrict__ w1, uint16_t* __restrict__ terms, int count) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < count; i += gridDim.x * blockDim.x) {
    const float w = w1[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    terms[i] = __bfloat16_as_ushort(hi);
    terms[count + i] = __bfloat16_as_ushort(mid);
    terms[2 * count + i] = __bfloat16_as_ushort(lo);
  }
}

__global__ void __launch_bounds__(192, 1) k_score_tc(const __grid_constant__ ScoreParams P) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ScoreSmem& S = *reinterpret_cast<ScoreSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * TM;
  const int chunk = blockIdx.y, n0 = chunk * TN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SST; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(&S.tmem_base, 32);
  if (warp >= 2) {
    const int t = threadIdx.x - 64;  // 0..127: stage this block's W2 columns
    S.w2c[t >> 5][t & 31] = P.w2[(t >> 5) * SH + n0 + (t & 31)];
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = S.tmem_base;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA
    for (int kb = 0; kb < NKB; ++kb) {
      const int s = kb % SST;
      const uint32_t ph = (kb / SST) & 1;
      if (!mbar_wait(&S.empty[s], ph ^ 1, P.err)) break;
      mbar_arrive_expect_tx(&S.full[s], A_BYTES + NPART * B_BYTES);
      tc::tma_load_2d(S.a[s], &P.tmap_x, kb * KB, m0, &S.full[s]);
#pragma unroll
      for (int p = 0; p < NPART; ++p)
        tc::tma_load_2d(S.b[s][p], &P.tmap_w, kb * KB, p * SH + n0, &S.full[s]);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    constexpr uint32_t idesc = tc::idesc_bf16(TM, TN, false, false);
    for (int kb = 0; kb < NKB; ++kb) {
      const int s = kb % SST;
      const uint32_t ph = (kb / SST) & 1;
      if (!mbar_wait(&S.full[s], ph, P.err)) break;
      tc::fence_after_sync();
      const uint32_t a0 = smem_u32(S.a[s]);
#pragma unroll
      for (int kk = 0; kk < KB / 16; ++kk) {
        const uint64_t ad = tc::desc_sw128(a0 + 32 * kk, 16, 1024);
#pragma unroll
        for (int p = 0; p < NPART; ++p) {
          const uint64_t bd = tc::desc_sw128(smem_u32(S.b[s][p]) + 32 * kk, 16, 1024);
          tc::mma_bf16_ss(tmem, ad, bd, idesc, (kb | kk | p) != 0);
        }
      }
      tc::commit(&S.empty[s]);  // the stage is free once these MMAs have read it
    }
    tc::commit(&S.acc_full);
  } else if (warp >= 2) {
    // ----------------------------------------------------------- epilogue
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    const int tok = m0 + 32 * quad + lane;
    const bool ok = mbar_wait(&S.acc_full, 0, P.err);
    tc::fence_after_sync();
    uint32_t h[32];
    tc::tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16), h);
    tc::tmem_wait_ld();
    if (ok && tok < P.n) {
      float s4[NG] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < TN; ++j) {
        const float x = __uint_as_float(h[j]);
        const float a = x / (1.0f + expf(-x));
#pragma unroll
        for (int g = 0; g < NG; ++g) s4[g] = fmaf(S.w2c[g][j], a, s4[g]);
      }
      *reinterpret_cast<float4*>(P.part + ((size_t)chunk * P.n + tok) * NG) =
          make_float4(s4[0], s4[1], s4[2], s4[3]);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 32);
  }
}

// s[t][g] = sum over the 8 hidden chunks, in chunk order.
__global__ void k_score_sum(const float* __restrict__ part, int n, float* __restrict__ s) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n * NG) return;
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < NCH; ++c) acc += part[(size_t)c * n * NG + i];
  s[i] = acc;
}

bool g_attr_done[64] = {false};
std::mutex g_attr_mu;

}  // namespace

// Scratch layout: the W1 terms (3 x 256 x 2560 BF16), then the partial scores.
size_t score_scratch_bytes(int n) {
  Carver c(nullptr);
  c.take<uint16_t>((size_t)NPART * SH * HID);
  c.take<float>((size_t)NCH * n * NG);
  return c.used();
}

int launch_score(const float* w1, const float* w2, const uint16_t* x, int n, float* s,
                 void* scratch, int32_t* err, cudaStream_t st) {
  if (n <= 0) return ER_OK;
  Carver c(scratch);
  uint16_t* terms = c.take<uint16_t>((size_t)NPART * SH * HID);
  float* part = c.take<float>((size_t)NCH * n * NG);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ER_ECUDA;
  {
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (!g_attr_done[dev]) {
      if (cudaFuncSetAttribute(k_score_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)sizeof(ScoreSmem) + 1024) != cudaSuccess)
        return ER_ECUDA;
      g_attr_done[dev] = true;
    }
  }
  ScoreParams P;
  if (!encode_bf16_2d(&P.tmap_x, x, HID, (uint64_t)n, HID * 2, KB, TM) ||
      !encode_bf16_2d(&P.tmap_w, terms, HID, (uint64_t)NPART * SH, HID * 2, KB, TN))
    return ER_ECUDA;
  P.w2 = w2;
  P.part = part;
  P.n = n;
  P.err = err;
  k_w1_split<<<148 * 4, 256, 0, st>>>(w1, terms, SH * HID);
  k_score_tc<<<dim3((n + TM - 1) / TM, NCH), 192, sizeof(ScoreSmem) + 1024, st>>>(P);
  k_score_sum<<<(n * NG + 255) / 256, 256, 0, st>>>(part, n, s);
  count_launches(3);
  return launch_status();
}

}  // namespace er

// ---------------------------------------------------------------------------
// Allocation-free variant.  The scratch normally lives in memory the caller
// passes in; here it lives in this fixed array, which every GPU that loads the
// library keeps for the life of the process (4 MiB: the W1 terms plus the
// partial scores of up to ER_SCORE_NOALLOC_MAX_TOKENS tokens).  Host code must
// not hand the array's name to a kernel: on the host it only stands in for the
// symbol, so its device address is looked up with cudaGetSymbolAddress, once
// per device.
static __device__ __align__(256) float g_score_noalloc_scratch[(size_t)16 *
                                                               ER_SCORE_NOALLOC_MAX_TOKENS *
                                                               er::SH];

namespace er {
namespace {

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
  if (!aligned16(w->w1) || !aligned16(x)) return ER_EINVAL;
  if (score_scratch_bytes(n) > sizeof(g_score_noalloc_scratch)) return ER_ECAPACITY;
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
  // every scratch word a call reads was written earlier in the same call: nothing to clear
  return launch_score(w->w1, w->w2, x, n, s, scratch, nullptr, (cudaStream_t)stream);
}

size_t er_score_workspace_bytes(int32_t n) {
  if (n < 1) return 0;
  return score_scratch_bytes(n);
}

int er_rma_score(const er_layer_weights* w, const er_bf16* x, int32_t n, float* s, void* ws,
                 size_t ws_bytes, er_stream_t stream) {
  if (!w || n < 0 || (n > 0 && (!w->w1 || !w->w2 || !x || !s || !ws))) return ER_EINVAL;
  if (n == 0) return ER_OK;
  if (!aligned16(w->w1) || !aligned16(ws) || !aligned16(x)) return ER_EINVAL;
  if (ws_bytes < er_score_workspace_bytes(n)) return ER_ECAPACITY;
  return launch_score(w->w1, w->w2, x, n, s, ws, nullptr, (cudaStream_t)stream);
}

}  // extern "C"
