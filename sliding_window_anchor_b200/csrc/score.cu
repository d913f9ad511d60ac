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
// is taken as three BF16 terms W1 ≈ hi + mid + lo (residual below 2^-24 of
// |W1|), so x·W1 is the sum of three exact BF16 products accumulated in FP32.
// The terms come prepared with the weights (er_score_split_w1), or are made
// in the workspace by each call.
//
// k_score_tc: a cluster of 8 CTAs splits K = 2560 into 8 parts of 320; each
// CTA owns 128 tokens x 64 hidden units of one part:
//   warp 0    : TMA — 64-wide K slices of x and of the three W1 terms
//               (128-byte swizzle, 4-stage mbarrier ring);
//   warp 1    : TMEM (64 columns) and MMA issue (M=128, N=64, K=16; 3 per
//               K step, one per term);
//   warps 2-5 : the 128x64 partial accumulator from TMEM into shared memory;
// then, after a cluster barrier, CTA r of the cluster sums rows 16r..16r+15
// over the 8 parts in rank order (distributed shared memory), applies SiLU
// and contracts with its 64 columns of W2 into 4 partial scores per token.
// k_score_sum adds the 4 quarters of the hidden units in a fixed order.
// Deterministic.
#include <mutex>

#include "common.cuh"
#include "tc.cuh"

namespace er {
namespace {

constexpr int TM = 128;                  // tokens per CTA (MMA M)
constexpr int TN = 64;                   // hidden units per CTA (MMA N)
constexpr int NQ = SH / TN;              // 4 hidden quarters
constexpr int KB = 64;                   // K slice: one 128-byte swizzled row
constexpr int KPARTS = 8;                // cluster size: parts of K
constexpr int KSL = HID / KB / KPARTS;   // 5 slices per part
constexpr int SST = 4;                   // pipeline stages
constexpr int NPART = 3;                 // BF16 terms of W1
constexpr int A_BYTES = TM * 128;        // 16 KB
constexpr int B_BYTES = TN * 128;        // 8 KB per term
constexpr int ROWS_PER_RANK = TM / KPARTS;  // 16 rows reduced by each CTA

static_assert(KSL * KB * KPARTS == HID, "K parts must tile the hidden size");

struct __align__(1024) ScoreSmem {
  unsigned char a[SST][A_BYTES];
  unsigned char b[SST][NPART][B_BYTES];
  // this part's 128 x 64 partial sums; row r keeps its 16-byte chunk c at
  // position c ^ (r & 7), so neither the row-wise writes nor the vector reads
  // of the reduction collide on banks
  float red[TM * TN];
  float w2c[NG][TN];
  uint64_t full[SST], empty[SST], acc_full;
  uint32_t tmem_base;
};

constexpr size_t SCORE_SMEM = sizeof(ScoreSmem) + 1024;
static_assert(SCORE_SMEM <= 232448, "shared memory above the per-block limit");

struct ScoreParams {
  CUtensorMap tmap_x;  // x [n][2560] BF16, box 64 x 128
  CUtensorMap tmap_w;  // W1 terms [3*256][2560] BF16, box 64 x 64
  const float* w2;
  float* part;         // [4][n][4]: per hidden quarter
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

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory word in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t dsmem_map(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ float4 dsmem_ld4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ int red_index(int row, int chunk) {
  return row * TN + ((chunk ^ (row & 7)) << 2);
}

// Every thread of every CTA of the cluster (release / acquire on shared memory).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__global__ void __cluster_dims__(KPARTS, 1, 1) __launch_bounds__(192, 1)
    k_score_tc(const __grid_constant__ ScoreParams P) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ScoreSmem& S = *reinterpret_cast<ScoreSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  grid_dep_trigger();  // the norm/RoPE kernel may set itself up (it waits for us)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // the K part
  const int m0 = blockIdx.y * TM;
  const int quarter = blockIdx.z, n0 = quarter * TN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SST; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(&S.tmem_base, TN);
  if (warp >= 2) {
    // this CTA's 64 columns of W2
    for (int t = threadIdx.x - 64; t < NG * TN; t += 128)
      S.w2c[t / TN][t % TN] = P.w2[(t / TN) * SH + n0 + (t % TN)];
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = S.tmem_base;
  bool ok = true;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA
    int issued = 0;
    for (int ks = 0; ks < KSL; ++ks) {
      const int s = ks % SST;
      const uint32_t ph = (ks / SST) & 1;
      if (!mbar_wait(&S.empty[s], ph ^ 1, P.err)) break;
      const int kx = ((int)rank * KSL + ks) * KB;
      mbar_arrive_expect_tx(&S.full[s], A_BYTES + NPART * B_BYTES);
      tc::tma_load_2d(S.a[s], &P.tmap_x, kx, m0, &S.full[s]);
#pragma unroll
      for (int p = 0; p < NPART; ++p)
        tc::tma_load_2d(S.b[s][p], &P.tmap_w, kx, p * SH + n0, &S.full[s]);
      ++issued;
    }
    // no copy may still be landing when the block exits
    for (int ks = max(0, issued - SST); ks < issued; ++ks)
      mbar_wait(&S.full[ks % SST], (ks / SST) & 1, P.err);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    constexpr uint32_t idesc = tc::idesc_bf16(TM, TN, false, false);
    for (int ks = 0; ks < KSL; ++ks) {
      const int s = ks % SST;
      const uint32_t ph = (ks / SST) & 1;
      if (!mbar_wait(&S.full[s], ph, P.err)) break;
      tc::fence_after_sync();
      const uint32_t a0 = smem_u32(S.a[s]);
#pragma unroll
      for (int kk = 0; kk < KB / 16; ++kk) {
        const uint64_t ad = tc::desc_sw128(a0 + 32 * kk, 16, 1024);
#pragma unroll
        for (int p = 0; p < NPART; ++p) {
          const uint64_t bd = tc::desc_sw128(smem_u32(S.b[s][p]) + 32 * kk, 16, 1024);
          tc::mma_bf16_ss(tmem, ad, bd, idesc, (ks | kk | p) != 0);
        }
      }
      tc::commit(&S.empty[s]);  // the stage is free once these MMAs have read it
    }
    tc::commit(&S.acc_full);
    mbar_wait(&S.acc_full, 0, P.err);  // nothing in flight on the tensor cores at exit
  } else if (warp >= 2) {
    // ---------------------------------------- partial accumulator -> smem
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    const int row = 32 * quad + lane;
    ok = __all_sync(0xffffffffu, mbar_wait(&S.acc_full, 0, P.err));
    if (ok) {
      tc::fence_after_sync();
#pragma unroll
      for (int cb = 0; cb < TN / 32; ++cb) {
        uint32_t h[32];
        tc::tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + 32 * cb, h);
        tc::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<float4*>(&S.red[red_index(row, 8 * cb + c)]) =
              make_float4(__uint_as_float(h[4 * c]), __uint_as_float(h[4 * c + 1]),
                          __uint_as_float(h[4 * c + 2]), __uint_as_float(h[4 * c + 3]));
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  cluster_sync();  // every part's partial sums are in its shared memory

  if (warp >= 2) {
    // rows 16*rank .. +15 of the tile: sum the 8 parts in rank order, SiLU, W2
    const int t = threadIdx.x - 64;        // 0..127
    const int rl = t >> 3, seg = t & 7;    // row within the rank's 16, 8-column segment
    const int row = ROWS_PER_RANK * (int)rank + rl;
    const uint32_t a0 = smem_u32(&S.red[red_index(row, 2 * seg)]);
    const uint32_t a1 = smem_u32(&S.red[red_index(row, 2 * seg + 1)]);
    // all 16 remote loads in flight, then the sum in rank order
    float4 v0[KPARTS], v1[KPARTS];
#pragma unroll
    for (uint32_t q = 0; q < KPARTS; ++q) {
      v0[q] = dsmem_ld4(dsmem_map(a0, q));
      v1[q] = dsmem_ld4(dsmem_map(a1, q));
    }
    float h[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < KPARTS; ++q) {
      h[0] += v0[q].x; h[1] += v0[q].y; h[2] += v0[q].z; h[3] += v0[q].w;
      h[4] += v1[q].x; h[5] += v1[q].y; h[6] += v1[q].z; h[7] += v1[q].w;
    }
    float s4[NG] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float a = h[c] / (1.0f + expf(-h[c]));
#pragma unroll
      for (int g = 0; g < NG; ++g) s4[g] = fmaf(S.w2c[g][seg * 8 + c], a, s4[g]);
    }
    // the 8 segments of a row sit in 8 consecutive lanes: fixed-order tree
#pragma unroll
    for (int o = 4; o >= 1; o >>= 1)
#pragma unroll
      for (int g = 0; g < NG; ++g) s4[g] += __shfl_xor_sync(0xffffffffu, s4[g], o);
    const int tok = m0 + row;
    if (seg == 0 && tok < P.n)
      *reinterpret_cast<float4*>(P.part + ((size_t)quarter * P.n + tok) * NG) =
          make_float4(s4[0], s4[1], s4[2], s4[3]);
  }
  cluster_sync();  // no CTA leaves while another still reads its shared memory
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TN);
  }
}

// s[t][g] = sum over the 4 hidden quarters, in quarter order.
__global__ void k_score_sum(const float* __restrict__ part, int n, float* __restrict__ s) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n * NG) return;
  float acc = 0.f;
#pragma unroll
  for (int q = 0; q < NQ; ++q) acc += part[(size_t)q * n * NG + i];
  s[i] = acc;
}

bool g_attr_done[64] = {false};
std::mutex g_attr_mu;

}  // namespace

// Where launch_score leaves the partial scores [4][n][4] in its scratch.
const float* score_partials(const void* scratch, int n) {
  Carver c(const_cast<void*>(scratch));
  c.take<uint16_t>((size_t)NPART * SH * HID);
  return c.take<float>((size_t)NQ * n * NG);
}

// Scratch layout: the W1 terms (3 x 256 x 2560 BF16; only used when the
// weights carry no prepared terms), then the partial scores.
size_t score_scratch_bytes(int n) {
  Carver c(nullptr);
  c.take<uint16_t>((size_t)NPART * SH * HID);
  c.take<float>((size_t)NQ * n * NG);
  return c.used();
}

// s == nullptr: leave the 4 quarter partials in the scratch (score_partials)
// for a consumer that adds them itself.
int launch_score(const float* w1, const uint16_t* w1_split, const float* w2, const uint16_t* x,
                 int n, float* s, void* scratch, int32_t* err, cudaStream_t st) {
  if (n <= 0) return ER_OK;
  Carver c(scratch);
  uint16_t* terms = c.take<uint16_t>((size_t)NPART * SH * HID);
  float* part = c.take<float>((size_t)NQ * n * NG);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ER_ECUDA;
  {
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (!g_attr_done[dev]) {
      if (cudaFuncSetAttribute(k_score_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)SCORE_SMEM) != cudaSuccess)
        return ER_ECUDA;
      g_attr_done[dev] = true;
    }
  }
  int launches = 2;
  if (!w1_split) {
    k_w1_split<<<148 * 4, 256, 0, st>>>(w1, terms, SH * HID);
    w1_split = terms;
    ++launches;
  }
  ScoreParams P;
  if (!encode_bf16_2d(&P.tmap_x, x, HID, (uint64_t)n, HID * 2, KB, TM) ||
      !encode_bf16_2d(&P.tmap_w, w1_split, HID, (uint64_t)NPART * SH, HID * 2, KB, TN))
    return ER_ECUDA;
  P.w2 = w2;
  P.part = part;
  P.n = n;
  P.err = err;
  k_score_tc<<<dim3(KPARTS, (n + TM - 1) / TM, NQ), 192, SCORE_SMEM, st>>>(P);
  if (s) {
    k_score_sum<<<(n * NG + 255) / 256, 256, 0, st>>>(part, n, s);
  } else {
    --launches;
  }
  count_launches(launches);
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

int er_score_split_w1(const float* w1, er_bf16* terms, er_stream_t stream) {
  if (!w1 || !terms || !aligned16(w1) || !aligned16(terms)) return ER_EINVAL;
  k_w1_split<<<148 * 4, 256, 0, (cudaStream_t)stream>>>(w1, terms, SH * HID);
  count_launches(1);
  return launch_status();
}

int er_prepare_qkv_score(const er_bf16* w_qkv, const float* w1, er_bf16* out,
                         er_stream_t stream) {
  if (!w_qkv || !w1 || !out || !aligned16(w_qkv) || !aligned16(w1) || !aligned16(out))
    return ER_EINVAL;
  const size_t qkv_bytes = (size_t)QKV * HID * sizeof(uint16_t);
  const uintptr_t a = reinterpret_cast<uintptr_t>(w_qkv), b = reinterpret_cast<uintptr_t>(out);
  if (a < b + (size_t)QKVS * HID * sizeof(uint16_t) && b < a + qkv_bytes) return ER_EINVAL;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(out, w_qkv, qkv_bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return ER_ECUDA;
  k_w1_split<<<148 * 4, 256, 0, st>>>(w1, out + (size_t)QKV * HID, SH * HID);
  count_launches(1);
  return launch_status();
}

int er_rma_score_noalloc(const er_layer_weights* w, const er_bf16* x, int32_t n, float* s,
                         er_stream_t stream) {
  if (!w || n < 0 || (n > 0 && (!w->w1 || !w->w2 || !x || !s))) return ER_EINVAL;
  if (n > ER_SCORE_NOALLOC_MAX_TOKENS) return ER_ECAPACITY;
  if (n == 0) return ER_OK;
  if (!aligned16(w->w1) || !aligned16(x) || (w->w1_split && !aligned16(w->w1_split)))
    return ER_EINVAL;
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
  int32_t* err = call_error_word();  // also a fixed device word: nothing allocated
  if (!err) return ER_ECUDA;
  // every scratch word a call reads was written earlier in the same call: nothing to clear
  return launch_score(w->w1, w->w1_split, w->w2, x, n, s, scratch, err, (cudaStream_t)stream);
}

size_t er_score_workspace_bytes(int32_t n) {
  if (n < 1) return 0;
  return score_scratch_bytes(n);
}

int er_rma_score_ex(const er_layer_weights* w, const er_bf16* x, int32_t n, float* s, void* ws,
                    size_t ws_bytes, int32_t* dev_error, er_stream_t stream) {
  if (!w || n < 0 || (n > 0 && (!w->w1 || !w->w2 || !x || !s || !ws))) return ER_EINVAL;
  if (n == 0) return ER_OK;
  if (!aligned16(w->w1) || !aligned16(ws) || !aligned16(x) ||
      (w->w1_split && !aligned16(w->w1_split)))
    return ER_EINVAL;
  if (ws_bytes < er_score_workspace_bytes(n)) return ER_ECAPACITY;
  int32_t* err = dev_error ? dev_error : call_error_word();
  if (!err) return ER_ECUDA;
  return launch_score(w->w1, w->w1_split, w->w2, x, n, s, ws, err, (cudaStream_t)stream);
}

int er_rma_score(const er_layer_weights* w, const er_bf16* x, int32_t n, float* s, void* ws,
                 size_t ws_bytes, er_stream_t stream) {
  return er_rma_score_ex(w, x, n, s, ws, ws_bytes, nullptr, stream);
}

}  // extern "C"
