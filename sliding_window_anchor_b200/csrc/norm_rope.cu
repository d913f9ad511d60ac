// norm_rope.cu — a2 (q/k RMS-norm + partial RoPE) and the a4 state writes
// that follow the projections.
//
// EdgeRock-4B 开源：72 MiB 固定 KV, §架构：递归、局部窗口与记忆锚点三件套:
// q and k carry a learned RMS-norm; rotary embedding covers 64 of the 256
// dims with base 1e7; v is neither normed nor rotated.  Pairing (i, i+32),
// eps 1e-6 and the directly applied gain are this library's reading.
//
// One warp owns one 256-wide head vector, 8 BF16 values per lane (one 16-byte
// load); lanes 0..7 hold the rotated dims and exchange pairs with xor 4.  The
// rotation angle pos * 1e7^(-2i/64) is formed and reduced in float64 so that
// positions up to 2^18 keep full angle accuracy (once per token in the layer
// kernel, shared by its head vectors); the rotation itself is fp32.
#include "common.cuh"
#include "params.cuh"

namespace er {
namespace {

__device__ __forceinline__ void load8(const uint16_t* src, float v[8]) {
  uint4 w = *reinterpret_cast<const uint4*>(src);
  v[0] = bf_lo(w.x); v[1] = bf_hi(w.x); v[2] = bf_lo(w.y); v[3] = bf_hi(w.y);
  v[4] = bf_lo(w.z); v[5] = bf_hi(w.z); v[6] = bf_lo(w.w); v[7] = bf_hi(w.w);
}

__device__ __forceinline__ void store8(uint16_t* dst, const float v[8]) {
  uint4 w;
  w.x = pack_bf2(v[0], v[1]); w.y = pack_bf2(v[2], v[3]);
  w.z = pack_bf2(v[4], v[5]); w.w = pack_bf2(v[6], v[7]);
  *reinterpret_cast<uint4*>(dst) = w;
}

// cos/sin of pos * 1e7^(-2i/64) for i = lane (0..31): the angle is formed and
// reduced in float64 (one evaluation per lane), then rounded to float.
__device__ __forceinline__ float2 rope_cs_lane(int32_t pos, int lane) {
  const double kLog2Theta = 23.253496664211536;  // log2(1e7)
  const double inv_freq = exp2(-(double)lane * (kLog2Theta / 32.0));
  double sn, cs;
  sincos((double)pos * inv_freq, &sn, &cs);
  return make_float2((float)cs, (float)sn);
}

// y = x / sqrt(mean(x^2) + 1e-6) * gain, then rotate (i, i+32), i < 32.
__device__ __forceinline__ void norm_rope_lane(float v[8], const uint16_t* gain, int32_t pos,
                                               int lane) {
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss * (1.0f / D) + 1e-6f);
  float g[8];
  load8(gain + lane * 8, g);
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = (v[e] * inv) * g[e];
  const float2 mycs = rope_cs_lane(pos, lane);
  float partner[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    partner[e] = __shfl_xor_sync(0xffffffffu, v[e], 4);
    // frequency index of this lane's element e (lanes 0..7): 8*(lane&3) + e
    const float c = __shfl_sync(0xffffffffu, mycs.x, (lane & 3) * 8 + e);
    const float sn = __shfl_sync(0xffffffffu, mycs.y, (lane & 3) * 8 + e);
    if (lane < 4) v[e] = v[e] * c - partner[e] * sn;        // dim i:    a cos - b sin
    else if (lane < 8) v[e] = v[e] * c + partner[e] * sn;   // dim i+32: b cos + a sin
  }
}

// The same with the 32 (cos, sin) pairs of the position already in `cs`
// (shared memory): the unfused layer kernel forms them once per token.
__device__ __forceinline__ void norm_rope_lane_cs(float v[8], const uint16_t* gain,
                                                  const float2* cs, int lane) {
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss * (1.0f / D) + 1e-6f);
  float g[8];
  load8(gain + lane * 8, g);
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = (v[e] * inv) * g[e];
  float partner[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    partner[e] = __shfl_xor_sync(0xffffffffu, v[e], 4);
    const float2 f = cs[(lane & 3) * 8 + e];
    if (lane < 4) v[e] = v[e] * f.x - partner[e] * f.y;        // dim i:    a cos - b sin
    else if (lane < 8) v[e] = v[e] * f.x + partner[e] * f.y;   // dim i+32: b cos + a sin
  }
}

__global__ void k_norm_rope(const uint16_t* x, uint16_t* y, int64_t n_rows, const uint16_t* gain,
                            const int32_t* pos) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  float v[8];
  load8(x + row * D + lane * 8, v);
  norm_rope_lane(v, gain, pos[row], lane);
  store8(y + row * D + lane * 8, v);
}

}  // namespace


// Grid (nq, 6) x 256 threads: warp slot hs = 0..47 covers, per token,
// q_swa 0..15 | k_swa 16..19 | v_swa 20..23 | q_rma 24..39 | k_rma 40..43 | v_rma 44..47.
__global__ void __launch_bounds__(256) k_post_proj(PostParams P) {
  __shared__ float2 s_cs[32];  // the rotation of this token's position, formed once
  grid_dep_trigger();  // a prefill read may set itself up meanwhile (it waits for us)
  const int lane = threadIdx.x & 31;
  const int hs = blockIdx.y * 8 + (threadIdx.x >> 5);
  const int qi = blockIdx.x;
  // the read that follows takes its work units from this counter; it waits for
  // this kernel to complete before the first one
  if (P.sched_reset && qi == 0 && hs == 0 && lane == 0) *P.sched_reset = 0;
  const int seq = P.prefill ? P.seq_fixed : P.seq_ids[qi];
  if (seq < 0 || seq >= P.s_max) {  // the same for the whole block
    if (hs == 0 && lane == 0) set_dev_error(P.err, ER_EINVAL);
    return;
  }
  const int32_t pos0 = P.meta[seq * 4 + 0];
  const int32_t pend0 = P.meta[seq * 4 + 1];
  const int32_t t = pos0 + (P.prefill ? qi : 0);
  if (threadIdx.x < 32) s_cs[lane] = rope_cs_lane(t, lane);
  __syncthreads();
  // launched behind the scorer / the projection GEMM: the angles above used only
  // metadata; the projections and the partial scores come from them
  grid_dep_wait();
  const int p_idx = pend0 + (P.prefill ? qi : 0);
  const bool state_ok = p_idx >= 0 && p_idx < PEND && t >= 0;
  if (!state_ok && hs == 40 && lane == 0) set_dev_error(P.err, ER_ECAPACITY);

  int col;
  const uint16_t* gain = nullptr;
  if (hs < 16) { col = OFF_Q_SWA + hs * D; gain = P.gq_swa; }
  else if (hs < 20) { col = OFF_K_SWA + (hs - 16) * D; gain = P.gk_swa; }
  else if (hs < 24) { col = OFF_V_SWA + (hs - 20) * D; }
  else if (hs < 40) { col = OFF_Q_RMA + (hs - 24) * D; gain = P.gq_rma; }
  else if (hs < 44) { col = OFF_K_RMA + (hs - 40) * D; gain = P.gk_rma; }
  else { col = OFF_V_RMA + (hs - 44) * D; }

  float v[8];
  if (P.proj_f32) {
    // FP32 sums of the fused GEMM, rounded to BF16 as a BF16-output GEMM would
    const float4* src = reinterpret_cast<const float4*>(P.proj_f32 + (size_t)qi * QKVS + col) +
                        lane * 2;
    const float4 a = src[0], b = src[1];
    v[0] = bf1(f2bf(a.x)); v[1] = bf1(f2bf(a.y)); v[2] = bf1(f2bf(a.z)); v[3] = bf1(f2bf(a.w));
    v[4] = bf1(f2bf(b.x)); v[5] = bf1(f2bf(b.y)); v[6] = bf1(f2bf(b.z)); v[7] = bf1(f2bf(b.w));
  } else {
    load8(P.proj + (size_t)qi * QKV + col + lane * 8, v);
  }
  if (gain) norm_rope_lane_cs(v, gain, s_cs, lane);

  uint16_t* dst = nullptr;
  if (hs < 16) {
    dst = P.q_swa + ((size_t)qi * NH + hs) * D;
  } else if (hs < 24) {
    const int g = (hs < 20) ? hs - 16 : hs - 20;
    const bool is_k = hs < 20;
    if (P.prefill) {
      dst = (is_k ? P.chunk_k : P.chunk_v) + ((size_t)g * P.nq + qi) * D;
    } else {
      if (t < 0) return;
      const size_t row = grp(seq, P.layer, g, P.L) * WIN + (size_t)(t % WIN);
      dst = (is_k ? P.win_k : P.win_v) + row * D;
    }
  } else if (hs < 40) {
    dst = P.q_rma + ((size_t)qi * NH + (hs - 24)) * D;
  } else {
    if (!state_ok) return;
    const int g = (hs < 44) ? hs - 40 : hs - 44;
    const size_t gi = grp(seq, P.layer, g, P.L);
    dst = ((hs < 44) ? P.pend_k : P.pend_v) + (gi * PEND + p_idx) * D;
    if (hs < 44) {
      float sc = 0.f;
      if (P.proj_f32) {
        // the score of group g from the fused GEMM: h_j = hi_j + mid_j + lo_j (the
        // three W1-term sums, smallest first), s_g = sum_j W2[g][j] SiLU(h_j);
        // lane covers j = 8 lane .. 8 lane + 7, then a fixed-order warp sum
        const float4* hrow =
            reinterpret_cast<const float4*>(P.proj_f32 + (size_t)qi * QKVS + QKV) + lane * 2;
        const float4* w2g = reinterpret_cast<const float4*>(P.w2 + g * 256) + lane * 2;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float4 hi = hrow[e], mid = hrow[64 + e], lo = hrow[128 + e], w2 = w2g[e];
          const float h0 = (lo.x + mid.x) + hi.x, h1 = (lo.y + mid.y) + hi.y;
          const float h2 = (lo.z + mid.z) + hi.z, h3 = (lo.w + mid.w) + hi.w;
          sc += w2.x * (h0 / (1.0f + expf(-h0))) + w2.y * (h1 / (1.0f + expf(-h1))) +
                w2.z * (h2 / (1.0f + expf(-h2))) + w2.w * (h3 / (1.0f + expf(-h3)));
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
      } else if (lane == 0) {
        // the separate scorer: its 4 quarter partials added in order
#pragma unroll
        for (int q = 0; q < 4; ++q) sc += P.s_part[((size_t)q * P.nq + qi) * NG + g];
      }
      if (lane == 0) {
        P.pend_score[gi * PEND + p_idx] = sc;
        P.pend_pos[gi * PEND + p_idx] = t;
      }
    }
  }
  store8(dst + lane * 8, v);
}

// Grid rows 0-2 hold the SWA head slots (q, k, v), rows 3-5 the RMA ones
// (q, k and v with the pending append); with the RMA switched off only the
// first three run.
int launch_post_proj(const PostParams& P, bool rma_off, cudaStream_t st) {
  if (P.nq <= 0) return ER_OK;
  // a programmatic launch (see grid_dep_wait above)
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.nq, rma_off ? 3 : 6);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k_post_proj, P) != cudaSuccess) return ER_ECUDA;
  count_launches(1);
  return launch_status();
}

}  // namespace er

using namespace er;

extern "C" int er_qk_norm_rope(const er_bf16* x, er_bf16* y, int64_t n_rows, const er_bf16* gain,
                               const int32_t* pos, er_stream_t stream) {
  if (n_rows < 0 || (n_rows > 0 && (!x || !y || !gain || !pos))) return ER_EINVAL;
  if (n_rows == 0) return ER_OK;
  if (!aligned16(x) || !aligned16(y) || !aligned16(gain)) return ER_EINVAL;
  const int64_t blocks = (n_rows + 7) / 8;
  if (blocks > 0x7FFFFFFF) return ER_EINVAL;
  k_norm_rope<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(x, y, n_rows, gain, pos);
  count_launches(1);
  return launch_status();
}
