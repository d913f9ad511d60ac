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
// rotation angle pos * 1e7^(-2i/64) is formed and reduced (to [-1/2, 1/2] turn)
// in float64 so that positions up to 2^18 keep full angle accuracy (once per
// token in the layer kernel, shared by its head vectors); the rotation itself
// is fp32.
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

// Turns per position of rotary frequency i: 1e7^(-2i/64) / (2 pi), i = 0..31,
// each the float64 nearest to the real value (printed to 17 digits).
__device__ const double kTurnsPerPos[32] = {
    0.15915494309189535, 0.09617675759898782,
    0.058119267441876246, 0.03512126351841045,
    0.02122365276477766, 0.012825376753422709,
    0.0077503288755374055, 0.004683495762645621,
    0.00283021958306234, 0.0017102914776258452,
    0.0010335229661843405, 0.0006245541976934049,
    0.00037741584717419774, 0.00022807103406603446,
    0.00013782250260398286, 8.32856408171725e-05,
    5.0329212104487035e-05, 3.0413761198270857e-05,
    1.8378926105679668e-05, 1.1106318702115607e-05,
    6.711508300522725e-06, 4.055740239059148e-06,
    2.450869186206985e-06, 1.4810514021707515e-06,
    8.949940160889103e-07, 5.408416532072578e-07,
    3.2682865872357e-07, 1.9750137869302395e-07,
    1.1934937021124886e-07, 7.212239359585222e-08,
    4.358330210530733e-08, 2.6337232136895232e-08,
};

// cos/sin of pos * 1e7^(-2i/64) for i = lane (0..31).  The angle is formed in
// turns in float64 and reduced there to [-1/2, 1/2] turn (for pos < 2^18 the
// product is within ~1e-11 turn), so the float64 sincospi that evaluates it
// never needs a large-argument reduction; the results are rounded to float.
__device__ __forceinline__ float2 rope_cs_lane(int32_t pos, int lane) {
  const double turns = (double)pos * kTurnsPerPos[lane];
  const double red = turns - rint(turns);
  double sn, cs;
  sincospi(2.0 * red, &sn, &cs);
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


// Grid (nq, 6) x 256 threads: warp slot hs = 8 blockIdx.y + warp covers, per
// token, q_swa 0..15 | k_swa 16..19 | v_swa 20..23 | q_rma 24..39 | k_rma 40..43
// | v_rma 44..47 (blockIdx.y < 3 only with the RMA off).  A one-block-per-token
// layout with six rows per warp was measured slower (its rows' norm/RoPE chains
// run in series, at half the resident warps).
namespace {

// The retention score of token qi for group g (warp-wide; lane 0's value is
// the one stored).  It needs no metadata, so k_post_proj forms it before its
// barrier, beside the metadata loads.
__device__ __forceinline__ float score_of(const PostParams& P, int qi, int g, int lane) {
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
  return sc;
}

// One head row: norm + RoPE where it has a gain, then its destination (sc: the
// group's score, for the k_rma rows).
__device__ __forceinline__ void post_row(const PostParams& P, int hs, int lane, int qi, int seq,
                                         int32_t t, int p_idx, bool state_ok,
                                         const float2* s_cs, float v[8], float sc) {
  const uint16_t* gain = nullptr;
  if (hs < 16) gain = P.gq_swa;
  else if (hs < 20) gain = P.gk_swa;
  else if (hs >= 24 && hs < 40) gain = P.gq_rma;
  else if (hs >= 40 && hs < 44) gain = P.gk_rma;
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
    // the pending record's home: its slot of the pending block, or, in the pooled
    // layout, the pool slot the group's slot list names for it
    size_t rec = gi * PEND + p_idx;
    if (P.pool) {
      const int slot = P.pend_pos[gi * PEND + p_idx];
      if (slot < 0 || slot >= POOL) {
        if (lane == 0) set_dev_error(P.err, ER_ECAPACITY);
        return;
      }
      rec = gi * POOL + slot;
    }
    dst = ((hs < 44) ? (P.pool ? P.bank_k : P.pend_k) : (P.pool ? P.bank_v : P.pend_v)) +
          rec * D;
    if (hs < 44) {
      if (lane == 0) {
        if (P.pool) {
          P.bank_score[rec] = sc;
          P.bank_pos[rec] = t;
        } else {
          P.pend_score[rec] = sc;
          P.pend_pos[rec] = t;
        }
      }
    }
  }
  store8(dst + lane * 8, v);
}

// Column of head row hs inside a projection row.
__device__ __forceinline__ int row_col(int hs) {
  if (hs < 16) return OFF_Q_SWA + hs * D;
  if (hs < 20) return OFF_K_SWA + (hs - 16) * D;
  if (hs < 24) return OFF_V_SWA + (hs - 20) * D;
  if (hs < 40) return OFF_Q_RMA + (hs - 24) * D;
  if (hs < 44) return OFF_K_RMA + (hs - 40) * D;
  return OFF_V_RMA + (hs - 44) * D;
}

}  // namespace

__global__ void __launch_bounds__(256, 8) k_post_proj(PostParams P) {
  __shared__ float2 s_cs[32];  // the rotation of this token's position
  __shared__ int s_tok[4];     // seq, t, p_idx, valid
  grid_dep_trigger();  // a prefill read may set itself up meanwhile (it waits for us)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int hs = blockIdx.y * 8 + warp;
  const int qi = blockIdx.x;
  // the read that follows takes its work units from this counter; it waits for
  // this kernel to complete before the first one
  if (P.sched_reset && qi == 0 && hs == 0 && lane == 0) *P.sched_reset = 0;
  if (warp == 0) {
    // metadata only (written before the kernel this one is launched behind)
    const int seq = P.prefill ? P.seq_fixed : P.seq_ids[qi];
    const bool valid = seq >= 0 && seq < P.s_max;
    int32_t t = 0, p_idx = 0;
    if (valid) {
      t = P.meta[seq * 4 + 0] + (P.prefill ? qi : 0);
      p_idx = P.meta[seq * 4 + 1] + (P.prefill ? qi : 0);
    }
    s_cs[lane] = rope_cs_lane(t, lane);
    if (lane == 0) {
      s_tok[0] = seq;
      s_tok[1] = t;
      s_tok[2] = p_idx;
      s_tok[3] = valid ? 1 : 0;
    }
  }
  // launched behind the scorer / the projection GEMM: the projections and the
  // partial scores come from them.  The row is loaded before the barrier so that
  // its latency overlaps warp 0's metadata and rotations.
  grid_dep_wait();
  float v[8];
  const int col = row_col(hs);
  if (P.proj_f32) {
    // FP32 sums of the fused GEMM, rounded to BF16 as a BF16-output GEMM would
    const float4* src =
        reinterpret_cast<const float4*>(P.proj_f32 + (size_t)qi * QKVS + col) + lane * 2;
    const float4 a = src[0], b = src[1];
    v[0] = bf1(f2bf(a.x)); v[1] = bf1(f2bf(a.y)); v[2] = bf1(f2bf(a.z)); v[3] = bf1(f2bf(a.w));
    v[4] = bf1(f2bf(b.x)); v[5] = bf1(f2bf(b.y)); v[6] = bf1(f2bf(b.z)); v[7] = bf1(f2bf(b.w));
  } else {
    load8(P.proj + (size_t)qi * QKV + col + lane * 8, v);
  }
  // the k_rma rows' score (no metadata needed)
  const float sc = (hs >= 40 && hs < 44) ? score_of(P, qi, hs - 40, lane) : 0.f;
  __syncthreads();
  if (!s_tok[3]) {  // the same for the whole block
    if (hs == 0 && lane == 0) set_dev_error(P.err, ER_EINVAL);
    return;
  }
  const int seq = s_tok[0];
  const int32_t t = s_tok[1];
  const int p_idx = s_tok[2];
  const bool state_ok = p_idx >= 0 && p_idx < PEND && t >= 0;
  if (!state_ok && hs == 40 && lane == 0) set_dev_error(P.err, ER_ECAPACITY);
  post_row(P, hs, lane, qi, seq, t, p_idx, state_ok, s_cs, v, sc);
}

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
