// attend.cu — a5, the two softmax reads of an SWA∥RMA layer.
//
// EdgeRock-4B 开源：72 MiB 固定 KV, §架构：递归、局部窗口与记忆锚点三件套: 16 query
// heads read 4 KV groups (head h reads group h/4), head dim 256; the 1024-
// position window runs in parallel with the anchor bank.  Reading fixed for
// this library: the RMA read is its own softmax over committed + pending
// records, with its own q, added to the SWA output before o_proj.
//
// Work item = (query, KV group, branch, split).  A branch's rows are one to
// three contiguous ranges of 512-byte K rows and V rows (window ring pieces,
// the chunk's own rows in prefill, bank, pending); they stream through shared
// memory in 64-row tiles.
//
// Persistent kernel, one 288-thread CTA per SM:
//   warp 8 (producer): lane 0 walks the CTA's items and issues one bulk copy
//     (cp.async.bulk, the TMA engine, no tensor map, no multicast) for the K
//     rows and one for the V rows of each tile into a 3-stage ring, with
//     completion counted as transaction bytes on the stage's mbarrier;
//   warps 0..7 (consumers): each takes 8 rows of every tile.  K·q for the
//     group's 4 heads uses packed FP32 FMA (FFMA2) with the logits reduced by
//     a 5-step transpose butterfly in which lane L ends with (row L/4, head
//     L%4); lane-dependent XOR indexing of rows and heads removes every select
//     from the butterfly.  Online softmax in base 2 (q pre-scaled by
//     log2(e)/16), P·V again with FFMA2.  At the item's last tile the 8 warps
//     merge through shared memory and write one partial (m, l, o).
// A second kernel merges the splits of both branches: o = o_swa + o_rma.
// Every wait is bounded (≈2 s) and records ER_ETIMEOUT instead of hanging.
#include <math.h>

#include "common.cuh"
#include "params.cuh"

namespace er {

bool profile_begin(cudaStream_t st, std::pair<cudaEvent_t, cudaEvent_t>* ev);
void profile_end(cudaStream_t st, std::pair<cudaEvent_t, cudaEvent_t> ev);

namespace {

constexpr int TR = 64;        // rows per tile
constexpr int NCW = 8;        // consumer warps (8 rows each)
constexpr int STAGES = 3;
constexpr int NTHREADS = (NCW + 1) * 32;
constexpr float kLog2eOver16 = 1.4426950408889634f / 16.0f;
constexpr int F_FIRST = 1, F_LAST = 2;

struct TileDesc {
  int rows;
  int flags;
};

struct __align__(128) AttnSmem {
  uint16_t k[STAGES][TR * D];
  uint16_t v[STAGES][TR * D];
  float merge_acc[NCW][HPG][D];
  float merge_ml[NCW][HPG][2];
  float2 pbuf[NCW][8][HPG];
  TileDesc desc[STAGES];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t merge_bar;
  volatile int abort_flag;
};

}  // namespace


namespace {

struct Range {
  const uint16_t* k;
  const uint16_t* v;
  int rows;
};

// Row ranges of one item; returns the number of ranges (0..3).
__device__ int item_ranges(const AttendParams& P, int qi, int g, int br, Range r[3]) {
  const int seq = P.prefill ? P.seq_fixed : P.seq_ids[qi];
  if (seq < 0 || seq >= P.s_max) return 0;
  const int32_t pos0 = P.meta[seq * 4 + 0];
  const int pend = P.meta[seq * 4 + 1];
  const int bank = min(max(P.meta[seq * 4 + 2], 0), BANK);
  const size_t gi = grp(seq, P.layer, g, P.L);
  int n = 0;
  if (br == 0) {
    const uint16_t* wk = P.win_k + gi * WIN * D;
    const uint16_t* wv = P.win_v + gi * WIN * D;
    if (!P.prefill) {
      // window positions [t-1023, t], t = pos0, all already in the ring
      const int nwin = min(pos0 + 1, WIN);
      r[n++] = Range{wk, wv, nwin};
    } else {
      const int t = pos0 + qi;
      const int lo = max(0, t - (WIN - 1));
      const int count = pos0 - lo;  // old ring positions lo..pos0-1
      if (count > 0) {
        const int s0 = lo % WIN;
        const int n1 = min(count, WIN - s0);
        r[n++] = Range{wk + (size_t)s0 * D, wv + (size_t)s0 * D, n1};
        if (count > n1) r[n++] = Range{wk, wv, count - n1};
      }
      r[n++] = Range{P.chunk_k + (size_t)g * P.nq * D, P.chunk_v + (size_t)g * P.nq * D, qi + 1};
    }
  } else {
    if (bank > 0)
      r[n++] = Range{P.bank_k + gi * BANK * D, P.bank_v + gi * BANK * D, bank};
    const int np = min(pend + (P.prefill ? qi : 0) + 1, PEND);
    if (np > 0) r[n++] = Range{P.pend_k + gi * PEND * D, P.pend_v + gi * PEND * D, np};
  }
  return n;
}

__device__ __forceinline__ void item_coords(const AttendParams& P, int item, int* qi, int* g,
                                            int* br, int* split) {
  *split = item % P.splits;
  int rest = item / P.splits;
  *br = rest & 1;
  rest >>= 1;
  *g = rest & 3;
  *qi = rest >> 2;
}

__global__ void __launch_bounds__(NTHREADS, 1) k_attend(AttendParams P) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  AttnSmem& S = *reinterpret_cast<AttnSmem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = P.nq * NG * 2 * P.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], NCW);
    }
    mbar_init(&S.merge_bar, NCW);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NCW) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    uint32_t tc = 0;
    for (int item = blockIdx.x; item < n_items && !S.abort_flag; item += gridDim.x) {
      int qi, g, br, split;
      item_coords(P, item, &qi, &g, &br, &split);
      Range r[3];
      const int nr = item_ranges(P, qi, g, br, r);
      int nt = 0;
      for (int i = 0; i < nr; ++i) nt += (r[i].rows + TR - 1) / TR;
      const int t0 = (int)((long)split * nt / P.splits);
      const int t1 = (int)((long)(split + 1) * nt / P.splits);
      int ri = 0, tile_in_range = 0, tix = 0;
      // advance to tile t0
      while (ri < nr && tix + (r[ri].rows + TR - 1) / TR <= t0) {
        tix += (r[ri].rows + TR - 1) / TR;
        ++ri;
      }
      tile_in_range = t0 - tix;
      const int emit = (t1 > t0) ? (t1 - t0) : 1;  // an empty item still sends one tile
      for (int e = 0; e < emit; ++e) {
        const int stage = tc % STAGES;
        const uint32_t phase = (tc / STAGES) & 1;
        if (!mbar_wait(&S.empty[stage], phase ^ 1, P.err)) {
          S.abort_flag = 1;
          break;
        }
        int rows = 0;
        const uint16_t *ks = nullptr, *vs = nullptr;
        if (t1 > t0) {
          const int off = tile_in_range * TR;
          rows = min(TR, r[ri].rows - off);
          ks = r[ri].k + (size_t)off * D;
          vs = r[ri].v + (size_t)off * D;
          if (++tile_in_range * TR >= r[ri].rows) {
            ++ri;
            tile_in_range = 0;
          }
        }
        S.desc[stage].rows = rows;
        S.desc[stage].flags = (e == 0 ? F_FIRST : 0) | (e == emit - 1 ? F_LAST : 0);
        if (rows > 0) {
          const uint32_t bytes = (uint32_t)rows * ROW_BYTES;
          mbar_arrive_expect_tx(&S.full[stage], 2 * bytes);
          bulk_g2s(S.k[stage], ks, bytes, &S.full[stage]);
          bulk_g2s(S.v[stage], vs, bytes, &S.full[stage]);
        } else {
          mbar_arrive(&S.full[stage]);
        }
        ++tc;
      }
    }
    // drain: the last tile of each stage must have landed before exit
    for (uint32_t i = (tc > STAGES ? tc - STAGES : 0); i < tc; ++i)
      mbar_wait(&S.full[i % STAGES], (i / STAGES) & 1, P.err);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int rx = (lane >> 2) & 7;  // row XOR of this lane
  const int hx = lane & 3;         // head XOR of this lane
  const int lr = lane >> 2;        // logit row held after the butterfly
  uint32_t tc = 0;
  uint32_t mphase = 0;
  bool aborted = false;

  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    int qi, g, br, split;
    item_coords(P, item, &qi, &g, &br, &split);
    // q for the group's 4 heads: dims 8*lane..8*lane+7, heads XOR-permuted, duplicated pairs
    float2 qd[HPG][8];
    {
      const uint16_t* qb = (br ? P.q_rma : P.q_swa) + ((size_t)qi * NH + g * HPG) * D + lane * 8;
#pragma unroll
      for (int h = 0; h < HPG; ++h) {
        const uint4 w = *reinterpret_cast<const uint4*>(qb + (size_t)(h ^ hx) * D);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = bf_lo(ws[e]) * kLog2eOver16, b = bf_hi(ws[e]) * kLog2eOver16;
          qd[h][2 * e] = make_float2(a, a);
          qd[h][2 * e + 1] = make_float2(b, b);
        }
      }
    }
    float m_run = -INFINITY, l_run = 0.f;
    float2 accv[HPG][4];
#pragma unroll
    for (int h = 0; h < HPG; ++h)
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) accv[h][wd] = make_float2(0.f, 0.f);

    while (true) {
      const int stage = tc % STAGES;
      const uint32_t phase = (tc / STAGES) & 1;
      if (!aborted && !mbar_wait(&S.full[stage], phase, P.err)) {
        aborted = true;
        S.abort_flag = 1;
      }
      const TileDesc d = S.desc[stage];
      const int nrows = aborted ? 0 : min(8, d.rows - 8 * warp);
      if (nrows > 0) {
        // ---- K phase: logits of 8 rows x 4 heads
        const char* kt = reinterpret_cast<const char*>(S.k[stage]) + (8 * warp) * ROW_BYTES +
                         lane * 16;
        float2 acc[4][HPG];
#pragma unroll
        for (int ip = 0; ip < 4; ++ip)
#pragma unroll
          for (int h = 0; h < HPG; ++h) acc[ip][h] = make_float2(0.f, 0.f);
#pragma unroll
        for (int ip = 0; ip < 4; ++ip) {
          const uint4 ka = lds128(kt + ((2 * ip) ^ rx) * ROW_BYTES);
          const uint4 kb = lds128(kt + ((2 * ip + 1) ^ rx) * ROW_BYTES);
          const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w};
          const uint32_t wb[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
          for (int wd = 0; wd < 4; ++wd) {
            const float2 lo = make_float2(bf_lo(wa[wd]), bf_lo(wb[wd]));
            const float2 hi = make_float2(bf_hi(wa[wd]), bf_hi(wb[wd]));
#pragma unroll
            for (int h = 0; h < HPG; ++h) {
              acc[ip][h] = __ffma2_rn(qd[h][2 * wd], lo, acc[ip][h]);
              acc[ip][h] = __ffma2_rn(qd[h][2 * wd + 1], hi, acc[ip][h]);
            }
          }
        }
        // transpose butterfly: lane L ends with (row L>>2, head L&3)
#pragma unroll
        for (int ip = 0; ip < 2; ++ip)
#pragma unroll
          for (int h = 0; h < HPG; ++h) {
            acc[ip][h].x += __shfl_xor_sync(0xffffffffu, acc[ip + 2][h].x, 16);
            acc[ip][h].y += __shfl_xor_sync(0xffffffffu, acc[ip + 2][h].y, 16);
          }
#pragma unroll
        for (int h = 0; h < HPG; ++h) {
          acc[0][h].x += __shfl_xor_sync(0xffffffffu, acc[1][h].x, 8);
          acc[0][h].y += __shfl_xor_sync(0xffffffffu, acc[1][h].y, 8);
        }
        float rr[HPG];
#pragma unroll
        for (int h = 0; h < HPG; ++h)
          rr[h] = acc[0][h].x + __shfl_xor_sync(0xffffffffu, acc[0][h].y, 4);
        rr[0] += __shfl_xor_sync(0xffffffffu, rr[2], 2);
        rr[1] += __shfl_xor_sync(0xffffffffu, rr[3], 2);
        rr[0] += __shfl_xor_sync(0xffffffffu, rr[1], 1);

        // ---- online softmax (base 2) for head hx
        const float s = (lr < nrows) ? rr[0] : -INFINITY;
        float mt = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, 4));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
        const float m_new = fmaxf(m_run, mt);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = exp2f(m_run - m_use);
        const float pr = exp2f(s - m_use);
        l_run = l_run * alpha + pr;
        m_run = m_new;
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
          for (int h = 0; h < HPG; ++h) {
            const float ah = __shfl_sync(0xffffffffu, alpha, h);
            const float2 a2 = make_float2(ah, ah);
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) accv[h][wd] = __fmul2_rn(accv[h][wd], a2);
          }
        }
        S.pbuf[warp][lr][hx] = make_float2(pr, pr);
        __syncwarp();

        // ---- V phase
        const char* vt = reinterpret_cast<const char*>(S.v[stage]) + (8 * warp) * ROW_BYTES +
                         lane * 16;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          if (r < nrows) {
            const uint4 vv = lds128(vt + r * ROW_BYTES);
            const float4 pa = lds128f(&S.pbuf[warp][r][0]);
            const float4 pb = lds128f(&S.pbuf[warp][r][2]);
            const float2 p2[HPG] = {make_float2(pa.x, pa.y), make_float2(pa.z, pa.w),
                                    make_float2(pb.x, pb.y), make_float2(pb.z, pb.w)};
            const uint32_t ws[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              const float2 val = make_float2(bf_lo(ws[wd]), bf_hi(ws[wd]));
#pragma unroll
              for (int h = 0; h < HPG; ++h) accv[h][wd] = __ffma2_rn(p2[h], val, accv[h][wd]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[stage]);
      ++tc;
      if (aborted || (d.flags & F_LAST)) break;
    }

    // ---- merge the 8 warps' partials of this item
    float lt = l_run;
    lt += __shfl_xor_sync(0xffffffffu, lt, 4);
    lt += __shfl_xor_sync(0xffffffffu, lt, 8);
    lt += __shfl_xor_sync(0xffffffffu, lt, 16);
    if (lane < HPG) {
      S.merge_ml[warp][lane][0] = m_run;
      S.merge_ml[warp][lane][1] = lt;
    }
#pragma unroll
    for (int h = 0; h < HPG; ++h) {
      float4* dst = reinterpret_cast<float4*>(&S.merge_acc[warp][h][lane * 8]);
      dst[0] = make_float4(accv[h][0].x, accv[h][0].y, accv[h][1].x, accv[h][1].y);
      dst[1] = make_float4(accv[h][2].x, accv[h][2].y, accv[h][3].x, accv[h][3].y);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.merge_bar);
    if (!mbar_wait(&S.merge_bar, mphase, P.err)) aborted = true;
    mphase ^= 1;
    {
      const int ct = warp * 32 + lane;
      const int h = ct >> 6, d0 = (ct & 63) * 4;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, S.merge_ml[w][h][0]);
      float Ls = 0.f;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < NCW; ++w) {
          const float f = exp2f(S.merge_ml[w][h][0] - M);
          Ls += S.merge_ml[w][h][1] * f;
          const float4 a = *reinterpret_cast<const float4*>(&S.merge_acc[w][h][d0]);
          o.x += a.x * f; o.y += a.y * f; o.z += a.z * f; o.w += a.w * f;
        }
      }
      *reinterpret_cast<float4*>(P.part_o + ((size_t)item * HPG + h) * D + d0) = o;
      if (d0 == 0) {
        P.part_ml[((size_t)item * HPG + h) * 2 + 0] = M;
        P.part_ml[((size_t)item * HPG + h) * 2 + 1] = Ls;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.merge_bar);
    if (!mbar_wait(&S.merge_bar, mphase, P.err)) aborted = true;
    mphase ^= 1;
    if (aborted) break;
  }
}

// Merge the splits of both branches for (query, head).
//  mode 0: o_swa, o_rma FP32 [nq][16][256]; mode 1: o_sum BF16 [nq][4096] = bf16(o_swa + o_rma)
__global__ void __launch_bounds__(256) k_attend_merge(const float* __restrict__ part_o,
                                                      const float* __restrict__ part_ml,
                                                      int splits, float* o_swa, float* o_rma,
                                                      uint16_t* o_sum) {
  const int qi = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
  const int g = h / HPG, hh = h % HPG;
  float ob[2];
#pragma unroll
  for (int br = 0; br < 2; ++br) {
    const size_t base = (((size_t)qi * NG + g) * 2 + br) * splits;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, part_ml[((base + s) * HPG + hh) * 2]);
    float Ls = 0.f, o = 0.f;
    if (M != -INFINITY) {
      for (int s = 0; s < splits; ++s) {
        const float m = part_ml[((base + s) * HPG + hh) * 2];
        const float f = exp2f(m - M);
        Ls += part_ml[((base + s) * HPG + hh) * 2 + 1] * f;
        o += part_o[((base + s) * HPG + hh) * D + d] * f;
      }
    }
    ob[br] = Ls > 0.f ? o / Ls : 0.f;
  }
  if (o_sum) {
    o_sum[(size_t)qi * OIN + h * D + d] = f2bf(ob[0] + ob[1]);
  } else {
    o_swa[((size_t)qi * NH + h) * D + d] = ob[0];
    o_rma[((size_t)qi * NH + h) * D + d] = ob[1];
  }
}

}  // namespace

// Splits per branch so that at least ~2 items per SM exist (deterministic in nq).
int attend_splits(int nq) {
  const int items = nq * NG * 2;
  int s = 1;
  while (items * s < 296 && s < 16) s <<= 1;
  return s;
}

size_t attend_part_floats(int nq) {
  return (size_t)nq * NG * 2 * attend_splits(nq) * HPG * D;
}
size_t attend_ml_floats(int nq) { return (size_t)nq * NG * 2 * attend_splits(nq) * HPG * 2; }

int launch_attend(const AttendParams& P0, float* o_swa, float* o_rma, uint16_t* o_sum,
                  cudaStream_t st) {
  if (P0.nq <= 0) return ER_OK;
  AttendParams P = P0;
  P.splits = attend_splits(P.nq);
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(k_attend, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(AttnSmem)) != cudaSuccess)
      return ER_ECUDA;
    attr_done[dev] = true;
  }
  const int n_items = P.nq * NG * 2 * P.splits;
  const int grid = min(n_items, num_sms());
  std::pair<cudaEvent_t, cudaEvent_t> ev;
  const bool timed = profile_begin(st, &ev);
  k_attend<<<grid, NTHREADS, sizeof(AttnSmem), st>>>(P);
  if (timed) profile_end(st, ev);
  count_launches(1);
  int rc = launch_status();
  if (rc != ER_OK) return rc;
  k_attend_merge<<<dim3(P.nq, NH), 256, 0, st>>>(P.part_o, P.part_ml, P.splits, o_swa, o_rma,
                                                  o_sum);
  count_launches(1);
  return launch_status();
}

}  // namespace er

using namespace er;

extern "C" {

size_t er_attend_workspace_bytes(int32_t B) {
  if (B < 0) return 0;
  Carver c(nullptr);
  c.take<float>(attend_part_floats(B));
  c.take<float>(attend_ml_floats(B));
  return c.used();
}

int er_swa_rma_attend(const er_state* st, int32_t layer, const int32_t* seq_ids, int32_t B,
                      const er_bf16* q_swa, const er_bf16* q_rma, float* o_swa, float* o_rma,
                      void* ws, size_t ws_bytes, er_stream_t stream) {
  if (!st || B < 0 || layer < 0 || layer >= st->n_layers) return ER_EINVAL;
  if (B == 0) return ER_OK;
  if (!seq_ids || !q_swa || !q_rma || !o_swa || !o_rma || !ws) return ER_EINVAL;
  if (ws_bytes < er_attend_workspace_bytes(B)) return ER_ECAPACITY;
  Carver c(ws);
  AttendParams P{};
  P.win_k = st->win_k; P.win_v = st->win_v;
  P.bank_k = st->bank_k; P.bank_v = st->bank_v;
  P.pend_k = st->pend_k; P.pend_v = st->pend_v;
  P.meta = st->meta; P.seq_ids = seq_ids;
  P.s_max = st->s_max; P.L = st->n_layers; P.layer = layer;
  P.q_swa = q_swa; P.q_rma = q_rma; P.nq = B; P.prefill = 0;
  P.part_o = c.take<float>(attend_part_floats(B));
  P.part_ml = c.take<float>(attend_ml_floats(B));
  P.err = st->dev_error;
  return launch_attend(P, o_swa, o_rma, nullptr, (cudaStream_t)stream);
}

}  // extern "C"
