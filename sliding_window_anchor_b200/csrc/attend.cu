// attend.cu — a5, the two softmax reads of an SWA∥RMA layer.
//
// EdgeRock-4B 开源：72 MiB 固定 KV, §架构：递归、局部窗口与记忆锚点三件套: 16 query
// heads read 4 KV groups (head h reads group h/4), head dim 256; the 1024-
// position window runs in parallel with the anchor bank.  Reading fixed for
// this library: the RMA read is its own softmax over committed + pending
// records, with its own q, added to the SWA output before o_proj.
//
// Work item = (query, KV group, branch, split).  A branch's rows are one or two
// contiguous ranges of 512-byte K rows and V rows (the window ring; bank and
// pending); they stream through shared memory in 64-row tiles.  (A prefill
// chunk's reads run in prefill_attn.cu.)
//
// Persistent kernel, one 160-thread CTA per SM:
//   warp 4 (producer): lane 0 takes the CTA's items from a work counter; for
//     each tile it arms the
//     stage's mbarrier with the transaction bytes and issues TMA tensor copies
//     (cp.async.bulk.tensor.2d, into this CTA only) of four 64x64 boxes of K rows and
//     four of V rows, 128-byte swizzled, plus the item's 4 query heads (one
//     plain bulk copy) with its first tile; 3-stage ring.
//   warps 0..3 (consumers): each takes 16 rows (keys) of every tile.  The
//     group's 4 heads share every K and V row, so the two contractions are
//     small dense matrix products and run on the tensor cores with
//     mma.m16n8k16 (BF16 in, FP32 accumulate), fragments read by ldmatrix from
//     the swizzled tiles without bank conflicts:
//       Sᵀ[16 keys x 8] = K[16 x 256] · Qᵀ  (heads 4..7 are zero padding)
//       Oᵀ[256 x 8]    += Vᵀ[256 x 16 keys] · Pᵀ[16 keys x 8]
//     P = exp2(S·log2e/16 - m) is split into a BF16 high part and a BF16
//     remainder, and both are multiplied (two MMAs), so P·V keeps ~16
//     significant bits instead of BF16's 8.  Online softmax in base 2 with the
//     rescale skipped while the running maximum holds.  At the item's last
//     tile the 4 warps merge through shared memory (their own rows of the
//     tile's K boxes) and write either the final output or one partial
//     (m, l, o) per split.
// Measured on B200 before this design: the same pipeline with CUDA-core FMAs
// reached 80% of the measured copy bandwidth, and 105% with the math removed,
// so the math, not the data path, was the limit.
// Small batches split each branch's rows (up to 16 ways, one item per work
// unit; with no more units than CTAs, CTA i takes unit i and touches no work
// counter), and a second kernel merges the splits of both branches.
// Every wait is bounded (≈2 s) and records ER_ETIMEOUT instead of hanging.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "params.cuh"
#include "tc.cuh"

namespace er {

bool profile_begin(cudaStream_t st, std::pair<cudaEvent_t, cudaEvent_t>* ev);
void profile_end(cudaStream_t st, std::pair<cudaEvent_t, cudaEvent_t> ev);

namespace {

constexpr int TR = 64;                  // rows per tile
constexpr int NCW = 4;                  // consumer warps, 16 rows each
constexpr int STAGES = 3;
constexpr int NTHREADS = (NCW + 1) * 32;
constexpr int BOX = 64 * 128;           // one 64-row x 64-dim box (8 KB, 128 B per row)
constexpr int TILE_BYTES = 4 * BOX;     // a 64-row K (or V) tile: four boxes
constexpr float kLog2eOver16 = 1.4426950408889634f / 16.0f;
constexpr int F_FIRST = 1, F_LAST = 2, F_END = 4;  // F_END: no more work for this CTA
constexpr int kMaxSplits = 16;          // splits of one (query, group, branch) read

struct TileDesc {
  int rows;
  int flags;
  int item;
  int row;  // the tile's first row in its tensor-mapped array
};

struct __align__(1024) AttnSmem {
  unsigned char k[STAGES][TILE_BYTES];  // the item's last K tile doubles as the merge area
  unsigned char v[STAGES][TILE_BYTES];
  uint16_t q[STAGES][HPG * D];         // the item's 4 query heads, sent with its first tile
  uint16_t pt[NCW][2][8][16];          // Pᵀ staging per warp: [hi/lo][head][key]
  float merge_ml[NCW][HPG][2];
  TileDesc desc[STAGES];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t merge_bar;
  volatile int abort_flag;
};

static_assert(sizeof(AttnSmem) + 1024 <= 232448,
              "shared memory above the 227 KB per-block limit");

// Rows [row, row + rows) of one of the tensor-mapped arrays.
struct Range {
  int map;
  int row;
  int rows;
};

// Row ranges of one item; returns the number of ranges (0..2), none empty.
__device__ int item_ranges(const AttendParams& P, int qi, int g, int br, Range r[2]) {
  const int seq = P.seq_ids[qi];
  if (seq < 0 || seq >= P.s_max) return 0;
  const int32_t pos0 = P.meta[seq * 4 + 0];
  const int pend = P.meta[seq * 4 + 1];
  const int bank = min(max(P.meta[seq * 4 + 2], 0), BANK);
  const int gi = (int)grp(seq, P.layer, g, P.L);
  int n = 0;
  if (br == 0) {
    // window positions [t-1023, t], t = pos0, all already in the ring (the
    // softmax does not depend on their order, so the ring is read as stored)
    const int nwin = min(pos0 + 1, WIN);
    if (nwin > 0) r[n++] = Range{TM_WIN, gi * WIN, nwin};
  } else {
    if (P.rma_off) return 0;  // the RMA switched off: an empty read, o_rma = 0
    if (P.pool) {
      // the whole pool of the group; free slots and later records are masked
      r[n++] = Range{TM_BANK, gi * POOL, POOL};
      return n;
    }
    if (bank > 0) r[n++] = Range{TM_BANK, gi * BANK, bank};
    const int np = min(pend + 1, PEND);
    if (np > 0) r[n++] = Range{TM_PEND, gi * PEND, np};
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

struct Tile {
  int map, row;
  int rows, flags, qi, g, br, item;
};

// The tiles of items begin..end-1, each the tiles of its split (or one empty
// tile when the split has no rows).
struct TileIter {
  const AttendParams* P;
  int item, item_end;
  Range r[2];
  int nr, ri, tile_in_range, e, emit, qi, g, br;
  bool has_rows;

  __device__ void init(const AttendParams* p, int begin, int end) {
    P = p;
    item = begin;
    item_end = end;
    start_item();
  }
  __device__ void start_item() {
    if (item >= item_end) return;
    int split;
    item_coords(*P, item, &qi, &g, &br, &split);
    nr = item_ranges(*P, qi, g, br, r);
    int nt = 0;
    for (int i = 0; i < nr; ++i) nt += (r[i].rows + TR - 1) / TR;
    const int t0 = (int)((long)split * nt / P->splits);
    const int t1 = (int)((long)(split + 1) * nt / P->splits);
    ri = 0;
    int tix = 0;
    while (ri < nr && tix + (r[ri].rows + TR - 1) / TR <= t0) {
      tix += (r[ri].rows + TR - 1) / TR;
      ++ri;
    }
    tile_in_range = t0 - tix;
    has_rows = t1 > t0;
    emit = has_rows ? t1 - t0 : 1;
    e = 0;
  }
  __device__ bool next(Tile* t) {
    if (item >= item_end) return false;
    t->item = item;
    t->qi = qi;
    t->g = g;
    t->br = br;
    t->rows = 0;
    t->map = 0;
    t->row = 0;
    if (has_rows) {
      const int off = tile_in_range * TR;
      t->rows = min(TR, r[ri].rows - off);
      t->map = r[ri].map;
      t->row = r[ri].row + off;
      if (++tile_in_range * TR >= r[ri].rows) {
        ++ri;
        tile_in_range = 0;
      }
    }
    t->flags = (e == 0 ? F_FIRST : 0) | (e == emit - 1 ? F_LAST : 0);
    if (++e == emit) {
      ++item;
      start_item();
    }
    return true;
  }
};

// ------------------------------------------------------- tensor-core helpers

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t r[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t r[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D = A·B + D, m16n8k16, BF16 operands, FP32 accumulators.
__device__ __forceinline__ void mma_bf16(float d[4], const uint32_t a[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One 64x64 box of a 2-D tensor map into shared memory (x: dims, y: rows).
// x is a multiple of 64 elements (128 B), as TMA requires.
__device__ __forceinline__ void tma_box(void* dst, const CUtensorMap* map, int x, int y,
                                        uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__global__ void __launch_bounds__(NTHREADS, 1) k_attend(const __grid_constant__ AttendParams P) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the swizzled boxes need 1024-byte aligned destinations
  AttnSmem& S = *reinterpret_cast<AttnSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
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
  // launched behind the kernel that writes q, the window slot and the pending
  // record (norm/RoPE): nothing above touched them
  grid_dep_wait();
  grid_dep_trigger();  // the split merge after this read may set itself up (it waits for us)

  // Work is handed out in units: two consecutive items when unsplit (a (query,
  // group)'s two branch items, read back to back by one CTA, which writes their
  // sum), one item when split (small batches: one or two tiles each, so every
  // SM gets some).  The producer takes the next unit from a counter in global
  // memory (zeroed before the launch) when it has issued the last one, so CTAs
  // that meet short items take more and all finish within about one unit of
  // each other.  Nothing waits on another CTA.
  const int upi = P.splits == 1 ? 2 : 1;
  const int n_units = n_items / upi;

  if (warp == NCW) {
    // ------------------------------------------------------------ producer
    // with no more units than CTAs (small batches) each CTA takes unit blockIdx.x
    // and no other: the counter's round trips stay off the short critical path
    const bool fixed = n_units <= (int)gridDim.x;
    bool first = true;
    auto take_unit = [&]() {
      if (fixed) {
        const int u = first ? (int)blockIdx.x : n_units;
        first = false;
        return u;
      }
      int u = 0;
      if (lane == 0) u = atomicAdd(P.sched, 1);
      u = __shfl_sync(0xffffffffu, u, 0);
      return (u < 0 || u > n_units) ? n_units : u;  // past the end: no more work
    };
    TileIter ld;
    int unit = take_unit();
    ld.init(&P, upi * unit, upi * min(unit + 1, n_units));
    Tile t;
    uint32_t tc = 0;
    while (true) {
      if (!ld.next(&t)) {
        if (unit >= n_units) break;
        unit = take_unit();
        ld.init(&P, upi * unit, upi * min(unit + 1, n_units));
        continue;
      }
      const int stage = tc % STAGES;
      const uint32_t phase = (tc / STAGES) & 1;
      if (lane == 0 && !mbar_wait(&S.empty[stage], phase ^ 1, P.err)) S.abort_flag = 1;
      __syncwarp();
      if (S.abort_flag) break;
      if (lane == 0) {
        const uint32_t qbytes = (t.flags & F_FIRST) ? HPG * ROW_BYTES : 0;
        // whole boxes always land (rows past the range are masked by the consumers,
        // rows past the array are zero-filled by TMA)
        const uint32_t bytes = (t.rows > 0 ? 2u * TILE_BYTES : 0u) + qbytes;
        S.desc[stage].rows = t.rows;
        S.desc[stage].flags = t.flags;
        S.desc[stage].item = t.item;
        S.desc[stage].row = t.row;
        if (bytes) mbar_arrive_expect_tx(&S.full[stage], bytes);
        else mbar_arrive(&S.full[stage]);
        if (qbytes)
          bulk_g2s(S.q[stage], (t.br ? P.q_rma : P.q_swa) + ((size_t)t.qi * NH + t.g * HPG) * D,
                   qbytes, &S.full[stage]);
        if (t.rows > 0) {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            tma_box(S.k[stage] + b * BOX, &P.tmap_k[t.map], 64 * b, t.row, &S.full[stage]);
            tma_box(S.v[stage] + b * BOX, &P.tmap_v[t.map], 64 * b, t.row, &S.full[stage]);
          }
        }
      }
      ++tc;
    }
    if (!S.abort_flag) {
      // the end marker: an empty tile the consumers stop at
      const int stage = tc % STAGES;
      const uint32_t phase = (tc / STAGES) & 1;
      if (lane == 0 && !mbar_wait(&S.empty[stage], phase ^ 1, P.err)) S.abort_flag = 1;
      __syncwarp();
      if (!S.abort_flag) {
        if (lane == 0) {
          S.desc[stage].rows = 0;
          S.desc[stage].flags = F_END;
          S.desc[stage].item = -1;
          mbar_arrive(&S.full[stage]);
        }
        ++tc;
      }
    }
    // drain: the last tile of each stage must have landed before exit
    if (lane == 0)
      for (uint32_t i = (tc > STAGES ? tc - STAGES : 0); i < tc; ++i)
        mbar_wait(&S.full[i % STAGES], (i / STAGES) & 1, P.err);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gq = lane >> 2;   // fragment row group: keys gq, gq+8 / head gq (B operands)
  const int cq = lane & 3;    // fragment column quad: heads 2cq, 2cq+1 / keys 2cq.. (B)
  const bool real_heads = cq < 2;   // lanes holding heads 0..3 of the C fragments
  const int row0 = 16 * warp;       // this warp's 16 rows of a tile
  // ldmatrix rows of this lane: QK reads keys row0 + (lane&7) + 8*((lane>>3)&1) at dim
  // chunk 2kk + (lane>>4); PV reads keys row0 + (lane&7) + 8*(lane>>4) at dim chunk
  // 2mt + ((lane>>3)&1).  In a 128B-swizzled box, 16-byte chunk c of row r sits at
  // chunk position c ^ (r & 7), and r & 7 == lane & 7 here.
  const int sw = lane & 7;
  const uint32_t row_qk = (uint32_t)(row0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * 128u;
  const int chunk_qk = lane >> 4;
  const uint32_t row_pv = (uint32_t)(row0 + (lane & 7) + 8 * (lane >> 4)) * 128u;
  const int chunk_pv = (lane >> 3) & 1;

  uint32_t tc = 0;
  uint32_t mphase = 0;
  bool aborted = false;
  float keep[8];  // normalized SWA output of the pair's first item (direct mode)
#pragma unroll
  for (int i = 0; i < 8; ++i) keep[i] = 0.f;

  int item = 0, qi = 0, g = 0, br = 0;
  int32_t tq = 0;  // pooled layout: the query's position (records after it are masked)
  while (true) {
    bool end = false;
    uint32_t qb[16][2];  // Qᵀ B fragments for the 16 k-steps (heads >= 4 are zero)
    float o[16][4];      // Oᵀ accumulators: dims 16mt + gq (+8) x heads 2cq (+1)
#pragma unroll
    for (int mt = 0; mt < 16; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[mt][i] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};  // heads 2cq, 2cq+1
    float l_run[2] = {0.f, 0.f};              // this lane's partial sums

    int last_stage = 0;
    while (true) {
      const int stage = tc % STAGES;
      const uint32_t phase = (tc / STAGES) & 1;
      if (!aborted && !mbar_wait(&S.full[stage], phase, P.err)) {
        aborted = true;
        S.abort_flag = 1;
      }
      const TileDesc d = S.desc[stage];
      if (!aborted && (d.flags & F_END)) {
        end = true;
        break;
      }
      const int nrows = aborted ? 0 : min(16, d.rows - row0);
      if (!aborted && (d.flags & F_FIRST)) {
        // a new item: its coordinates come with its first tile
        int split;
        item = d.item;
        item_coords(P, item, &qi, &g, &br, &split);
        if (P.pool) {
          const int seq = P.seq_ids[qi];
          tq = (seq >= 0 && seq < P.s_max) ? P.meta[seq * 4 + 0] : -1;
        }
        const uint16_t* q = S.q[stage];
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
          qb[kk][0] = gq < HPG ? *reinterpret_cast<const uint32_t*>(q + gq * D + 16 * kk + 2 * cq)
                               : 0u;
          qb[kk][1] = gq < HPG
                          ? *reinterpret_cast<const uint32_t*>(q + gq * D + 16 * kk + 8 + 2 * cq)
                          : 0u;
        }
      }
      if (nrows > 0) {
        const uint32_t kbase = smem_u32(S.k[stage]);
        const uint32_t vbase = smem_u32(S.v[stage]);
        if (nrows < 16) {
          // rows past the tile's end hold stale bytes: zero this warp's V rows there so
          // that p = 0 times them stays 0 in the tensor-core sum
          for (int r = nrows; r < 16; ++r)  // a whole row: 4 boxes x 8 chunks = 32 lanes
            *reinterpret_cast<uint4*>(S.v[stage] + (lane >> 3) * BOX + (row0 + r) * 128 +
                                      (lane & 7) * 16) = make_uint4(0, 0, 0, 0);
          __syncwarp();
        }
        // ---- Sᵀ = K · Qᵀ over 256 dims (two accumulators to halve the chain)
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 16; kk += 2) {
          uint32_t a[4], a2[4];
          const int c0 = 2 * kk + chunk_qk, c1 = 2 * (kk + 1) + chunk_qk;  // 0..31
          ldsm_x4(kbase + (c0 >> 3) * BOX + row_qk + (((c0 & 7) ^ sw) << 4), a);
          ldsm_x4(kbase + (c1 >> 3) * BOX + row_qk + (((c1 & 7) ^ sw) << 4), a2);
          mma_bf16(sa, a, qb[kk][0], qb[kk][1]);
          mma_bf16(sb, a2, qb[kk + 1][0], qb[kk + 1][1]);
        }
        // s[i]: keys gq (i<2) / gq+8 (i>=2), heads 2cq + (i&1); base-2 logits
        float s[4];
        bool vis[2] = {gq < nrows, gq + 8 < nrows};
        if (P.pool && br) {
          // pool slots: a free slot, or a record after the query, is not read
          const int32_t* pp = P.bank_pos + d.row + row0;
          vis[0] = vis[0] && pp[gq] <= tq;
          vis[1] = vis[1] && pp[gq + 8] <= tq;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
          s[i] = vis[i >> 1] ? (sa[i] + sb[i]) * kLog2eOver16 : -INFINITY;
        // ---- online softmax for this lane's two heads (8 lanes share each pair)
        float alpha[2], pv[4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float mt = fmaxf(s[j], s[j + 2]);
          mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
          mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
          mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
          const float m_new = fmaxf(m_run[j], mt);
          const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
          alpha[j] = exp2f(m_run[j] - m_use);
          pv[j] = exp2f(s[j] - m_use);
          pv[j + 2] = exp2f(s[j + 2] - m_use);
          l_run[j] = l_run[j] * alpha[j] + pv[j] + pv[j + 2];
          m_run[j] = m_new;
        }
        if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
          for (int mt = 0; mt < 16; ++mt) {
            o[mt][0] *= alpha[0];
            o[mt][1] *= alpha[1];
            o[mt][2] *= alpha[0];
            o[mt][3] *= alpha[1];
          }
        }
        // ---- Pᵀ to shared memory as BF16 high part + BF16 remainder
        if (real_heads) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int key = (i < 2) ? gq : gq + 8;
            const int head = 2 * cq + (i & 1);
            const __nv_bfloat16 hi = __float2bfloat16_rn(pv[i]);
            const __nv_bfloat16 lo = __float2bfloat16_rn(pv[i] - __bfloat162float(hi));
            S.pt[warp][0][head][key] = __bfloat16_as_ushort(hi);
            S.pt[warp][1][head][key] = __bfloat16_as_ushort(lo);
          }
        }
        __syncwarp();
        uint32_t bh0 = 0, bh1 = 0, bl0 = 0, bl1 = 0;
        if (gq < HPG) {
          bh0 = *reinterpret_cast<const uint32_t*>(&S.pt[warp][0][gq][2 * cq]);
          bh1 = *reinterpret_cast<const uint32_t*>(&S.pt[warp][0][gq][2 * cq + 8]);
          bl0 = *reinterpret_cast<const uint32_t*>(&S.pt[warp][1][gq][2 * cq]);
          bl1 = *reinterpret_cast<const uint32_t*>(&S.pt[warp][1][gq][2 * cq + 8]);
        }
        // ---- Oᵀ += Vᵀ · Pᵀ, 16 dim tiles of 16
#pragma unroll
        for (int mt = 0; mt < 16; ++mt) {
          uint32_t a[4];
          const int c = 2 * mt + chunk_pv;  // 0..31
          ldsm_x4_t(vbase + (c >> 3) * BOX + row_pv + (((c & 7) ^ sw) << 4), a);
          mma_bf16(o[mt], a, bh0, bh1);
          mma_bf16(o[mt], a, bl0, bl1);
        }
        __syncwarp();  // Pᵀ staging is rewritten by the next tile
        if (nrows < 16) fence_proxy_async_smem();  // zeroed rows are refilled by TMA later
      }
      ++tc;
      if (aborted || (d.flags & F_LAST)) {
        last_stage = stage;  // released after the merge, which reuses its K buffer
        break;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[stage]);
    }
    if (end) break;

    // ---- merge the 4 warps' partials of this item
    // merge slot of (warp, head): 1 KB inside this warp's own rows of K box `head`
    unsigned char* kl = S.k[last_stage];
    auto slot = [&](int w, int h) { return reinterpret_cast<float*>(kl + h * BOX + w * 2048); };
    float lt[2] = {l_run[0], l_run[1]};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      lt[j] += __shfl_xor_sync(0xffffffffu, lt[j], 4);
      lt[j] += __shfl_xor_sync(0xffffffffu, lt[j], 8);
      lt[j] += __shfl_xor_sync(0xffffffffu, lt[j], 16);
    }
    if (lane < 2) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        S.merge_ml[warp][2 * lane + j][0] = m_run[j];
        S.merge_ml[warp][2 * lane + j][1] = lt[j];
      }
    }
    if (real_heads) {
#pragma unroll
      for (int mt = 0; mt < 16; ++mt) {
        const int d0 = 16 * mt + gq;
        slot(warp, 2 * cq)[d0] = o[mt][0];
        slot(warp, 2 * cq + 1)[d0] = o[mt][1];
        slot(warp, 2 * cq)[d0 + 8] = o[mt][2];
        slot(warp, 2 * cq + 1)[d0 + 8] = o[mt][3];
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.merge_bar);
    if (!mbar_wait(&S.merge_bar, mphase, P.err)) aborted = true;
    mphase ^= 1;
    {
      const int ct = warp * 32 + lane;        // 128 threads: head ct/32, dims 8*(ct%32)..
      const int h = ct >> 5, d0 = (ct & 31) * 8;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, S.merge_ml[w][h][0]);
      float Ls = 0.f, acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < NCW; ++w) {
          const float f = exp2f(S.merge_ml[w][h][0] - M);
          Ls += S.merge_ml[w][h][1] * f;
          const float* sl = slot(w, h);
          const float4 a = *reinterpret_cast<const float4*>(sl + d0);
          const float4 b = *reinterpret_cast<const float4*>(sl + d0 + 4);
          acc[0] += a.x * f; acc[1] += a.y * f; acc[2] += a.z * f; acc[3] += a.w * f;
          acc[4] += b.x * f; acc[5] += b.y * f; acc[6] += b.z * f; acc[7] += b.w * f;
        }
      }
      if (aborted) {
        // a wait ran out (error recorded): the item index may be stale, write nothing
      } else if (P.direct) {
        const float rcp = Ls > 0.f ? 1.0f / Ls : 0.f;
        const size_t oi = ((size_t)qi * NH + g * HPG + h) * D + d0;
        if (P.o_sum == nullptr) {
          float* dst = (br ? P.o_rma : P.o_swa) + oi;
          *reinterpret_cast<float4*>(dst) =
              make_float4(acc[0] * rcp, acc[1] * rcp, acc[2] * rcp, acc[3] * rcp);
          *reinterpret_cast<float4*>(dst + 4) =
              make_float4(acc[4] * rcp, acc[5] * rcp, acc[6] * rcp, acc[7] * rcp);
        } else if (br == 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i) keep[i] = acc[i] * rcp;
        } else {
          uint4 packed;
          packed.x = pack_bf2(keep[0] + acc[0] * rcp, keep[1] + acc[1] * rcp);
          packed.y = pack_bf2(keep[2] + acc[2] * rcp, keep[3] + acc[3] * rcp);
          packed.z = pack_bf2(keep[4] + acc[4] * rcp, keep[5] + acc[5] * rcp);
          packed.w = pack_bf2(keep[6] + acc[6] * rcp, keep[7] + acc[7] * rcp);
          *reinterpret_cast<uint4*>(P.o_sum + oi) = packed;
        }
      } else {
        float* dst = P.part_o + ((size_t)item * HPG + h) * D + d0;
        *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
        if (d0 == 0) {
          P.part_ml[((size_t)item * HPG + h) * 2 + 0] = M;
          P.part_ml[((size_t)item * HPG + h) * 2 + 1] = Ls;
        }
      }
    }
    fence_proxy_async_smem();  // the merge wrote the K buffer that TMA refills next
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.merge_bar);
    if (!mbar_wait(&S.merge_bar, mphase, P.err)) aborted = true;
    mphase ^= 1;
    if (lane == 0) mbar_arrive(&S.empty[last_stage]);
    if (aborted) break;
  }
}


// Merge the splits of both branches for (query, head).
//  mode 0: o_swa, o_rma FP32 [nq][16][256]; mode 1: o_sum BF16 [nq][4096] = bf16(o_swa + o_rma)
// Every split's (m, l) and output element is requested before the first is
// used (the loads of both branches are independent), so a merge costs one
// round trip to L2 rather than one per split.  A programmatic launch: its
// blocks wait beside the read's last CTAs (grid_dep_wait).
template <int SPLITS>
__global__ void __launch_bounds__(256) k_attend_merge(const float* __restrict__ part_o,
                                                      const float* __restrict__ part_ml,
                                                      float* o_swa, float* o_rma,
                                                      uint16_t* o_sum) {
  const int qi = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
  const int g = h / HPG, hh = h % HPG;
  grid_dep_wait();     // the partials come from the read before
  grid_dep_trigger();  // o_proj may start streaming its weights
  float m[2][SPLITS], l[2][SPLITS], o[2][SPLITS];
#pragma unroll
  for (int br = 0; br < 2; ++br) {
    const size_t base = (((size_t)qi * NG + g) * 2 + br) * SPLITS;
#pragma unroll
    for (int s = 0; s < SPLITS; ++s) {
      const float2 ml = *reinterpret_cast<const float2*>(part_ml + ((base + s) * HPG + hh) * 2);
      m[br][s] = ml.x;
      l[br][s] = ml.y;
      o[br][s] = part_o[((base + s) * HPG + hh) * D + d];
    }
  }
  float ob[2];
#pragma unroll
  for (int br = 0; br < 2; ++br) {
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < SPLITS; ++s) M = fmaxf(M, m[br][s]);
    float Ls = 0.f, acc = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int s = 0; s < SPLITS; ++s) {
        const float f = exp2f(m[br][s] - M);
        Ls += l[br][s] * f;
        acc += o[br][s] * f;
      }
    }
    ob[br] = Ls > 0.f ? acc / Ls : 0.f;
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
  while (items * s < 296 && s < kMaxSplits) s <<= 1;
  return s;
}

size_t attend_part_floats(int nq) {
  return (size_t)nq * NG * 2 * attend_splits(nq) * HPG * D;
}
size_t attend_ml_floats(int nq) { return (size_t)nq * NG * 2 * attend_splits(nq) * HPG * 2; }

namespace {

// 2-D map of `rows` contiguous 512-byte BF16 rows; 64x64 boxes, 128-byte swizzle.
bool encode_rows(CUtensorMap* m, const void* base, uint64_t rows) {
  return encode_bf16_2d(m, base, D, rows, ROW_BYTES, 64, 64);
}

}  // namespace

// P0.sched must be 0 when the kernel starts: zero_sched makes this call clear it
// first (a memset on st); the layer path has k_post_proj clear it instead.
int launch_attend(const AttendParams& P0, float* o_swa, float* o_rma, uint16_t* o_sum,
                  bool zero_sched, cudaStream_t st) {
  if (P0.nq <= 0) return ER_OK;
  if (!P0.sched) return ER_EINVAL;
  if (zero_sched && cudaMemsetAsync(P0.sched, 0, sizeof(int), st) != cudaSuccess) return ER_ECUDA;
  AttendParams P = P0;
  P.splits = attend_splits(P.nq);
  const uint64_t groups = (uint64_t)P.s_max * P.L * NG;
  const uint64_t bank_rows = P.pool ? (uint64_t)POOL : (uint64_t)BANK;
  bool ok = encode_rows(&P.tmap_k[TM_WIN], P.win_k, groups * WIN) &&
            encode_rows(&P.tmap_v[TM_WIN], P.win_v, groups * WIN) &&
            encode_rows(&P.tmap_k[TM_BANK], P.bank_k, groups * bank_rows) &&
            encode_rows(&P.tmap_v[TM_BANK], P.bank_v, groups * bank_rows) &&
            (P.pool || (encode_rows(&P.tmap_k[TM_PEND], P.pend_k, groups * PEND) &&
                        encode_rows(&P.tmap_v[TM_PEND], P.pend_v, groups * PEND)));
  if (!ok) return ER_ECUDA;
  {
    // the shared-memory opt-in, once per device (calls may come from several threads)
    static std::mutex mu;
    static bool attr_done[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ER_ECUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_done[dev]) {
      if (cudaFuncSetAttribute(k_attend, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)sizeof(AttnSmem) + 1024) != cudaSuccess)
        return ER_ECUDA;
      attr_done[dev] = true;
    }
  }
  const int n_items = P.nq * NG * 2 * P.splits;
  const int grid = min(P.splits == 1 ? n_items / 2 : n_items, num_sms());
  P.direct = P.splits == 1 ? 1 : 0;
  P.o_swa = o_swa;
  P.o_rma = o_rma;
  P.o_sum = o_sum;
  std::pair<cudaEvent_t, cudaEvent_t> ev;
  const bool timed = profile_begin(st, &ev);
  // a programmatic launch: the CTAs may start while the kernel before still runs
  // and wait for it (grid_dep_wait) before reading anything it writes
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = sizeof(AttnSmem) + 1024;
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k_attend, P) != cudaSuccess) {
    if (timed) profile_end(st, ev);
    return ER_ECUDA;
  }
  if (timed) profile_end(st, ev);
  count_launches(1);
  int rc = launch_status();
  if (rc != ER_OK || P.direct) return rc;
  cfg.gridDim = dim3(P.nq, NH);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  auto merge = P.splits == 2   ? k_attend_merge<2>
               : P.splits == 4 ? k_attend_merge<4>
               : P.splits == 8 ? k_attend_merge<8>
                               : k_attend_merge<16>;
  if (cudaLaunchKernelEx(&cfg, merge, (const float*)P.part_o, (const float*)P.part_ml, o_swa,
                         o_rma, o_sum) != cudaSuccess)
    return ER_ECUDA;
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
  c.take<int>(1);
  return c.used();
}

int er_swa_rma_attend(const er_state* st, int32_t layer, const int32_t* seq_ids, int32_t B,
                      const er_bf16* q_swa, const er_bf16* q_rma, float* o_swa, float* o_rma,
                      void* ws, size_t ws_bytes, er_stream_t stream) {
  if (!st || B < 0 || layer < 0 || layer >= st->n_layers) return ER_EINVAL;
  if (B == 0) return ER_OK;
  if (!seq_ids || !q_swa || !q_rma || !o_swa || !o_rma || !ws) return ER_EINVAL;
  if (!aligned16(q_swa) || !aligned16(q_rma) || !aligned16(o_swa) || !aligned16(o_rma) ||
      !aligned16(ws))
    return ER_EINVAL;
  if (ws_bytes < er_attend_workspace_bytes(B)) return ER_ECAPACITY;
  Carver c(ws);
  AttendParams P{};
  P.win_k = st->win_k; P.win_v = st->win_v;
  P.bank_k = st->bank_k; P.bank_v = st->bank_v;
  P.pend_k = st->pend_k; P.pend_v = st->pend_v;
  P.meta = st->meta; P.seq_ids = seq_ids;
  P.s_max = st->s_max; P.L = st->n_layers; P.layer = layer;
  P.q_swa = q_swa; P.q_rma = q_rma; P.nq = B;
  P.part_o = c.take<float>(attend_part_floats(B));
  P.part_ml = c.take<float>(attend_ml_floats(B));
  P.sched = c.take<int>(1);
  P.err = st->dev_error;
  P.pool = st->pool;
  P.bank_pos = st->bank_pos;
  return launch_attend(P, o_swa, o_rma, nullptr, true, (cudaStream_t)stream);
}

}  // extern "C"
