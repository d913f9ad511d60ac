// proj.cu — the layer's dense projections on the 5th-generation tensor cores:
// a1 (x·W_qkvᵀ, with the prepared weights also the scorer's three W1 terms, so
// a3's W1·x) and a6 (o·W_oᵀ, the shared o_proj).  Layer shapes from
// EdgeRock-4B 开源：72 MiB 固定 KV, §架构：递归、局部窗口与记忆锚点三件套
// (hidden 2560; 16 q heads and 4 KV groups of width 256 per branch).
//
// Y[t][f] = Σ_k X[t][k] · W[f][k]: X [T][K] and W [F][K] BF16 row-major (the
// nn.Linear layout), FP32 accumulation; features below `nbf` go out as BF16
// (round to nearest even) to Yb [T][ldb], the others as FP32 to Yf [T][ldf]
// (the fused q/k/v + W1-term projection keeps only the scorer's sums in FP32).
//
// The MMA's M is the feature dimension: a CTA pair (2-CTA cluster, tcgen05
// cta_group::2) owns 256 features (128 per CTA, in its TMEM lanes) and the
// tokens are the MMA's N, so one kernel serves a single decode token (a
// weight stream) up to 512 tokens (compute-bound).  Work is cut into units of
// (feature tile of 256, token chunk, 64-wide K step); the pairs of a
// persistent grid (one CTA per SM) take contiguous, equal shares of the
// units in tile-major order ("stream-K"), so every SM does the same work
// whatever the tile count.  A tile split between pairs is finished by the
// pair holding its first K step, which reaches it last in its share: the
// pairs holding its later K steps (at the start of theirs) leave FP32
// partial sums in the workspace and raise a flag; the finishing pair, whose
// pipeline buffers are free by then, pulls them in with bulk copies (32
// tokens at a time, double-buffered), adds them to its own in K order
// (deterministic), writes Y and lowers the flags.  Every wait is bounded
// (≈2 s) and records ER_ETIMEOUT.
//
// Per CTA: warp 4 — TMA (W: one 64 x 128 box of its 128 features; X: the
// chunk's tokens split between the two CTAs, N/2 rows each, 128- or 32-row
// boxes; every copy lands in this CTA and counts on the even CTA's barrier);
// warp 5 — TMEM (512 columns: two accumulators of up to 256 tokens, so a
// chunk's epilogue overlaps the next chunk's MMAs) and, in the even CTA, the
// MMA issue (M=256, N=chunk, K=16, both operands K-major, 128-byte swizzle);
// warps 0-3 — the epilogue, one feature (TMEM lane) per thread.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "tc.cuh"

namespace er {
namespace {

constexpr int PJ_THREADS = 192;
constexpr int PJ_MAXST = 8;
constexpr int W_BOX_BYTES = 128 * 128;  // 128 features x 64 K of BF16
constexpr int XBIG = 128, XSMALL = 32, XTINY = 8;  // X box rows
constexpr int PJ_SMEM_LIMIT = 232448;
constexpr int EB = 16;                  // tokens per epilogue block
constexpr int EB_BYTES = EB * 128 * 4;  // one block of 128 FP32 features: 8 KB
constexpr int PJ_STAGE_OUT = 2 * EB_BYTES;  // the two staging buffers of the stores
constexpr int PJ_MAXRING = 16;
constexpr uint64_t kFlagTag = 0xE5C0DE0000000000ull;
constexpr uint64_t kDrainNs = 200000;

struct ProjPlan {
  int T, F, K, KB;
  int n_ft;      // feature tiles of 256
  int chunk;     // tokens per chunk (multiple of 16, <= 512)
  int n_tc;      // chunks: ceil(T16 / chunk)
  int T16;       // T rounded up to 16
  int P;         // pairs
  int U;         // units: n_ft * n_tc * KB (< 2^17 for every layer shape)
  int max_acc;   // accumulators per chunk (1: chunk <= 256, else 2)
  int x_acc_bytes;  // shared-memory bytes of one accumulator's X rows per CTA
  int stage_bytes, stages;
  int nq_max;       // most contributor pairs of one tile
  int ring;         // a finishing pair's partial-block slots in the idle stage memory
};

struct ProjParams {
  CUtensorMap w_map;    // W [F][K], box 64 x 128
  CUtensorMap x_big;    // X [T][K], box 64 x 128
  CUtensorMap x_small;  // X [T][K], box 64 x 32
  CUtensorMap x_tiny;   // X [T][K], box 64 x 8
  ProjPlan plan;
  uint16_t* yb;         // BF16 [T][ldb]: features 0 .. nbf-1
  float* yf;            // FP32 [T][ldf]: features nbf .. F-1 (column f - nbf)
  int nbf, ldb, ldf;
  float* part;          // [P][2][chunk][128] FP32 partial sums
  unsigned long long* flags;  // [P][2]
  uint32_t epoch;
  int32_t* err;
};

enum : int { SEG_DIRECT = 0, SEG_OWNER = 1, SEG_CONTRIB = 2 };

struct Seg {
  int ft, tc, tok0, ntok, kb0, nkb, role;
  int q_first, q_last;  // SEG_OWNER: the pairs whose partials complete the tile
};

// First unit of a pair's share (32-bit: U * P stays below 2^31).
__host__ __device__ inline int share_begin(const ProjPlan& p, int pair) {
  return (int)((unsigned)p.U * (unsigned)pair / (unsigned)p.P);
}

// The segments of one pair's share, in order.
struct SegIter {
  const ProjPlan* p;
  int pair;
  int cur, end;
  __host__ __device__ void init(const ProjPlan* pl, int pr) {
    p = pl;
    pair = pr;
    cur = share_begin(*pl, pr);
    end = share_begin(*pl, pr + 1);
  }
  __host__ __device__ bool next(Seg& s) {
    if (cur >= end) return false;
    const int tile = cur / p->KB;
    const int kb0 = cur % p->KB;
    const int tile_end = (tile + 1) * p->KB;
    const int seg_end = end < tile_end ? end : tile_end;
    s.ft = tile / p->n_tc;
    s.tc = tile % p->n_tc;
    s.tok0 = s.tc * p->chunk;
    const int rem = p->T16 - s.tok0;
    s.ntok = rem < p->chunk ? rem : p->chunk;
    s.kb0 = kb0;
    s.nkb = seg_end - cur;
    s.q_first = s.q_last = -1;
    if (kb0 > 0) {
      s.role = SEG_CONTRIB;
    } else if (seg_end == tile_end) {
      s.role = SEG_DIRECT;
    } else {
      s.role = SEG_OWNER;
      s.q_first = pair + 1;
      int q = pair + 1;
      while (q + 1 < p->P && share_begin(*p, q + 1) < tile_end) ++q;
      s.q_last = q;
    }
    cur = seg_end;
    return true;
  }
};

// Shared-memory bytes of r X rows loaded in 128-, 32- or 8-row boxes.
__host__ __device__ inline int x_rows_bytes(int r) {
  return r == XBIG ? XBIG * 128
                   : r >= XSMALL ? ((r + XSMALL - 1) / XSMALL) * XSMALL * 128
                                 : ((r + XTINY - 1) / XTINY) * XTINY * 128;
}

__device__ __forceinline__ int seg_acc(const Seg& s) { return (s.ntok + 255) >> 8; }
__device__ __forceinline__ int acc_n(const Seg& s, int j) { return min(256, s.ntok - 256 * j); }

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Generic-proxy writes to this CTA's shared memory become visible to the TMA.
__device__ __forceinline__ void fence_async_smem_cta() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// AND of a predicate over the `n` threads that meet at named barrier `id`.
__device__ __forceinline__ bool bar_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PJ_THREADS, 1)
    k_proj(const __grid_constant__ ProjParams P) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const ProjPlan& pl = P.plan;
  const int NST = pl.stages, SB = pl.stage_bytes;
  struct Bars {
    uint64_t full[PJ_MAXST], empty[PJ_MAXST], tfull[2], tempty[2], mma_done, pbar[PJ_MAXRING];
    uint32_t tmem_base;
    volatile int failed;
    int qlist[PJ_MAXRING];  // a finishing pair's contributors (non-empty shares), in K order
  };
  unsigned char* stg = base + NST * SB;  // two staging buffers for the stores
  Bars& B = *reinterpret_cast<Bars*>(stg + PJ_STAGE_OUT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_rank();
  const uint32_t lead = rank & ~1u, peer = rank ^ 1u;
  const int pair = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&B.full[s], 2);   // one arrival (with the byte count) per CTA
      mbar_init(&B.empty[s], 1);  // the MMAs that read the stage have completed
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&B.tfull[b], 1);
      mbar_init(&B.tempty[b], 8);  // four epilogue warps of each CTA
    }
    mbar_init(&B.mma_done, 1);
    for (int r = 0; r < PJ_MAXRING; ++r) mbar_init(&B.pbar[r], 1);
    B.failed = 0;
    fence_mbar_init();
  }
  if (warp == 5) tc::tmem_alloc_pair(&B.tmem_base, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::cluster_sync();
  tc::fence_after_sync();
  // launched behind the kernel that writes X: nothing above touched it
  grid_dep_wait();
  grid_dep_trigger();
  const uint32_t tmem = B.tmem_base;
  SegIter it;
  it.init(&pl, pair);
  Seg sg;

  if (warp == 4) {
    // ----------------------------------------------------------------- TMA
    if (lane == 0) {
      int step = 0;
      while (!B.failed && it.next(sg)) {
        const int na = seg_acc(sg);
        uint32_t bytes = W_BOX_BYTES;
        for (int j = 0; j < na; ++j) bytes += x_rows_bytes(acc_n(sg, j) / 2);
        for (int kb = sg.kb0; kb < sg.kb0 + sg.nkb; ++kb, ++step) {
          const int s = step % NST;
          if (!mbar_wait(&B.empty[s], ((step / NST) & 1) ^ 1, P.err)) {
            B.failed = 1;
            break;
          }
          unsigned char* st = base + (size_t)s * SB;
          const uint32_t fb = tc::map_to_rank(&B.full[s], lead);
          tc::mbar_arrive_expect_tx_cluster(fb, bytes);
          tc::tma_load_2d_pair(st, &P.w_map, 64 * kb, 256 * sg.ft + 128 * (int)rank, fb);
          for (int j = 0; j < na; ++j) {
            const int r = acc_n(sg, j) / 2;
            const int y0 = sg.tok0 + 256 * j + (int)rank * r;
            unsigned char* dst = st + W_BOX_BYTES + j * pl.x_acc_bytes;
            if (r == XBIG) {
              tc::tma_load_2d_pair(dst, &P.x_big, 64 * kb, y0, fb);
            } else if (r >= XSMALL) {
              for (int b = 0; b * XSMALL < r; ++b)
                tc::tma_load_2d_pair(dst + b * XSMALL * 128, &P.x_small, 64 * kb,
                                     y0 + b * XSMALL, fb);
            } else {
              for (int b = 0; b * XTINY < r; ++b)
                tc::tma_load_2d_pair(dst + b * XTINY * 128, &P.x_tiny, 64 * kb,
                                     y0 + b * XTINY, fb);
            }
          }
        }
      }
    }
  } else if (warp == 5) {
    // --------------------------------------------- MMA (even CTA, one thread)
    if (lane == 0 && rank == lead) {
      int step = 0, accn = 0;
      bool ok = true;
      while (ok && !B.failed && it.next(sg)) {
        const int na = seg_acc(sg);
        // two accumulators at most, kept in registers (no dynamic indexing)
        const int b0 = accn & 1, b1 = (accn + 1) & 1;
        ok = mbar_wait(&B.tempty[b0], ((accn >> 1) & 1) ^ 1, P.err);
        if (ok && na > 1) ok = mbar_wait(&B.tempty[b1], (((accn + 1) >> 1) & 1) ^ 1, P.err);
        if (!ok) break;
        const uint32_t d0 = tmem + 256u * b0, d1 = tmem + 256u * b1;
        const uint32_t id0 = tc::idesc_bf16(256, acc_n(sg, 0), false, false);
        const uint32_t id1 = na > 1 ? tc::idesc_bf16(256, acc_n(sg, 1), false, false) : 0u;
        tc::fence_after_sync();
        for (int kb = 0; kb < sg.nkb; ++kb, ++step) {
          const int s = step % NST;
          ok = mbar_wait(&B.full[s], (step / NST) & 1, P.err);
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t a0 = smem_u32(base + (size_t)s * SB);
          const uint32_t x0 = a0 + W_BOX_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_pair_bf16_ss(d0, tc::desc_sw128(a0 + 32 * kk, 16, 1024),
                                 tc::desc_sw128(x0 + 32 * kk, 16, 1024), id0,
                                 (kb > 0 || kk > 0) ? 1u : 0u);
          if (na > 1) {
            const uint32_t x1 = x0 + pl.x_acc_bytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc::mma_pair_bf16_ss(d1, tc::desc_sw128(a0 + 32 * kk, 16, 1024),
                                   tc::desc_sw128(x1 + 32 * kk, 16, 1024), id1,
                                   (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc::commit_pair(tc::map_to_rank(&B.empty[s], rank));
          tc::commit_pair(tc::map_to_rank(&B.empty[s], peer));
        }
        if (!ok) break;
        tc::commit_pair(tc::map_to_rank(&B.tfull[b0], rank));
        tc::commit_pair(tc::map_to_rank(&B.tfull[b0], peer));
        if (na > 1) {
          tc::commit_pair(tc::map_to_rank(&B.tfull[b1], rank));
          tc::commit_pair(tc::map_to_rank(&B.tfull[b1], peer));
        }
        accn += na;
      }
      if (!ok) B.failed = 1;
      tc::commit_pair(tc::map_to_rank(&B.mma_done, rank));
      mbar_wait(&B.mma_done, 0, P.err);  // nothing of the pair's on the tensor cores at exit
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Blocks of 16 tokens: TMEM -> registers (-> plus the partials of the pairs
    // that finish this tile) -> a staging buffer (two, alternating) -> 16-byte
    // stores of whole row segments (the TMA engine stays with the operand
    // loads; stores queued behind them waited microseconds).  The four warps take
    // every decision together
    // (bar.red over their 128 threads), so they always meet at the same named
    // barriers.
    const uint32_t lane_addr = (uint32_t)(32 * warp) << 16;
    const int fl = 32 * warp + lane;  // this thread's feature within the CTA's 128
    const int ep = threadIdx.x;       // 0..127
    const int R = pl.ring;
    const uint32_t slot_bytes = (uint32_t)pl.nq_max * EB_BYTES;
    int accn = 0, pk = 0, nst = 0;    // accumulators drained, partial blocks, stores issued
    bool ok = true;
    while (ok && it.next(sg)) {
      const int na = seg_acc(sg);
      const int f0 = 256 * sg.ft + 128 * (int)rank;  // the CTA's first feature
      const bool fp32_y = f0 >= P.nbf;
      int nq = 0;  // contributors (pairs with a non-empty share) of an owner's tile
      if (sg.role == SEG_OWNER) {
        // the pairs holding the tile's later K steps must have left their partials
        bool got = true;
        if (ep == 0) {
          const unsigned long long want = kFlagTag | P.epoch;
          int n = 0;
          for (int q = sg.q_first; q <= sg.q_last; ++q)
            if (share_begin(pl, q) != share_begin(pl, q + 1) && n < PJ_MAXRING) B.qlist[n++] = q;
          for (int qi = 0; qi < n && got; ++qi) {
            const unsigned long long* fp = P.flags + 2 * B.qlist[qi] + rank;
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_u64(fp) != want) {
              if (globaltimer_ns() - t0 > kWaitLimitNs || B.failed) {
                set_dev_error(P.err, ER_ETIMEOUT);
                got = false;
                break;
              }
            }
          }
          // the bulk copies below read what those pairs stored
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        ok = bar_and(1, 128, got);
        if (!ok) break;
        for (int q = sg.q_first; q <= sg.q_last; ++q)
          if (share_begin(pl, q) != share_begin(pl, q + 1)) ++nq;
      }
      for (int j = 0; j < na; ++j) {
        const int b = (accn + j) & 1;
        ok = bar_and(1, 128, mbar_wait(&B.tfull[b], ((accn + j) >> 1) & 1, P.err));
        if (!ok) break;
        tc::fence_after_sync();
        const int nj = acc_n(sg, j);
        const int nblk = nj / EB;
        // an owner's partial blocks: block k of every contributor into ring slot
        // (pk + k) % R (the stage memory, idle once this segment's MMAs are done)
        auto issue = [&](int k) {
          const int u = pk + k, slot = u % R;
          const int tl = 256 * j + k * EB;  // first token of the block in the chunk
          mbar_arrive_expect_tx(&B.pbar[slot], (uint32_t)(nq * EB_BYTES));
          for (int qi = 0; qi < nq; ++qi)
            bulk_g2s(base + (size_t)slot * slot_bytes + (size_t)qi * EB_BYTES,
                     P.part + (((size_t)B.qlist[qi] * 2 + rank) * pl.chunk + tl) * 128,
                     EB_BYTES, &B.pbar[slot]);
        };
        if (sg.role == SEG_OWNER && ep == 0)
          for (int k = 0; k < R - 1 && k < nblk; ++k) issue(k);
        uint32_t r[32];
        for (int k = 0; k < nblk; ++k) {
          if ((k & 1) == 0) {
            tc::tmem_ld32(tmem + lane_addr + 256u * b + k * EB, r);
            tc::tmem_wait_ld();
          }
          float v[EB];
#pragma unroll
          for (int c = 0; c < EB; ++c) v[c] = __uint_as_float((k & 1) ? r[EB + c] : r[c]);
          if (sg.role == SEG_OWNER) {
            const int u = pk + k;
            if (!mbar_wait(&B.pbar[u % R], (u / R) & 1, P.err)) B.failed = 1;
            const float* src = reinterpret_cast<const float*>(base + (size_t)(u % R) * slot_bytes);
            for (int qi = 0; qi < nq; ++qi)
#pragma unroll
              for (int c = 0; c < EB; ++c) v[c] += src[qi * (EB * 128) + c * 128 + fl];
          }
          // stage the block ([16 tokens][128 features]; a thread writes its
          // feature's column), then store it with coalesced 16-byte writes
          unsigned char* sb = stg + (nst & 1) * EB_BYTES;
          const bool f32 = sg.role == SEG_CONTRIB || fp32_y;
          if (f32) {
#pragma unroll
            for (int c = 0; c < EB; ++c) reinterpret_cast<float*>(sb)[c * 128 + fl] = v[c];
          } else {
#pragma unroll
            for (int c = 0; c < EB; ++c) reinterpret_cast<uint16_t*>(sb)[c * 128 + fl] = f2bf(v[c]);
          }
          // the block is staged; the ring slot of the previous block has been read
          named_bar_sync(1, 128);
          if (sg.role == SEG_OWNER && ep == 0 && k + R - 1 < nblk) issue(k + R - 1);
          const int tl = 256 * j + k * EB;  // the chunk's token in row 0 of the block
          if (sg.role == SEG_CONTRIB) {
            // 16 x 512 B, contiguous in the pair's partial buffer
            float4* dst = reinterpret_cast<float4*>(
                P.part + (((size_t)pair * 2 + rank) * pl.chunk + tl) * 128);
#pragma unroll
            for (int i = 0; i < EB * 32 / 128; ++i)
              __stcg(dst + ep + 128 * i, reinterpret_cast<const float4*>(sb)[ep + 128 * i]);
          } else if (fp32_y) {
            // 32 chunks of 16 B per token row
#pragma unroll
            for (int i = 0; i < EB * 32 / 128; ++i) {
              const int ci = ep + 128 * i, row = ci >> 5, col = ci & 31;
              const int tok = sg.tok0 + tl + row;
              if (tok < pl.T)
                *reinterpret_cast<float4*>(P.yf + (size_t)tok * P.ldf + (f0 - P.nbf) + 4 * col) =
                    reinterpret_cast<const float4*>(sb)[ci];
            }
          } else {
            // 16 chunks of 16 B per token row
#pragma unroll
            for (int i = 0; i < EB * 16 / 128; ++i) {
              const int ci = ep + 128 * i, row = ci >> 4, col = ci & 15;
              const int tok = sg.tok0 + tl + row;
              if (tok < pl.T)
                *reinterpret_cast<uint4*>(P.yb + (size_t)tok * P.ldb + f0 + 8 * col) =
                    reinterpret_cast<const uint4*>(sb)[ci];
            }
          }
          ++nst;
        }
        if (sg.role == SEG_OWNER) pk += nblk;
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive_cluster(tc::map_to_rank(&B.tempty[b], lead));
        ok = bar_and(1, 128, !B.failed);
        if (!ok) break;
      }
      accn += na;
      if (!ok) break;
      if (sg.role == SEG_CONTRIB) {
        // the partial is complete: raise this CTA's flag for the finishing pair
        __threadfence();
        named_bar_sync(1, 128);
        if (ep == 0) st_release_u64(P.flags + 2 * pair + rank, kFlagTag | P.epoch);
      } else if (sg.role == SEG_OWNER) {
        // every partial has been read: lower the flags for the next launch
        named_bar_sync(1, 128);
        if (ep == 0)
          for (int q = sg.q_first; q <= sg.q_last; ++q) P.flags[2 * q + rank] = 0ull;
      }
    }
    if (!ok) B.failed = 1;
  }
  tc::fence_before_sync();
  __syncthreads();
  if (B.failed) {
    // a wait gave up: give copies that may still be in flight time to land
    const uint64_t tw = globaltimer_ns();
    while (globaltimer_ns() - tw < kDrainNs) {
    }
  }
  tc::cluster_sync();  // the pair's MMAs are done with both CTAs' memory
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(tmem, 512);
  }
}

// ------------------------------------------------------------------ plan

int x_acc_bytes_for(int chunk) { return x_rows_bytes((chunk > 256 ? 256 : chunk) / 2); }

// Cost estimate of a plan in SM cycles: per pair, each K step costs the longer
// of its MMAs and its copies (one SM's TMA brings ~27 B per cycle from HBM and
// ~65 B per cycle from L2; a weight slice comes from HBM the first time, from L2
// when another token chunk of the same tile has fetched it), plus the output
// stores, a finishing pair's partial reads and a fixed cost per segment.
double plan_cost(const ProjPlan& p) {
  constexpr double kFlopPerCycle = 7700.0;   // BF16 tensor rate per SM
  constexpr double kHbmBytesPerCycle = 27.0;
  constexpr double kL2BytesPerCycle = 65.0;
  constexpr double kStoreBytesPerCycle = 60.0;
  constexpr double kSegCycles = 1500.0;
  double worst = 0.0;
  for (int pr = 0; pr < p.P; ++pr) {
    SegIter it;
    it.init(&p, pr);
    Seg s;
    double c = 0.0;
    while (it.next(s)) {
      const double mma = 2.0 * 128.0 * s.ntok * 64.0 / kFlopPerCycle;
      double xb = 0.0;
      for (int j = 0; j * 256 < s.ntok; ++j)
        xb += x_rows_bytes((s.ntok - 256 * j > 256 ? 256 : s.ntok - 256 * j) / 2);
      const double w = W_BOX_BYTES / (s.tc == 0 ? kHbmBytesPerCycle : kL2BytesPerCycle);
      const double fetch = w + xb / kL2BytesPerCycle;
      c += s.nkb * (mma > fetch ? mma : fetch) + kSegCycles;
      const double tile_bytes = s.ntok * 128.0 * 4.0;  // FP32 sums of one CTA
      if (s.role == SEG_OWNER)
        c += (double)(s.q_last - s.q_first + 1) * tile_bytes / kL2BytesPerCycle;
      c += (s.role == SEG_CONTRIB ? tile_bytes : tile_bytes / 2) / kStoreBytesPerCycle;
    }
    if (c > worst) worst = c;
  }
  return worst;
}

ProjPlan make_plan(int T, int F, int K, int pairs, int chunk) {
  ProjPlan p{};
  p.T = T;
  p.F = F;
  p.K = K;
  p.KB = K / 64;
  p.n_ft = F / 256;
  p.T16 = (T + 15) / 16 * 16;
  p.chunk = chunk;
  p.n_tc = (p.T16 + chunk - 1) / chunk;
  p.P = pairs;
  p.U = p.n_ft * p.n_tc * p.KB;
  p.max_acc = chunk > 256 ? 2 : 1;
  p.x_acc_bytes = x_acc_bytes_for(chunk);
  p.stage_bytes = W_BOX_BYTES + p.max_acc * p.x_acc_bytes;
  // alignment slack, barriers, the staging buffers of the stores
  const int room = PJ_SMEM_LIMIT - 2048 - PJ_STAGE_OUT;
  p.stages = room / p.stage_bytes;
  if (p.stages > PJ_MAXST) p.stages = PJ_MAXST;
  p.nq_max = 0;
  for (int pr = 0; pr < p.P; ++pr) {
    SegIter it;
    it.init(&p, pr);
    Seg s;
    while (it.next(s))
      if (s.role == SEG_OWNER) {
        int n = 0;
        for (int q = s.q_first; q <= s.q_last; ++q)
          if (share_begin(p, q) != share_begin(p, q + 1)) ++n;
        if (n > p.nq_max) p.nq_max = n;
      }
  }
  p.ring = 0;
  if (p.nq_max > 0) {
    p.ring = (int)((long)p.stages * p.stage_bytes / ((long)p.nq_max * EB_BYTES));
    if (p.ring > PJ_MAXRING) p.ring = PJ_MAXRING;
  } else {
    p.ring = 2;
  }
  return p;
}

// A finishing pair borrows the stage memory for at least two ring slots of
// partial blocks.
bool plan_fits(const ProjPlan& p) {
  return p.stages >= 2 && p.ring >= 2 && p.nq_max <= PJ_MAXRING;
}

ProjPlan choose_plan(int T, int F, int K, int pairs) {
  const int T16 = (T + 15) / 16 * 16;
  ProjPlan best{};
  double best_cost = 0.0;
  bool have = false;
  int cands[12];
  int nc = 0;
  if (T16 <= 512) cands[nc++] = T16;
  for (int c : {512, 384, 256, 192, 128, 96, 64, 48, 32, 16})
    if (c < T16) cands[nc++] = c;
  // small problems may leave pairs idle rather than split a tile many ways
  for (int np = pairs; np >= 1; np = np > 1 ? (np + 1) / 2 : 0) {
    for (int i = 0; i < nc; ++i) {
      ProjPlan p = make_plan(T, F, K, np, cands[i]);
      if (!plan_fits(p)) continue;
      const double cost = plan_cost(p);
      if (!have || cost < best_cost) {
        best = p;
        best_cost = cost;
        have = true;
      }
    }
    if (np == 1) break;
  }
  return best;
}

struct PlanKey {
  int T, F, K, pairs;
  bool operator==(const PlanKey& o) const {
    return T == o.T && F == o.F && K == o.K && pairs == o.pairs;
  }
};

std::mutex g_plan_mu;
struct PlanEntry {
  PlanKey key;
  ProjPlan plan;
};
PlanEntry g_plans[64];
int g_n_plans = 0;

ProjPlan plan_for(int T, int F, int K, int pairs) {
  std::lock_guard<std::mutex> lock(g_plan_mu);
  const PlanKey key{T, F, K, pairs};
  for (int i = 0; i < g_n_plans; ++i)
    if (g_plans[i].key == key) return g_plans[i].plan;
  ProjPlan p = choose_plan(T, F, K, pairs);
  if (g_n_plans < 64) g_plans[g_n_plans++] = PlanEntry{key, p};
  return p;
}

int pairs_of_device() { return num_sms() / 2; }

// W tensor maps by (pointer, rows, columns): weights stay put between calls.
struct WMapEntry {
  const void* ptr;
  int F, K;
  CUtensorMap map;
};
std::mutex g_wmap_mu;
WMapEntry g_wmaps[128];
int g_n_wmaps = 0, g_wmap_next = 0;

bool w_map_for(const uint16_t* W, int F, int K, CUtensorMap* out) {
  std::lock_guard<std::mutex> lock(g_wmap_mu);
  for (int i = 0; i < g_n_wmaps; ++i)
    if (g_wmaps[i].ptr == W && g_wmaps[i].F == F && g_wmaps[i].K == K) {
      *out = g_wmaps[i].map;
      return true;
    }
  CUtensorMap m;
  if (!encode_bf16_2d(&m, W, (uint64_t)K, (uint64_t)F, (uint64_t)K * 2, 64, 128)) return false;
  WMapEntry& e = g_n_wmaps < 128 ? g_wmaps[g_n_wmaps++] : g_wmaps[(g_wmap_next++) % 128];
  e = WMapEntry{W, F, K, m};
  *out = m;
  return true;
}

std::mutex g_attr_mu;
bool g_attr_done[64] = {false};
std::atomic<uint32_t> g_epoch{1};

}  // namespace

int launch_gemv(const uint16_t* X, int T, const uint16_t* W, int F, int K, void* Y, bool yf32,
                int ldy, cudaStream_t st);

// Workspace of one projection: the partial sums of the pairs that hand a tile
// to another (one chunk of 256 features each) and their flags.
size_t proj_workspace_bytes(int T, int F, int K) {
  if (T <= 0) return 0;
  const ProjPlan p = plan_for(T, F, K, pairs_of_device());
  Carver c(nullptr);
  c.take<float>((size_t)p.P * 2 * p.chunk * 128);
  c.take<unsigned long long>((size_t)p.P * 2);
  return c.used();
}

// Y = X · Wᵀ (see the top of this file): features f < nbf to yb [T][ldb] as
// BF16, the others to yf [T][ldf] as FP32 (column f - nbf).  F a multiple of
// 256, K of 64, nbf of 256 (0..F); X, W, yb, yf 16-byte aligned; ws at least
// proj_workspace_bytes(T, F, K), 256-byte aligned.  A flag counts as raised
// only when it holds this launch's tag, and the finishing pair lowers it
// again, so the workspace needs no clearing.
int launch_proj(const uint16_t* X, int T, const uint16_t* W, int F, int K, uint16_t* yb,
                int ldb, int nbf, float* yf, int ldf, void* ws, int32_t* err, cudaStream_t st) {
  if (T <= 0) return ER_OK;
  if (F % 256 || K % 64 || nbf % 256 || nbf < 0 || nbf > F) return ER_EINVAL;
  if ((nbf > 0 && (!yb || ldb < nbf)) || (nbf < F && (!yf || ldf < F - nbf))) return ER_EINVAL;
  ProjParams P{};
  P.plan = plan_for(T, F, K, pairs_of_device());
  if (P.plan.stages < 2) return ER_EINVAL;
  if (!w_map_for(W, F, K, &P.w_map)) return ER_ECUDA;
  if (!encode_bf16_2d(&P.x_big, X, (uint64_t)K, (uint64_t)T, (uint64_t)K * 2, 64, XBIG) ||
      !encode_bf16_2d(&P.x_small, X, (uint64_t)K, (uint64_t)T, (uint64_t)K * 2, 64, XSMALL) ||
      !encode_bf16_2d(&P.x_tiny, X, (uint64_t)K, (uint64_t)T, (uint64_t)K * 2, 64, XTINY))
    return ER_ECUDA;
  if ((nbf > 0 && ((uintptr_t)yb & 15u || ldb % 8)) || (nbf < F && ((uintptr_t)yf & 15u || ldf % 4)))
    return ER_EINVAL;
  Carver c(ws);
  P.part = c.take<float>((size_t)P.plan.P * 2 * P.plan.chunk * 128);
  P.flags = c.take<unsigned long long>((size_t)P.plan.P * 2);
  P.yb = yb;
  P.yf = yf;
  P.nbf = nbf;
  P.ldb = ldb;
  P.ldf = ldf;
  P.epoch = g_epoch.fetch_add(1, std::memory_order_relaxed) & 0xFFFFFFu;
  P.err = err;
  const int smem = P.plan.stages * P.plan.stage_bytes + PJ_STAGE_OUT + 2048;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ER_ECUDA;
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (!g_attr_done[dev]) {
      if (cudaFuncSetAttribute(k_proj, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               PJ_SMEM_LIMIT) != cudaSuccess)
        return ER_ECUDA;
      g_attr_done[dev] = true;
    }
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * P.plan.P);
  cfg.blockDim = dim3(PJ_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k_proj, P) != cudaSuccess) return ER_ECUDA;
  count_launches(1);
  return launch_status();
}

}  // namespace er

using namespace er;

extern "C" {

size_t er_linear_workspace_bytes(int32_t T, int32_t F, int32_t K) {
  if (T < 1 || F < 256 || F % 256 || K < 64 || K % 64) return 0;
  return proj_workspace_bytes(T, F, K);
}

int er_linear(const er_bf16* x, int32_t T, const er_bf16* w, int32_t F, int32_t K, void* y,
              int32_t y_fp32, int32_t ldy, void* ws, size_t ws_bytes, int32_t* dev_error,
              er_stream_t stream) {
  if (T < 0 || F < 256 || F % 256 || K < 64 || K % 64 || ldy < F) return ER_EINVAL;
  if (y_fp32 != 0 && y_fp32 != 1) return ER_EINVAL;
  if (T == 0) return ER_OK;
  if (!x || !w || !y || !ws) return ER_EINVAL;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) || ((uintptr_t)ws & 255u)) return ER_EINVAL;
  if (ws_bytes < er_linear_workspace_bytes(T, F, K)) return ER_ECAPACITY;
  int32_t* err = dev_error ? dev_error : call_error_word();
  if (!err) return ER_ECUDA;
  const bool bf = y_fp32 == 0;
  if (T <= kGemvMaxTokensAll)
    return launch_gemv(x, T, w, F, K, y, !bf, ldy, (cudaStream_t)stream);
  return launch_proj(x, T, w, F, K, bf ? static_cast<uint16_t*>(y) : nullptr, ldy, bf ? F : 0,
                     bf ? nullptr : static_cast<float*>(y), ldy, ws, err, (cudaStream_t)stream);
}

}  // extern "C"
