// prefill_attn.cu — a8's two reads on the 5th-generation tensor cores.
//
// EdgeRock-4B 开源：72 MiB 固定 KV, §架构：递归、局部窗口与记忆锚点三件套 (16 query
// heads over 4 KV groups, head dim 256, a 1024-position window beside the
// anchor bank) with the reading fixed for this library: the RMA read is its
// own softmax over committed + pending records, summed with the SWA read
// before o_proj.  In a prefill chunk of T tokens starting at stream position
// t0, query token i (position t = t0 + i) reads
//   SWA: positions max(0, t-1023) .. t — older ones from the window ring (slot
//        pos mod 1024, not yet overwritten by this chunk), the chunk's own
//        rows j <= i;
//   RMA: the c committed anchors and pending records 0 .. p0+i (the chunk's
//        candidates were appended at p0 .. p0+T-1 before the reads).
//
// Work item = (64 tokens x the group's 4 heads = 256 query rows, KV group,
// branch, split of the key tiles).  An item runs on a CTA pair (a 2-CTA
// cluster) whose tensor-core MMAs span both SMs (tcgen05 cta_group::2): each
// CTA keeps 128 query rows (its 32 tokens), their S, P and O in its own TMEM,
// and fetches HALF of every key tile — 64 of its 128 keys, 128 of V's 256
// dims — so the pair reads each K/V byte once for 256 query rows (one SM's
// TMA engine delivers ~40 B per cycle; a whole tile per 128 rows left the
// loop waiting on it).  Keys stream in tiles of 128 rows aligned to 128-slot
// boundaries of the ring, the chunk, the bank or the pending block (so a TMA
// box never wraps); rows a query may not see are masked in the softmax.
//   warp 4    : TMA — Q once (a 4-D map picks the group's heads out of
//               [T][16][256]), then this CTA's K halves (2 stages);
//   warp 6    : TMA — this CTA's V halves (2 stages);
//   warp 5    : TMEM (512 columns in both CTAs: O 0..255, two S buffers of 128
//               FP32 columns; a tile's P, as BF16 pairs, overwrites the first
//               half of its S buffer); in the even CTA one thread issues
//               S = Q·Kᵀ (M=256, N=128, K=256) and, one tile behind,
//               O += P·V (M=256, N=256, K=128, P read from TMEM, V MN-major),
//               and commits each to both CTAs;
//   warps 0-3 : one thread per query row: S from TMEM, mask, online softmax
//               in base 2, P = exp2(s - m) rounded to BF16 and stored back to
//               TMEM.  The running maximum is raised only when a tile's
//               maximum exceeds it by more than 2^8; then the row of O is
//               rescaled in TMEM (after the previous PV has completed).  At the
//               end O / l and (m, l) go out in FP32 through a staging tile.
// Both CTAs' loads count on the even CTA's barriers; each softmax warp of
// both CTAs arrives (once per tile) on the even CTA's P-ready barrier.  Every copy
// lands in one CTA only.  An item's key tiles are split over NSPLIT pairs; a second
// kernel merges the splits of each branch by their (m, l), adds the two
// branches and rounds to BF16 for o_proj, and moves the chunk's window rows
// into the ring (after every read of the chunk).
// Every mbarrier wait is bounded (≈2 s) and records ER_ETIMEOUT instead of
// hanging.
#include <math.h>

#include <mutex>
#include <utility>

#include "common.cuh"
#include "tc.cuh"

namespace er {

bool profile_begin(cudaStream_t st, std::pair<cudaEvent_t, cudaEvent_t>* ev);
void profile_end(cudaStream_t st, std::pair<cudaEvent_t, cudaEvent_t> ev);

namespace {

constexpr int PQ_TOK = 32;               // tokens per CTA
constexpr int PAIR_TOK = 2 * PQ_TOK;     // tokens per CTA pair
constexpr int PM = 128;                  // query rows per CTA (half the MMA's M)
constexpr int PKT = 128;                 // keys per key tile
constexpr int KH = PKT / 2;              // keys of a tile each CTA holds
constexpr int SLICE = PM * 128;          // 128 rows x 64 BF16: one Q slice
constexpr int KSL = KH * 128;            // 64 keys x 64 dims: one K slice, 8 KB
constexpr int KHALF = 4 * KSL;           // this CTA's half of a K tile, 32 KB
constexpr int VSL = PKT * 128;           // 128 keys x 64 dims: one V slice, 16 KB
constexpr int VHALF = 2 * VSL;           // this CTA's half of a V tile (128 dims), 32 KB
constexpr int KST = 2, VST = 2;          // stages
constexpr int MAX_TILES = WIN / PKT + PEND / PKT;  // 10
constexpr int PF_THREADS = 224;
// TMEM: O in columns 0..255, two S buffers of 128 FP32 columns; a tile's P
// (128 keys as 64 columns of BF16 pairs) overwrites the first half of its own S
// buffer once the softmax has read it
constexpr uint32_t TMEM_COLS = 512, TM_O = 0, TM_S = 256;
constexpr float SCALE_LOG2 = 1.4426950408889634f / 16.0f;  // log2(e) / sqrt(256)
constexpr float RESCALE_AT = 8.0f;
constexpr int NSPLIT = 2;                // key tiles of an item split over this many pairs
constexpr uint64_t kDrainNs = 200000;    // after a timeout: let copies in flight land

enum : int { KIND_RING = 0, KIND_CHUNK = 1, KIND_BANK = 2, KIND_PEND = 3 };

struct PTile {
  int kind, row0, base;
  int full;  // every key of the tile is visible to every query row of the item
};

struct __align__(1024) PrefillSmem {
  unsigned char q[4][SLICE];     // this CTA's 128 query rows, 4 slices of 64 dims (64 KB)
  unsigned char k[KST][KHALF];   // K halves (64 KB)
  unsigned char v[VST][VHALF];   // V halves (32 KB)
  // used in the even CTA: both CTAs' copies and softmax warps arrive here
  uint64_t q_full, k_full[KST], v_full[VST], p_full[2], mma_done;
  // used in both CTAs: the even CTA's MMAs commit here
  uint64_t k_empty[KST], s_full[2], pv_done[2];
  uint32_t tmem_base;
  int ntiles, meta_ok, failed;
  PTile tiles[MAX_TILES];
};

constexpr size_t PF_SMEM = sizeof(PrefillSmem) + 1024;
static_assert(PF_SMEM <= 232448, "shared memory above the per-block limit");
static_assert(4 * 32 * 32 * 4 <= KHALF, "epilogue staging must fit a K stage");

struct PrefillParams {
  CUtensorMap tmap_q[2];  // q_swa, q_rma: {256, 4 heads, 4 groups, T}, box {64, 4, 1, 32}
  CUtensorMap tmap_k[4];  // ring, chunk, bank, pending K rows; box 64 dims x 64 rows
  CUtensorMap tmap_v[4];  // the same V rows; box 64 dims x 128 rows
  const int32_t* meta;
  int seq, s_max, L, layer, T;
  int pool;                 // pooled layout: the RMA read takes the group's 1280 pool slots
  const int32_t* bank_pos;  // pooled layout: each slot's source position (free: FREE_POS)
  float* out;   // FP32 [2 branches][NSPLIT][T][16][256]: each split's O / l
  float2* ml;   // [2][NSPLIT][T][16]: each split's (running maximum m in log2 units, l)
  int32_t* err;
};

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

// The key tiles one work item (tokens i0 .. i0+63) reads, in streaming order.
// In the pooled layout the RMA tiles are the group's 10 pool tiles (kind
// KIND_BANK over the pool rows), masked by each slot's source position.
__device__ int build_tiles(PTile* tl, int br, int g, int i0, int T, int t0, int p0, int c,
                           int gi, int pool) {
  const int i_last = min(T, i0 + PAIR_TOK) - 1;
  int n = 0;
  if (br == 0) {
    // ring tiles holding at least one position the item's first query still sees;
    // slot w = t0 mod 1024 holds the oldest position t0-1024, slot w-1 the newest
    // t0-1; elsewhere positions rise by one per slot
    const int lo_first = max(0, t0 + i0 - (WIN - 1));
    const int lo_last = max(0, t0 + i_last - (WIN - 1));
    const int w = t0 & (WIN - 1);
    for (int rt = 0; rt < WIN / PKT && t0 > 0; ++rt) {
      const int a = rt * PKT, z = a + PKT - 1;
      const int pos_a = t0 - WIN + ((a - t0) & (WIN - 1));
      const int pos_z = t0 - WIN + ((z - t0) & (WIN - 1));
      const int oldest = (w >= a && w <= z) ? t0 - WIN : pos_a;
      const int newest = (w > a && w <= z) ? t0 - 1 : pos_z;
      if (newest >= lo_first)
        tl[n++] = {KIND_RING, gi * WIN + a, a, oldest >= lo_last ? 1 : 0};
    }
    for (int ct = 0; ct * PKT <= i_last; ++ct)
      tl[n++] = {KIND_CHUNK, g * T + ct * PKT, ct * PKT, ct * PKT + PKT - 1 <= i0 ? 1 : 0};
  } else if (pool) {
    for (int bt = 0; bt < POOL / PKT; ++bt) tl[n++] = {KIND_BANK, gi * POOL + bt * PKT, bt * PKT, 0};
  } else {
    for (int bt = 0; bt * PKT < c; ++bt)
      tl[n++] = {KIND_BANK, gi * BANK + bt * PKT, bt * PKT, bt * PKT + PKT <= c ? 1 : 0};
    for (int pt = 0; pt * PKT <= p0 + i_last; ++pt)
      tl[n++] = {KIND_PEND, gi * PEND + pt * PKT, pt * PKT, pt * PKT + PKT - 1 <= p0 + i0 ? 1 : 0};
  }
  return n;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PF_THREADS, 1)
    k_prefill_attn(const __grid_constant__ PrefillParams P) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  PrefillSmem& S = *reinterpret_cast<PrefillSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_rank();  // 0: issues the MMAs; 1: its peer
  const uint32_t lead = rank & ~1u, peer = rank ^ 1u;
  const int i0 = (blockIdx.x >> 1) * PAIR_TOK;  // the pair's first token
  const int g = blockIdx.y;
  const int br = blockIdx.z / NSPLIT, split = blockIdx.z % NSPLIT;
  const int T = P.T;
  const int t0 = P.meta[P.seq * 4 + 0];
  const int p0 = P.meta[P.seq * 4 + 1];
  const int c = P.meta[P.seq * 4 + 2];
  const int gi = (int)grp(P.seq, P.layer, g, P.L);

  if (threadIdx.x == 0) {
    mbar_init(&S.q_full, 2);
    for (int b = 0; b < KST; ++b) {
      mbar_init(&S.k_full[b], 2);
      mbar_init(&S.k_empty[b], 1);
    }
    for (int b = 0; b < VST; ++b) mbar_init(&S.v_full[b], 2);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.s_full[b], 1);
      mbar_init(&S.p_full[b], 2 * 4);  // one arrival per softmax warp of each CTA
      mbar_init(&S.pv_done[b], 1);
    }
    mbar_init(&S.mma_done, 1);
    fence_mbar_init();
    const bool meta_ok = t0 >= 0 && p0 >= 0 && c >= 0 && c <= BANK && p0 + T <= PEND;
    int nt = 0;
    if (meta_ok) {
      // this pair's contiguous share of the item's tiles (both CTAs build the same list)
      const int all = build_tiles(S.tiles, br, g, i0, T, t0, p0, c, gi, P.pool);
      const int tb = all * split / NSPLIT, te = all * (split + 1) / NSPLIT;
      for (int j = tb; j < te; ++j) S.tiles[j - tb] = S.tiles[j];
      nt = te - tb;
    } else if (rank == 0) {
      set_dev_error(P.err, ER_ECAPACITY);
    }
    S.ntiles = nt;
    S.meta_ok = meta_ok ? 1 : 0;
    S.failed = 0;
  }
  if (warp == 5) tc::tmem_alloc_pair(&S.tmem_base, TMEM_COLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::cluster_sync();  // both CTAs' barriers initialised, TMEM held by both
  tc::fence_after_sync();
  // launched behind the norm/RoPE kernel that writes q, the chunk rows and the
  // pending records: everything above read only metadata written earlier
  grid_dep_wait();
  grid_dep_trigger();  // the combine kernel may launch (it waits for this grid)
  const uint32_t tmem = S.tmem_base;
  const int n = S.ntiles;

  if (warp == 4) {
    // ------------------------------------------------ Q + K halves (both CTAs)
    if (lane == 0 && n > 0) {
      tc::mbar_arrive_expect_tx_cluster(tc::map_to_rank(&S.q_full, lead), 4 * SLICE);
      for (int d = 0; d < 4; ++d)
        tc::tma_load_4d_pair(S.q[d], &P.tmap_q[br], 64 * d, 0, g, i0 + PQ_TOK * (int)rank,
                             tc::map_to_rank(&S.q_full, lead));
      for (int j = 0; j < n; ++j) {
        const int b = j % KST;
        if (!mbar_wait(&S.k_empty[b], ((j / KST) & 1) ^ 1, P.err)) {
          S.failed = 1;
          break;
        }
        const PTile tl = S.tiles[j];
        const uint32_t full = tc::map_to_rank(&S.k_full[b], lead);
        tc::mbar_arrive_expect_tx_cluster(full, KHALF);
        for (int d = 0; d < 4; ++d)
          tc::tma_load_2d_pair(S.k[b] + d * KSL, &P.tmap_k[tl.kind], 64 * d,
                               tl.row0 + KH * (int)rank, full);
      }
    }
  } else if (warp == 6) {
    // ---------------------------------------------------- V halves (both CTAs)
    if (lane == 0 && n > 0) {
      for (int j = 0; j < n; ++j) {
        const int b = j % VST;
        if (!mbar_wait(&S.pv_done[b], ((j / VST) & 1) ^ 1, P.err)) {
          S.failed = 1;
          break;
        }
        const PTile tl = S.tiles[j];
        const uint32_t full = tc::map_to_rank(&S.v_full[b], lead);
        tc::mbar_arrive_expect_tx_cluster(full, VHALF);
        for (int d = 0; d < 2; ++d)
          tc::tma_load_2d_pair(S.v[b] + d * VSL, &P.tmap_v[tl.kind], 64 * (2 * (int)rank + d),
                               tl.row0, full);
      }
    }
  } else if (warp == 5) {
    // --------------------------------------------- MMA (even CTA, one thread)
    if (lane == 0 && n > 0 && rank == lead) {
      constexpr uint32_t idesc_s = tc::idesc_bf16(2 * PM, PKT, false, false);
      constexpr uint32_t idesc_pv = tc::idesc_bf16(2 * PM, 256, false, true);
      bool ok = mbar_wait(&S.q_full, 0, P.err);
      for (int j = 0; ok && j <= n; ++j) {
        if (j < n) {
          // S buffer b last held P_{j-2}; P·V_{j-2} was issued before this MMA, and
          // the MMAs of one thread run in issue order
          const int b = j & 1, kb = j % KST;
          ok = mbar_wait(&S.k_full[kb], (j / KST) & 1, P.err);
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t d_s = tmem + TM_S + PKT * b;
#pragma unroll
          for (int kk = 0; kk < 16; ++kk) {
            const uint64_t a =
                tc::desc_sw128(smem_u32(S.q[kk >> 2]) + 32 * (kk & 3), 16, 1024);
            const uint64_t bd =
                tc::desc_sw128(smem_u32(S.k[kb]) + (kk >> 2) * KSL + 32 * (kk & 3), 16, 1024);
            tc::mma_pair_bf16_ss(d_s, a, bd, idesc_s, kk > 0);
          }
          tc::commit_pair(tc::map_to_rank(&S.s_full[b], rank));
          tc::commit_pair(tc::map_to_rank(&S.s_full[b], peer));
          tc::commit_pair(tc::map_to_rank(&S.k_empty[kb], rank));
          tc::commit_pair(tc::map_to_rank(&S.k_empty[kb], peer));
        }
        if (j >= 1) {
          const int jj = j - 1, b = jj & 1, vb = jj % VST;
          ok = mbar_wait(&S.v_full[vb], (jj / VST) & 1, P.err) &&
               mbar_wait(&S.p_full[b], (jj >> 1) & 1, P.err);
          if (!ok) break;
          tc::fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < PKT / 16; ++kk) {
            // P from TMEM (the first half of S buffer b; 16 keys = 8 columns per
            // step); this CTA's V half as the MN-major B operand: 64-dim blocks VSL
            // apart, 8-key groups 1 KB apart
            const uint64_t bd = tc::desc_sw128(smem_u32(S.v[vb]) + 2048 * kk, VSL, 1024);
            tc::mma_pair_bf16_ts(tmem + TM_O, tmem + TM_S + PKT * b + 8 * kk, bd, idesc_pv,
                                 (jj > 0 || kk > 0) ? 1u : 0u);
          }
          tc::commit_pair(tc::map_to_rank(&S.pv_done[b], rank));
          tc::commit_pair(tc::map_to_rank(&S.pv_done[b], peer));
        }
      }
      if (!ok) S.failed = 1;
      // nothing of the pair's may still run on the tensor cores at exit
      tc::commit_pair(tc::map_to_rank(&S.mma_done, rank));
      mbar_wait(&S.mma_done, 0, P.err);
    }
  } else {
    // ------------------------------------------------------ softmax, rows
    const int r = threadIdx.x;  // 0..127 = TMEM lane
    const int i = i0 + PQ_TOK * (int)rank + (r >> 2), hh = r & 3;
    const int t = t0 + i;
    const uint32_t lane_addr = (uint32_t)(32 * warp) << 16;
    // ring slot u = (slot - t0) mod 1024 holds position t0 - 1024 + u: visible from
    // u >= uth on; other kinds: key index base + k visible up to hi_*
    const int uth = max(0, t - (WIN - 1)) - (t0 - WIN);
    const int hi_chunk = i, hi_bank = c - 1, hi_pend = p0 + i;
    float m = -INFINITY, l = 0.f;  // m in log2 units (scores x log2(e)/16)
    bool ok = n > 0;
    for (int j = 0; ok && j < n; ++j) {
      const int b = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      ok = warp_all(mbar_wait(&S.s_full[b], ph, P.err));
      if (!ok) break;
      tc::fence_after_sync();
      float s[PKT];
#pragma unroll
      for (int cb = 0; cb < PKT / 32; ++cb) {
        uint32_t raw[32];
        tc::tmem_ld32(tmem + lane_addr + TM_S + PKT * b + 32 * cb, raw);
        tc::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) s[32 * cb + k] = __uint_as_float(raw[k]);
      }

      const PTile tl = S.tiles[j];
      if (!tl.full) {
        if (P.pool && tl.kind == KIND_BANK) {
          // a free slot, or a record after this query, is not read
          const int4* pp = reinterpret_cast<const int4*>(P.bank_pos + tl.row0);
#pragma unroll
          for (int k4 = 0; k4 < PKT / 4; ++k4) {
            const int4 q4 = pp[k4];
            if (q4.x > t) s[4 * k4 + 0] = -INFINITY;
            if (q4.y > t) s[4 * k4 + 1] = -INFINITY;
            if (q4.z > t) s[4 * k4 + 2] = -INFINITY;
            if (q4.w > t) s[4 * k4 + 3] = -INFINITY;
          }
        } else if (tl.kind == KIND_RING) {
          const int ub = tl.base - t0;
#pragma unroll
          for (int k = 0; k < PKT; ++k)
            if (((ub + k) & (WIN - 1)) < uth) s[k] = -INFINITY;
        } else {
          const int khi =
              (tl.kind == KIND_CHUNK ? hi_chunk : tl.kind == KIND_BANK ? hi_bank : hi_pend) -
              tl.base;
#pragma unroll
          for (int k = 0; k < PKT; ++k)
            if (k > khi) s[k] = -INFINITY;
        }
      }
      float mt = s[0];
#pragma unroll
      for (int k = 1; k < PKT; ++k) mt = fmaxf(mt, s[k]);
      const float m_new = fmaxf(m, mt * SCALE_LOG2);
      const bool need = (m != -INFINITY) && (m_new > m + RESCALE_AT);
      if (__any_sync(0xffffffffu, need)) {
        // O holds P_0..P_{j-1}·V: wait for the last of those products, then rescale
        ok = warp_all(mbar_wait(&S.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, P.err));
        if (!ok) break;
        tc::fence_after_sync();
        const float f = need ? ex2_approx(m - m_new) : 1.f;
#pragma unroll 1
        for (int cb = 0; cb < 8; ++cb) {
          uint32_t o[32];
          tc::tmem_ld32(tmem + lane_addr + TM_O + 32 * cb, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tc::tmem_st32(tmem + lane_addr + TM_O + 32 * cb, o);
        }
        tc::tmem_wait_st();
        if (need) l *= f;
      }
      if (need || m == -INFINITY) m = m_new;
      const float msub = m == -INFINITY ? 0.f : m;
      uint32_t pk[PKT / 2];
      float lsum = 0.f;
#pragma unroll
      for (int k = 0; k < PKT; k += 2) {
        const float pa = ex2_approx(fmaf(s[k], SCALE_LOG2, -msub));
        const float pb = ex2_approx(fmaf(s[k + 1], SCALE_LOG2, -msub));
        lsum += pa + pb;
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(pa, pb);
        pk[k >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      l += lsum;
      // P_j over the first half of S_j's buffer (this thread has read all of S_j)
      {
        uint32_t half[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) half[e] = pk[e];
        tc::tmem_st32(tmem + lane_addr + TM_S + PKT * b, half);
#pragma unroll
        for (int e = 0; e < 32; ++e) half[e] = pk[32 + e];
        tc::tmem_st32(tmem + lane_addr + TM_S + PKT * b + 32, half);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive_cluster(tc::map_to_rank(&S.p_full[b], lead));
    }
    if (ok) ok = warp_all(mbar_wait(&S.pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1, P.err));
    if (!ok && n > 0 && lane == 0) S.failed = 1;
    // this split's partial result: O / l and (m, l); a split without keys for the
    // row (or without tiles) leaves O = 0, m = -inf, l = 0
    const size_t row = ((size_t)(br * NSPLIT + split) * T + i) * NH + 4 * g + hh;
    if (ok) {
      // every MMA and copy of the pair is complete: the K stages serve as a 4 KB
      // staging tile per warp, so each store instruction writes 4 whole 128-byte
      // row segments (row r keeps its 16-byte chunk c at position c ^ (r & 7))
      tc::fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      float* stage = reinterpret_cast<float*>(S.k[0]) + warp * (32 * 32);
      const int q8 = lane & 7;
#pragma unroll 1
      for (int cb = 0; cb < 8; ++cb) {
        uint32_t o[32];
        tc::tmem_ld32(tmem + lane_addr + TM_O + 32 * cb, o);
        tc::tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          *reinterpret_cast<float4*>(stage + lane * 32 + ((cc ^ (lane & 7)) << 2)) =
              make_float4(__uint_as_float(o[4 * cc]) * inv, __uint_as_float(o[4 * cc + 1]) * inv,
                          __uint_as_float(o[4 * cc + 2]) * inv,
                          __uint_as_float(o[4 * cc + 3]) * inv);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = 4 * k + (lane >> 3);      // row of this warp's 32
          const int rg = 32 * warp + rr;           // row of this CTA's 128
          const int ti = i0 + PQ_TOK * (int)rank + (rg >> 2);
          if (ti < T) {
            const size_t grow = ((size_t)(br * NSPLIT + split) * T + ti) * NH + 4 * g + (rg & 3);
            *reinterpret_cast<float4*>(P.out + grow * D + 32 * cb + 4 * q8) =
                *reinterpret_cast<const float4*>(stage + rr * 32 + ((q8 ^ (rr & 7)) << 2));
          }
        }
        __syncwarp();
      }
      if (i < T) P.ml[row] = make_float2(m, l);
    } else if (n == 0 && S.meta_ok && i < T) {
      float4* dst = reinterpret_cast<float4*>(P.out + row * D);
      for (int e = 0; e < D / 4; ++e) dst[e] = make_float4(0.f, 0.f, 0.f, 0.f);
      P.ml[row] = make_float2(-INFINITY, 0.f);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (S.failed) {
    // a wait gave up: give copies that may still be in flight time to land
    const uint64_t tw = globaltimer_ns();
    while (globaltimer_ns() - tw < kDrainNs) {
    }
  }
  tc::cluster_sync();  // the pair's MMAs are done with both CTAs' memory
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// o_sum[t][h*256 + d] = bf16(o_swa + o_rma), each branch the merge of its
// NSPLIT partial reads weighted by l·2^(m - M); 8 values per thread.  Every
// read of the chunk is done by now, so the same launch also moves the chunk's
// window rows into the ring (slot (t0 + i) mod 1024): 256 16-byte pieces per
// token (4 groups x K, V x 32).
struct RingWrite {
  const uint16_t *chunk_k, *chunk_v;  // [4][T][256]
  uint16_t *win_k, *win_v;
  const int32_t* meta;
  int seq, s_max, L, layer;
};

__global__ void k_prefill_combine(const float* __restrict__ out, const float2* __restrict__ ml,
                                  int T, int nbr, uint16_t* __restrict__ o_sum, RingWrite rw) {
  grid_dep_wait();  // the partial reads of the kernel before
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= T * (OIN / 8)) return;
  {
    const int tok = idx / (OIN / 8), piece = idx % (OIN / 8);
    if (piece < NG * 2 * 32 && rw.seq >= 0 && rw.seq < rw.s_max) {
      const int g = piece >> 6, is_v = (piece >> 5) & 1, lane = piece & 31;
      const int t = rw.meta[rw.seq * 4 + 0] + tok;
      if (t >= 0) {
        const size_t row = grp(rw.seq, rw.layer, g, rw.L) * WIN + (size_t)(t % WIN);
        const uint4* src =
            reinterpret_cast<const uint4*>((is_v ? rw.chunk_v : rw.chunk_k) +
                                           ((size_t)g * T + tok) * D);
        reinterpret_cast<uint4*>((is_v ? rw.win_v : rw.win_k) + row * D)[lane] = src[lane];
      }
    }
  }
  const int row = idx / (D / 8);  // token * 16 + head
  const int d0 = (idx % (D / 8)) * 8;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int br = 0; br < nbr; ++br) {
    // every split's (m, l) and partial row are loaded up front (all in bounds),
    // so the loads overlap; a split without keys (l = 0) is skipped, never
    // multiplied, whatever its row holds
    float2 v[NSPLIT];
    float4 x0[NSPLIT], x1[NSPLIT];
#pragma unroll
    for (int sp = 0; sp < NSPLIT; ++sp) {
      v[sp] = ml[(size_t)(br * NSPLIT + sp) * T * NH + row];
      const float4* src = reinterpret_cast<const float4*>(
          out + ((size_t)(br * NSPLIT + sp) * T * NH + row) * D + d0);
      x0[sp] = src[0];
      x1[sp] = src[1];
    }
    float M = -INFINITY;
#pragma unroll
    for (int sp = 0; sp < NSPLIT; ++sp)
      if (v[sp].y > 0.f) M = fmaxf(M, v[sp].x);
    float w[NSPLIT], wsum = 0.f;
#pragma unroll
    for (int sp = 0; sp < NSPLIT; ++sp) {
      w[sp] = v[sp].y > 0.f ? exp2f(v[sp].x - M) * v[sp].y : 0.f;
      wsum += w[sp];
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
    for (int sp = 0; sp < NSPLIT; ++sp) {
      if (w[sp] == 0.f) continue;
      const float ws = w[sp] * inv;
      acc[0] += ws * x0[sp].x; acc[1] += ws * x0[sp].y;
      acc[2] += ws * x0[sp].z; acc[3] += ws * x0[sp].w;
      acc[4] += ws * x1[sp].x; acc[5] += ws * x1[sp].y;
      acc[6] += ws * x1[sp].z; acc[7] += ws * x1[sp].w;
    }
  }
  uint4 pk;
  uint32_t* pw = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
    pw[q] = *reinterpret_cast<const uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(o_sum + (size_t)idx * 8) = pk;
}

bool g_pf_attr[64] = {false};
std::mutex g_pf_mu;

}  // namespace

// Workspace FP32 floats for the partial reads of a T-token chunk: O / l per
// (branch, split, token, head), then (m, l) pairs.
size_t prefill_out_floats(int T) {
  return (size_t)2 * NSPLIT * T * OIN + (size_t)2 * NSPLIT * T * NH * 2;
}

int launch_prefill_attend(const er_state* st, int layer, int seq, int T, const uint16_t* q_swa,
                          const uint16_t* q_rma, const uint16_t* chunk_k,
                          const uint16_t* chunk_v, float* out, uint16_t* o_sum, bool rma_off,
                          cudaStream_t stream) {
  if (T < 1 || T > PEND) return ER_EINVAL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ER_ECUDA;
  {
    std::lock_guard<std::mutex> lock(g_pf_mu);
    if (!g_pf_attr[dev]) {
      if (cudaFuncSetAttribute(k_prefill_attn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)PF_SMEM) != cudaSuccess)
        return ER_ECUDA;
      g_pf_attr[dev] = true;
    }
  }
  PrefillParams P;
  const uint64_t rows_win = (uint64_t)st->s_max * st->n_layers * NG * WIN;
  const uint64_t rows_pend = (uint64_t)st->s_max * st->n_layers * NG * PEND;
  const uint64_t qd[4] = {D, 4, NG, (uint64_t)T};
  const uint64_t qs[3] = {D * 2, 4 * D * 2, NH * D * 2};
  const uint32_t qb[4] = {64, 4, 1, PQ_TOK};
  bool ok = encode_bf16(&P.tmap_q[0], q_swa, 4, qd, qs, qb) &&
            encode_bf16(&P.tmap_q[1], q_rma, 4, qd, qs, qb);
  // the pooled layout has no pending arrays: its pool (bank) map stands in for
  // the unused pending one
  const uint64_t rows_bank =
      (uint64_t)st->s_max * st->n_layers * NG * (st->pool ? POOL : BANK);
  const uint16_t* kb[4] = {st->win_k, chunk_k, st->bank_k, st->pool ? st->bank_k : st->pend_k};
  const uint16_t* vb[4] = {st->win_v, chunk_v, st->bank_v, st->pool ? st->bank_v : st->pend_v};
  const uint64_t rows[4] = {rows_win, (uint64_t)NG * T, rows_bank, rows_pend};
  for (int m = 0; m < 4; ++m)
    ok = ok && encode_bf16_2d(&P.tmap_k[m], kb[m], D, rows[m], ROW_BYTES, 64, KH) &&
         encode_bf16_2d(&P.tmap_v[m], vb[m], D, rows[m], ROW_BYTES, 64, PKT);
  if (!ok) return ER_ECUDA;
  P.meta = st->meta;
  P.seq = seq;
  P.s_max = st->s_max;
  P.L = st->n_layers;
  P.layer = layer;
  P.T = T;
  P.pool = st->pool;
  P.bank_pos = st->bank_pos;
  P.out = out;
  P.ml = reinterpret_cast<float2*>(out + (size_t)2 * NSPLIT * T * OIN);
  P.err = st->dev_error;
  // branch 0 (SWA) and, unless the RMA is switched off, branch 1
  const int nbr = rma_off ? 1 : 2;
  // x: CTA pairs (2-CTA clusters), one per 64 tokens
  const dim3 grid(2 * ((T + PAIR_TOK - 1) / PAIR_TOK), NG, nbr * NSPLIT);
  std::pair<cudaEvent_t, cudaEvent_t> ev;
  const bool timed = profile_begin(stream, &ev);
  // both kernels launch programmatically: they may start while their
  // predecessor runs, and wait for it (grid_dep_wait) before its outputs
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(PF_THREADS);
  cfg.dynamicSmemBytes = PF_SMEM;
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  const bool launched = cudaLaunchKernelEx(&cfg, k_prefill_attn, P) == cudaSuccess;
  if (timed) profile_end(stream, ev);
  const int nv = T * (OIN / 8);
  RingWrite rw;
  rw.chunk_k = chunk_k;
  rw.chunk_v = chunk_v;
  rw.win_k = st->win_k;
  rw.win_v = st->win_v;
  rw.meta = st->meta;
  rw.seq = seq;
  rw.s_max = st->s_max;
  rw.L = st->n_layers;
  rw.layer = layer;
  cudaLaunchConfig_t cfg2 = {};
  cfg2.gridDim = dim3((nv + 255) / 256);
  cfg2.blockDim = dim3(256);
  cfg2.dynamicSmemBytes = 0;
  cfg2.stream = stream;
  cfg2.attrs = pdl;
  cfg2.numAttrs = 1;
  if (!launched ||
      cudaLaunchKernelEx(&cfg2, k_prefill_combine, (const float*)out, (const float2*)P.ml, T,
                         nbr, o_sum, rw) != cudaSuccess)
    return ER_ECUDA;
  count_launches(2);
  return launch_status();
}

}  // namespace er
