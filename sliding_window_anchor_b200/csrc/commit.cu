// commit.cu — a7, the RMA anchor-bank commit, and a4's standalone append.
//
// EdgeRock-4B 开源：72 MiB 固定 KV, §架构：… and neodrop.ai "内存还会跌吗？…",
// §三段记忆，只记值得记的: pending candidates are merged with the committed bank
// once 256 have gathered; each KV group independently keeps the 1024 records
// with the highest scores (groups may keep the same source positions); kept
// anchors are never rewritten.  Ties go to the lower source position (the
// reading fixed for this library), -0 ranks as +0 and NaN below every number.
//
// One 256-thread block per (sequence, layer, group), up to 4 blocks per SM:
//  1. 64-bit keys (ordered score << 32 | ~position) for the ≤1280 records;
//     key 0 (padding, empty slots) ranks below every real record;
//  2. the kept set: when no ranked list is requested, a radix select on 8-bit
//     digits finds the K-th largest key (K = min(1024, c+p)), usually in two
//     or three histogram passes; when the ranked list is requested, a bitonic
//     sort (descending) of 2048 keys, 8 per thread in registers: partner
//     strides below 8 inside a thread, 8..128 across lanes (shuffles), 256 and
//     up through shared memory;
//  3. flags for the kept records; two block scans give the evicted bank slots
//     (ascending) and the pending winners (ascending);
//  4. each warp moves winners' K and V rows (512 B each, 16 B per lane) into
//     their target slots, with the score and position, four rows in flight.
// Launches with few merges run as clusters of 8 CTAs that repeat steps 1-3
// and split step 4 (a cluster barrier keeps every key read ahead of the first
// bank write).  The layer calls split the commit in two launches instead:
// steps 1-3 (k_commit_plan) while the read runs, step 4 (k_commit_move) after
// it.
// Surviving anchors are not touched, so the write traffic is only the moved
// records.
#include "common.cuh"
#include "params.cuh"

namespace er {
namespace {

constexpr int NSORT = 2048;
constexpr int CT = 256;   // threads per commit block
constexpr int EPT = NSORT / CT;  // 8 keys per thread
constexpr int CW = CT / 32;      // warps per block
constexpr int SPB = 32;   // most sequences one block looks after (decode path)
constexpr int REPL = 8;   // CTAs per cluster sharing the moves of a few merges

__device__ __forceinline__ uint32_t ordered_score(float s) {
  uint32_t u = __float_as_uint(s);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;             // -0 -> +0
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0;  // NaN: lowest
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t rec_key(float s, int32_t pos) {
  return ((uint64_t)ordered_score(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)pos);
}

// Exclusive scan over the CT threads of a block; *total gets the sum.
__device__ int block_scan_excl(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < CW ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < CW; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < CW) warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  const int base = warp ? warp_sums[warp - 1] : 0;
  *total = warp_sums[CW - 1];
  __syncthreads();
  return base + x - v;
}

// Compare-exchange toward descending order when `desc`, ascending otherwise.
__device__ __forceinline__ void cas(uint64_t& ka, uint32_t& sa, uint64_t& kb, uint32_t& sb,
                                    bool desc) {
  if (desc ? (ka < kb) : (ka > kb)) {
    const uint64_t tk = ka;
    ka = kb;
    kb = tk;
    const uint32_t ts = sa;
    sa = sb;
    sb = ts;
  }
}

// Bitonic sort (descending) of 2048 keys held 8 per thread: element i = 8*tid + e.
__device__ void sort2048(uint64_t (&key)[EPT], uint32_t (&src)[EPT], uint64_t* skey,
                         uint16_t* ssrc) {
  const int tid = threadIdx.x, lane = tid & 31;
#pragma unroll
  for (int k = 2; k <= NSORT; k <<= 1) {
    int j = k >> 1;
    if (j >= 256) {
      // strides that cross warps: through shared memory, disjoint pairs per thread
      __syncthreads();
#pragma unroll
      for (int e = 0; e < EPT; ++e) {
        skey[tid * EPT + e] = key[e];
        ssrc[tid * EPT + e] = (uint16_t)src[e];
      }
      __syncthreads();
#pragma unroll
      for (; j >= 256; j >>= 1) {
#pragma unroll
        for (int q = 0; q < (NSORT / 2) / CT; ++q) {
          const int pr = q * CT + tid;  // pair index 0..1023
          const int i = ((pr & ~(j - 1)) << 1) | (pr & (j - 1));
          const int m = i | j;
          uint64_t a = skey[i], b = skey[m];
          uint32_t sa = ssrc[i], sb = ssrc[m];
          cas(a, sa, b, sb, (i & k) == 0);
          skey[i] = a;
          skey[m] = b;
          ssrc[i] = (uint16_t)sa;
          ssrc[m] = (uint16_t)sb;
        }
        __syncthreads();
      }
#pragma unroll
      for (int e = 0; e < EPT; ++e) {
        key[e] = skey[tid * EPT + e];
        src[e] = ssrc[tid * EPT + e];
      }
    }
#pragma unroll
    for (; j >= EPT; j >>= 1) {
      // partner element i ^ j is element e of lane lane ^ (j / 8)
      const int pl = j / EPT;
      const bool lower = (lane & pl) == 0;
      const bool desc = ((tid * EPT) & k) == 0;
      const bool keep_max = lower == desc;
#pragma unroll
      for (int e = 0; e < EPT; ++e) {
        const uint64_t b = __shfl_xor_sync(0xffffffffu, key[e], pl);
        const uint32_t sb = __shfl_xor_sync(0xffffffffu, src[e], pl);
        const bool take = keep_max ? (b > key[e]) : (b < key[e]);
        if (take) {
          key[e] = b;
          src[e] = sb;
        }
      }
    }
#pragma unroll
    for (; j >= 1; j >>= 1) {
#pragma unroll
      for (int e = 0; e < EPT; ++e) {
        if ((e & j) == 0)
          cas(key[e], src[e], key[e | j], src[e | j], ((tid * EPT + e) & k) == 0);
      }
    }
  }
}

}  // namespace


// K-th largest of the block's keys (keys unique, 0 = padding), by radix select on
// 8-bit digits from the top: each pass histograms the digit of the keys that
// still match the chosen prefix, and a suffix scan over the 256 bins finds the
// bin holding rank K.  Returns a (prefix, shift) pair such that a key is among
// the top K exactly when (key >> shift) >= (prefix >> shift).
__device__ void radix_select(const uint64_t (&key)[5], int K, int* hist, int* warp_sums,
                             int* sel, uint64_t* out_prefix, int* out_shift) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t prefix = 0, mask = 0;
  int need = K;
  int shift = 64;
  while (shift > 0) {
    shift -= 8;
    hist[tid] = 0;
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 5; ++q)
      if (key[q] != 0 && (key[q] & mask) == prefix)
        atomicAdd(&hist[(int)((key[q] >> shift) & 255u)], 1);
    __syncthreads();
    // inclusive suffix sum S(i) = sum_{d >= i} hist[d], thread i = bin 255 - tid
    const int bin = 255 - tid;
    int x = hist[bin];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_sums[w];
    const int S = base + x;              // keys with digit >= bin
    const int above = S - hist[bin];     // keys with digit > bin
    if (S >= need && above < need) {
      sel[0] = bin;
      sel[1] = above;
      sel[2] = hist[bin];
    }
    __syncthreads();
    const int b = sel[0];
    need -= sel[1];
    prefix |= (uint64_t)b << shift;
    mask |= (uint64_t)255 << shift;
    const int in_bin = sel[2];
    __syncthreads();  // sel and hist are rewritten by the next pass
    if (in_bin == need) break;  // every key of the boundary bin is kept
  }
  *out_prefix = prefix;
  *out_shift = shift;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

// Every thread of every CTA of the cluster (a cluster of one is the block).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Step 2 in the select form (no ranked list wanted): flag[i] = 1 for the K
// kept records (bank i < c, pending BANK + j, j < p; in the pooled layout the
// occupied pool slots i).  flag must be cleared and synchronised before; every
// thread of the block calls it.
__device__ void select_kept(const CommitParams& P, size_t gi, int c, int p, int K, uint8_t* flag,
                            int* hist, int* warp_sums, int* sel) {
  const int tid = threadIdx.x;
  uint64_t key5[5];  // records tid + 256*q (bank 0..1023, then pending)
#pragma unroll
  for (int q = 0; q < 5; ++q) {
    const int i = tid + CT * q;
    uint64_t kv = 0;
    if (P.pool) {
      // pool slot i: a record unless free
      const int32_t pos = P.bank_pos[gi * POOL + i];
      if (pos != FREE_POS) kv = rec_key(P.bank_score[gi * POOL + i], pos);
    } else if (i < BANK) {
      if (i < c) kv = rec_key(P.bank_score[gi * BANK + i], P.bank_pos[gi * BANK + i]);
    } else if (i - BANK < p) {
      kv = rec_key(P.pend_score[gi * PEND + (i - BANK)], P.pend_pos[gi * PEND + (i - BANK)]);
    }
    key5[q] = kv;
  }
  uint64_t prefix = 0;
  int shift = 64;
  if (c + p > BANK) radix_select(key5, K, hist, warp_sums, sel, &prefix, &shift);
#pragma unroll
  for (int q = 0; q < 5; ++q)
    if (key5[q] != 0 && (shift >= 64 || (key5[q] >> shift) >= (prefix >> shift)))
      flag[tid + CT * q] = 1;
}

// Step 3: from the kept flags (synchronised), the move list: winner w, in
// ascending pending index, goes from pending slot move_src[w] to the w-th
// evicted bank slot (ascending), or past the bank's end while it is not full.
// Returns the number of winners; the lists are synchronised on return.
__device__ int plan_moves(int c, int p, const uint8_t* flag, int16_t* evict_list,
                          int16_t* move_src, int16_t* move_dst, int* warp_sums) {
  const int tid = threadIdx.x;
  int ev[4], nev = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int slot = tid * 4 + q;
    ev[q] = (slot < c && !flag[slot]) ? 1 : 0;
    nev += ev[q];
  }
  int total_evict = 0;
  int er = block_scan_excl(nev, warp_sums, &total_evict);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (ev[q]) evict_list[er++] = (int16_t)(tid * 4 + q);
  int total_win = 0;
  const int wn = (tid < p && flag[BANK + tid]) ? 1 : 0;
  const int w_rank = block_scan_excl(wn, warp_sums, &total_win);
  __syncthreads();
  if (wn) {
    const int dst = w_rank < total_evict ? (int)evict_list[w_rank] : c + (w_rank - total_evict);
    move_src[w_rank] = (int16_t)tid;
    move_dst[w_rank] = (int16_t)dst;
  }
  __syncthreads();
  return total_win;
}

// Step 3 in the pooled layout: the evicted records' slots (occupied, not kept,
// ascending) into evict_list, and the next block's slot list (the 256 lowest
// slots free after the merge, ascending) into slot_list.  Returns the number
// evicted; the lists are synchronised on return.
__device__ int plan_pool(const CommitParams& P, size_t gi, const uint8_t* flag,
                         int16_t* evict_list, int16_t* slot_list, int* warp_sums) {
  const int tid = threadIdx.x;
  int ev[5], fr[5], nev = 0, nfr = 0;
#pragma unroll
  for (int q = 0; q < 5; ++q) {
    const int slot = tid * 5 + q;
    const bool occ = P.bank_pos[gi * POOL + slot] != FREE_POS;
    ev[q] = (occ && !flag[slot]) ? 1 : 0;
    fr[q] = (!occ || ev[q]) ? 1 : 0;
    nev += ev[q];
    nfr += fr[q];
  }
  int total_ev = 0, total_fr = 0;
  int er = block_scan_excl(nev, warp_sums, &total_ev);
  int fi = block_scan_excl(nfr, warp_sums, &total_fr);
#pragma unroll
  for (int q = 0; q < 5; ++q) {
    if (ev[q]) evict_list[er++] = (int16_t)(tid * 5 + q);
    if (fr[q]) {
      if (fi < PEND) slot_list[fi] = (int16_t)(tid * 5 + q);
      ++fi;
    }
  }
  __syncthreads();
  return total_ev;
}

// Step 4 in the pooled layout: free the evicted slots and install the slot list.
__device__ void apply_pool(const CommitParams& P, size_t gi, int n_ev, const int16_t* evict_list,
                           const int16_t* slot_list) {
  for (int w = threadIdx.x; w < n_ev; w += CT) {
    P.bank_pos[gi * POOL + evict_list[w]] = FREE_POS;
    P.bank_score[gi * POOL + evict_list[w]] = 0.f;
  }
  for (int j = threadIdx.x; j < PEND; j += CT) P.slots[gi * PEND + j] = slot_list[j];
}

// Step 4 for the winners this block's warps own: warp `mover` of `movers`
// takes winners mover, mover + movers, ...; 16 bytes per lane per row, MV rows
// per warp in flight (every load issued before the first store).  The lists
// are in shared memory.
__device__ void move_winners(const CommitParams& P, size_t gi, int total_win,
                             const int16_t* move_src, const int16_t* move_dst, int mover,
                             int movers) {
  constexpr int MV = 4;
  const int lane = threadIdx.x & 31;
  for (int w0 = mover; w0 < total_win; w0 += MV * movers) {
    uint4 kr[MV], vr[MV];
    int src[MV];
#pragma unroll
    for (int q = 0; q < MV; ++q) {
      const int w = w0 + q * movers;
      src[q] = w < total_win ? (int)move_src[w] : -1;
      kr[q] = vr[q] = make_uint4(0, 0, 0, 0);
      if (src[q] >= 0) {
        kr[q] = reinterpret_cast<const uint4*>(P.pend_k + (gi * PEND + src[q]) * D)[lane];
        vr[q] = reinterpret_cast<const uint4*>(P.pend_v + (gi * PEND + src[q]) * D)[lane];
      }
    }
#pragma unroll
    for (int q = 0; q < MV; ++q) {
      if (src[q] < 0) continue;
      const int dst = move_dst[w0 + q * movers];
      reinterpret_cast<uint4*>(P.bank_k + (gi * BANK + dst) * D)[lane] = kr[q];
      reinterpret_cast<uint4*>(P.bank_v + (gi * BANK + dst) * D)[lane] = vr[q];
      if (lane == 0) {
        P.bank_score[gi * BANK + dst] = P.pend_score[gi * PEND + src[q]];
        P.bank_pos[gi * BANK + dst] = P.pend_pos[gi * PEND + src[q]];
      }
    }
  }
}

// Metadata of a block's run of sequences, read in one parallel load so that
// the (many) sequences with nothing to commit cost no serial global-memory
// latency.  Threads tid < nb fill slot tid.
__device__ __forceinline__ void load_run(const CommitParams& P, int b0, int nb, int* blk_seq,
                                         int* blk_c, int* blk_p) {
  const int tid = threadIdx.x;
  if (tid < nb) {
    const int seq = P.seq_fixed >= 0 ? P.seq_fixed : P.seq_ids[b0 + tid];
    blk_seq[tid] = seq;
    blk_c[tid] = 0;
    blk_p[tid] = 0;
    if (seq >= 0 && seq < P.s_max) {
      blk_c[tid] = P.meta[seq * 4 + 2];
      blk_p[tid] = P.meta[seq * 4 + 1] + P.p_add;
    }
  }
}

// The checks every form of the commit makes for sequence slot bi: returns true
// when (seq, c, p) is a merge to run.
__device__ __forceinline__ bool merge_due(const CommitParams& P, int seq, int c, int p) {
  const int tid = threadIdx.x;
  if (seq < 0 || seq >= P.s_max) {
    if (tid == 0 && blockIdx.y == 0) set_dev_error(P.err, ER_EINVAL);
    return false;
  }
  if (P.only_if_full && p != PEND) return false;
  if (c < 0 || c > BANK || p < 0 || p > PEND) {
    if (tid == 0) set_dev_error(P.err, ER_ECAPACITY);
    return false;
  }
  return true;
}

__global__ void __launch_bounds__(CT, 4) k_commit(CommitParams P) {
  __shared__ uint64_t skey[NSORT];
  __shared__ uint16_t ssrc[NSORT];
  __shared__ uint8_t flag[BANK + PEND];
  __shared__ int16_t evict_list[BANK];
  __shared__ int16_t move_src[PEND], move_dst[PEND];
  __shared__ int warp_sums[CW];
  __shared__ int blk_seq[SPB], blk_c[SPB], blk_p[SPB];
  __shared__ int hist[256];
  __shared__ int sel[4];

  const int l = P.layer0 + blockIdx.y / NG;
  const int g = blockIdx.y % NG;
  const int tid = threadIdx.x;
  // the CTAs of a cluster work on the same merges: each computes the same kept set
  // and move list, and moves its share of the winners (rank r takes winners
  // r*8+warp, r*8+warp + 8*ranks, ...)
  const int rank = (int)cluster_ctarank(), nranks = (int)cluster_nctarank();
  // each cluster owns a run of `per_block` listed sequences
  const int b0 = (blockIdx.x / nranks) * P.per_block;
  const int nb = min(P.per_block, P.n - b0);
  load_run(P, b0, nb, blk_seq, blk_c, blk_p);
  __syncthreads();
  for (int bi = 0; bi < nb; ++bi) {
    const int b = b0 + bi;
    const int seq = blk_seq[bi];
    const int c = blk_c[bi];
    const int p = blk_p[bi];
    if (!merge_due(P, seq, c, p)) continue;
    const size_t gi = grp(seq, l, g, P.L);

    const int K = min(BANK, c + p);
    for (int i = tid; i < BANK + PEND; i += CT) flag[i] = 0;
    __syncthreads();  // flags cleared before they are set
    if (P.kept == nullptr) {
      // only the kept set is needed: radix-select the K-th largest key
      select_kept(P, gi, c, p, K, flag, hist, warp_sums, sel);
    } else {
      // the ranked list is wanted: full bitonic sort, elements 8*tid .. 8*tid+7
      uint64_t key[EPT];
      uint32_t src[EPT];
#pragma unroll
      for (int e = 0; e < EPT; ++e) {
        const int i = tid * EPT + e;
        uint64_t kv = 0;
        if (P.pool) {
          if (i < POOL) {
            const int32_t pos = P.bank_pos[gi * POOL + i];
            if (pos != FREE_POS) kv = rec_key(P.bank_score[gi * POOL + i], pos);
          }
        } else if (i < c) {
          kv = rec_key(P.bank_score[gi * BANK + i], P.bank_pos[gi * BANK + i]);
        } else if (i >= BANK && i < BANK + p) {
          kv = rec_key(P.pend_score[gi * PEND + (i - BANK)], P.pend_pos[gi * PEND + (i - BANK)]);
        }
        key[e] = kv;
        src[e] = (uint32_t)i;
      }
      sort2048(key, src, skey, ssrc);
      // rank r = 8*tid + e
#pragma unroll
      for (int e = 0; e < EPT; ++e)
        if (tid * EPT + e < K) flag[src[e]] = 1;
      if (rank == 0 && tid * EPT < BANK) {
        int32_t* kp = P.kept + (((size_t)b * P.nlayers + (l - P.layer0)) * NG + g) * BANK;
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
          const int r = tid * EPT + e;
          kp[r] = r < K ? (int32_t)src[e] : -1;
        }
      }
    }
    __syncthreads();
    if (P.pool) {
      // nothing moves: free the evicted slots, list the next block's slots
      const int n_ev = plan_pool(P, gi, flag, evict_list, move_dst, warp_sums);
      cluster_sync_all();
      if (rank == 0) apply_pool(P, gi, n_ev, evict_list, move_dst);
      __syncthreads();
      continue;
    }
    const int total_win = plan_moves(c, p, flag, evict_list, move_src, move_dst, warp_sums);
    // no CTA of the cluster writes the bank before every CTA has read this merge's keys
    cluster_sync_all();
    move_winners(P, gi, total_win, move_src, move_dst, rank * CW + (tid >> 5), CW * nranks);
    __syncthreads();  // shared arrays are reused by the next sequence
  }
}

// The layer calls' commit in two launches: k_commit_plan (steps 1-3, the move
// lists into `plan`) runs beside the read, which leaves the keys and the bank
// alone; k_commit_move (step 4) runs after the read, beside o_proj.  One block
// per (run of SPB sequences, layer, group) plans; MOVE_CTAS blocks per run
// share the moves.
constexpr int MOVE_CTAS = 8;

__global__ void __launch_bounds__(CT, 4) k_commit_plan(CommitParams P, MovePlan* plan) {
  __shared__ uint8_t flag[BANK + PEND];
  __shared__ int16_t evict_list[BANK];
  __shared__ int16_t move_src[PEND], move_dst[PEND];
  __shared__ int warp_sums[CW];
  __shared__ int blk_seq[SPB], blk_c[SPB], blk_p[SPB];
  __shared__ int hist[256];
  __shared__ int sel[4];
  const int lg = blockIdx.y, l = P.layer0 + lg / NG, g = lg % NG;
  const int nlg = P.nlayers * NG;
  const int tid = threadIdx.x;
  const int b0 = blockIdx.x * SPB;
  const int nb = min(SPB, P.n - b0);
  load_run(P, b0, nb, blk_seq, blk_c, blk_p);
  __syncthreads();
  for (int bi = 0; bi < nb; ++bi) {
    MovePlan& mp = plan[(size_t)(b0 + bi) * nlg + lg];
    const int seq = blk_seq[bi];
    const int c = blk_c[bi];
    const int p = blk_p[bi];
    if (!merge_due(P, seq, c, p)) {
      if (tid == 0) {
        mp.n = 0;
        mp.commit = 0;
      }
      continue;
    }
    const size_t gi = grp(seq, l, g, P.L);
    for (int i = tid; i < BANK + PEND; i += CT) flag[i] = 0;
    __syncthreads();
    select_kept(P, gi, c, p, min(BANK, c + p), flag, hist, warp_sums, sel);
    __syncthreads();
    if (P.pool) {
      const int n_ev = plan_pool(P, gi, flag, evict_list, move_dst, warp_sums);
      for (int w = tid; w < n_ev; w += CT) mp.src[w] = evict_list[w];
      for (int j = tid; j < PEND; j += CT) mp.dst[j] = move_dst[j];
      if (tid == 0) {
        mp.n = n_ev;
        mp.commit = 1;
      }
      __syncthreads();
      continue;
    }
    const int total_win = plan_moves(c, p, flag, evict_list, move_src, move_dst, warp_sums);
    for (int w = tid; w < total_win; w += CT) {
      mp.src[w] = move_src[w];
      mp.dst[w] = move_dst[w];
    }
    if (tid == 0) {
      mp.n = total_win;
      mp.commit = 1;
    }
    __syncthreads();  // shared arrays are reused by the next sequence
  }
}

__global__ void __launch_bounds__(CT, 4) k_commit_move(CommitParams P, const MovePlan* plan) {
  __shared__ int16_t move_src[PEND], move_dst[PEND];
  __shared__ int blk_seq[SPB], blk_n[SPB], blk_commit[SPB];
  const int lg = blockIdx.y, l = P.layer0 + lg / NG, g = lg % NG;
  const int nlg = P.nlayers * NG;
  const int tid = threadIdx.x;
  const int run = blockIdx.x / MOVE_CTAS, r = blockIdx.x % MOVE_CTAS;
  const int b0 = run * SPB;
  const int nb = min(SPB, P.n - b0);
  if (tid < nb) {
    blk_seq[tid] = P.seq_fixed >= 0 ? P.seq_fixed : P.seq_ids[b0 + tid];
    blk_n[tid] = plan[(size_t)(b0 + tid) * nlg + lg].n;
    blk_commit[tid] = plan[(size_t)(b0 + tid) * nlg + lg].commit;
  }
  __syncthreads();
  if (P.pool) {
    // nothing moves: the first CTA of each run frees the evicted slots and
    // installs the slot lists
    if (r == 0)
      for (int bi = 0; bi < nb; ++bi) {
        if (!blk_commit[bi]) continue;
        const MovePlan& mp = plan[(size_t)(b0 + bi) * nlg + lg];
        apply_pool(P, grp(blk_seq[bi], l, g, P.L), blk_n[bi], mp.src, mp.dst);
      }
    return;
  }
  for (int bi = 0; bi < nb; ++bi) {
    const int n = blk_n[bi];
    if (n <= 0) continue;  // planned as a merge only for a valid, full sequence
    const MovePlan& mp = plan[(size_t)(b0 + bi) * nlg + lg];
    for (int w = tid; w < n; w += CT) {
      move_src[w] = mp.src[w];
      move_dst[w] = mp.dst[w];
    }
    __syncthreads();
    move_winners(P, grp(blk_seq[bi], l, g, P.L), n, move_src, move_dst,
                 r * CW + (tid >> 5), CW * MOVE_CTAS);
    __syncthreads();  // the lists are reused by the next sequence
  }
}

__global__ void k_commit_finish(int32_t* meta, const int32_t* seq_ids, int n, int s_max) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= n) return;
  const int s = seq_ids[b];
  if (s < 0 || s >= s_max) return;
  int32_t* m = meta + (size_t)s * 4;
  m[2] = min(BANK, m[2] + m[1]);
  m[1] = 0;
}

// Device-gated commits (a layer call: few merges per launch) and small explicit
// ones run as clusters of REPL CTAs that split each merge's row moves; large
// explicit batches (every block busy) run one CTA per merge.
int launch_commit(const CommitParams& P, cudaStream_t st) {
  if (P.n <= 0) return ER_OK;
  CommitParams Q = P;
  Q.per_block = P.only_if_full ? SPB : 1;
  const int runs = (P.n + Q.per_block - 1) / Q.per_block;
  const int repl = (P.only_if_full || P.n * P.nlayers <= 16) ? REPL : 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(runs * repl, P.nlayers * NG);
  cfg.blockDim = dim3(CT);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = repl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k_commit, Q) != cudaSuccess) return ER_ECUDA;
  count_launches(1);
  return launch_status();
}

// The layer calls' commit (only_if_full, no ranked list): plan beside the read,
// move after it.  plan: [n][nlayers * 4] MovePlan, caller scratch.
size_t commit_plan_bytes(int n, int nlayers) {
  return (size_t)n * nlayers * NG * sizeof(MovePlan);
}

int launch_commit_plan(const CommitParams& P, MovePlan* plan, cudaStream_t st) {
  if (P.n <= 0) return ER_OK;
  if (!P.only_if_full || P.kept || !plan) return ER_EINVAL;
  CommitParams Q = P;
  Q.per_block = SPB;
  const int runs = (P.n + SPB - 1) / SPB;
  k_commit_plan<<<dim3(runs, P.nlayers * NG), CT, 0, st>>>(Q, plan);
  count_launches(1);
  return launch_status();
}

int launch_commit_move(const CommitParams& P, const MovePlan* plan, cudaStream_t st) {
  if (P.n <= 0) return ER_OK;
  if (!plan) return ER_EINVAL;
  CommitParams Q = P;
  Q.per_block = SPB;
  const int runs = (P.n + SPB - 1) / SPB;
  k_commit_move<<<dim3(runs * MOVE_CTAS, P.nlayers * NG), CT, 0, st>>>(Q, plan);
  count_launches(1);
  return launch_status();
}

// ------------------------------------------------------------- a4: append

struct AppendParams {
  uint16_t *pend_k, *pend_v;
  float* pend_score;
  int32_t* pend_pos;  // pooled layout: the slot lists
  int pool;
  uint16_t *bank_k, *bank_v;
  float* bank_score;
  int32_t* bank_pos;
  const int32_t* meta;
  const int32_t* seq_ids;
  int n, s_max, L, layer;
  const uint16_t *k, *v;
  const float* s;
  const int32_t* pos;
  int32_t* err;
};

// block per sequence, warp w: rows k0..k3 (w < 4), v0..v3 (w >= 4)
__global__ void __launch_bounds__(256) k_append(AppendParams P) {
  const int b = blockIdx.x, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seq = P.seq_ids[b];
  if (seq < 0 || seq >= P.s_max) {
    if (threadIdx.x == 0) set_dev_error(P.err, ER_EINVAL);
    return;
  }
  const int p = P.meta[seq * 4 + 1];
  if (p >= PEND) {
    if (threadIdx.x == 0) set_dev_error(P.err, ER_ECAPACITY);
    return;
  }
  const int g = w & 3;
  const size_t gi = grp(seq, P.layer, g, P.L);
  const uint4* srcp =
      reinterpret_cast<const uint4*>((w < 4 ? P.k : P.v) + ((size_t)b * NG + g) * D);
  if (P.pool) {
    // the record's pool slot comes from the group's slot list
    const int slot = P.pend_pos[gi * PEND + p];
    if (slot < 0 || slot >= POOL) {
      if (lane == 0) set_dev_error(P.err, ER_ECAPACITY);
      return;
    }
    uint4* dstp = reinterpret_cast<uint4*>((w < 4 ? P.bank_k : P.bank_v) + (gi * POOL + slot) * D);
    dstp[lane] = srcp[lane];
    if (w < 4 && lane == 0) {
      P.bank_score[gi * POOL + slot] = P.s[b * NG + g];
      P.bank_pos[gi * POOL + slot] = P.pos[b];
    }
    return;
  }
  uint4* dstp = reinterpret_cast<uint4*>((w < 4 ? P.pend_k : P.pend_v) + (gi * PEND + p) * D);
  dstp[lane] = srcp[lane];
  if (w < 4 && lane == 0) {
    P.pend_score[gi * PEND + p] = P.s[b * NG + g];
    P.pend_pos[gi * PEND + p] = P.pos[b];
  }
}

}  // namespace er

using namespace er;

extern "C" {

int er_rma_commit(const er_state* st, int32_t layer, const int32_t* seq_ids, int32_t n,
                  int32_t* kept, er_stream_t stream) {
  if (!st || n < 0 || (n > 0 && !seq_ids) || layer < -1 || layer >= st->n_layers)
    return ER_EINVAL;
  if (n == 0) return ER_OK;
  CommitParams P;
  P.bank_k = st->bank_k; P.bank_v = st->bank_v;
  P.pend_k = st->pend_k; P.pend_v = st->pend_v;
  P.bank_score = st->bank_score; P.pend_score = st->pend_score;
  P.bank_pos = st->bank_pos; P.pend_pos = st->pend_pos;
  P.meta = st->meta; P.seq_ids = seq_ids; P.seq_fixed = -1;
  P.n = n; P.s_max = st->s_max; P.L = st->n_layers;
  P.layer0 = layer < 0 ? 0 : layer;
  P.nlayers = layer < 0 ? st->n_layers : 1;
  P.p_add = 0; P.only_if_full = 0;
  P.kept = kept; P.err = st->dev_error;
  P.pool = st->pool; P.slots = st->pend_pos;
  cudaStream_t s = (cudaStream_t)stream;
  int rc = launch_commit(P, s);
  if (rc != ER_OK || layer >= 0) return rc;
  k_commit_finish<<<(n + 127) / 128, 128, 0, s>>>(st->meta, seq_ids, n, st->s_max);
  count_launches(1);
  return launch_status();
}

int er_rma_append_pending(const er_state* st, int32_t layer, const int32_t* seq_ids, int32_t n,
                          const er_bf16* k, const er_bf16* v, const float* s,
                          const int32_t* pos, er_stream_t stream) {
  if (!st || n < 0 || layer < 0 || layer >= st->n_layers) return ER_EINVAL;
  if (n > 0 && (!seq_ids || !k || !v || !s || !pos)) return ER_EINVAL;
  if (n == 0) return ER_OK;
  if (!aligned16(k) || !aligned16(v)) return ER_EINVAL;
  AppendParams P;
  P.pend_k = st->pend_k; P.pend_v = st->pend_v;
  P.pend_score = st->pend_score; P.pend_pos = st->pend_pos;
  P.pool = st->pool; P.bank_k = st->bank_k; P.bank_v = st->bank_v;
  P.bank_score = st->bank_score; P.bank_pos = st->bank_pos;
  P.meta = st->meta; P.seq_ids = seq_ids;
  P.n = n; P.s_max = st->s_max; P.L = st->n_layers; P.layer = layer;
  P.k = k; P.v = v; P.s = s; P.pos = pos; P.err = st->dev_error;
  k_append<<<n, 256, 0, (cudaStream_t)stream>>>(P);
  count_launches(1);
  return launch_status();
}

}  // extern "C"
