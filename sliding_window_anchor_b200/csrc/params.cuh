// params.cuh — launch parameters shared between the kernels and the layer
// orchestration (layer.cu).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace er {

struct PostParams {
  const uint16_t* proj;      // [nq][12288] BF16 (separate scorer), or
  const float* proj_f32;     // [nq][13056] FP32: q/k/v sums, then hi/mid/lo W1-term sums
  const float* s_part;       // separate scorer: [4 hidden quarters][nq][4] partial scores
  const float* w2;           // fused: W2 [4][256] FP32
  int nq;
  const uint16_t *gq_swa, *gk_swa, *gq_rma, *gk_rma;
  uint16_t *q_swa, *q_rma;  // [nq][16][256] each
  uint16_t *win_k, *win_v, *pend_k, *pend_v;
  float* pend_score;
  int32_t* pend_pos;           // pooled layout: the groups' slot lists
  int pool;                    // the pooled layout: records go to bank_* at their slot
  uint16_t *bank_k, *bank_v;
  float* bank_score;
  int32_t* bank_pos;
  const int32_t* meta;
  const int32_t* seq_ids;
  int s_max, L, layer;
  int prefill;                 // 0: token b of sequence seq_ids[b]; 1: token i of seq_fixed
  int seq_fixed;
  uint16_t *chunk_k, *chunk_v; // prefill: [4][nq][256] window rows of the chunk
  int* sched_reset;            // decode: the read's work counter, zeroed here (or NULL)
  int32_t* err;
};

// Tensor maps of the row arrays the decode read streams (2-D views [rows][256]
// BF16, 64x64 boxes, 128-byte swizzle): K and V of window, bank, pending.
enum { TM_WIN = 0, TM_BANK = 1, TM_PEND = 2, TM_COUNT = 3 };

struct AttendParams {
  CUtensorMap tmap_k[TM_COUNT];
  CUtensorMap tmap_v[TM_COUNT];
  const uint16_t *win_k, *win_v, *bank_k, *bank_v, *pend_k, *pend_v;
  const int32_t* meta;
  const int32_t* seq_ids;
  int s_max, L, layer;
  const uint16_t* q_swa;  // [nq][16][256], normed and rotated
  const uint16_t* q_rma;  // [nq][16][256]
  int nq;                 // query b = the token of sequence seq_ids[b] at its meta pos
  int splits;
  float* part_o;   // [items][4][256]
  float* part_ml;  // [items][4][2]
  // direct output (splits == 1): the CTA that reads a (query, group)'s SWA item
  // reads its RMA item next and writes the final result itself
  int direct;
  float *o_swa, *o_rma;  // FP32 [nq][16][256] (standalone read), or
  uint16_t* o_sum;       // BF16 [nq][4096] = bf16(o_swa + o_rma) (layer path)
  int rma_off;           // the RMA read sees no records (o_rma = 0)
  int pool;              // pooled layout: the RMA read takes a group's 1280 pool slots
  const int32_t* bank_pos;  // pooled layout: per slot the source position (free: FREE_POS)
  int* sched;            // work counter, 0 at launch (the CTAs take units from it)
  int32_t* err;
};

// One merge's move list (the layer calls' two-launch commit): winner w moves
// from pending slot src[w] to bank slot dst[w]; n = 0 when nothing commits.
// In the pooled layout: src[0..n) are the pool slots of the evicted records
// and dst[0..256) the next block's slot list; commit = 1 when the merge ran.
struct MovePlan {
  int32_t n;
  int32_t commit;
  int16_t src[256];
  int16_t dst[256];
};

struct CommitParams {
  uint16_t *bank_k, *bank_v;
  const uint16_t *pend_k, *pend_v;
  float* bank_score;
  const float* pend_score;
  int32_t* bank_pos;
  const int32_t* pend_pos;
  const int32_t* meta;
  const int32_t* seq_ids;  // [n], or ignored when seq_fixed >= 0 (then n == 1)
  int seq_fixed;
  int n, s_max, L;
  int layer0, nlayers;
  int p_add;         // pending records = meta.pend + p_add
  int only_if_full;  // commit only when that count is 256
  int per_block;     // sequences per block (set at launch)
  int32_t* kept;     // optional [n][nlayers][4][1024]
  int32_t* err;
  int pool;          // the pooled layout: bank_* hold 1280 slots, pend_pos the slot lists
  int32_t* slots;    // pooled layout: [s_max][L][4][256] slot lists (the state's pend_pos)
};

}  // namespace er
