/*
 * edgerock.h — C ABI of the B200 (sm_100a) SWA∥RMA hot path of EdgeRock-4B.
 *
 * What the layer is (page title, section):
 *  [F-arch] fluxbbs.com "EdgeRock-4B 开源：72 MiB 固定 KV，AIME 82.9 分",
 *           §架构：递归、局部窗口与记忆锚点三件套 — hidden 2560; the eight
 *           sliding-window layers run a 1024-position window in parallel with
 *           Rock Memory Anchors (RMA); 16 query heads over 4 KV groups, head
 *           dim 256, learned RMS-norm on q and k, RoPE on 64 of the 256 dims
 *           with base 1e7, values neither rotated nor normed; a bias-free FP32
 *           scorer 2560→256→4 gives one retention score per KV group; each
 *           group keeps its own top records, groups may share positions;
 *           candidates gather in blocks of 256 and the bank keeps 1024.
 *  [F-mem]  same page, §72 MiB 是怎么算出来的 — every part of the state has a
 *           hard capacity: 32 MiB committed anchors, 8 MiB pending block,
 *           32 MiB window, 72 MiB per sequence whatever its length.
 *  [N-rma]  neodrop.ai "内存还会跌吗？KV Cache砍掉99%，单卡吞吐飙6倍…",
 *           §三段记忆，只记值得记的 — a writer makes one candidate per token, a
 *           scorer rates it; at 256 candidates they are compared with the bank
 *           and only the 1024 best are kept, for each of the four KV groups;
 *           kept anchors are independent and never change.
 *  Readings fixed where the pages are silent: SiLU between the two scorer
 *  matmuls; the RMA read is its own softmax over committed + pending records
 *  with its own q/k/v projections, added to the SWA output before one shared
 *  o_proj; ties in the top-k go to the lower source position.
 *
 * Conventions for every entry point:
 *  - Pointers named in a signature are DEVICE pointers unless marked (host).
 *    The caller allocates and frees all memory (state, weights, inputs,
 *    outputs, workspace); the library never allocates or frees device memory
 *    itself (cuBLAS keeps its own handle memory; er_rma_score_noalloc's scratch
 *    and the library's error word are fixed device arrays) and never
 *    synchronises the stream,
 *    except er_last_device_error and er_last_call_error, which read one word
 *    back.
 *  - Work is enqueued on `stream` (a cudaStream_t; 0 = legacy default).  A
 *    layer call may also run part of its work (the commit, beside the read
 *    and o_proj) on a side stream that the library assigns to each caller
 *    stream (16 per device; past 16 caller streams, some share one), forked
 *    from and joined back to `stream` inside the call, so everything still
 *    completes in `stream` order and the call can be captured in a CUDA
 *    graph; calls on different caller streams do not wait on each other.
 *    The first layer call on a device creates that device's side streams,
 *    events and cuBLAS handle, and the first call of each kind its kernel
 *    attributes: make one such call on the device before capturing on it.
 *  - Those per-device resources, and the device addresses of the library's
 *    fixed device arrays, are made once per device and process and are not
 *    made again after cudaDeviceReset: do not call the library on a device
 *    that was reset in the same process.
 *  - A workspace (`ws`) is a call's scratch; in the layer calls it also holds
 *    the read's work counter and the commit's move lists, which live from the
 *    call's first kernel to its last.  Calls that may run at the same time
 *    (other streams, other threads) need workspaces of their own; calls
 *    ordered on one stream can share one.
 *  - Return value: ER_OK, or a negative ER_E* code.  Host-side argument checks
 *    happen before anything is enqueued; a failed check enqueues nothing.
 *    Conditions only the device can see (a sequence id out of range, a full
 *    pending block, a prefill chunk crossing the block boundary, a bounded
 *    wait that gave up) skip the affected work and record the first such
 *    code in a device error word: the state's (read with
 *    er_last_device_error), or, for the calls that take no state, the
 *    library's own word (read with er_last_call_error).  No kernel traps.
 *  - BF16 values are raw bfloat16 bit patterns (er_bf16).
 */
#ifndef EDGEROCK_H
#define EDGEROCK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t er_bf16;
typedef struct CUstream_st* er_stream_t; /* same type as cudaStream_t */

/* Layer shape [F-arch], capacities [F-mem]/[N-rma]. */
#define ER_HIDDEN 2560
#define ER_Q_HEADS 16
#define ER_KV_GROUPS 4
#define ER_HEADS_PER_GROUP 4
#define ER_HEAD_DIM 256
#define ER_MAX_LAYERS 8
#define ER_WINDOW 1024
#define ER_BANK 1024
#define ER_PENDING 256
#define ER_ROPE_DIMS 64
#define ER_SCORE_HIDDEN 256
#define ER_QKV_ROWS 12288 /* 4096 + 1024 + 1024 (SWA) + 4096 + 1024 + 1024 (RMA) */
#define ER_QKV_SCORE_ROWS 13056 /* ER_QKV_ROWS + the three BF16 terms of W1 (3 x 256) */
#define ER_O_IN 4096      /* 16 heads x 256 */

enum {
  ER_OK = 0,
  ER_EINVAL = -1,    /* bad argument (null pointer, size or index out of range) */
  ER_ECAPACITY = -2, /* pending block full, batch above capacity, workspace too small */
  ER_ECUDA = -3,     /* a CUDA launch or runtime call failed */
  ER_EDEVICE = -4,   /* returned by er_last_device_error when the device word is set */
  ER_ETIMEOUT = -5   /* device word only: a bounded wait inside a kernel gave up */
};

/* Per-sequence fixed-capacity state, carved out of ONE caller allocation by
 * er_state_carve.  Layouts ([seq] is the state row, not a batch index):
 *   win_k, win_v   BF16  [s_max][n_layers][4][1024][256]  ring: position t in slot t % 1024
 *   bank_k, bank_v BF16  [s_max][n_layers][4][1024][256]  committed anchors, slots [0, bank_count)
 *   pend_k, pend_v BF16  [s_max][n_layers][4][256][256]   pending block, slots [0, pend_count)
 *   bank_score     FP32  [s_max][n_layers][4][1024]       score of each committed record
 *   pend_score     FP32  [s_max][n_layers][4][256]
 *   bank_pos       INT32 [s_max][n_layers][4][1024]       source position of each record
 *   pend_pos       INT32 [s_max][n_layers][4][256]
 *   meta           INT32 [s_max][4] = {pos, pend_count, bank_count, 0}; pos is the
 *                  position of the next token; the counts are shared by every
 *                  layer and group because every token appends to each.
 *   dev_error      INT32 [4]: first device-side error code (0 = none).
 * K rows are stored already RMS-normed and rotated at their source position.
 */
typedef struct er_state {
  er_bf16 *win_k, *win_v, *bank_k, *bank_v, *pend_k, *pend_v;
  float *bank_score, *pend_score;
  int32_t *bank_pos, *pend_pos;
  int32_t *meta;
  int32_t *dev_error;
  int32_t s_max;
  int32_t n_layers;
  int32_t pool; /* 1: the pooled anchor layout (ER_STATE_POOL), 0: the layout above */
} er_state;

/* The pooled anchor layout (a variant of the commit that moves no K/V row).
 * The committed bank and the pending block of a group share ONE pool of 1280
 * rows, with the same K/V bytes as bank + pending:
 *   bank_k, bank_v BF16  [s_max][n_layers][4][1280][256]  pool rows
 *   bank_score     FP32  [s_max][n_layers][4][1280]       score of the record in a slot
 *   bank_pos       INT32 [s_max][n_layers][4][1280]       its source position, or
 *                                                         0x7FFFFFFF for a free slot
 *   pend_pos       INT32 [s_max][n_layers][4][256]        slot list: pending record j
 *                                                         of the block lives in pool
 *                                                         slot pend_pos[j]
 *   pend_k, pend_v, pend_score: NULL.
 * A record never moves once written.  A commit ranks the records of the
 * occupied slots exactly as in the other layout and keeps the same records
 * [F-arch], [N-rma]; it marks the slots of the evicted ones free and lists
 * the 256 lowest free slots (ascending) as the next block's slots.  The reads
 * take the whole pool of a group and skip free slots and records a query may
 * not see (source position above the query's).  meta is unchanged. */
#define ER_STATE_POOL 1u

/* One SWA∥RMA layer's weights (device, caller-owned), nn.Linear layout [out][in]:
 *   w_qkv BF16 [12288][2560]: rows q_swa 0..4095 | k_swa 4096..5119 | v_swa 5120..6143 |
 *                             q_rma 6144..10239 | k_rma 10240..11263 | v_rma 11264..12287
 *   w_o   BF16 [2560][4096]  shared o_proj
 *   q_norm_swa, k_norm_swa, q_norm_rma, k_norm_rma: BF16 [256] RMS-norm gains
 *                             (one per head dim, shared by all heads of the branch)
 *   w1    FP32 [256][2560], w2 FP32 [4][256]: the scorer, bias-free.
 *   w1_split (optional, may be NULL): BF16 [3][256][2560], w1 written as three
 *                             BF16 terms by er_score_split_w1 (prepared once per
 *                             weight set); NULL makes every scorer call split
 *                             w1 again into its workspace.
 *   w_qkv_score (optional, may be NULL): BF16 [13056][2560], rows 0..12287 equal
 *                             to w_qkv and rows 12288..13055 the three W1 terms in
 *                             w1_split's layout (er_prepare_qkv_score writes it).
 *                             When set, the layer calls take a1 and the W1·x
 *                             product of a3 from ONE GEMM over it (FP32 output;
 *                             the projections are then rounded to BF16, the same
 *                             values a BF16-output GEMM gives) and apply SiLU and
 *                             W2 in the norm/RoPE kernel, so no separate scorer
 *                             launch runs (calls with ER_FLAG_RMA_OFF score
 *                             nothing and project from w_qkv with BF16 output).
 *                             w_qkv, w1 and w1_split must still be
 *                             valid (the standalone er_rma_score reads them); a
 *                             caller can point w_qkv and w1_split into this
 *                             buffer so the layer holds one copy. */
typedef struct er_layer_weights {
  const er_bf16* w_qkv;
  const er_bf16* w_o;
  const er_bf16 *q_norm_swa, *k_norm_swa, *q_norm_rma, *k_norm_rma;
  const float* w1;
  const float* w2;
  const er_bf16* w1_split;
  const er_bf16* w_qkv_score;
} er_layer_weights;

/* ---------------------------------------------------------------- state */

/* Bytes er_state_carve needs for s_max (1..4096) sequences of n_layers (1..8) layers:
 * 72 MiB of K/V per sequence at 8 layers [F-mem], plus scores, positions,
 * metadata and alignment.  Returns 0 on bad arguments.  Host-only. */
size_t er_state_bytes(int32_t s_max, int32_t n_layers);

/* Fills *out with pointers into [base, base+bytes) (device memory, caller
 * owned, 256-byte aligned).  Touches no memory.  ER_EINVAL if bytes is too
 * small, base is unaligned, or sizes are out of range. */
int er_state_carve(void* base, size_t bytes, int32_t s_max, int32_t n_layers, er_state* out);

/* The same with layout flags: 0, or ER_STATE_POOL for the pooled anchor layout
 * (other bits: 0 bytes / ER_EINVAL). */
size_t er_state_bytes_ex(int32_t s_max, int32_t n_layers, uint32_t flags);
int er_state_carve_ex(void* base, size_t bytes, int32_t s_max, int32_t n_layers, uint32_t flags,
                      er_state* out);

/* Empties the listed sequences: meta := {0, 0, 0, 0}, i.e. the stream start
 * of [F-mem]: a window, bank and pending block of fixed capacity, all empty.
 * In the pooled layout it also marks every pool slot free and lists slots
 * 0..255 for the first block.  seq_ids: device int32 [n].  Row contents are
 * left as they are (unread until written). */
int er_state_init(const er_state* st, const int32_t* seq_ids, int32_t n, er_stream_t stream);

/* End of one step of T tokens for the listed sequences, after every layer's
 * call [N-rma]: every token left one candidate per group in the pending
 * block, and a block of 256 is merged into a bank of at most 1024.  So:
 * pos += T; pend_count += T, and a block that reached 256 (which every layer
 * has committed) empties: pend_count := 0, bank_count := min(1024,
 * bank_count + 256).  T in 1..256. */
int er_advance(const er_state* st, const int32_t* seq_ids, int32_t n, int32_t T,
               er_stream_t stream);

/* Flags of the *_ex calls.
 *   ER_FLAG_RMA_OFF: the pages' ablation with every RMA module switched off
 *   at inference time, recurrent layers and local attention kept (fluxbbs.com
 *   "EdgeRock-4B 开源：72 MiB 固定 KV" §消融：关掉 RMA 会发生什么; neodrop.ai
 *   §三段记忆，只记值得记的).  The layer calls then take o_rma = 0 and skip the score, the
 *   pending append and the commit; er_advance_ex moves only the position, so
 *   the anchor bank, the pending block and their counters stay as they were.
 *   Use it for every layer of a step and for that step's advance. */
#define ER_FLAG_RMA_OFF 1u

/* er_advance with flags (0 or ER_FLAG_RMA_OFF; other bits: ER_EINVAL). */
int er_advance_ex(const er_state* st, const int32_t* seq_ids, int32_t n, int32_t T,
                  uint32_t flags, er_stream_t stream);

/* Copies the state's device error word to *code (host) and clears it;
 * synchronises `stream`.  Returns ER_OK when the word was 0, else ER_EDEVICE.
 * (The capacities that the device checks are those of [F-mem]: a full
 * pending block or a chunk crossing it reports ER_ECAPACITY here.) */
int er_last_device_error(const er_state* st, int32_t* code, er_stream_t stream);

/* The same for the library's own error word, which the calls that take no
 * state record into: er_rma_score (and er_rma_score_ex with dev_error NULL),
 * er_rma_score_noalloc, and er_wait_selftest with st NULL.  One word per
 * device, shared by every such call in the process: it holds the first code
 * recorded since the last read.  Synchronises `stream`. */
int er_last_call_error(int32_t* code, er_stream_t stream);

/* Diagnostic for the failure path, no part of the method: one thread waits on
 * a fresh mbarrier (one expected arrival) through the bounded wait that every
 * kernel of the library uses for its pipeline barriers.  arrive = 1 completes
 * the barrier first (the wait returns at once, nothing is recorded); arrive =
 * 0 leaves it incomplete, so the wait gives up after ~2 s and records
 * ER_ETIMEOUT in st's device error word (st NULL: the library's own word, read
 * by er_last_call_error); the kernel then exits and the context stays usable.
 * ER_EINVAL for another arrive value. */
int er_wait_selftest(const er_state* st, int32_t arrive, er_stream_t stream);

/* ------------------------------------------------------- hot-path steps */

/* a2 — RMS-norm with gain, then rotary embedding of dims [0, 64) at each
 * row's position [F-arch]: y = x / sqrt(mean(x^2) + 1e-6) * gain, then for
 * i < 32 the pair (i, i+32) turns by pos * 1e7^(-2i/64).  x, y: BF16
 * [n_rows][256] (may alias); gain: BF16 [256]; pos: INT32 [n_rows]. */
int er_qk_norm_rope(const er_bf16* x, er_bf16* y, int64_t n_rows, const er_bf16* gain,
                    const int32_t* pos, er_stream_t stream);

/* a1 / a6 — a projection of the layer's shapes on its own [F-arch]: y = x · wᵀ
 * with x BF16 [T][K] and w BF16 [F][K] (row-major, the nn.Linear layout), BF16
 * products accumulated in FP32 on the tensor cores by this library's own
 * kernels: up to 32 tokens a weight-streaming kernel (mma.m16n8k16 tiles, the
 * one the layer calls use for decode batches of up to 8 sequences), above
 * that a tcgen05 GEMM (CTA pairs, work split over all SMs along K); y is BF16
 * (y_fp32 = 0, round to nearest even) or FP32 (y_fp32 = 1), [T][ldy] with
 * ldy >= F.  The shapes are those of x·W_qkvᵀ (F = 12288, or 13056 with the
 * scorer's W1 terms, K = 2560) and of the shared o_proj (F = 2560, K = 4096).
 * (For more than 8 tokens the layer calls take these products from cuBLAS,
 * measured faster at their token counts.)  F a multiple of 256, K of
 * 64, T >= 0; x, w, y 16-byte aligned; ws 256-byte aligned, at least
 * er_linear_workspace_bytes(T, F, K) (0 for bad sizes), reusable by calls
 * ordered on one stream.  The summation order is fixed for given (T, F, K):
 * the same inputs give the same bits.  A bounded wait that gives up records
 * ER_ETIMEOUT in *dev_error (NULL: the library's own word). */
size_t er_linear_workspace_bytes(int32_t T, int32_t F, int32_t K);
int er_linear(const er_bf16* x, int32_t T, const er_bf16* w, int32_t F, int32_t K, void* y,
              int32_t y_fp32, int32_t ldy, void* ws, size_t ws_bytes, int32_t* dev_error,
              er_stream_t stream);

/* a3 — retention scores [F-arch], [N-rma]: s = W2 · SiLU(W1 · x) with FP32
 * accuracy: W1 is taken as three BF16 terms hi + mid + lo (residual below
 * 2^-24 |W1|), each product with the BF16 x is exact and accumulates in FP32;
 * partial sums are added in a fixed order (deterministic).
 * x: BF16 [n][2560]; s: FP32 [n][4] (one per KV group); n may be 0.
 * ws: scratch of er_score_workspace_bytes(n) bytes (room for the W1 terms when
 * w->w1_split is NULL, and the partial scores; contents on return are
 * unspecified). */
size_t er_score_workspace_bytes(int32_t n);

/* Writes w1 (FP32 [256][2560]) as three BF16 terms hi, mid, lo into terms
 * (BF16 [3][256][2560], caller-owned device memory, 16-byte aligned): hi =
 * bf16(w1), mid = bf16(w1 - hi), lo = bf16(w1 - hi - mid).  The result is the
 * optional er_layer_weights.w1_split. */
int er_score_split_w1(const float* w1, er_bf16* terms, er_stream_t stream);

/* Builds er_layer_weights.w_qkv_score: copies w_qkv (BF16 [12288][2560]) into
 * rows 0..12287 of out (BF16 [13056][2560], caller-owned device memory,
 * 16-byte aligned, not overlapping w_qkv) and writes w1's three BF16 terms
 * (as er_score_split_w1) into rows 12288..13055.  Stream-ordered; ER_EINVAL
 * on NULL or unaligned pointers. */
int er_prepare_qkv_score(const er_bf16* w_qkv, const float* w1, er_bf16* out,
                         er_stream_t stream);
int er_rma_score(const er_layer_weights* w, const er_bf16* x, int32_t n, float* s, void* ws,
                 size_t ws_bytes, er_stream_t stream);

/* er_rma_score with an explicit device error word: a bounded wait inside the
 * scorer that gives up (its scores are then not valid) records ER_ETIMEOUT in
 * *dev_error (a caller-owned device int32, e.g. a state's dev_error; NULL
 * means the library's own word, as for er_rma_score). */
int er_rma_score_ex(const er_layer_weights* w, const er_bf16* x, int32_t n, float* s, void* ws,
                    size_t ws_bytes, int32_t* dev_error, er_stream_t stream);

/* a3 without caller scratch.  The pages describe nothing like this; it exists
 * for callers that cannot hand the library any device memory beyond the
 * inputs and outputs, so cannot provide er_rma_score's workspace: for example
 * a host program whose device memory is all owned by another framework's
 * caching allocator, or a plugin interface that only receives tensor pointers
 * and may not call cudaMalloc itself.  Same result as er_rma_score.
 *  - Its scratch (W1 split into three BF16 terms, 3.75 MiB, when w->w1_split
 *    is NULL, plus 4 partial scores per token and group, 16 KiB at 256
 *    tokens) lives in one fixed 4 MiB device array inside the library, which
 *    every GPU that loads the library holds until the process exits.
 *  - n above ER_SCORE_NOALLOC_MAX_TOKENS returns ER_ECAPACITY; nothing runs.
 *  - The first call on a device (with that device current) looks the array's
 *    device address up with cudaGetSymbolAddress and caches it; make that
 *    first call before any stream capture on the device.
 *  - Nothing is allocated or freed: no cudaMalloc, no cudaFree.
 *  - Every call shares the one array: calls whose work overlaps on the GPU
 *    (different streams, or different threads on one device) race and give
 *    wrong scores; serialise them.  The array keeps the last call's contents;
 *    no part of it needs to start at zero.
 *  - A bounded wait that gives up records ER_ETIMEOUT in the library's own
 *    error word (a fixed device word too), read with er_last_call_error. */
#define ER_SCORE_NOALLOC_MAX_TOKENS 256
int er_rma_score_noalloc(const er_layer_weights* w, const er_bf16* x, int32_t n, float* s,
                         er_stream_t stream);

/* a4 — appends one candidate record per KV group for each listed sequence at
 * its pend_count slot of `layer` [N-rma]: k, v BF16 [n][4][256] (k already
 * normed and rotated), s FP32 [n][4], pos INT32 [n].  Metadata is not
 * changed (er_advance does that once per step).  A sequence whose block is
 * already full is skipped and records ER_ECAPACITY on the device. */
int er_rma_append_pending(const er_state* st, int32_t layer, const int32_t* seq_ids, int32_t n,
                          const er_bf16* k, const er_bf16* v, const float* s,
                          const int32_t* pos, er_stream_t stream);

/* a7 — commit [F-arch], [N-rma]: for each listed sequence and each KV group
 * independently, the bank_count committed and pend_count pending records are
 * ranked by (score descending, source position ascending; -0 ranks as +0,
 * NaN below every number) and the top min(1024, bank_count + pend_count)
 * stay.  Surviving anchors do not move; evicted bank slots in ascending order,
 * then slots bank_count, bank_count+1, ..., receive the pending winners in
 * ascending pending order.
 *   layer >= 0: that layer only; metadata untouched (a decode step commits
 *               each layer, then er_advance empties the block).
 *   layer == -1: every layer, then pend_count := 0 and
 *               bank_count := min(1024, bank_count + pend_count).
 *   kept (optional, may be NULL): INT32 [n][layers][4][1024], the kept
 *   records in rank order as indices 0..1023 (bank slot) / 1024+j (pending
 *   j), -1 padded; `layers` is n_layers for layer == -1, else 1. */
int er_rma_commit(const er_state* st, int32_t layer, const int32_t* seq_ids, int32_t n,
                  int32_t* kept, er_stream_t stream);

/* a5 — the two reads of a decode step, for B sequences whose current token
 * (position pos) has already been written to the window and appended at
 * pending slot pend_count: for head h of group h/4,
 *   o_swa = softmax(q_swa·Kᵀ/16)·V over window positions [pos-1023, pos];
 *   o_rma = softmax(q_rma·Kᵀ/16)·V over bank slots [0, bank_count) and
 *           pending slots [0, pend_count]  (o = 0 over an empty list).
 * q_swa, q_rma: BF16 [B][16][256] (normed, rotated); o_swa, o_rma: FP32
 * [B][16][256].  ws: workspace of er_attend_workspace_bytes(B) bytes. */
size_t er_attend_workspace_bytes(int32_t B);
int er_swa_rma_attend(const er_state* st, int32_t layer, const int32_t* seq_ids, int32_t B,
                      const er_bf16* q_swa, const er_bf16* q_rma, float* o_swa, float* o_rma,
                      void* ws, size_t ws_bytes, er_stream_t stream);

/* a1–a7 — one decode step of one layer for B sequences (one token each at
 * its meta pos), the SWA∥RMA layer of [F-arch] with the memory rules of
 * [N-rma]: q/k/v projections of both branches, norm + RoPE, scores,
 * window write (slot pos % 1024), pending append, the two reads,
 * out = W_o · bf16(o_swa + o_rma), and the commit of this layer for every
 * sequence whose block this token fills (pend_count + 1 == 256), decided on
 * the device.  x, out: BF16 [B][2560].  ws: er_decode_workspace_bytes(B).
 * A step is one call per layer followed by one er_advance(T=1). */
size_t er_decode_workspace_bytes(int32_t B);
int er_swa_rma_decode(const er_state* st, const er_layer_weights* w, int32_t layer,
                      const int32_t* seq_ids, int32_t B, const er_bf16* x, er_bf16* out,
                      void* ws, size_t ws_bytes, er_stream_t stream);

/* a8 — a prefill chunk of T tokens (1..256) of one sequence (state row
 * seq_id, a host int) at positions pos..pos+T-1: the layer of [F-arch] run
 * causally over a chunk, each token appending its candidate [N-rma] within
 * the capacities of [F-mem].  Requires
 * pend_count + T <= 256 (checked on the device).  Token i reads, causally,
 * window positions [t-1023, t] (old ring entries and the chunk's own tokens)
 * and the bank plus pending slots [0, pend_count + i]; the chunk enters the
 * ring after every read; the layer commits if the chunk fills the block.
 * x, out: BF16 [T][2560]; ws: er_prefill_workspace_bytes(T).  Follow the
 * chunk's calls for every layer with er_advance(T). */
size_t er_prefill_workspace_bytes(int32_t T);
int er_swa_rma_prefill_chunk(const er_state* st, const er_layer_weights* w, int32_t layer,
                             int32_t seq_id, const er_bf16* x, int32_t T, er_bf16* out,
                             void* ws, size_t ws_bytes, er_stream_t stream);

/* The two layer calls with flags (0 or ER_FLAG_RMA_OFF; other bits:
 * ER_EINVAL).  With ER_FLAG_RMA_OFF: out = W_o · bf16(o_swa), the window is
 * written and read as usual, and the RMA memory (scores, pending block, bank,
 * their counters) is neither read by the attention nor written; a prefill
 * chunk still obeys pend_count + T <= 256.  Same workspace sizes.  The
 * flag-less calls above are these with flags = 0. */
int er_swa_rma_decode_ex(const er_state* st, const er_layer_weights* w, int32_t layer,
                         const int32_t* seq_ids, int32_t B, const er_bf16* x, er_bf16* out,
                         void* ws, size_t ws_bytes, uint32_t flags, er_stream_t stream);
int er_swa_rma_prefill_chunk_ex(const er_state* st, const er_layer_weights* w, int32_t layer,
                                int32_t seq_id, const er_bf16* x, int32_t T, er_bf16* out,
                                void* ws, size_t ws_bytes, uint32_t flags, er_stream_t stream);

/* ------------------------------------------------------ instrumentation */

/* Human-readable name of an ER_* code (static string). */
const char* er_error_string(int code);

/* Number of kernels this library has launched since load (all threads). */
uint64_t er_launch_count(void);

/* When enabled, launches of the read kernels (the a5 decode read and the a8
 * prefill read) are bracketed by CUDA events on their own stream;
 * er_profile_read returns the summed milliseconds and the number of timed
 * launches since the last reset (it synchronises the events).
 * Host-side bookkeeping only; not thread-safe. */
int er_profile_enable(int enable);
int er_profile_read(double* ms_total, int64_t* launches, int reset);

#ifdef __cplusplus
}
#endif

#endif /* EDGEROCK_H */
