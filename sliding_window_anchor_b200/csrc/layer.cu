// layer.cu — one SWA∥RMA layer step: decode (a1–a7) and a prefill chunk (a8).
//
// Order of a decode step (the reading fixed for this library, consistent with
// EdgeRock-4B 开源：72 MiB 固定 KV §架构 and neodrop.ai §三段记忆): project, score,
// norm + RoPE, write the window slot and append the pending record, read both
// branches, o_proj, then commit this layer for sequences whose block the token
// filled.  A prefill chunk writes its window rows only after every token read,
// because the chunk's early tokens still see ring positions its late tokens
// would overwrite (the prefill read kernel's second launch moves them).
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "params.cuh"

namespace er {

int gemm_bf16_xwt(const uint16_t* X, const uint16_t* W, uint16_t* Y, int M, int N, int K,
                  cudaStream_t st);
int gemm_bf16_xwt_f32(const uint16_t* X, const uint16_t* W, float* Y, int M, int N, int K,
                      int ldy, cudaStream_t st);
int launch_gemv(const uint16_t* X, int T, const uint16_t* W, int F, int K, void* Y, bool yf32,
                int ldy, cudaStream_t st);
int launch_score(const float* w1, const uint16_t* w1_split, const float* w2, const uint16_t* x,
                 int n, float* s, void* scratch, int32_t* err, cudaStream_t st);
size_t score_scratch_bytes(int n);
const float* score_partials(const void* scratch, int n);
int launch_post_proj(const PostParams& P, bool rma_off, cudaStream_t st);
int launch_attend(const AttendParams& P, float* o_swa, float* o_rma, uint16_t* o_sum,
                  bool zero_sched, cudaStream_t st);
size_t commit_plan_bytes(int n, int nlayers);
int launch_commit_plan(const CommitParams& P, MovePlan* plan, cudaStream_t st);
int launch_commit_move(const CommitParams& P, const MovePlan* plan, cudaStream_t st);
size_t attend_part_floats(int nq);
size_t attend_ml_floats(int nq);
size_t prefill_out_floats(int T);
int launch_prefill_attend(const er_state* st, int layer, int seq, int T, const uint16_t* q_swa,
                          const uint16_t* q_rma, const uint16_t* chunk_k,
                          const uint16_t* chunk_v, float* out, uint16_t* o_sum, bool rma_off,
                          cudaStream_t stream);

}  // namespace er

namespace er {
namespace {

// A batch of at most this many tokens streams the weights through the
// library's own GEMV kernel (the product is bound by reading the weights);
// larger ones go to cuBLAS.
constexpr int kGemvMaxTokens = 8;

// Y[M,N] = X[M,K] · W[N,K]ᵀ, BF16 out (row stride N).
int project_bf16(const uint16_t* X, const uint16_t* W, uint16_t* Y, int M, int N, int K,
                 cudaStream_t st) {
  if (M <= kGemvMaxTokens) return launch_gemv(X, M, W, N, K, Y, false, N, st);
  return gemm_bf16_xwt(X, W, Y, M, N, K, st);
}

// The same with FP32 out of row stride ldy.
int project_f32(const uint16_t* X, const uint16_t* W, float* Y, int M, int N, int K, int ldy,
                cudaStream_t st) {
  if (M <= kGemvMaxTokens) return launch_gemv(X, M, W, N, K, Y, true, ldy, st);
  return gemm_bf16_xwt_f32(X, W, Y, M, N, K, ldy, st);
}

struct LayerWs {
  void* proj;  // BF16 [nq][12288], or FP32 [nq][13056] with the fused weights
  unsigned char* score_scratch;
  uint16_t *q_swa, *q_rma;
  uint16_t *chunk_k, *chunk_v;
  float *part_o, *part_ml;  // decode: split partials of the reads
  int* sched;                // decode: the read's work counter
  float* pf_out;             // prefill: FP32 branch outputs [2][T][4096]
  uint16_t* o_sum;
  MovePlan* plan;            // the commit's move lists, one per (sequence, group)
  size_t bytes;
};

LayerWs carve_ws(void* base, int nq, bool prefill) {
  Carver c(base);
  LayerWs w;
  w.proj = c.take<float>((size_t)nq * QKVS);
  w.score_scratch = c.take<unsigned char>(score_scratch_bytes(nq));
  w.q_swa = c.take<uint16_t>((size_t)nq * NH * D);
  w.q_rma = c.take<uint16_t>((size_t)nq * NH * D);
  w.chunk_k = prefill ? c.take<uint16_t>((size_t)NG * nq * D) : nullptr;
  w.chunk_v = prefill ? c.take<uint16_t>((size_t)NG * nq * D) : nullptr;
  w.part_o = prefill ? nullptr : c.take<float>(attend_part_floats(nq));
  w.part_ml = prefill ? nullptr : c.take<float>(attend_ml_floats(nq));
  w.sched = prefill ? nullptr : c.take<int>(1);
  w.pf_out = prefill ? c.take<float>(prefill_out_floats(nq)) : nullptr;
  w.o_sum = c.take<uint16_t>((size_t)nq * OIN);
  w.plan = reinterpret_cast<MovePlan*>(
      c.take<unsigned char>(commit_plan_bytes(prefill ? 1 : nq, 1)));
  w.bytes = c.used();
  return w;
}

// Steps of a layer call that run beside other work on a side stream: the
// commit's planning beside the read (it reads only scores and positions, which
// the read leaves alone) and its row moves beside o_proj (anchor rows vs the
// read output), and, in a prefill chunk with unprepared weights, the scorer
// beside the q/k/v projection (both only read x).  Each caller stream has a
// side stream and fork/join events of its own, taken between forks and a join
// on the caller's stream, so a call's work still completes in the caller's
// stream order (and stays capturable), and calls on different caller streams
// share nothing: no lock is held across them and no stream waits on another
// caller's work.
struct Side {
  std::mutex mu;  // the events are re-recorded by every call that uses this entry
  cudaStream_t caller = nullptr;
  bool bound = false;
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, fork2 = nullptr, join = nullptr;
};
constexpr int kSidesPerDevice = 16;
struct DeviceSides {
  bool made = false;
  Side side[kSidesPerDevice];
};
DeviceSides g_sides[64];
std::mutex g_side_mu;

// The side resources of `caller` on the current device.  The device's pool is
// made by its first layer call (before any capture); later calls only bind a
// caller stream to a free entry, or, past 16 caller streams, share one.
Side* side_for(cudaStream_t caller) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_side_mu);
  DeviceSides& ds = g_sides[dev];
  if (!ds.made) {
    for (Side& sd : ds.side)
      if (cudaStreamCreateWithFlags(&sd.stream, cudaStreamNonBlocking) != cudaSuccess ||
          cudaEventCreateWithFlags(&sd.fork, cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&sd.fork2, cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&sd.join, cudaEventDisableTiming) != cudaSuccess)
        return nullptr;
    ds.made = true;
  }
  for (Side& sd : ds.side)
    if (sd.bound && sd.caller == caller) return &sd;
  for (Side& sd : ds.side)
    if (!sd.bound) {
      sd.bound = true;
      sd.caller = caller;
      return &sd;
    }
  return &ds.side[(reinterpret_cast<uintptr_t>(caller) >> 4) % kSidesPerDevice];
}

bool weights_ok(const er_layer_weights* w) {
  return w && w->w_qkv && w->w_o && w->q_norm_swa && w->k_norm_swa && w->q_norm_rma &&
         w->k_norm_rma && w->w1 && w->w2 && aligned16(w->w_qkv) && aligned16(w->w_o) &&
         aligned16(w->q_norm_swa) && aligned16(w->k_norm_swa) && aligned16(w->q_norm_rma) &&
         aligned16(w->k_norm_rma) && aligned16(w->w1) && aligned16(w->w2) &&
         (!w->w1_split || aligned16(w->w1_split)) &&
         (!w->w_qkv_score || aligned16(w->w_qkv_score));
}

int run_layer(const er_state* st, const er_layer_weights* w, int layer, const int32_t* seq_ids,
              int seq_fixed, int nq, const uint16_t* x, uint16_t* out, void* ws, size_t ws_bytes,
              uint32_t flags, cudaStream_t s) {
  const bool prefill = seq_fixed >= 0;
  const bool rma_off = (flags & ER_FLAG_RMA_OFF) != 0;
  LayerWs W = carve_ws(ws, nq, prefill);
  if (ws_bytes < W.bytes) return ER_ECAPACITY;
  int rc;
  Side* sd = side_for(s);
  if (!sd) return ER_ECUDA;
  // with the RMA off nothing is scored: the plain BF16 projection is cheaper
  const bool fused = w->w_qkv_score != nullptr && !rma_off;
  uint16_t* proj_bf = static_cast<uint16_t*>(W.proj);
  float* proj_f = static_cast<float*>(W.proj);
  if (fused) {
    // a1 and a3's W1·x in one GEMM, FP32 out
    if ((rc = project_f32(x, w->w_qkv_score, proj_f, nq, QKVS, HID, QKVS, s)) != ER_OK)
      return rc;
  } else if (rma_off) {
    // a1: all six projections in one GEMM
    if ((rc = project_bf16(x, w->w_qkv, proj_bf, nq, QKV, HID, s)) != ER_OK) return rc;
  } else if (!prefill) {
    // a1, then a3 (FP32 scores; the partials stay in the scratch, k_post_proj
    // adds them).  Measured: beside a batch's a1 GEMM, which fills the GPU, the
    // scorer slowed the decode step, so here they run in turn.
    if ((rc = project_bf16(x, w->w_qkv, proj_bf, nq, QKV, HID, s)) != ER_OK) return rc;
    if ((rc = launch_score(w->w1, w->w1_split, w->w2, x, nq, nullptr, W.score_scratch,
                           st->dev_error, s)) != ER_OK)
      return rc;
  } else {
    // a prefill chunk: a3 on the side stream beside a1 (both read only x)
    std::lock_guard<std::mutex> lock(sd->mu);  // the events are re-recorded by every call
    if (cudaEventRecord(sd->fork, s) != cudaSuccess ||
        cudaStreamWaitEvent(sd->stream, sd->fork, 0) != cudaSuccess)
      return ER_ECUDA;
    const int rc_score = launch_score(w->w1, w->w1_split, w->w2, x, nq, nullptr,
                                      W.score_scratch, st->dev_error, sd->stream);
    const int rc_proj = project_bf16(x, w->w_qkv, proj_bf, nq, QKV, HID, s);
    if (cudaEventRecord(sd->join, sd->stream) != cudaSuccess ||
        cudaStreamWaitEvent(s, sd->join, 0) != cudaSuccess)
      return ER_ECUDA;
    if ((rc = rc_score != ER_OK ? rc_score : rc_proj) != ER_OK) return rc;
  }
  // a2 + a4: norm/RoPE, window write (decode) or chunk rows (prefill), pending append
  PostParams pp{};
  pp.proj = fused ? nullptr : proj_bf;
  pp.proj_f32 = fused ? proj_f : nullptr;
  pp.s_part = fused ? nullptr : score_partials(W.score_scratch, nq);
  pp.w2 = w->w2;
  pp.nq = nq;
  pp.gq_swa = w->q_norm_swa; pp.gk_swa = w->k_norm_swa;
  pp.gq_rma = w->q_norm_rma; pp.gk_rma = w->k_norm_rma;
  pp.q_swa = W.q_swa; pp.q_rma = W.q_rma;
  pp.win_k = st->win_k; pp.win_v = st->win_v; pp.pend_k = st->pend_k; pp.pend_v = st->pend_v;
  pp.pend_score = st->pend_score; pp.pend_pos = st->pend_pos;
  pp.pool = st->pool; pp.bank_k = st->bank_k; pp.bank_v = st->bank_v;
  pp.bank_score = st->bank_score; pp.bank_pos = st->bank_pos;
  pp.meta = st->meta; pp.seq_ids = seq_ids; pp.s_max = st->s_max; pp.L = st->n_layers;
  pp.layer = layer; pp.prefill = prefill ? 1 : 0; pp.seq_fixed = seq_fixed;
  pp.chunk_k = W.chunk_k; pp.chunk_v = W.chunk_v; pp.err = st->dev_error;
  pp.sched_reset = W.sched;
  if ((rc = launch_post_proj(pp, rma_off, s)) != ER_OK) return rc;
  // a7, planned: the layer's commit where the block is now full (decided on the
  // device) works out its kept set and move lists on the side stream -- in a
  // decode batch while the reads run (a long, dynamically scheduled kernel that
  // absorbs the shared SMs), in a prefill chunk after its reads (short, with a
  // fixed CTA per tile: sharing SMs lengthened it) beside the combine and
  // o_proj -- and the rows move after the reads, beside a6 (the shared o_proj)
  CommitParams cp{};
  cp.bank_k = st->bank_k; cp.bank_v = st->bank_v; cp.pend_k = st->pend_k; cp.pend_v = st->pend_v;
  cp.bank_score = st->bank_score; cp.pend_score = st->pend_score;
  cp.bank_pos = st->bank_pos; cp.pend_pos = st->pend_pos;
  cp.meta = st->meta; cp.seq_ids = seq_ids; cp.seq_fixed = seq_fixed;
  cp.n = prefill ? 1 : nq; cp.s_max = st->s_max; cp.L = st->n_layers;
  cp.layer0 = layer; cp.nlayers = 1; cp.p_add = prefill ? nq : 1; cp.only_if_full = 1;
  cp.kept = nullptr; cp.err = st->dev_error;
  cp.pool = st->pool; cp.slots = st->pend_pos;
  // the events are re-recorded by every call: hold the side stream from the
  // first fork to the join
  std::unique_lock<std::mutex> lock(sd->mu, std::defer_lock);
  int rc_plan = ER_OK;
  if (!rma_off) {
    lock.lock();
    if (!prefill) {
      if (cudaEventRecord(sd->fork, s) != cudaSuccess ||
          cudaStreamWaitEvent(sd->stream, sd->fork, 0) != cudaSuccess)
        return ER_ECUDA;
      rc_plan = launch_commit_plan(cp, W.plan, sd->stream);
    }
  }
  // a5 / a8: both reads, merged into bf16(o_swa + o_rma)
  int rc_read;
  if (prefill) {
    rc_read = launch_prefill_attend(st, layer, seq_fixed, nq, W.q_swa, W.q_rma, W.chunk_k,
                                    W.chunk_v, W.pf_out, W.o_sum, rma_off, s);
  } else {
    AttendParams ap{};
    ap.win_k = st->win_k; ap.win_v = st->win_v; ap.bank_k = st->bank_k; ap.bank_v = st->bank_v;
    ap.pend_k = st->pend_k; ap.pend_v = st->pend_v; ap.meta = st->meta; ap.seq_ids = seq_ids;
    ap.s_max = st->s_max; ap.L = st->n_layers; ap.layer = layer;
    ap.q_swa = W.q_swa; ap.q_rma = W.q_rma; ap.nq = nq;
    ap.rma_off = rma_off ? 1 : 0;
    ap.pool = st->pool; ap.bank_pos = st->bank_pos;
    ap.part_o = W.part_o; ap.part_ml = W.part_ml; ap.sched = W.sched; ap.err = st->dev_error;
    // k_post_proj above zeroed the work counter
    rc_read = launch_attend(ap, nullptr, nullptr, W.o_sum, false, s);
  }
  if (rma_off)
    return rc_read != ER_OK ? rc_read : project_bf16(W.o_sum, w->w_o, out, nq, HID, OIN, s);
  // the moves wait for the reads (they overwrite evicted anchor rows); after a
  // failed launch nothing moves, but the side stream still joins
  int rc_move = ER_OK;
  bool joined_ok = cudaEventRecord(sd->fork2, s) == cudaSuccess &&
                   cudaStreamWaitEvent(sd->stream, sd->fork2, 0) == cudaSuccess;
  if (prefill && joined_ok && rc_read == ER_OK)
    rc_plan = launch_commit_plan(cp, W.plan, sd->stream);
  if (joined_ok && rc_plan == ER_OK && rc_read == ER_OK)
    rc_move = launch_commit_move(cp, W.plan, sd->stream);
  const int rc_proj =
      rc_read == ER_OK
          ? project_bf16(W.o_sum, w->w_o, out, nq, HID, OIN, s)
          : ER_OK;
  // join: the caller's stream waits for the side stream whatever happened above
  joined_ok = cudaEventRecord(sd->join, sd->stream) == cudaSuccess &&
              cudaStreamWaitEvent(s, sd->join, 0) == cudaSuccess && joined_ok;
  if (!joined_ok) return ER_ECUDA;
  for (int r : {rc_plan, rc_read, rc_move, rc_proj})
    if (r != ER_OK) return r;
  return ER_OK;
}

}  // namespace
}  // namespace er

using namespace er;

extern "C" {

size_t er_decode_workspace_bytes(int32_t B) {
  if (B < 1) return 0;
  return carve_ws(nullptr, B, false).bytes;
}

size_t er_prefill_workspace_bytes(int32_t T) {
  if (T < 1 || T > PEND) return 0;
  return carve_ws(nullptr, T, true).bytes;
}

int er_swa_rma_decode_ex(const er_state* st, const er_layer_weights* w, int32_t layer,
                         const int32_t* seq_ids, int32_t B, const er_bf16* x, er_bf16* out,
                         void* ws, size_t ws_bytes, uint32_t flags, er_stream_t stream) {
  if (!st || B < 0 || layer < 0 || layer >= st->n_layers) return ER_EINVAL;
  if (flags & ~ER_FLAG_RMA_OFF) return ER_EINVAL;
  if (B == 0) return ER_OK;
  if (B > st->s_max) return ER_ECAPACITY;
  if (!weights_ok(w) || !seq_ids || !x || !out || !ws) return ER_EINVAL;
  if (!aligned16(x) || !aligned16(out) || !aligned16(ws)) return ER_EINVAL;
  return run_layer(st, w, layer, seq_ids, -1, B, x, out, ws, ws_bytes, flags,
                   (cudaStream_t)stream);
}

int er_swa_rma_decode(const er_state* st, const er_layer_weights* w, int32_t layer,
                      const int32_t* seq_ids, int32_t B, const er_bf16* x, er_bf16* out,
                      void* ws, size_t ws_bytes, er_stream_t stream) {
  return er_swa_rma_decode_ex(st, w, layer, seq_ids, B, x, out, ws, ws_bytes, 0u, stream);
}

int er_swa_rma_prefill_chunk_ex(const er_state* st, const er_layer_weights* w, int32_t layer,
                                int32_t seq_id, const er_bf16* x, int32_t T, er_bf16* out,
                                void* ws, size_t ws_bytes, uint32_t flags, er_stream_t stream) {
  if (!st || layer < 0 || layer >= st->n_layers || T < 1 || T > PEND) return ER_EINVAL;
  if (flags & ~ER_FLAG_RMA_OFF) return ER_EINVAL;
  if (seq_id < 0 || seq_id >= st->s_max) return ER_EINVAL;
  if (!weights_ok(w) || !x || !out || !ws) return ER_EINVAL;
  if (!aligned16(x) || !aligned16(out) || !aligned16(ws)) return ER_EINVAL;
  return run_layer(st, w, layer, nullptr, seq_id, T, x, out, ws, ws_bytes, flags,
                   (cudaStream_t)stream);
}

int er_swa_rma_prefill_chunk(const er_state* st, const er_layer_weights* w, int32_t layer,
                             int32_t seq_id, const er_bf16* x, int32_t T, er_bf16* out,
                             void* ws, size_t ws_bytes, er_stream_t stream) {
  return er_swa_rma_prefill_chunk_ex(st, w, layer, seq_id, x, T, out, ws, ws_bytes, 0u, stream);
}

}  // extern "C"
