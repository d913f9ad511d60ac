// state.cu — state carving, per-sequence metadata kernels, error word,
// launch accounting and the optional timing of the read kernel.
//
// The state's capacities are hard limits (EdgeRock-4B 开源：72 MiB 固定 KV,
// §72 MiB 是怎么算出来的): window 1024, bank 1024 and pending 256 rows per
// (layer, group), K and V in BF16, so a sequence holds 72 MiB at 8 layers
// whatever its length.
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace er {

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ER_OK : ER_ECUDA;
}

int num_sms() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

namespace {

struct StateLayout {
  size_t win, bank, pend, bscore, pscore, bpos, ppos, meta, err, total;
};

// pool = 0: the bank (1024 rows per group) and the pending block (256) apart;
// pool = 1: one pool of 1280 rows per group holding both, with a 256-entry
// slot list per group in place of the pending arrays (same K/V bytes).
bool layout_of(int32_t s_max, int32_t n_layers, int pool, StateLayout* L) {
  // row indices of every array stay below 2^31 (TMA coordinates are 32-bit): 4096
  // sequences are 288 GiB of state, more than one GPU holds
  if (s_max < 1 || s_max > 4096 || n_layers < 1 || n_layers > ER_MAX_LAYERS) return false;
  Carver c(nullptr);
  size_t g = (size_t)s_max * n_layers * NG;
  const size_t bank_rows = pool ? (size_t)POOL : (size_t)BANK;
  L->win = (size_t)c.take<uint16_t>(g * WIN * D);
  c.take<uint16_t>(g * WIN * D);  // win_v
  L->bank = (size_t)c.take<uint16_t>(g * bank_rows * D);
  c.take<uint16_t>(g * bank_rows * D);  // bank_v
  L->pend = pool ? 0 : (size_t)c.take<uint16_t>(g * PEND * D);
  if (!pool) c.take<uint16_t>(g * PEND * D);  // pend_v
  L->bscore = (size_t)c.take<float>(g * bank_rows);
  L->pscore = pool ? 0 : (size_t)c.take<float>(g * PEND);
  L->bpos = (size_t)c.take<int32_t>(g * bank_rows);
  L->ppos = (size_t)c.take<int32_t>(g * PEND);  // pool: the slot list
  L->meta = (size_t)c.take<int32_t>((size_t)s_max * 4);
  L->err = (size_t)c.take<int32_t>(64);
  L->total = c.used();
  return true;
}

// The pooled layout's stream start: every pool slot free (position FREE_POS),
// the first block's records going to slots 0..255.
// A read weighs a skipped record by exactly 0, which a NaN in its V row would
// still spoil, so the V rows of the pool start at zero too.
__global__ void k_pool_init(float* score, int32_t* pos, int32_t* slots, uint16_t* bank_v,
                            const int32_t* seq_ids, int n, int s_max, int L) {
  const int b = blockIdx.x, lg = blockIdx.y;
  const int seq = seq_ids[b];
  if (seq < 0 || seq >= s_max) return;  // recorded by k_state_init
  const size_t gi = (size_t)seq * L * NG + lg;
  for (int i = threadIdx.x; i < POOL; i += blockDim.x) {
    score[gi * POOL + i] = 0.f;
    pos[gi * POOL + i] = FREE_POS;
  }
  for (int j = threadIdx.x; j < PEND; j += blockDim.x) slots[gi * PEND + j] = j;
  uint4* v = reinterpret_cast<uint4*>(bank_v + gi * POOL * D);
  for (int i = threadIdx.x; i < POOL * D / 8; i += blockDim.x) v[i] = make_uint4(0, 0, 0, 0);
}

__global__ void k_state_init(int32_t* meta, const int32_t* seq_ids, int n, int s_max,
                             int32_t* err) {
  int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= n) return;
  int s = seq_ids[b];
  if (s < 0 || s >= s_max) {
    set_dev_error(err, ER_EINVAL);
    return;
  }
  meta[s * 4 + 0] = 0;
  meta[s * 4 + 1] = 0;
  meta[s * 4 + 2] = 0;
  meta[s * 4 + 3] = 0;
}

// End of a step of T tokens: the position moves on; a block that reached 256
// was committed by every layer during the step and empties.  With the RMA
// switched off only the position moves.
__global__ void k_advance(int32_t* meta, const int32_t* seq_ids, int n, int T, int s_max,
                          int rma_off, int32_t* err) {
  int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= n) return;
  int s = seq_ids[b];
  if (s < 0 || s >= s_max) {
    set_dev_error(err, ER_EINVAL);
    return;
  }
  int32_t* m = meta + (size_t)s * 4;
  if (rma_off) {
    m[0] += T;
    return;
  }
  int pend = m[1] + T;
  if (pend > PEND) {
    set_dev_error(err, ER_ECAPACITY);
    return;
  }
  m[0] += T;
  if (pend == PEND) {
    m[1] = 0;
    m[2] = min(BANK, m[2] + PEND);
  } else {
    m[1] = pend;
  }
}

// ------------------------------------------------------ read-kernel timing
struct ProfileState {
  std::mutex mu;
  bool enabled = false;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pending;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pool;
  double ms = 0.0;
  int64_t launches = 0;
};
ProfileState& prof() {
  static ProfileState p;
  return p;
}

}  // namespace

bool profile_begin(cudaStream_t st, std::pair<cudaEvent_t, cudaEvent_t>* ev) {
  ProfileState& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.enabled) return false;
  if (p.pool.empty()) {
    cudaEvent_t a, b;
    if (cudaEventCreate(&a) != cudaSuccess) return false;
    if (cudaEventCreate(&b) != cudaSuccess) {
      cudaEventDestroy(a);
      return false;
    }
    p.pool.push_back({a, b});
  }
  *ev = p.pool.back();
  p.pool.pop_back();
  cudaEventRecord(ev->first, st);
  return true;
}

void profile_end(cudaStream_t st, std::pair<cudaEvent_t, cudaEvent_t> ev) {
  ProfileState& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  cudaEventRecord(ev.second, st);
  p.pending.push_back(ev);
}

// One thread waits on a fresh one-arrival mbarrier through the bounded wait
// every kernel of the library uses; with arrive = 0 nothing completes the
// barrier, so the wait must give up (~2 s) and record ER_ETIMEOUT.
__global__ void k_wait_selftest(int32_t* err, int arrive) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (arrive) mbar_arrive(&bar);
  mbar_wait(&bar, 0, err);
}

}  // namespace er

// The error word of the calls that take no state (the standalone scorers): a
// fixed device word inside the library, one per GPU that loads it.  Host code
// cannot hand its name to a kernel (on the host it only stands in for the
// symbol), so call_error_word() looks its device address up once per device.
static __device__ __align__(16) int32_t g_call_error[4];

namespace er {
namespace {
std::mutex g_call_error_mu;
int32_t* g_call_error_ptr[64] = {nullptr};
}  // namespace

int32_t* call_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_call_error_mu);
  if (!g_call_error_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_call_error) != cudaSuccess || !p) return nullptr;
    g_call_error_ptr[dev] = static_cast<int32_t*>(p);
  }
  return g_call_error_ptr[dev];
}

namespace {
// Copies a device error word to the host, clears it, waits for both.
int read_and_clear(int32_t* word, int32_t* code, cudaStream_t s) {
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, word, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return ER_ECUDA;
  if (cudaMemsetAsync(word, 0, sizeof(int32_t), s) != cudaSuccess) return ER_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ER_ECUDA;
  *code = h;
  return h == 0 ? ER_OK : ER_EDEVICE;
}
}  // namespace
}  // namespace er

using namespace er;

extern "C" {

int er_wait_selftest(const er_state* st, int32_t arrive, er_stream_t stream) {
  if ((st && !st->dev_error) || (arrive != 0 && arrive != 1)) return ER_EINVAL;
  int32_t* err = st ? st->dev_error : call_error_word();
  if (!err) return ER_ECUDA;
  k_wait_selftest<<<1, 32, 0, (cudaStream_t)stream>>>(err, arrive);
  count_launches(1);
  return launch_status();
}

int er_last_call_error(int32_t* code, er_stream_t stream) {
  if (!code) return ER_EINVAL;
  int32_t* word = call_error_word();
  if (!word) return ER_ECUDA;
  return read_and_clear(word, code, (cudaStream_t)stream);
}

size_t er_state_bytes_ex(int32_t s_max, int32_t n_layers, uint32_t flags) {
  StateLayout L;
  if (flags & ~ER_STATE_POOL) return 0;
  return layout_of(s_max, n_layers, (flags & ER_STATE_POOL) ? 1 : 0, &L) ? L.total : 0;
}

size_t er_state_bytes(int32_t s_max, int32_t n_layers) {
  return er_state_bytes_ex(s_max, n_layers, 0u);
}

int er_state_carve_ex(void* base, size_t bytes, int32_t s_max, int32_t n_layers, uint32_t flags,
                      er_state* out) {
  StateLayout L;
  const int pool = (flags & ER_STATE_POOL) ? 1 : 0;
  if ((flags & ~ER_STATE_POOL) || !base || !out || !layout_of(s_max, n_layers, pool, &L))
    return ER_EINVAL;
  if (((uintptr_t)base & 255u) != 0 || bytes < L.total) return ER_EINVAL;
  char* b = (char*)base;
  size_t g = (size_t)s_max * n_layers * NG;
  const size_t bank_rows = pool ? (size_t)POOL : (size_t)BANK;
  out->win_k = (er_bf16*)(b + L.win);
  out->win_v = out->win_k + g * WIN * D;
  out->bank_k = (er_bf16*)(b + L.bank);
  out->bank_v = out->bank_k + g * bank_rows * D;
  out->pend_k = pool ? nullptr : (er_bf16*)(b + L.pend);
  out->pend_v = pool ? nullptr : out->pend_k + g * PEND * D;
  out->bank_score = (float*)(b + L.bscore);
  out->pend_score = pool ? nullptr : (float*)(b + L.pscore);
  out->bank_pos = (int32_t*)(b + L.bpos);
  out->pend_pos = (int32_t*)(b + L.ppos);
  out->meta = (int32_t*)(b + L.meta);
  out->dev_error = (int32_t*)(b + L.err);
  out->s_max = s_max;
  out->n_layers = n_layers;
  out->pool = pool;
  return ER_OK;
}

int er_state_carve(void* base, size_t bytes, int32_t s_max, int32_t n_layers, er_state* out) {
  return er_state_carve_ex(base, bytes, s_max, n_layers, 0u, out);
}

int er_state_init(const er_state* st, const int32_t* seq_ids, int32_t n, er_stream_t stream) {
  if (!st || !st->meta || (n > 0 && !seq_ids) || n < 0) return ER_EINVAL;
  if (n == 0) return ER_OK;
  cudaStream_t s = (cudaStream_t)stream;
  k_state_init<<<(n + 127) / 128, 128, 0, s>>>(st->meta, seq_ids, n, st->s_max, st->dev_error);
  count_launches(1);
  if (st->pool) {
    k_pool_init<<<dim3(n, st->n_layers * NG), 256, 0, s>>>(st->bank_score, st->bank_pos,
                                                          st->pend_pos, st->bank_v, seq_ids, n,
                                                          st->s_max, st->n_layers);
    count_launches(1);
  }
  return launch_status();
}

int er_advance_ex(const er_state* st, const int32_t* seq_ids, int32_t n, int32_t T,
                  uint32_t flags, er_stream_t stream) {
  if (!st || !st->meta || (n > 0 && !seq_ids) || n < 0 || T < 1 || T > PEND) return ER_EINVAL;
  if (flags & ~ER_FLAG_RMA_OFF) return ER_EINVAL;
  if (n == 0) return ER_OK;
  k_advance<<<(n + 127) / 128, 128, 0, (cudaStream_t)stream>>>(
      st->meta, seq_ids, n, T, st->s_max, (flags & ER_FLAG_RMA_OFF) ? 1 : 0, st->dev_error);
  count_launches(1);
  return launch_status();
}

int er_advance(const er_state* st, const int32_t* seq_ids, int32_t n, int32_t T,
               er_stream_t stream) {
  return er_advance_ex(st, seq_ids, n, T, 0u, stream);
}

int er_last_device_error(const er_state* st, int32_t* code, er_stream_t stream) {
  if (!st || !st->dev_error || !code) return ER_EINVAL;
  return read_and_clear(st->dev_error, code, (cudaStream_t)stream);
}

const char* er_error_string(int code) {
  switch (code) {
    case ER_OK: return "ok";
    case ER_EINVAL: return "invalid argument";
    case ER_ECAPACITY: return "capacity exceeded";
    case ER_ECUDA: return "CUDA error";
    case ER_EDEVICE: return "device-side error recorded";
    case ER_ETIMEOUT: return "bounded device wait timed out";
    default: return "unknown error";
  }
}

uint64_t er_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int er_profile_enable(int enable) {
  ProfileState& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  p.enabled = enable != 0;
  return ER_OK;
}

int er_profile_read(double* ms_total, int64_t* launches, int reset) {
  ProfileState& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  for (auto& ev : p.pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(ev.second) != cudaSuccess) return ER_ECUDA;
    if (cudaEventElapsedTime(&ms, ev.first, ev.second) != cudaSuccess) return ER_ECUDA;
    p.ms += ms;
    p.launches += 1;
    p.pool.push_back(ev);
  }
  p.pending.clear();
  if (ms_total) *ms_total = p.ms;
  if (launches) *launches = p.launches;
  if (reset) {
    p.ms = 0.0;
    p.launches = 0;
  }
  return ER_OK;
}

}  // extern "C"
