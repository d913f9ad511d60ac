// common.cuh — shapes, BF16 helpers, device error word, mbarrier / bulk-copy
// primitives (hand-written PTX for sm_100a) and host launch bookkeeping.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "edgerock.h"

namespace er {

// Layer shape (EdgeRock-4B 开源：72 MiB 固定 KV, §架构：递归、局部窗口与记忆锚点三件套).
constexpr int D = ER_HEAD_DIM;          // 256
constexpr int HID = ER_HIDDEN;          // 2560
constexpr int NH = ER_Q_HEADS;          // 16
constexpr int NG = ER_KV_GROUPS;        // 4
constexpr int HPG = ER_HEADS_PER_GROUP; // 4
constexpr int WIN = ER_WINDOW;          // 1024
constexpr int BANK = ER_BANK;           // 1024
constexpr int PEND = ER_PENDING;        // 256
constexpr int ROPE = ER_ROPE_DIMS;      // 64
constexpr int SH = ER_SCORE_HIDDEN;     // 256
constexpr int QKV = ER_QKV_ROWS;        // 12288
constexpr int QKVS = ER_QKV_SCORE_ROWS; // 13056: q/k/v rows + the 3 x 256 W1-term rows
constexpr int OIN = ER_O_IN;            // 4096
constexpr int ROW_BYTES = D * 2;        // one BF16 K or V row
// The pooled state layout: bank and pending block share 1280 rows per group; a
// free pool slot holds this position (above every stream position).
constexpr int POOL = BANK + PEND;       // 1280
constexpr int kGemvMaxTokensAll = 32;   // largest token count the GEMV kernel takes
constexpr int32_t FREE_POS = 0x7FFFFFFF;

// Column offsets of the six projections inside one [QKV] projection row.
constexpr int OFF_Q_SWA = 0, OFF_K_SWA = 4096, OFF_V_SWA = 5120;
constexpr int OFF_Q_RMA = 6144, OFF_K_RMA = 10240, OFF_V_RMA = 11264;

// Per-(seq, layer, group) base index.
__host__ __device__ __forceinline__ size_t grp(int s, int l, int g, int L) {
  return ((size_t)s * L + l) * NG + g;
}

// ------------------------------------------------------------ BF16 bits

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf1(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }
__device__ __forceinline__ uint16_t f2bf(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  return (uint32_t)f2bf(lo) | ((uint32_t)f2bf(hi) << 16);
}

// ------------------------------------------------------ device error word

__device__ __forceinline__ void set_dev_error(int32_t* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// -------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialisation may start while its
// predecessor on the stream is still running; it must pass grid_dep_wait()
// before touching anything the predecessor writes.  grid_dep_trigger() lets a
// kernel's dependents launch before it has finished (they still wait for all of
// its memory operations in grid_dep_wait).  Both are no-ops for a plain launch.
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ----------------------------------------------- mbarrier + bulk copies

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: gives up after ~2 s, records ER_ETIMEOUT and returns false.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      set_dev_error(err, ER_ETIMEOUT);
      return false;
    }
  }
  return true;
}

// Contiguous global -> shared bulk copy (TMA engine, no tensor map, into this
// CTA only), completion signalled on `bar` as transaction bytes.
// dst/src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(smem_u32(p)));
  return r;
}

__device__ __forceinline__ float4 lds128f(const void* p) {
  float4 r;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "r"(smem_u32(p)));
  return r;
}

// ------------------------------------------------------------ host side

// Vector loads and bulk copies need 16-byte aligned rows; entry points reject
// pointers that are not (ER_EINVAL) instead of letting a kernel fault.
inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

void count_launches(int n);                 // bookkeeping for er_launch_count
int launch_status();                        // ER_OK or ER_ECUDA after a launch
int num_sms();                              // SMs of the current device (cached)
int32_t* call_error_word();                 // device address of the stateless calls' error word

// Workspace carving: 256-byte aligned sub-buffers.  With a null base the
// returned "pointers" are the byte offsets themselves (layout computation).
struct Carver {
  uintptr_t base;
  size_t off = 0;
  explicit Carver(void* b) : base((uintptr_t)b) {}
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~(size_t)255;
    T* p = reinterpret_cast<T*>(base + off);
    off += count * sizeof(T);
    return p;
  }
  size_t used() const { return (off + 255) & ~(size_t)255; }
};

}  // namespace er
