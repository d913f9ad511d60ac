// tma.cu — host-side TMA tensor-map encoding (driver entry point looked up
// once through the runtime, so the library does not link libcuda).
#include <mutex>

#include "tc.cuh"

namespace er {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Encoded maps by their arguments: the read kernels' maps cover the state's
// arrays and a call's workspace, whose pointers stay the same from call to
// call, so a repeated call finds its maps here instead of encoding them again.
struct MapKey {
  const void* base;
  uint64_t dims[5], strides[4];
  uint32_t box[5];
  int rank, kind;
  bool operator==(const MapKey& o) const {
    if (base != o.base || rank != o.rank || kind != o.kind) return false;
    for (int i = 0; i < rank; ++i)
      if (dims[i] != o.dims[i] || box[i] != o.box[i]) return false;
    for (int i = 0; i + 1 < rank; ++i)
      if (strides[i] != o.strides[i]) return false;
    return true;
  }
};
constexpr int kMapCache = 512;
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  bool used;
};
std::mutex g_map_mu;
MapEntry g_maps[kMapCache];
int g_map_next = 0;

bool cache_find(const MapKey& k, CUtensorMap* out) {
  std::lock_guard<std::mutex> lock(g_map_mu);
  for (int i = 0; i < kMapCache; ++i)
    if (g_maps[i].used && g_maps[i].key == k) {
      *out = g_maps[i].map;
      return true;
    }
  return false;
}

void cache_put(const MapKey& k, const CUtensorMap& m) {
  std::lock_guard<std::mutex> lock(g_map_mu);
  MapEntry& e = g_maps[g_map_next];
  g_map_next = (g_map_next + 1) % kMapCache;
  e.key = k;
  e.map = m;
  e.used = true;
}

MapKey make_key(const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                const uint32_t* box, int kind) {
  MapKey k{};
  k.base = base;
  k.rank = rank;
  k.kind = kind;
  for (int i = 0; i < rank && i < 5; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
  }
  for (int i = 0; i + 1 < rank && i < 4; ++i) k.strides[i] = strides[i];
  return k;
}

}  // namespace

bool encode_bf16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box) {
  if (rank < 2 || rank > 5) return false;
  const MapKey key = make_key(base, rank, dims, strides_bytes, box, 0);
  if (cache_find(key, m)) return true;
  auto fn = encode_fn();
  if (!fn || rank < 2 || rank > 5 || ((uintptr_t)base & 15u)) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    if (dims[i] == 0) return false;
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) {
    if (strides_bytes[i] & 15u) return false;
    st[i] = strides_bytes[i];
  }
  if (fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), d, st, bx, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  cache_put(key, *m);
  return true;
}

bool encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                    uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows) {
  const uint64_t kd[2] = {cols, rows}, ks[1] = {pitch_bytes};
  const uint32_t kb[2] = {box_cols, box_rows};
  const MapKey key = make_key(base, 2, kd, ks, kb, 1);
  if (cache_find(key, m)) return true;
  auto fn = encode_fn();
  if (!fn || rows == 0 || cols == 0 || ((uintptr_t)base & 15u) || (pitch_bytes & 15u))
    return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)pitch_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  if (fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  cache_put(key, *m);
  return true;
}

// Host: a 2-D map for TMA stores of [box_rows][box_cols] blocks from plain
// (unswizzled) row-major shared memory into a BF16 or FP32 matrix; rows past
// `rows` are not written.
bool encode_store_2d(CUtensorMap* m, const void* base, bool fp32, uint64_t cols, uint64_t rows,
                     uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn || rows == 0 || cols == 0 || ((uintptr_t)base & 15u) || (pitch_bytes & 15u))
    return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)pitch_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace er
