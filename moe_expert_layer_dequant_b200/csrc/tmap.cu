// cuTensorMapEncodeTiled through the runtime's driver entry point.
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>
#include <unordered_map>

#include "tmap.cuh"

namespace moeffn {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_once;

void resolve() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

// Encoded maps are cached by their full description: layer calls reuse the
// same weights (and often the same activation buffers) call after call.
struct Key {
  uint64_t base, inner, rows, stride;
  uint32_t dt, box_inner, box_rows, swz;
  bool operator==(const Key& o) const { return std::memcmp(this, &o, sizeof(Key)) == 0; }
};
struct KeyHash {
  size_t operator()(const Key& k) const {
    uint64_t h = 1469598103934665603ull;
    const unsigned char* p = reinterpret_cast<const unsigned char*>(&k);
    for (size_t i = 0; i < sizeof(Key); ++i) h = (h ^ p[i]) * 1099511628211ull;
    return (size_t)h;
  }
};
std::mutex g_cache_mu;
std::unordered_map<Key, CUtensorMap, KeyHash> g_cache;
constexpr size_t kCacheMax = 8192;

cudaError_t encode_uncached(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                            uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz);

}  // namespace

cudaError_t encode_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                           uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  Key k;
  std::memset(&k, 0, sizeof(k));
  k.base = reinterpret_cast<uint64_t>(base);
  k.inner = inner;
  k.rows = rows;
  k.stride = row_stride_bytes;
  k.dt = (uint32_t)dt;
  k.box_inner = box_inner;
  k.box_rows = box_rows;
  k.swz = (uint32_t)swz;
  {
    std::lock_guard<std::mutex> lk(g_cache_mu);
    auto it = g_cache.find(k);
    if (it != g_cache.end()) {
      *m = it->second;
      return cudaSuccess;
    }
  }
  const cudaError_t e = encode_uncached(m, dt, base, inner, rows, row_stride_bytes, box_inner, box_rows, swz);
  if (e == cudaSuccess) {
    std::lock_guard<std::mutex> lk(g_cache_mu);
    if (g_cache.size() >= kCacheMax) g_cache.clear();
    g_cache.emplace(k, *m);
  }
  return e;
}

namespace {

cudaError_t encode_uncached(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                            uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  std::call_once(g_once, resolve);
  if (g_encode == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

}  // namespace moeffn
