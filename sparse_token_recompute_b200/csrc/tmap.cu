// TMA tensor-map encoding with a small cache.  A denoising step launches the
// same GEMMs and attention on the same buffers every step; encoding a map is a
// driver call, so maps are remembered by (address, shape, box) and reused.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>
#include <unordered_map>

#include "internal.h"

namespace dllm {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

struct Key {
  uintptr_t ptr;
  uint64_t rows, cols;
  uint32_t box_rows;
  int dev;
  bool operator==(const Key& o) const {
    return ptr == o.ptr && rows == o.rows && cols == o.cols && box_rows == o.box_rows &&
           dev == o.dev;
  }
};
struct KeyHash {
  size_t operator()(const Key& k) const {
    size_t h = k.ptr * 0x9E3779B97F4A7C15ull;
    h ^= (k.rows + 0x632BE59BD9B4E019ull) + (h << 6) + (h >> 2);
    h ^= (k.cols * 31 + k.box_rows) + (h << 6) + (h >> 2);
    h ^= (size_t)k.dev;
    return h;
  }
};

std::mutex g_mu;
std::unordered_map<Key, CUtensorMap, KeyHash> g_cache;

}  // namespace

bool tmap_bf16_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols,
                  uint32_t box_rows) {
  if (!ptr || rows == 0 || cols == 0 || (cols % 8) || (reinterpret_cast<uintptr_t>(ptr) & 15))
    return false;
  int dev = 0;
  cudaGetDevice(&dev);
  const Key k{reinterpret_cast<uintptr_t>(ptr), rows, cols, box_rows, dev};
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_cache.find(k);
    if (it != g_cache.end()) {
      *m = it->second;
      return true;
    }
  }
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  if (fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_cache.size() > 8192) g_cache.clear();
  g_cache.emplace(k, *m);
  return true;
}

}  // namespace dllm
