// Partial attention for callers that cannot allocate device memory.
//
// dllm_attention_bf16 takes a caller workspace for its scratch: one status word
// and the per-sequence offsets of the compact query rows.  Some callers have no
// way to provide one:
//   * code that runs while a CUDA graph is being captured -- cudaMalloc is not
//     a stream operation, cannot be captured, and may synchronise the device;
//   * serving processes that carve all device memory into fixed pools before
//     they start, so nothing may allocate on the request path;
//   * plugins handed only the tensors they compute on.
// dllm_attention_bf16_noalloc keeps that scratch in a fixed array in the
// library's own device memory instead (about 16 KB for DLLM_NOALLOC_MAX_SEQS
// sequences, held by every GPU that loads the library until the process exits).
//
// Host code cannot use the array's name as a device address: on the host it
// names a host-side stand-in.  The device address is looked up once per
// device with cudaGetSymbolAddress, with that device current, on the first
// call made on it; make that first call before any stream capture.  Every call
// shares the array, so calls that may overlap on the GPU (different streams,
// or different host threads on one device) race on it and must be ordered by
// the caller.
#include <mutex>

#include "../../include/dllm.h"
#include "internal.h"

namespace {

constexpr int kMaxSeqs = DLLM_NOALLOC_MAX_SEQS;
constexpr int kOffsetBase = 64;  // status word at [0]; offsets start 256 bytes in

// [0] device status word (cleared by every call), [64 .. 64 + B] row offsets
// (rewritten by every call)
static __device__ __align__(256) int g_noalloc_scratch[kOffsetBase + kMaxSeqs + 1];

std::mutex g_mu;
int* g_addr[64] = {};

// device address of g_noalloc_scratch on the current device (set up once per device)
cudaError_t scratch_address(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = static_cast<int*>(p);
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

extern "C" dllm_status dllm_attention_bf16_noalloc(const void* q, const void* k_cache,
                                                   const void* v_cache, void* o,
                                                   const int32_t* count, int B, int k_cap, int N,
                                                   int n_heads, int n_kv_heads, int head_dim,
                                                   dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (B < 0 || k_cap < 1 || N < 0 || n_heads <= 0 || n_kv_heads <= 0) return DLLM_ERR_INVALID_ARG;
  if (B > kMaxSeqs) return DLLM_ERR_CAPACITY;  // the fixed scratch holds kMaxSeqs offsets
  if (n_heads % n_kv_heads) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (head_dim != 64 && head_dim != 128) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || N == 0) return DLLM_OK;
  if (!q || !k_cache || !v_cache || !o || !count) return DLLM_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
    return DLLM_ERR_INVALID_ARG;
  int* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return DLLM_ERR_CUDA;
  int* status = scratch;
  int* row_off = scratch + kOffsetBase;
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return DLLM_ERR_CUDA;
  dllm::launch_row_map(nullptr, count, B, k_cap, N, row_off, nullptr, nullptr, status, s);
  const cudaError_t e = dllm::launch_attention_tc(
      static_cast<const __nv_bfloat16*>(q), B * k_cap, static_cast<const __nv_bfloat16*>(k_cache),
      static_cast<const __nv_bfloat16*>(v_cache), static_cast<__nv_bfloat16*>(o), row_off, B,
      k_cap, N, n_heads, n_kv_heads, head_dim, status, s);
  if (e != cudaSuccess) return DLLM_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? DLLM_OK : DLLM_ERR_CUDA;
}
