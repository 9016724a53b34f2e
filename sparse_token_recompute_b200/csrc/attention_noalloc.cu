// Partial attention for callers that cannot allocate device memory.
//
// dllm_attention_bf16 takes a caller workspace for its scratch: one status word
// and the per-sequence offsets of the compact query rows.  Some callers have no
// way to provide one:
//   * serving processes that carve all device memory into fixed pools before
//     they start, so nothing may allocate on the request path (cudaMalloc can
//     also synchronise the device, which stalls every stream in flight);
//   * plugins and operators handed only the tensors they compute on, with no
//     allocator of their own.
// dllm_attention_bf16_noalloc keeps that scratch in a fixed array in the
// library's own device memory instead (about 16 KB for DLLM_NOALLOC_MAX_SEQS
// sequences, held by every GPU that loads the library until the process exits).
//
// Host code cannot use the array's name as a device address: on the host it
// names a host-side stand-in.  The device address is looked up with
// cudaGetSymbolAddress, with the device current, on the first call made in
// each device context (and again if the context changes, e.g. after a
// cudaDeviceReset); later calls in the context reuse it.  Every call
// shares the array, so calls that may overlap on the GPU (different streams,
// or different host threads on one device) race on it and must be ordered by
// the caller.  Like dllm_attention_bf16, this entry point never splits a
// sequence's keys among CTAs (the split needs a partial-output scratch far
// larger than the fixed array); the attention inside a step does, so with few
// query tiles -- one or two sequences of a few hundred selected rows -- it runs
// fewer CTAs than the step's attention and can be slower.
#include <cuda.h>
#include <cudaTypedefs.h>

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
struct Slot {
  CUcontext ctx;  // the context the address was looked up in
  int* addr;
};
Slot g_slot[64] = {};

// the driver's cuCtxGetCurrent, reached through the runtime (no link-time libcuda)
PFN_cuCtxGetCurrent_v4000 ctx_current_fn() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
  });
  return fn;
}

// device address of g_noalloc_scratch in the current device context (looked up once
// per device and context)
cudaError_t scratch_address(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  auto get_ctx = ctx_current_fn();
  if (!get_ctx) return cudaErrorUnknown;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
  std::lock_guard<std::mutex> lk(g_mu);
  Slot& sl = g_slot[dev];
  if (!sl.addr || !ctx || sl.ctx != ctx) {
    // the lookup also makes the device's primary context current when none was
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorUnknown;
    sl.addr = static_cast<int*>(p);
    sl.ctx = ctx;
  }
  *out = sl.addr;
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
