// Memory-bound and bookkeeping kernels of the selected-token step (sm_100a):
// importance scores, max-softmax confidence, radix top-k / threshold
// compaction, confidence unmasking, compact-row bookkeeping, gather with the
// hidden-reference scatter, RMSNorm, the RoPE table, the LM-head merge, and
// the fp32 pieces of the layer for DLLM_F32 models.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dllm {

namespace {

// ---------------------------------------------------------------- block scan helpers

// inclusive scan of one int per thread across the block (blockDim.x <= 1024)
__device__ int block_inclusive_scan(int v, int* warp_tot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) warp_tot[w] = v;
  __syncthreads();
  if (w == 0) {
    int t = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += u;
    }
    if (lane < nw) warp_tot[lane] = t;  // inclusive totals per warp
  }
  __syncthreads();
  const int add = w > 0 ? warp_tot[w - 1] : 0;
  const int r = v + add;
  __syncthreads();  // warp_tot may be reused by the caller
  return r;
}

__device__ int block_sum_int(int v, int* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[w] = v;
  __syncthreads();
  int t = 0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < nw; ++i) t += red[i];
    red[32] = t;
  }
  __syncthreads();
  t = red[32];
  __syncthreads();
  return t;
}

__device__ int block_min_int(int v, int* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) red[w] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = red[0];
    for (int i = 1; i < nw; ++i) t = min(t, red[i]);
    red[32] = t;
  }
  __syncthreads();
  const int r = red[32];
  __syncthreads();
  return r;
}

// Order-preserving key of a float for "larger first": NaN -> 0 (below all),
// -0 -> +0, otherwise the standard sign-flip mapping (-inf -> 0x007FFFFF).
__device__ __forceinline__ uint32_t order_key(float x) {
  if (isnan(x)) return 0u;
  if (x == 0.0f) x = 0.0f;
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- score

template <typename T>
__device__ __forceinline__ void load_vec8(const T* p, float* f);
template <>
__device__ __forceinline__ void load_vec8<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
  unpack8(__ldg(reinterpret_cast<const uint4*>(p)), f);
}
template <>
__device__ __forceinline__ void load_vec8<float>(const float* p, float* f) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Variation of one row against its reference, by one warp (every lane gets
// the result).  Accumulates |h|^2, |r|^2, |h-r|^2, |h-r|_1 and bitwise
// equality; 1 - cos is evaluated as (|h-r|^2 - (|h|-|r|)^2) / (2 |h| |r|),
// which equals 1 - h.r/(|h||r|) and stays accurate when the rows are close.
template <typename T>
__device__ __forceinline__ float row_variation(const T* __restrict__ hc, const T* __restrict__ hr,
                                               int d, int kind, int lane) {
  float nc = 0.f, nr = 0.f, dd = 0.f, l1 = 0.f;
  int eq = 1;
  // U vector pairs per lane in flight before any arithmetic
  constexpr int U = 4;
  for (int base = lane * 8; base < d; base += 32 * 8 * U) {
    float a[U][8], b[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * 256;
      if (i < d) {
        load_vec8<T>(hc + i, a[u]);
        load_vec8<T>(hr + i, b[u]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) a[u][j] = b[u][j] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float df = a[u][j] - b[u][j];
        nc = fmaf(a[u][j], a[u][j], nc);
        nr = fmaf(b[u][j], b[u][j], nr);
        dd = fmaf(df, df, dd);
        l1 += fabsf(df);
        eq &= (__float_as_uint(a[u][j]) == __float_as_uint(b[u][j]));
      }
  }
  nc = warp_sum(nc);
  nr = warp_sum(nr);
  dd = warp_sum(dd);
  l1 = warp_sum(l1);
  eq = warp_and(eq);
  float v;
  if (eq) {
    v = 0.0f;
  } else if (kind == DLLM_SCORE_COS) {
    const float a = sqrtf(nc), b = sqrtf(nr);
    const float nn = a * b;
    if (nn > 0.0f) {
      const float t = a - b;
      v = (dd - t * t) / (2.0f * nn);
      v = fminf(fmaxf(v, 0.0f), 2.0f);
    } else {
      v = 1.0f;
    }
  } else {
    v = nr > 0.0f ? l1 / (sqrtf((float)d) * sqrtf(nr)) : INFINITY;
  }
  return v;
}

// One warp per row of [B, N].
template <typename T>
__global__ void __launch_bounds__(256) score_kernel(const T* __restrict__ h_cur,
                                                    const T* __restrict__ embed,
                                                    const int32_t* __restrict__ tokens,
                                                    const T* __restrict__ h_ref, int rows, int N,
                                                    int d, const float* __restrict__ conf,
                                                    const uint8_t* __restrict__ masked,
                                                    const int32_t* __restrict__ mask_tokens,
                                                    int mask_id, float alpha, int kind,
                                                    float* __restrict__ scores, int vocab,
                                                    int lo, int* status) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  if (row % N < lo) {  // never a candidate (response-only step): not scored
    if (lane == 0) scores[row] = -INFINITY;
    return;
  }
  const T* hc;
  if (tokens) {
    int t = tokens[row];
    if (t < 0 || t >= vocab) {
      if (lane == 0) raise_status(status, DEV_BAD_INDEX);
      t = t < 0 ? 0 : vocab - 1;
    }
    hc = embed + (size_t)t * d;
  } else {
    hc = h_cur + (size_t)row * d;
  }
  const float v = row_variation<T>(hc, h_ref + (size_t)row * d, d, kind, lane);
  if (lane == 0) {
    const bool is_m =
        masked ? (masked[row] != 0) : (mask_tokens ? mask_tokens[row] == mask_id : false);
    const float c = is_m ? conf[row] : 0.0f;
    scores[row] = alpha * c + (1.0f - alpha) * v;
  }
}

// The second skip point: one warp per compact row r < M (device count) of
// sequence b = row_seq[r] at position p = row_pos[r]; x[r] against
// h_ref[b, p]; the score lands at scores[b * k_cap + (r - row_off[b])].
template <typename T>
__global__ void __launch_bounds__(256) score_rows_kernel(
    const T* __restrict__ x, const T* __restrict__ h_ref, const int* __restrict__ row_off,
    const int* __restrict__ row_pos, const int* __restrict__ row_seq, const int* __restrict__ M,
    int cap, int N, int d, int k_cap, const float* __restrict__ conf,
    const int32_t* __restrict__ tokens, int mask_id, float alpha, int kind,
    float* __restrict__ scores) {
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= cap || r >= *M) return;
  const int b = row_seq[r], p = row_pos[r];
  const size_t g = (size_t)b * N + p;
  const float v = row_variation<T>(x + (size_t)r * d, h_ref + g * d, d, kind, lane);
  if (lane == 0) {
    const float c = tokens[g] == mask_id ? conf[g] : 0.0f;
    scores[(size_t)b * k_cap + (r - row_off[b])] = alpha * c + (1.0f - alpha) * v;
  }
}

// ---------------------------------------------------------------- confidence

struct SoftStat {
  float m, s;
  int a;
};
__device__ __forceinline__ SoftStat soft_merge(SoftStat x, SoftStat y) {
  SoftStat r;
  r.m = fmaxf(x.m, y.m);
  if (r.m == -INFINITY) {
    r.s = 0.f;
  } else {
    r.s = (x.m == -INFINITY ? 0.f : x.s * expf(x.m - r.m)) +
          (y.m == -INFINITY ? 0.f : y.s * expf(y.m - r.m));
  }
  r.a = (x.m > y.m) ? x.a : ((y.m > x.m) ? y.a : min(x.a, y.a));
  return r;
}

// 2^x with the hardware approximation (relative error about 2^-22), flushing
// subnormal results to zero; the confidence sums need no more than that
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// statistics (max, sum of exp(z - max), first argmax) of one logits row, block-wide
template <typename T>
__device__ SoftStat row_softstat(const T* z, int V, SoftStat* red) {
  // Chunks of U vectors of 8 per thread: U loads in flight; per chunk a max tree,
  // the argmax searched only when the chunk raises the running maximum, one
  // rescale, and exp(x) as 2^(x log2 e).
  constexpr int U = 4;
  constexpr float LOG2E = 1.4426950408889634f;
  SoftStat st{-INFINITY, 0.f, 0x7fffffff};
  const int stride = blockDim.x * 8;
  for (int base = threadIdx.x * 8; base < V; base += stride * U) {
    float f[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * stride;
      if (i < V) {
        load_vec8<T>(z + i, f[u]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) f[u][j] = -INFINITY;
      }
    }
    float mq[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      mq[u] = fmaxf(fmaxf(fmaxf(f[u][0], f[u][1]), fmaxf(f[u][2], f[u][3])),
                    fmaxf(fmaxf(f[u][4], f[u][5]), fmaxf(f[u][6], f[u][7])));
    const float cm = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
    if (cm == -INFINITY) continue;
    if (cm > st.m) {
      // first (lowest) index holding the new maximum
      int ca = 0x7fffffff;
#pragma unroll
      for (int u = U - 1; u >= 0; --u)
#pragma unroll
        for (int j = 7; j >= 0; --j)
          if (f[u][j] == cm) ca = base + u * stride + j;
      st.s = (st.m == -INFINITY) ? 0.f : st.s * ex2_approx((st.m - cm) * LOG2E);
      st.m = cm;
      st.a = ca;
    }
    const float mL = st.m * LOG2E;
    float sv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j) sv[j & 3] += ex2_approx(fmaf(f[u][j], LOG2E, -mL));
    st.s += (sv[0] + sv[1]) + (sv[2] + sv[3]);
  }
  // warp merge
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    SoftStat y;
    y.m = __shfl_xor_sync(0xffffffffu, st.m, o);
    y.s = __shfl_xor_sync(0xffffffffu, st.s, o);
    y.a = __shfl_xor_sync(0xffffffffu, st.a, o);
    st = soft_merge(st, y);
  }
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = st;
  __syncthreads();
  if (threadIdx.x == 0) {
    SoftStat t = red[0];
    for (int i = 1; i < nw; ++i) t = soft_merge(t, red[i]);
    red[32] = t;
  }
  __syncthreads();
  const SoftStat r = red[32];
  __syncthreads();
  return r;
}

__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Statistics of one logits row, block-wide, in few instructions per logit: each
// thread keeps a running (max, sum) over chunks of 4 vectors of 8 (three-input
// maxima; the exponent argument and the sum two lanes per instruction); the first
// index of the maximum is not tracked in the loop: once the block knows the row's
// maximum, the threads whose own maximum equals it read the chunk where they first
// met it again (from cache) and report its first position.  Measured against a
// variant that tracked the argmax per chunk: 139 -> 129 us for 8192 rows of 32768
// bf16 logits; staging rows through shared memory with bulk copies (164 us) and
// computing half the exponentials with a polynomial on the FMA pipe (184 us) were
// slower: the kernel is bound by instruction issue and the special-function unit.
template <typename T>
__device__ SoftStat row_softstat_lean(const T* z, int V, SoftStat* red) {
  constexpr int U = 4;
  constexpr float LOG2E = 1.4426950408889634f;
  float m = -INFINITY;
  int m_base = 0;  // first element of the chunk that last raised m
  float2 s2 = make_float2(0.f, 0.f);
  const int stride = blockDim.x * 8;
  for (int base = threadIdx.x * 8; base < V; base += stride * U) {
    float f[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * stride;
      if (i < V) {
        load_vec8<T>(z + i, f[u]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) f[u][j] = -INFINITY;
      }
    }
    float cm = m;
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int j = 0; j < 8; j += 2) cm = fmax3f(cm, f[u][j], f[u][j + 1]);
    if (cm == -INFINITY) continue;
    if (cm > m) {  // rescale the running sum to the new maximum
      const float sc = m == -INFINITY ? 0.f : ex2_approx((m - cm) * LOG2E);
      s2.x *= sc;
      s2.y *= sc;
      m = cm;
      m_base = base;
    }
    const float2 l2 = make_float2(LOG2E, LOG2E);
    const float2 nm = make_float2(-m * LOG2E, -m * LOG2E);
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float2 x = fma_f32x2(make_float2(f[u][j], f[u][j + 1]), l2, nm);
        s2 = add_f32x2(s2, make_float2(ex2_approx(x.x), ex2_approx(x.y)));
      }
  }
  SoftStat st{m, s2.x + s2.y, 0x7fffffff};
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    SoftStat y;
    y.m = __shfl_xor_sync(0xffffffffu, st.m, o);
    y.s = __shfl_xor_sync(0xffffffffu, st.s, o);
    y.a = 0x7fffffff;
    st = soft_merge(st, y);
  }
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = st;
  __syncthreads();
  if (threadIdx.x == 0) {
    SoftStat t = red[0];
    for (int i = 1; i < nw; ++i) t = soft_merge(t, red[i]);
    red[32] = t;
  }
  __syncthreads();
  SoftStat r = red[32];
  // first position of the maximum: threads whose own maximum is the row's scan the
  // chunk where they first met it (earlier chunks held only smaller values)
  int a = 0x7fffffff;
  if (m == r.m && m != -INFINITY) {
    float f[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = m_base + u * stride;
      if (i < V) {
        load_vec8<T>(z + i, f[u]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) f[u][j] = -INFINITY;
      }
    }
#pragma unroll
    for (int u = U - 1; u >= 0; --u)
#pragma unroll
      for (int j = 7; j >= 0; --j)
        if (f[u][j] == m) a = m_base + u * stride + j;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w].a = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = red[0].a;
    for (int i = 1; i < nw; ++i) t = min(t, red[i].a);
    red[32].a = t;
  }
  __syncthreads();
  r.a = red[32].a;
  __syncthreads();
  return r;
}

template <typename T>
__global__ void __launch_bounds__(256) confidence_kernel(const T* __restrict__ logits,
                                                         const int32_t* __restrict__ logit_pos,
                                                         int Mm, int V, int N,
                                                         float* __restrict__ conf,
                                                         int32_t* __restrict__ pred) {
  __shared__ SoftStat red[33];
  const int r = blockIdx.x;  // b * Mm + j
  const int b = r / Mm;
  const SoftStat st = row_softstat_lean<T>(logits + (size_t)r * V, V, red);
  if (threadIdx.x == 0) {
    const int p = logit_pos[r];
    if (p >= 0 && p < N) {
      conf[(size_t)b * N + p] = 1.0f / st.s;
      if (pred) pred[(size_t)b * N + p] = st.a;
    }
  }
}

// logits [cap, V] fp32 of the LM rows (DLLM_F32 models)
__global__ void __launch_bounds__(256) confidence_rows_f32_kernel(
    const float* __restrict__ logits, int V, const int* __restrict__ lm_rows,
    const int* __restrict__ n_lm, const int* __restrict__ row_pos,
    const int* __restrict__ row_seq, int N, float* __restrict__ conf,
    int32_t* __restrict__ pred) {
  __shared__ SoftStat red[33];
  const int j = blockIdx.x;
  if (j >= *n_lm) return;
  const SoftStat st = row_softstat<float>(logits + (size_t)j * V, V, red);
  if (threadIdx.x == 0) {
    const int r = lm_rows[j];
    const size_t o = (size_t)row_seq[r] * N + row_pos[r];
    conf[o] = 1.0f / st.s;
    pred[o] = st.a;
  }
}

// merge of the per-tile statistics written by the LM-head GEMM epilogue
__global__ void __launch_bounds__(128) lm_merge_kernel(const float* __restrict__ part, int tiles,
                                                       const int* __restrict__ lm_rows,
                                                       const int* __restrict__ n_lm, int cap,
                                                       const int* __restrict__ row_pos,
                                                       const int* __restrict__ row_seq, int N,
                                                       float* __restrict__ conf,
                                                       int32_t* __restrict__ pred) {
  const int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (j >= *n_lm || j >= cap) return;
  const float* p = part + (size_t)j * tiles * 3;
  SoftStat st{-INFINITY, 0.f, 0x7fffffff};
  // each lane's tiles lane, lane + 32, ... in order; eight of them loaded at once
  constexpr int U = 8;
  for (int t0 = lane; t0 < tiles; t0 += 32 * U) {
    SoftStat y[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = t0 + 32 * u;
      if (t < tiles) y[u] = SoftStat{p[3 * t], p[3 * t + 1], __float_as_int(p[3 * t + 2])};
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (t0 + 32 * u < tiles) st = soft_merge(st, y[u]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    SoftStat y;
    y.m = __shfl_xor_sync(0xffffffffu, st.m, o);
    y.s = __shfl_xor_sync(0xffffffffu, st.s, o);
    y.a = __shfl_xor_sync(0xffffffffu, st.a, o);
    st = soft_merge(st, y);
  }
  if (lane == 0) {
    const int r = lm_rows[j];
    const size_t o = (size_t)row_seq[r] * N + row_pos[r];
    conf[o] = 1.0f / st.s;
    pred[o] = st.a;
  }
}

// ---------------------------------------------------------------- select

constexpr int SEL_THREADS = 1024;
constexpr int SEL_MAX_PER_THREAD = 16;  // N <= 16384

// Candidates are the positions lo <= i < len (len = lens[b], or N without
// lens): all of them for top-k, those with a score above tau for the
// threshold mode; a bit per element marks them.
__global__ void __launch_bounds__(SEL_THREADS) select_kernel(const float* __restrict__ scores,
                                                             int N, int lo,
                                                             const int* __restrict__ lens,
                                                             int mode, int k, float tau,
                                                             int32_t* __restrict__ idx,
                                                             int32_t* __restrict__ count,
                                                             int k_cap, int* status) {
  __shared__ int hist[256];
  __shared__ int red[33];
  __shared__ int s_digit, s_above;
  const int b = blockIdx.x;
  const float* sc = scores + (size_t)b * N;
  const int E = (N + SEL_THREADS - 1) / SEL_THREADS;
  const int len = lens ? min(max(lens[b], 0), N) : N;
  const int i0 = threadIdx.x * E;  // contiguous chunk keeps position order for the scans
  uint32_t key[SEL_MAX_PER_THREAD];
  uint32_t candm = 0u;
  int n_cand = 0;
#pragma unroll
  for (int e = 0; e < SEL_MAX_PER_THREAD; ++e) {
    key[e] = 0u;
    const int i = i0 + e;
    if (e < E && i < len && i >= lo) {
      const float x = sc[i];
      if (mode == DLLM_SELECT_TOPK || x > tau) {  // NaN compares false
        key[e] = order_key(x);
        candm |= 1u << e;
        ++n_cand;
      }
    }
  }
  int total = block_sum_int(n_cand, red);
  int keff;
  if (mode == DLLM_SELECT_TOPK) {
    keff = min(min(k, total), k_cap);
  } else {
    keff = min(total, k_cap);
    if (total > k_cap && threadIdx.x == 0) raise_status(status, DEV_CAPACITY);
  }
  if (keff <= 0) {
    if (threadIdx.x == 0) count[b] = 0;
    return;
  }
  // radix select of the keff-th largest key, 8 bits per pass from the top
  uint32_t prefix = 0u, pmask = 0u;
  int remaining = keff;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < SEL_MAX_PER_THREAD; ++e) {
      if ((candm >> e) & 1u) {
        if ((key[e] & pmask) == prefix) atomicAdd(&hist[(key[e] >> shift) & 255u], 1);
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // warp-parallel search from the top bin: lane l owns bins 255-8l .. 248-8l;
      // an exclusive suffix sum over lanes gives the count above each lane's bins
      const int lane = threadIdx.x;
      int cnt[8], own = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnt[q] = hist[255 - 8 * lane - q];
        own += cnt[q];
      }
      int incl = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int above = incl - own;  // count in higher bins than this lane's
      // the lane whose bins cross `remaining` finds the digit
      if (above < remaining && above + own >= remaining) {
        int dg = -1;
#pragma unroll
        for (int q = 0; q < 8; ++q) {  // static indices: cnt[] stays in registers
          if (dg < 0) {
            if (above + cnt[q] >= remaining)
              dg = 255 - 8 * lane - q;
            else
              above += cnt[q];
          }
        }
        s_digit = dg;
        s_above = above;
      }
    }
    __syncthreads();
    remaining -= s_above;
    prefix |= (uint32_t)s_digit << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = prefix;  // keff-th largest key; take `remaining` ties, lowest positions first
  int n_tie = 0;
#pragma unroll
  for (int e = 0; e < SEL_MAX_PER_THREAD; ++e)
    n_tie += (((candm >> e) & 1u) && key[e] == T) ? 1 : 0;
  const int tie_incl = block_inclusive_scan(n_tie, red);
  int tie_rank = tie_incl - n_tie;
  bool sel[SEL_MAX_PER_THREAD];
  int n_sel = 0;
#pragma unroll
  for (int e = 0; e < SEL_MAX_PER_THREAD; ++e) {
    sel[e] = false;
    if ((candm >> e) & 1u) {
      if (key[e] > T) {
        sel[e] = true;
      } else if (key[e] == T) {
        sel[e] = tie_rank < remaining;
        ++tie_rank;
      }
      n_sel += sel[e] ? 1 : 0;
    }
  }
  const int sel_incl = block_inclusive_scan(n_sel, red);
  int o = sel_incl - n_sel;
  int32_t* out = idx + (size_t)b * k_cap;
#pragma unroll
  for (int e = 0; e < SEL_MAX_PER_THREAD; ++e)
    if (sel[e]) out[o++] = i0 + e;
  if (threadIdx.x == blockDim.x - 1) count[b] = sel_incl;
}

// ---------------------------------------------------------------- second skip point

// positions of the rows kept at the second skip point: seg_idx[b, i] indexes
// sequence b's compact segment; pos[b, i] = row_pos[row_off[b] + seg_idx[b, i]]
__global__ void __launch_bounds__(256) seg_positions_kernel(const int32_t* __restrict__ seg_idx,
                                                            const int32_t* __restrict__ count,
                                                            const int* __restrict__ row_off,
                                                            const int* __restrict__ row_pos,
                                                            int k2_cap, int32_t* __restrict__ pos) {
  const int b = blockIdx.x;
  const int n = min(count[b], k2_cap), base = row_off[b], len = row_off[b + 1] - base;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int j = seg_idx[(size_t)b * k2_cap + i];
    pos[(size_t)b * k2_cap + i] = (j >= 0 && j < len) ? row_pos[base + j] : -1;
  }
}

// x2[r2] = x[r] for the old compact row r of the same sequence and position
// (binary search in the old segment, ascending by position); h_ref2 of the row
// is refreshed with it.  A position not in the old segment raises DEV_BAD_INDEX
// and leaves the row zero.
template <typename T>
__global__ void __launch_bounds__(128) gather_narrow_kernel(
    const T* __restrict__ x, const int* __restrict__ row_off, const int* __restrict__ row_pos,
    const int* __restrict__ row_off2, const int* __restrict__ row_pos2,
    const int* __restrict__ row_seq2, const int* __restrict__ M2, int N, int d,
    T* __restrict__ x2, T* __restrict__ h_ref2, int* status) {
  const int r2 = blockIdx.x;
  if (r2 >= *M2) return;
  const int b = row_seq2[r2], p = row_pos2[r2];
  int lo = row_off[b], hi = row_off[b + 1] - 1, src = -1;
  while (lo <= hi) {
    const int mid = (lo + hi) >> 1;
    const int q = row_pos[mid];
    if (q == p) {
      src = mid;
      break;
    }
    if (q < p) lo = mid + 1; else hi = mid - 1;
  }
  T* dst = x2 + (size_t)r2 * d;
  T* ref = h_ref2 + ((size_t)b * N + p) * d;
  if (src < 0) {
    if (threadIdx.x == 0) raise_status(status, DEV_BAD_INDEX);
    for (int i = threadIdx.x; i < d; i += blockDim.x) dst[i] = T(0.f);
    return;
  }
  const T* a = x + (size_t)src * d;
  constexpr int V = 16 / sizeof(T);
  if (d % V == 0) {
    for (int i = threadIdx.x * V; i < d; i += blockDim.x * V) {
      const uint4 v = *reinterpret_cast<const uint4*>(a + i);
      *reinterpret_cast<uint4*>(dst + i) = v;
      *reinterpret_cast<uint4*>(ref + i) = v;
    }
  } else {
    for (int i = threadIdx.x; i < d; i += blockDim.x) dst[i] = ref[i] = a[i];
  }
}

// ---------------------------------------------------------------- unmask

// The n_unmask most confident masked positions of the current block; with
// tau > 0, all masked positions with conf > tau when that is more (the top
// max(n_unmask, #above) positions).  pos_out / forced rows hold pos_cap entries.
__global__ void __launch_bounds__(1024) unmask_kernel(const float* __restrict__ conf,
                                                      const int32_t* __restrict__ pred,
                                                      int32_t* __restrict__ tokens, int N,
                                                      int mask_id, int gen_start, int block_len,
                                                      int n_unmask, float tau, int pos_cap,
                                                      int32_t* __restrict__ pos_out,
                                                      const int32_t* __restrict__ forced) {
  __shared__ int red[33];
  __shared__ uint32_t skey[1024];
  __shared__ unsigned char smask[1024];
  const int b = blockIdx.x;
  int32_t* tk = tokens + (size_t)b * N;
  const float* cf = conf + (size_t)b * N;
  const int32_t* pr = pred + (size_t)b * N;
  int32_t* po = pos_out ? pos_out + (size_t)b * pos_cap : nullptr;
  if (forced) {
    for (int j = threadIdx.x; j < pos_cap; j += blockDim.x) {
      const int p = forced[(size_t)b * pos_cap + j];
      if (p >= 0 && p < N) tk[p] = pr[p];
      if (po) po[j] = (p >= 0 && p < N) ? p : -1;
    }
    return;
  }
  int first = N;
  for (int p = gen_start + threadIdx.x; p < N; p += blockDim.x)
    if (tk[p] == mask_id) first = min(first, p);
  first = block_min_int(first, red);
  if (first >= N || n_unmask <= 0) {
    if (po)
      for (int j = threadIdx.x; j < pos_cap; j += blockDim.x) po[j] = -1;
    return;
  }
  const int blk = gen_start + ((first - gen_start) / block_len) * block_len;
  const int L = min(block_len, N - blk);
  const int t = threadIdx.x;
  bool is_m = false;
  uint32_t mykey = 0u;
  if (t < L) {
    is_m = tk[blk + t] == mask_id;
    mykey = order_key(cf[blk + t]);
    skey[t] = mykey;
    smask[t] = is_m ? 1 : 0;
  }
  __syncthreads();
  int take = n_unmask;
  if (tau > 0.f) {
    const bool above = t < L && is_m && cf[blk + t] > tau;  // NaN compares false
    take = max(take, block_sum_int(above ? 1 : 0, red));
  }
  take = min(take, pos_cap);
  bool sel = false;
  if (t < L && is_m) {
    int rank = 0;
    for (int j = 0; j < L; ++j) {
      if (!smask[j]) continue;
      const uint32_t kj = skey[j];
      rank += (kj > mykey || (kj == mykey && j < t)) ? 1 : 0;
    }
    sel = rank < take;
  }
  const int incl = block_inclusive_scan(sel ? 1 : 0, red);
  __shared__ int s_total;
  if (threadIdx.x == blockDim.x - 1) s_total = incl;
  __syncthreads();
  if (sel) {
    const int p = blk + t;
    tk[p] = pr[p];
    if (po) po[incl - 1] = p;
  }
  if (po)
    for (int j = s_total + threadIdx.x; j < pos_cap; j += blockDim.x) po[j] = -1;
}

// start of each sequence's current block: the block holding the first masked
// position >= gen_start (-1 when none is left)
__global__ void __launch_bounds__(256) block_start_kernel(const int32_t* __restrict__ tokens,
                                                          int N, int mask_id, int gen_start,
                                                          int block_len,
                                                          int32_t* __restrict__ out) {
  __shared__ int red[33];
  const int b = blockIdx.x;
  const int32_t* tk = tokens + (size_t)b * N;
  int first = N;
  for (int p = gen_start + threadIdx.x; p < N; p += blockDim.x)
    if (tk[p] == mask_id) first = min(first, p);
  first = block_min_int(first, red);
  if (threadIdx.x == 0)
    out[b] = first >= N ? -1 : gen_start + ((first - gen_start) / block_len) * block_len;
}

// ---------------------------------------------------------------- row bookkeeping

__global__ void __launch_bounds__(1024) row_map_kernel(const int32_t* __restrict__ idx,
                                                       const int32_t* __restrict__ count, int B,
                                                       int k_cap, int N, int* __restrict__ row_off,
                                                       int* __restrict__ row_pos,
                                                       int* __restrict__ row_seq, int* status) {
  __shared__ int red[33];
  __shared__ int s_carry;
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  for (int b0 = 0; b0 < B; b0 += blockDim.x) {
    const int b = b0 + threadIdx.x;
    int c = 0;
    if (b < B) {
      c = count[b];
      if (c < 0 || c > k_cap) {
        raise_status(status, DEV_CAPACITY);
        c = c < 0 ? 0 : k_cap;
      }
    }
    const int incl = block_inclusive_scan(c, red);
    const int carry = s_carry;
    if (b < B) row_off[b] = carry + incl - c;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) s_carry = carry + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) row_off[B] = s_carry;
  __syncthreads();
  if (!idx) return;  // offsets only
  for (int b = 0; b < B; ++b) {
    int c = count[b];
    c = c < 0 ? 0 : (c > k_cap ? k_cap : c);
    const int off = row_off[b];
    for (int j = threadIdx.x; j < c; j += blockDim.x) {
      int p = idx[(size_t)b * k_cap + j];
      const bool bad = p < 0 || p >= N || (j > 0 && idx[(size_t)b * k_cap + j - 1] >= p);
      if (bad) {
        raise_status(status, DEV_BAD_INDEX);
        p = p < 0 ? 0 : (p >= N ? N - 1 : p);
      }
      row_pos[off + j] = p;
      row_seq[off + j] = b;
    }
  }
}

__global__ void row_map_dense_kernel(int B, int N, int* row_off, int* row_pos, int* row_seq) {
  const size_t total = (size_t)B * N;
  for (size_t r = blockIdx.x * (size_t)blockDim.x + threadIdx.x; r < total;
       r += (size_t)gridDim.x * blockDim.x) {
    row_pos[r] = (int)(r % N);
    row_seq[r] = (int)(r / N);
  }
  if (blockIdx.x == 0)
    for (int b = threadIdx.x; b <= B; b += blockDim.x) row_off[b] = b * N;
}

template <typename T>
__global__ void __launch_bounds__(256) gather_rows_kernel(
    const T* __restrict__ src_full, const T* __restrict__ embed,
    const int32_t* __restrict__ tokens, const int* __restrict__ row_pos,
    const int* __restrict__ row_seq, const int* __restrict__ M_dev, int M_cap, int N, int d,
    T* __restrict__ x, T* __restrict__ h_ref, int vocab, int* status) {
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int M = M_dev ? min(*M_dev, M_cap) : M_cap;
  if (r >= M) return;
  const size_t src_row = (size_t)row_seq[r] * N + row_pos[r];
  const T* src;
  if (tokens) {
    int t = tokens[src_row];
    if (t < 0 || t >= vocab) {
      if (lane == 0) raise_status(status, DEV_BAD_INDEX);
      t = t < 0 ? 0 : vocab - 1;
    }
    src = embed + (size_t)t * d;
  } else {
    src = src_full + src_row * d;
  }
  constexpr int VEC = 16 / sizeof(T);
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  uint4* x4 = reinterpret_cast<uint4*>(x + (size_t)r * d);
  uint4* h4 = h_ref ? reinterpret_cast<uint4*>(h_ref + src_row * d) : nullptr;
  for (int i = lane; i < d / VEC; i += 32) {
    const uint4 v = __ldg(s4 + i);
    x4[i] = v;
    if (h4) h4[i] = v;
  }
}

template <typename T>
__device__ __forceinline__ void rmsnorm_row(const T* __restrict__ x, const T* __restrict__ g,
                                            T* __restrict__ o, int d, float eps) {
  const int lane = threadIdx.x & 31;
  float ss = 0.f;
  if constexpr (sizeof(T) == 2) {
    if (d <= 256 * 16) {
      // bf16: the row and the gains stay packed in registers (16 + 16 vectors of 8
      // per lane); every load of both is issued before the first use, so a row
      // costs one memory round trip
      uint4 xr[16], gr[16];
#pragma unroll
      for (int v = 0; v < 16; ++v) {
        const int i = lane * 8 + v * 256;
        if (i < d) {
          xr[v] = __ldg(reinterpret_cast<const uint4*>(x + i));
          gr[v] = __ldg(reinterpret_cast<const uint4*>(g + i));
        }
      }
#pragma unroll
      for (int v = 0; v < 16; ++v) {
        if (lane * 8 + v * 256 < d) {
          float f[8];
          unpack8(xr[v], f);
#pragma unroll
          for (int j = 0; j < 8; ++j) ss = fmaf(f[j], f[j], ss);
        }
      }
      ss = warp_sum(ss);
      const float s = rsqrtf(ss / (float)d + eps);
#pragma unroll
      for (int v = 0; v < 16; ++v) {
        const int i = lane * 8 + v * 256;
        if (i < d) {
          float f[8], w[8];
          unpack8(xr[v], f);
          unpack8(gr[v], w);
#pragma unroll
          for (int j = 0; j < 8; ++j) f[j] = f[j] * s * w[j];
          *reinterpret_cast<uint4*>(o + i) = pack8(f);
        }
      }
      return;
    }
  }
  if (d <= 256 * 16) {
    // whole row in registers (up to 16 vectors of 8 per lane): every load is
    // issued before the first use, then the row is normalised from registers
    float f[16][8];
#pragma unroll
    for (int v = 0; v < 16; ++v) {
      const int i = lane * 8 + v * 256;
      if (i < d) load_vec8<T>(x + i, f[v]);
    }
#pragma unroll
    for (int v = 0; v < 16; ++v) {
      if (lane * 8 + v * 256 < d) {
#pragma unroll
        for (int j = 0; j < 8; ++j) ss = fmaf(f[v][j], f[v][j], ss);
      }
    }
    ss = warp_sum(ss);
    const float s = rsqrtf(ss / (float)d + eps);
#pragma unroll
    for (int v = 0; v < 16; ++v) {
      const int i = lane * 8 + v * 256;
      if (i < d) {
        float w[8];
        load_vec8<T>(g + i, w);
#pragma unroll
        for (int j = 0; j < 8; ++j) f[v][j] = f[v][j] * s * w[j];
        if constexpr (sizeof(T) == 2) {
          *reinterpret_cast<uint4*>(o + i) = pack8(f[v]);
        } else {
          float4* o4 = reinterpret_cast<float4*>(o + i);
          o4[0] = make_float4(f[v][0], f[v][1], f[v][2], f[v][3]);
          o4[1] = make_float4(f[v][4], f[v][5], f[v][6], f[v][7]);
        }
      }
    }
    return;
  }
  for (int i = lane * 8; i < d; i += 256) {
    float f[8];
    load_vec8<T>(x + i, f);
#pragma unroll
    for (int j = 0; j < 8; ++j) ss = fmaf(f[j], f[j], ss);
  }
  ss = warp_sum(ss);
  const float s = rsqrtf(ss / (float)d + eps);
  for (int i = lane * 8; i < d; i += 256) {
    float f[8], w[8];
    load_vec8<T>(x + i, f);
    load_vec8<T>(g + i, w);
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = f[j] * s * w[j];
    if constexpr (sizeof(T) == 2) {
      *reinterpret_cast<uint4*>(o + i) = pack8(f);
    } else {
      float4* o4 = reinterpret_cast<float4*>(o + i);
      o4[0] = make_float4(f[0], f[1], f[2], f[3]);
      o4[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const T* __restrict__ x,
                                                      const T* __restrict__ g, T* __restrict__ o,
                                                      const int* __restrict__ M_dev, int M_cap,
                                                      int d, float eps) {
  griddep_launch_dependents();  // the next GEMM may start streaming its weights
  griddep_wait();               // x is written by the kernel before
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int M = M_dev ? min(*M_dev, M_cap) : M_cap;
  if (r >= M) return;
  rmsnorm_row<T>(x + (size_t)r * d, g, o + (size_t)r * d, d, eps);
}

template <typename T>
__global__ void __launch_bounds__(256) rmsnorm_rows_kernel(const T* __restrict__ x,
                                                           const T* __restrict__ g,
                                                           T* __restrict__ o,
                                                           const int* __restrict__ rows,
                                                           const int* __restrict__ n_rows,
                                                           int cap, int d, float eps) {
  const int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (j >= min(*n_rows, cap)) return;
  rmsnorm_row<T>(x + (size_t)rows[j] * d, g, o + (size_t)j * d, d, eps);
}

__global__ void rope_table_kernel(float2* table, int N, int hd, double theta) {
  const int half = hd / 2;
  const size_t total = (size_t)N * half;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int p = (int)(i / half), j = (int)(i % half);
    const double inv = pow(theta, -2.0 * j / hd);
    double sn, cs;
    sincos((double)p * inv, &sn, &cs);
    table[i] = make_float2((float)cs, (float)sn);
  }
}

__global__ void __launch_bounds__(1024) masked_rows_kernel(const int32_t* __restrict__ tokens,
                                                           int mask_id,
                                                           const int* __restrict__ row_pos,
                                                           const int* __restrict__ row_seq,
                                                           const int* __restrict__ M_dev,
                                                           int M_cap, int N, int* __restrict__ out,
                                                           int* __restrict__ n_out) {
  __shared__ int red[33];
  __shared__ int s_carry;
  const int M = M_dev ? min(*M_dev, M_cap) : M_cap;
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  for (int r0 = 0; r0 < M; r0 += blockDim.x) {
    const int r = r0 + threadIdx.x;
    const int f = (r < M && tokens[(size_t)row_seq[r] * N + row_pos[r]] == mask_id) ? 1 : 0;
    const int incl = block_inclusive_scan(f, red);
    const int carry = s_carry;
    if (f) out[carry + incl - 1] = r;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) s_carry = carry + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_out = s_carry;
}

// ---------------------------------------------------------------- DyLLM FFN gate

// One warp per compact row r < M: the row's attention output o[r] against the
// context cached at its last pass, ctx[b, p] (1 - cos); salient when all_rows
// or 1 - cos > tau; the cache takes o[r].
template <typename T>
__global__ void __launch_bounds__(256) ffn_gate_kernel(const T* __restrict__ o, T* __restrict__ ctx,
                                                       const int* __restrict__ row_pos,
                                                       const int* __restrict__ row_seq,
                                                       const int* __restrict__ M_dev, int M_cap,
                                                       int N, int q, float tau, int all_rows,
                                                       const uint8_t* __restrict__ forced,
                                                       int* __restrict__ flag) {
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int M = M_dev ? min(*M_dev, M_cap) : M_cap;
  if (r >= M) return;
  const T* a = o + (size_t)r * q;
  T* c = ctx + ((size_t)row_seq[r] * N + row_pos[r]) * q;
  const float v = row_variation<T>(a, c, q, DLLM_SCORE_COS, lane);
  __syncwarp();
  for (int i = lane; i < q; i += 32) c[i] = a[i];
  if (lane == 0) flag[r] = (all_rows || (forced ? forced[r] != 0 : v > tau)) ? 1 : 0;
}

// rows r < M with flag[r] -> list (ascending) and count; inv[r] = position in the
// list or -1
__global__ void __launch_bounds__(1024) flag_compact_kernel(const int* __restrict__ flag,
                                                            const int* __restrict__ M_dev,
                                                            int M_cap, int* __restrict__ list,
                                                            int* __restrict__ inv,
                                                            int* __restrict__ n_out) {
  __shared__ int red[33];
  __shared__ int s_carry;
  const int M = M_dev ? min(*M_dev, M_cap) : M_cap;
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  for (int r0 = 0; r0 < M; r0 += blockDim.x) {
    const int r = r0 + threadIdx.x;
    const int f = (r < M && flag[r]) ? 1 : 0;
    const int incl = block_inclusive_scan(f, red);
    const int carry = s_carry;
    if (r < M) {
      inv[r] = f ? carry + incl - 1 : -1;
      if (f) list[carry + incl - 1] = r;
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) s_carry = carry + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_out = s_carry;
}

// x[r] = x[r] + f, with f = the FFN output just computed for a salient row (also
// written to the row's cache) or the cached one; one block per row
template <typename T>
__global__ void __launch_bounds__(128) ffn_combine_kernel(T* __restrict__ x,
                                                          const T* __restrict__ f_new,
                                                          T* __restrict__ f_cache,
                                                          const int* __restrict__ inv,
                                                          const int* __restrict__ row_pos,
                                                          const int* __restrict__ row_seq,
                                                          const int* __restrict__ M_dev,
                                                          int M_cap, int N, int d) {
  const int r = blockIdx.x;
  const int M = M_dev ? min(*M_dev, M_cap) : M_cap;
  if (r >= M) return;
  const int j = inv[r];
  T* fc = f_cache + ((size_t)row_seq[r] * N + row_pos[r]) * d;
  T* xr = x + (size_t)r * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    T f;
    if (j >= 0) {
      f = f_new[(size_t)j * d + i];
      fc[i] = f;
    } else {
      f = fc[i];
    }
    xr[i] = T((float)xr[i] + (float)f);
  }
}

// ---------------------------------------------------------------- DyLLM approximate attention

// Rows r < M of a per-row cache [B, N, words] (32-bit words) <-> compact rows
// [cap, words]: to_cache = 1 scatters compact -> cache, 0 gathers cache -> compact.
// One block per compact row.
__global__ void __launch_bounds__(128) row_words_kernel(uint32_t* __restrict__ cache,
                                                        uint32_t* __restrict__ compact,
                                                        const int* __restrict__ row_pos,
                                                        const int* __restrict__ row_seq,
                                                        const int* __restrict__ M_dev, int M_cap,
                                                        int N, int words, int to_cache) {
  const int r = blockIdx.x;
  const int M = M_dev ? min(*M_dev, M_cap) : M_cap;
  if (r >= M) return;
  uint32_t* c = cache + ((size_t)row_seq[r] * N + row_pos[r]) * words;
  uint32_t* x = compact + (size_t)r * words;
  if ((words & 3) == 0) {
    uint4* c4 = reinterpret_cast<uint4*>(c);
    uint4* x4 = reinterpret_cast<uint4*>(x);
    for (int i = threadIdx.x; i < (words >> 2); i += blockDim.x) {
      if (to_cache) c4[i] = x4[i]; else x4[i] = c4[i];
    }
  } else {
    for (int i = threadIdx.x; i < words; i += blockDim.x) {
      if (to_cache) c[i] = x[i]; else x[i] = c[i];
    }
  }
}

// flags[seq * N + pos] = 1 for the compact rows r < M (the buffer is cleared first)
__global__ void __launch_bounds__(256) mark_rows_kernel(const int* __restrict__ row_pos,
                                                        const int* __restrict__ row_seq,
                                                        const int* __restrict__ M_dev, int M_cap,
                                                        int N, uint8_t* __restrict__ flags) {
  const int M = M_dev ? min(*M_dev, M_cap) : M_cap;
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < M; r += gridDim.x * blockDim.x)
    flags[(size_t)row_seq[r] * N + row_pos[r]] = 1;
}

// off[b] = b * N for b <= B: every row of every sequence, in cache order
__global__ void seq_offsets_kernel(int B, int N, int* off) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b <= B; b += gridDim.x * blockDim.x)
    off[b] = b * N;
}

__global__ void copy_idx_kernel(const int32_t* src_idx, const int32_t* src_count,
                                int32_t* dst_idx, int32_t* dst_count, int B, int k_cap) {
  const size_t total = (size_t)B * k_cap;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x)
    dst_idx[i] = src_idx[i];
  if (blockIdx.x == 0)
    for (int b = threadIdx.x; b < B; b += blockDim.x) dst_count[b] = src_count[b];
}

// ---------------------------------------------------------------- fp32 layer pieces

// C[M,N] = A[M,K] B[N,K]^T (+ R[M,N]); 64x64 tile, 256 threads, 4x4 per thread
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A,
                                                       const float* __restrict__ Bm,
                                                       float* __restrict__ C,
                                                       const float* __restrict__ R,
                                                       const int* __restrict__ M_dev, int M_cap,
                                                       int N, int K) {
  __shared__ float As[16][65];
  __shared__ float Bs[16][65];
  const int M = M_dev ? min(*M_dev, M_cap) : M_cap;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  if (m0 >= M) return;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      const int r = i / 16, kk = i % 16;
      As[kk][r] = (m0 + r < M && k0 + kk < K) ? A[(size_t)(m0 + r) * K + k0 + kk] : 0.f;
      Bs[kk][r] = (n0 + r < N && k0 + kk < K) ? Bm[(size_t)(n0 + r) * K + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (R) v += R[(size_t)m * N + n];
      C[(size_t)m * N + n] = v;
    }
  }
}

__global__ void qkv_post_f32_kernel(const float* __restrict__ qr, const float* __restrict__ kr,
                                    const float* __restrict__ vr, float* __restrict__ q,
                                    float* __restrict__ kc, float* __restrict__ vc,
                                    const int* __restrict__ row_pos,
                                    const int* __restrict__ row_seq, const int* __restrict__ M_dev,
                                    int M_cap, int Nseq, int Hq, int Hkv, int hd,
                                    const float2* __restrict__ rope) {
  const int r = blockIdx.x;
  const int M = M_dev ? min(*M_dev, M_cap) : M_cap;
  if (r >= M) return;
  const int pos = row_pos[r], seq = row_seq[r];
  const int half = hd / 2;
  const size_t cache_row = ((size_t)seq * Nseq + pos) * Hkv * hd;
  for (int i = threadIdx.x; i < (Hq + 2 * Hkv) * half; i += blockDim.x) {
    const int h = i / half, j = i % half;
    const float* src;
    float* dst;
    bool rot = rope != nullptr;
    if (h < Hq) {
      src = qr + (size_t)r * Hq * hd + h * hd;
      dst = q + (size_t)r * Hq * hd + h * hd;
    } else if (h < Hq + Hkv) {
      src = kr + (size_t)r * Hkv * hd + (h - Hq) * hd;
      dst = kc + cache_row + (h - Hq) * hd;
    } else {
      src = vr + (size_t)r * Hkv * hd + (h - Hq - Hkv) * hd;
      dst = vc + cache_row + (h - Hq - Hkv) * hd;
      rot = false;
    }
    const float x1 = src[j], x2 = src[j + half];
    if (rot) {
      const float2 t = rope[(size_t)pos * half + j];
      dst[j] = x1 * t.x - x2 * t.y;
      dst[j + half] = x2 * t.x + x1 * t.y;
    } else {
      dst[j] = x1;
      dst[j + half] = x2;
    }
  }
}

__global__ void swiglu_f32_kernel(const float* __restrict__ g, const float* __restrict__ u,
                                  float* __restrict__ a, const int* __restrict__ M_dev, int M_cap,
                                  int F) {
  const int M = M_dev ? min(*M_dev, M_cap) : M_cap;
  const size_t total = (size_t)M * F;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const float x = g[i];
    a[i] = x / (1.0f + expf(-x)) * u[i];
  }
}

// one block per (row, head): scores of all keys in shared memory, softmax, P V
__global__ void __launch_bounds__(128) attention_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ kc, const float* __restrict__ vc,
    float* __restrict__ o, const int* __restrict__ row_seq, const int* __restrict__ M_dev,
    int M_cap, int Nseq, int Hq, int Hkv, int hd) {
  extern __shared__ float s_p[];
  __shared__ float red[33];
  const int r = blockIdx.x, h = blockIdx.y;
  const int M = M_dev ? min(*M_dev, M_cap) : M_cap;
  if (r >= M) return;
  const int seq = row_seq[r], g = (h * Hkv) / Hq;
  const float* qv = q + ((size_t)r * Hq + h) * hd;
  const float scale = rsqrtf((float)hd);
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < Nseq; j += blockDim.x) {
    const float* kv = kc + (((size_t)seq * Nseq + j) * Hkv + g) * hd;
    float s = 0.f;
    for (int e = 0; e < hd; ++e) s = fmaf(qv[e], kv[e], s);
    s *= scale;
    s_p[j] = s;
    mx = fmaxf(mx, s);
  }
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = red[0];
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) t = fmaxf(t, red[i]);
    red[32] = t;
  }
  __syncthreads();
  mx = red[32];
  __syncthreads();
  float sum = 0.f;
  for (int j = threadIdx.x; j < Nseq; j += blockDim.x) {
    const float e = expf(s_p[j] - mx);
    s_p[j] = e;
    sum += e;
  }
  sum = warp_sum(sum);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    red[32] = t;
  }
  __syncthreads();
  const float inv = 1.0f / red[32];
  for (int e = threadIdx.x; e < hd; e += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < Nseq; ++j)
      acc = fmaf(s_p[j], vc[(((size_t)seq * Nseq + j) * Hkv + g) * hd + e], acc);
    o[((size_t)r * Hq + h) * hd + e] = acc * inv;
  }
}

inline int grid_for(size_t n, int threads, int cap = 148 * 16) {
  size_t g = (n + threads - 1) / threads;
  if (g < 1) g = 1;
  if (g > (size_t)cap) g = cap;
  return (int)g;
}

}  // namespace

// ---------------------------------------------------------------- launchers

template <typename T>
void launch_score(const T* h_cur, const T* embed, const int32_t* tokens, const T* h_ref, int B,
                  int N, int d, const float* conf, const uint8_t* masked,
                  const int32_t* mask_tokens, int mask_id, float alpha, int kind, float* scores,
                  int vocab, int lo, int* status, cudaStream_t s) {
  const int rows = B * N;
  if (rows <= 0) return;
  ProfScope prof("score", s);
  score_kernel<T><<<(rows + 7) / 8, 256, 0, s>>>(h_cur, embed, tokens, h_ref, rows, N, d, conf,
                                                 masked, mask_tokens, mask_id, alpha, kind,
                                                 scores, vocab, lo, status);
}
template void launch_score<float>(const float*, const float*, const int32_t*, const float*, int,
                                  int, int, const float*, const uint8_t*, const int32_t*, int,
                                  float, int, float*, int, int, int*, cudaStream_t);
template void launch_score<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                          const int32_t*, const __nv_bfloat16*, int, int, int,
                                          const float*, const uint8_t*, const int32_t*, int, float,
                                          int, float*, int, int, int*, cudaStream_t);

template <typename T>
void launch_confidence(const T* logits, const int32_t* logit_pos, int B, int Mm, int V, int N,
                       float* conf, int32_t* pred, cudaStream_t s) {
  if (B * Mm <= 0) return;
  ProfScope prof("confidence", s);
  confidence_kernel<T><<<B * Mm, 256, 0, s>>>(logits, logit_pos, Mm, V, N, conf, pred);
}
template void launch_confidence<float>(const float*, const int32_t*, int, int, int, int, float*,
                                       int32_t*, cudaStream_t);
template void launch_confidence<__nv_bfloat16>(const __nv_bfloat16*, const int32_t*, int, int, int,
                                               int, float*, int32_t*, cudaStream_t);

void launch_select(const float* scores, int B, int N, int lo, int mode, int k, float tau,
                   int32_t* idx, int32_t* count, int k_cap, int* status, cudaStream_t s,
                   const int* lens) {
  if (B <= 0) return;
  ProfScope prof("select", s);
  select_kernel<<<B, SEL_THREADS, 0, s>>>(scores, N, lo, lens, mode, k, tau, idx, count, k_cap,
                                          status);
}

template <typename T>
void launch_score_rows(const T* x, const T* h_ref, const int* row_off, const int* row_pos,
                       const int* row_seq, const int* M, int cap, int N, int d, int k_cap,
                       const float* conf, const int32_t* tokens, int mask_id, float alpha,
                       int kind, float* scores, cudaStream_t s) {
  if (cap <= 0) return;
  ProfScope prof("score2", s);
  score_rows_kernel<T><<<(cap + 7) / 8, 256, 0, s>>>(x, h_ref, row_off, row_pos, row_seq, M, cap,
                                                     N, d, k_cap, conf, tokens, mask_id, alpha,
                                                     kind, scores);
}
template void launch_score_rows<float>(const float*, const float*, const int*, const int*,
                                       const int*, const int*, int, int, int, int, const float*,
                                       const int32_t*, int, float, int, float*, cudaStream_t);
template void launch_score_rows<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                               const int*, const int*, const int*, const int*,
                                               int, int, int, int, const float*, const int32_t*,
                                               int, float, int, float*, cudaStream_t);

void launch_seg_positions(const int32_t* seg_idx, const int32_t* count, const int* row_off,
                          const int* row_pos, int B, int k2_cap, int32_t* pos, cudaStream_t s) {
  if (B <= 0) return;
  seg_positions_kernel<<<B, 256, 0, s>>>(seg_idx, count, row_off, row_pos, k2_cap, pos);
}

template <typename T>
void launch_gather_narrow(const T* x, const int* row_off, const int* row_pos,
                          const int* row_off2, const int* row_pos2, const int* row_seq2,
                          const int* M2, int cap2, int N, int d, T* x2, T* h_ref2, int* status,
                          cudaStream_t s) {
  if (cap2 <= 0) return;
  ProfScope prof("gather", s);
  gather_narrow_kernel<T><<<cap2, 128, 0, s>>>(x, row_off, row_pos, row_off2, row_pos2, row_seq2,
                                               M2, N, d, x2, h_ref2, status);
}
template void launch_gather_narrow<float>(const float*, const int*, const int*, const int*,
                                          const int*, const int*, const int*, int, int, int,
                                          float*, float*, int*, cudaStream_t);
template void launch_gather_narrow<__nv_bfloat16>(const __nv_bfloat16*, const int*, const int*,
                                                  const int*, const int*, const int*, const int*,
                                                  int, int, int, __nv_bfloat16*, __nv_bfloat16*,
                                                  int*, cudaStream_t);

void launch_unmask(const float* conf, const int32_t* pred, int32_t* tokens, int B, int N,
                   int mask_id, int gen_start, int block_len, int n_unmask, float tau,
                   int pos_cap, int32_t* pos_out, const int32_t* forced, cudaStream_t s) {
  if (B <= 0) return;
  ProfScope prof("unmask", s);
  unmask_kernel<<<B, 1024, 0, s>>>(conf, pred, tokens, N, mask_id, gen_start, block_len, n_unmask,
                                   tau, pos_cap, pos_out, forced);
}

void launch_block_start(const int32_t* tokens, int B, int N, int mask_id, int gen_start,
                        int block_len, int32_t* out, cudaStream_t s) {
  if (B <= 0) return;
  ProfScope prof("block_start", s);
  block_start_kernel<<<B, 256, 0, s>>>(tokens, N, mask_id, gen_start, block_len, out);
}

void launch_row_map(const int32_t* idx, const int32_t* count, int B, int k_cap, int N,
                    int* row_off, int* row_pos, int* row_seq, int* status, cudaStream_t s) {
  ProfScope prof("row_map", s);
  row_map_kernel<<<1, 1024, 0, s>>>(idx, count, B, k_cap, N, row_off, row_pos, row_seq, status);
}

void launch_row_map_dense(int B, int N, int* row_off, int* row_pos, int* row_seq,
                          cudaStream_t s) {
  ProfScope prof("row_map", s);
  row_map_dense_kernel<<<grid_for((size_t)B * N, 256), 256, 0, s>>>(B, N, row_off, row_pos,
                                                                    row_seq);
}

template <typename T>
void launch_ffn_gate(const T* o, T* ctx, const int* row_pos, const int* row_seq,
                     const int* M_dev, int M_cap, int N, int q, float tau, int all_rows,
                     const uint8_t* forced, int* flag, int* list, int* inv, int* n_sal,
                     cudaStream_t s) {
  if (M_cap <= 0) return;
  ProfScope prof("ffn_gate", s);
  ffn_gate_kernel<T><<<(M_cap + 7) / 8, 256, 0, s>>>(o, ctx, row_pos, row_seq, M_dev, M_cap, N, q,
                                                     tau, all_rows, forced, flag);
  flag_compact_kernel<<<1, 1024, 0, s>>>(flag, M_dev, M_cap, list, inv, n_sal);
}
template void launch_ffn_gate<float>(const float*, float*, const int*, const int*, const int*, int,
                                     int, int, float, int, const uint8_t*, int*, int*, int*, int*,
                                     cudaStream_t);
template void launch_ffn_gate<__nv_bfloat16>(const __nv_bfloat16*, __nv_bfloat16*, const int*,
                                             const int*, const int*, int, int, int, float, int,
                                             const uint8_t*, int*, int*, int*, int*,
                                             cudaStream_t);

template <typename T>
void launch_ffn_combine(T* x, const T* f_new, T* f_cache, const int* inv, const int* row_pos,
                        const int* row_seq, const int* M_dev, int M_cap, int N, int d,
                        cudaStream_t s) {
  if (M_cap <= 0) return;
  ProfScope prof("ffn_combine", s);
  ffn_combine_kernel<T><<<M_cap, 128, 0, s>>>(x, f_new, f_cache, inv, row_pos, row_seq, M_dev,
                                              M_cap, N, d);
}
template void launch_ffn_combine<float>(float*, const float*, float*, const int*, const int*,
                                        const int*, const int*, int, int, int, cudaStream_t);
template void launch_ffn_combine<__nv_bfloat16>(__nv_bfloat16*, const __nv_bfloat16*,
                                                __nv_bfloat16*, const int*, const int*,
                                                const int*, const int*, int, int, int,
                                                cudaStream_t);

void launch_row_words(void* cache, void* compact, const int* row_pos, const int* row_seq,
                      const int* M_dev, int M_cap, int N, int row_bytes, bool to_cache,
                      cudaStream_t s) {
  if (M_cap <= 0 || row_bytes <= 0) return;
  ProfScope prof(to_cache ? "scatter_rows" : "gather_rows_cache", s);
  row_words_kernel<<<M_cap, 128, 0, s>>>(static_cast<uint32_t*>(cache),
                                         static_cast<uint32_t*>(compact), row_pos, row_seq,
                                         M_dev, M_cap, N, row_bytes / 4, to_cache ? 1 : 0);
}

void launch_mark_rows(const int* row_pos, const int* row_seq, const int* M_dev, int M_cap, int B,
                      int N, uint8_t* flags, cudaStream_t s) {
  ProfScope prof("mark_rows", s);
  cudaMemsetAsync(flags, 0, (size_t)B * N, s);
  if (M_cap > 0)
    mark_rows_kernel<<<grid_for((size_t)M_cap, 256), 256, 0, s>>>(row_pos, row_seq, M_dev, M_cap,
                                                                  N, flags);
}

void launch_seq_offsets(int B, int N, int* off, cudaStream_t s) {
  seq_offsets_kernel<<<grid_for((size_t)B + 1, 256), 256, 0, s>>>(B, N, off);
}

void launch_copy_idx(const int32_t* src_idx, const int32_t* src_count, int32_t* dst_idx,
                     int32_t* dst_count, int B, int k_cap, cudaStream_t s) {
  ProfScope prof("copy_idx", s);
  copy_idx_kernel<<<grid_for((size_t)B * k_cap, 256), 256, 0, s>>>(src_idx, src_count, dst_idx,
                                                                   dst_count, B, k_cap);
}

template <typename T>
void launch_gather_rows(const T* src_full, const T* embed, const int32_t* tokens,
                        const int* row_pos, const int* row_seq, const int* M_dev, int M_cap,
                        int N, int d, T* x, T* h_ref, int vocab, int* status, cudaStream_t s) {
  if (M_cap <= 0) return;
  ProfScope prof("gather", s);
  gather_rows_kernel<T><<<(M_cap + 7) / 8, 256, 0, s>>>(src_full, embed, tokens, row_pos,
                                                        row_seq, M_dev, M_cap, N, d, x, h_ref,
                                                        vocab, status);
}
template void launch_gather_rows<float>(const float*, const float*, const int32_t*, const int*,
                                        const int*, const int*, int, int, int, float*, float*,
                                        int, int*, cudaStream_t);
template void launch_gather_rows<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                const int32_t*, const int*, const int*,
                                                const int*, int, int, int, __nv_bfloat16*,
                                                __nv_bfloat16*, int, int*, cudaStream_t);

template <typename T>
void launch_rmsnorm(const T* x, const T* g, T* out, const int* M_dev, int M_cap, int d, float eps,
                    cudaStream_t s) {
  if (M_cap <= 0) return;
  ProfScope prof("rmsnorm", s);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((M_cap + 7) / 8));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  cudaLaunchKernelEx(&cfg, rmsnorm_kernel<T>, x, g, out, M_dev, M_cap, d, eps);
}
template void launch_rmsnorm<float>(const float*, const float*, float*, const int*, int, int,
                                    float, cudaStream_t);
template void launch_rmsnorm<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                            __nv_bfloat16*, const int*, int, int, float,
                                            cudaStream_t);

template <typename T>
void launch_rmsnorm_rows(const T* x, const T* g, T* out, const int* rows, const int* n_rows,
                         int cap, int d, float eps, cudaStream_t s) {
  if (cap <= 0) return;
  ProfScope prof("rmsnorm", s);
  rmsnorm_rows_kernel<T><<<(cap + 7) / 8, 256, 0, s>>>(x, g, out, rows, n_rows, cap, d, eps);
}
template void launch_rmsnorm_rows<float>(const float*, const float*, float*, const int*,
                                         const int*, int, int, float, cudaStream_t);
template void launch_rmsnorm_rows<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                 __nv_bfloat16*, const int*, const int*, int, int,
                                                 float, cudaStream_t);

void launch_rope_table(float2* table, int N, int hd, float theta, cudaStream_t s) {
  ProfScope prof("rope_table", s);
  rope_table_kernel<<<grid_for((size_t)N * hd / 2, 256), 256, 0, s>>>(table, N, hd,
                                                                      (double)theta);
}

void launch_masked_rows(const int32_t* tokens, int mask_id, const int* row_pos,
                        const int* row_seq, const int* M_dev, int M_cap, int N, int* lm_rows,
                        int* n_lm, cudaStream_t s) {
  ProfScope prof("masked_rows", s);
  masked_rows_kernel<<<1, 1024, 0, s>>>(tokens, mask_id, row_pos, row_seq, M_dev, M_cap, N,
                                        lm_rows, n_lm);
}

void launch_lm_merge(const float* lm_part, int tiles, const int* lm_rows, const int* n_lm,
                     int cap, const int* row_pos, const int* row_seq, int N, float* conf,
                     int32_t* pred, cudaStream_t s) {
  if (cap <= 0) return;
  ProfScope prof("lm_merge", s);
  lm_merge_kernel<<<(cap + 3) / 4, 128, 0, s>>>(lm_part, tiles, lm_rows, n_lm, cap, row_pos,
                                                row_seq, N, conf, pred);
}

void launch_gemm_f32(const float* A, const float* B, float* C, const float* R, const int* M_dev,
                     int M_cap, int N, int K, cudaStream_t s) {
  if (M_cap <= 0) return;
  ProfScope prof("gemm_f32", s);
  dim3 grid((N + 63) / 64, (M_cap + 63) / 64);
  gemm_f32_kernel<<<grid, 256, 0, s>>>(A, B, C, R, M_dev, M_cap, N, K);
}

void launch_qkv_post_f32(const float* q_raw, const float* k_raw, const float* v_raw,
                         float* q_out, float* kc, float* vc, const int* row_pos,
                         const int* row_seq, const int* M_dev, int M_cap, int Nseq, int Hq,
                         int Hkv, int hd, const float2* rope, cudaStream_t s) {
  if (M_cap <= 0) return;
  ProfScope prof("qkv_post_f32", s);
  qkv_post_f32_kernel<<<M_cap, 256, 0, s>>>(q_raw, k_raw, v_raw, q_out, kc, vc, row_pos, row_seq,
                                            M_dev, M_cap, Nseq, Hq, Hkv, hd, rope);
}

void launch_swiglu_f32(const float* g, const float* u, float* a, const int* M_dev, int M_cap,
                       int F, cudaStream_t s) {
  if (M_cap <= 0) return;
  ProfScope prof("swiglu_f32", s);
  swiglu_f32_kernel<<<grid_for((size_t)M_cap * F, 256), 256, 0, s>>>(g, u, a, M_dev, M_cap, F);
}

void launch_attention_f32(const float* q, const float* kc, const float* vc, float* o,
                          const int* row_seq, const int* M_dev, int M_cap, int Nseq, int Hq,
                          int Hkv, int hd, cudaStream_t s) {
  if (M_cap <= 0) return;
  ProfScope prof("attention_f32", s);
  const size_t smem = (size_t)Nseq * sizeof(float);
  if (ensure_smem_attr<attention_f32_kernel>(64 * 1024) != cudaSuccess) return;
  dim3 grid(M_cap, Hq);
  attention_f32_kernel<<<grid, 128, smem, s>>>(q, kc, vc, o, row_seq, M_dev, M_cap, Nseq, Hq, Hkv,
                                               hd);
}

void launch_confidence_rows_f32(const float* logits, int V, const int* lm_rows, const int* n_lm,
                                int cap, const int* row_pos, const int* row_seq, int N,
                                float* conf, int32_t* pred, cudaStream_t s) {
  if (cap <= 0) return;
  ProfScope prof("confidence", s);
  confidence_rows_f32_kernel<<<cap, 256, 0, s>>>(logits, V, lm_rows, n_lm, row_pos, row_seq, N,
                                                 conf, pred);
}

}  // namespace dllm
