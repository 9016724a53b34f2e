// Tensor-core GEMM for the selected-row projections, sm_100a.
//
//   C[M, N] = A[M, K] * B[N, K]^T     bf16 operands, fp32 accumulation in TMEM
//
// A holds the compact (gathered) rows of the selected tokens, B a weight
// matrix [out, in].  Structure:
//   * persistent CTAs (one per SM), static round-robin over work units; a
//     unit is (m-tile of 128 rows, n-tile of BN columns, K split);
//   * warp 0: TMA producer (128-byte-swizzled boxes of 64 K-elements into a
//     STAGES-deep ring, one mbarrier pair per stage);
//   * warp 1: allocates TMEM and issues tcgen05.mma (M=128, N=BN, K=16) from
//     a single thread; two accumulator buffers of BN fp32 columns so the
//     epilogue of one unit overlaps the main loop of the next;
//   * warps 2-5: epilogue, one TMEM lane quadrant each (thread = one row),
//     fused per use: plain store, residual add, SwiGLU, RoPE + K/V cache
//     scatter, or the LM-head online softmax statistics;
//   * weight-streaming shapes may split K across the CTAs of a thread-block
//     cluster: each CTA stages its fp32 partial tile in shared memory and the
//     cluster reduces it over distributed shared memory in split order, so
//     the result does not depend on timing;
//   * tensor-bound plain, residual and QKV GEMMs run on CTA pairs instead
//     (gemm_pair_kernel: tcgen05 cta_group::2, 256 x 256 tiles).
// No TMA multicast is used anywhere.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dllm {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;


constexpr int NUM_THREADS = 192;
constexpr int EPI_THREADS = 128;

__host__ __device__ constexpr int stages_for(int bn) { return bn >= 256 ? 4 : (bn >= 128 ? 6 : 8); }
__host__ __device__ constexpr int tmem_cols_for(int bn) { return 2 * bn < 32 ? 32 : 2 * bn; }
__host__ __device__ constexpr size_t smem_bytes_for(int bn) {
  return (size_t)stages_for(bn) * (BM * BK * 2 + bn * BK * 2) + 1024 + 256;
}

struct Params {
  int M_cap;
  const int* M_dev;
  int N;  // output columns of the GEMM (SWIGLU: 2F)
  int K;
  int tiles_n;
  int splits;
  int kb_total;
  int kb_per_split;
  int seg0, seg1;  // column boundaries of B segments
  __nv_bfloat16* out;
  int ldo;
  __nv_bfloat16* kc;
  __nv_bfloat16* vc;
  const int* row_pos;
  const int* row_seq;
  int Nseq;
  int q_cols, kv_cols, hd;
  const float2* rope;
  float* lm_part;
  int V;
  int a_tx;  // bytes one A box delivers (fewer than a full 128-row tile when M_cap < 128)
  int prefetch_b;  // issue the first unit's weight tiles before waiting on the previous kernel
  int raster_g;    // row tiles (pairs, in the CTA-pair kernel) per raster group
  int stall_test;  // CTA-pair kernel, tests only: CTA 1 withholds its first stage
  int krot;        // walk each tile's k-blocks from a tile-dependent start (weight streaming)
  int* status;
};

// G: row tiles per raster group (the group's A rows stay in L2 while its CTAs sweep
// every column tile)
__device__ __forceinline__ void decode_unit(int u, int m_tiles, int tiles_n, int splits, int& m,
                                            int& n, int& s, int G = 32) {
  s = u % splits;
  const int t = u / splits;
  const int per_group = G * tiles_n;
  const int g = t / per_group;
  const int first_m = g * G;
  const int gsz = min(m_tiles - first_m, G);
  const int r = t - g * per_group;
  m = first_m + r % gsz;
  n = r / gsz;
}

// The i-th k-block of a unit whose K range is [kb0, kb0 + nkb), for output tile n.
// With krot the walk starts at a tile-dependent block and wraps around, so that
// CTAs streaming different weight tiles at the same time read different column
// ranges of their rows (the same accumulation, in another order); measured ~3%
// faster on weight-streaming GEMMs and slower on tensor-bound ones.
__device__ __forceinline__ int kb_at(int i, int kb0, int nkb, int n, int krot) {
  if (!krot) return kb0 + i;
  int j = i + (n * 5) % nkb;
  if (j >= nkb) j -= nkb;
  return kb0 + j;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

// ---------------------------------------------------------------- cluster / DSMEM
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// the address of the same shared-memory offset in CTA `rank` of this cluster
__device__ __forceinline__ uint32_t mapa_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
// every thread of every CTA in the cluster
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// ---------------------------------------------------------------- epilogues
// `ld(c, v)` fills v[0..31] with fp32 columns [c, c+32) of this thread's row
// in the tile; every lane of the warp must call it (TMEM loads are warp-wide).

template <int BN, int EPI, class Loader>
__device__ __forceinline__ void epilogue_tile(const Params& p, int row, bool row_ok, int m, int n,
                                              Loader&& ld) {
  if constexpr (EPI == EPI_STORE || EPI == EPI_RESID) {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      float v[32];
      ld(c, v);
      const int col = n * BN + c;
      if (row_ok) {
        __nv_bfloat16* o = p.out + (size_t)row * p.ldo + col;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          if (col + j < p.N) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = v[j + i];
            if constexpr (EPI == EPI_RESID) {
              float r[8];
              unpack8(*reinterpret_cast<const uint4*>(o + j), r);
#pragma unroll
              for (int i = 0; i < 8; ++i) f[i] += r[i];
            }
            *reinterpret_cast<uint4*>(o + j) = pack8(f);
          }
        }
      }
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    const int F = p.N >> 1;
#pragma unroll 1
    for (int c = 0; c < BN / 2; c += 32) {
      float g[32], u[32];
      ld(c, g);
      ld(BN / 2 + c, u);
      const int col = n * (BN / 2) + c;
      if (row_ok) {
        __nv_bfloat16* o = p.out + (size_t)row * p.ldo + col;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          if (col + j < F) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = silu_f(g[j + i]) * u[j + i];
            *reinterpret_cast<uint4*>(o + j) = pack8(f);
          }
        }
      }
    }
  } else if constexpr (EPI == EPI_QKV) {
    const int n0 = n * BN;
    int pos = 0, seq = 0;
    if (row_ok) {
      pos = p.row_pos[row];
      seq = p.row_seq[row];
    }
    __nv_bfloat16* dst;
    bool rot;
    if (n0 < p.q_cols) {
      dst = p.out + (size_t)row * p.ldo + n0;
      rot = p.rope != nullptr;
    } else if (n0 < p.q_cols + p.kv_cols) {
      dst = p.kc + ((size_t)seq * p.Nseq + pos) * p.kv_cols + (n0 - p.q_cols);
      rot = p.rope != nullptr;
    } else {
      dst = p.vc + ((size_t)seq * p.Nseq + pos) * p.kv_cols + (n0 - p.q_cols - p.kv_cols);
      rot = false;
    }
    if (!rot) {
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        ld(c, v);
        if (row_ok) {
#pragma unroll
          for (int j = 0; j < 32; j += 8)
            *reinterpret_cast<uint4*>(dst + c + j) = pack8(v + j);
        }
      }
    } else {
      const int half = p.hd >> 1;
#pragma unroll 1
      for (int h0 = 0; h0 < BN; h0 += p.hd) {
#pragma unroll 1
        for (int c = 0; c < half; c += 32) {
          float x1[32], x2[32];
          ld(h0 + c, x1);
          ld(h0 + half + c, x2);
          if (row_ok) {
            const float2* cs = p.rope + (size_t)pos * half + c;
            float y1[32], y2[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float2 t = cs[i];
              y1[i] = x1[i] * t.x - x2[i] * t.y;
              y2[i] = x2[i] * t.x + x1[i] * t.y;
            }
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              *reinterpret_cast<uint4*>(dst + h0 + c + j) = pack8(y1 + j);
              *reinterpret_cast<uint4*>(dst + h0 + half + c + j) = pack8(y2 + j);
            }
          }
        }
      }
    }
  } else if constexpr (EPI == EPI_LMHEAD) {
    float mx = -INFINITY, sm = 0.0f;
    int arg = 0;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      float v[32];
      ld(c, v);
      const int col0 = n * BN + c;
      float cm = -INFINITY;
      int ca = col0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (col0 + i < p.V && v[i] > cm) {
          cm = v[i];
          ca = col0 + i;
        }
      }
      const float nm = fmaxf(mx, cm);
      if (nm != -INFINITY) {
        sm = (mx == -INFINITY) ? 0.0f : sm * expf(mx - nm);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (col0 + i < p.V) sm += expf(v[i] - nm);
      }
      if (cm > mx) arg = ca;
      mx = nm;
    }
    if (row_ok) {
      float* o = p.lm_part + ((size_t)row * p.tiles_n + n) * 3;
      o[0] = mx;
      o[1] = sm;
      o[2] = __int_as_float(arg);
    }
  }
}

// ---------------------------------------------------------------- kernel

template <int BN, int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ CUtensorMap tmB2, const Params p) {
  constexpr int STAGES = stages_for(BN);
  constexpr int A_BYTES = BM * BK * 2;
  constexpr int B_BYTES = BN * BK * 2;
  constexpr uint32_t TMEM_COLS = tmem_cols_for(BN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain[1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[STAGES + s]); };
  auto tfull_bar = [&](int a) { return smem_u32(&bars[2 * STAGES + a]); };
  auto tempty_bar = [&](int a) { return smem_u32(&bars[2 * STAGES + 2 + a]); };
  const uint32_t drain_bar = smem_u32(&bars[2 * STAGES + 4]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), EPI_THREADS);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (EPI == EPI_SWIGLU || EPI == EPI_QKV) tma_prefetch_desc(&tmB1);
    if (EPI == EPI_QKV) tma_prefetch_desc(&tmB2);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the next kernel may start its CTAs on SMs this grid leaves free
  griddep_launch_dependents();

  // weight (B) tile of k-block kb of output tile n into a stage
  auto load_b = [&](uint32_t b_dst, uint32_t bar, int kb, int n) {
    if constexpr (EPI == EPI_SWIGLU) {
      tma_load_2d(b_dst, &tmB0, bar, kb * BK, n * (BN / 2));
      tma_load_2d(b_dst + (BN / 2) * BK * 2, &tmB1, bar, kb * BK, n * (BN / 2));
    } else if constexpr (EPI == EPI_QKV) {
      const int n0 = n * BN;
      if (n0 < p.seg0)
        tma_load_2d(b_dst, &tmB0, bar, kb * BK, n0);
      else if (n0 < p.seg1)
        tma_load_2d(b_dst, &tmB1, bar, kb * BK, n0 - p.seg0);
      else
        tma_load_2d(b_dst, &tmB2, bar, kb * BK, n0 - p.seg1);
    } else {
      tma_load_2d(b_dst, &tmB0, bar, kb * BK, n * BN);
    }
  };

  // Weights never depend on earlier kernels: with a single row tile by
  // capacity, the producer starts streaming this CTA's first weight tiles
  // before it waits for the kernel that writes A (and the row count).
  int npre = 0, pre_n = 0, pre_kb0 = 0, pre_nkb = 1;
  if (p.prefetch_b && warp == 0 && lane == 0 && (int)blockIdx.x < p.tiles_n * p.splits) {
    int m, s;
    decode_unit(blockIdx.x, 1, p.tiles_n, p.splits, m, pre_n, s, p.raster_g);
    pre_kb0 = s * p.kb_per_split;
    pre_nkb = max(1, min(pre_kb0 + p.kb_per_split, p.kb_total) - pre_kb0);
    npre = max(0, min(STAGES, min(pre_kb0 + p.kb_per_split, p.kb_total) - pre_kb0));
    for (int i = 0; i < npre; ++i) {  // fresh stages: no empty wait
      mbar_arrive_expect_tx(full_bar(i), (uint32_t)p.a_tx + B_BYTES);
      load_b(smem_u32(sB + i * B_BYTES), full_bar(i), kb_at(i, pre_kb0, pre_nkb, pre_n, p.krot), pre_n);
    }
  }
  griddep_wait();

  int M = p.M_cap;
  if (p.M_dev) {
    M = *p.M_dev;
    if (M > p.M_cap || M < 0) {
      if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(p.status, DEV_BAD_SHAPE);
      M = M < 0 ? 0 : p.M_cap;
    }
  }
  const int m_tiles = (M + BM - 1) / BM;
  const int n_units = m_tiles * p.tiles_n * p.splits;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = npre % STAGES;
      uint32_t phase = npre == STAGES ? 1u : 0u;
      uint32_t issued = 0;
      uint32_t issue_phase = 0;
      bool ok = true;
      // the A halves of the pre-issued stages (row tile 0); when this CTA has no
      // unit after all (no rows), they only complete the stages before exit
      for (int i = 0; i < npre; ++i) {
        tma_load_2d(smem_u32(sA + i * A_BYTES), &tmA, full_bar(i),
                    kb_at(i, pre_kb0, pre_nkb, pre_n, p.krot) * BK, 0);
        issued |= 1u << i;
      }
      if (npre > 0 && (int)blockIdx.x >= n_units) {
        for (int i = 0; i < npre; ++i) mbar_wait_drain(full_bar(i), 0, p.status);
        npre = 0;
      }
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        int m, n, s;
        decode_unit(u, m_tiles, p.tiles_n, p.splits, m, n, s, p.raster_g);
        const int kb0 = s * p.kb_per_split;
        const int nkb = min(kb0 + p.kb_per_split, p.kb_total) - kb0;
        for (int i = (u == (int)blockIdx.x ? npre : 0); i < nkb; ++i) {
          const int kb = kb_at(i, kb0, nkb, n, p.krot);
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(stage), (uint32_t)p.a_tx + B_BYTES);
          const uint32_t a_dst = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * B_BYTES);
          tma_load_2d(a_dst, &tmA, full_bar(stage), kb * BK, m * BM);
          load_b(b_dst, full_bar(stage), kb, n);
          issued |= 1u << stage;
          if (phase) issue_phase |= 1u << stage; else issue_phase &= ~(1u << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // drain: every load this thread issued must land before the block exits
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s)) mbar_wait_drain(full_bar(s), (issue_phase >> s) & 1u, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued_any = false;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        int m, n, s;
        decode_unit(u, m_tiles, p.tiles_n, p.splits, m, n, s, p.raster_g);
        const int kb0 = s * p.kb_per_split;
        const int kb1 = min(kb0 + p.kb_per_split, p.kb_total);
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {  // stages arrive in the producer's k order
          if (!mbar_wait(full_bar(stage), phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            tc_mma_bf16(d_tmem, umma_desc_k_sw128(a_base + k * 32),
                        umma_desc_k_sw128(b_base + k * 32), idesc,
                        (kb > kb0 || k > 0) ? 1u : 0u);
          }
          issued_any = true;
          tc_commit(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok && issued_any) {
        tc_commit(drain_bar);
        mbar_wait_drain(drain_bar, 0, p.status);
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int quad = warp & 3;  // TMEM lanes [32*quad, 32*quad+32)
    const int r_in_tile = quad * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      int m, n, s;
      decode_unit(u, m_tiles, p.tiles_n, p.splits, m, n, s, p.raster_g);
      // warp-uniform outcome: TMEM loads below are warp-collective
      const bool ok = __all_sync(0xffffffffu,
                                 mbar_wait(tfull_bar(acc), acc_phase, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      const int row = m * BM + r_in_tile;
      const bool row_ok = row < M;
      const uint32_t t_row = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
      if (p.splits == 1) {
        epilogue_tile<BN, EPI>(p, row, row_ok, m, n,
                               [&](int c, float* v) { tmem_ld_32x32b_x32(t_row + c, v); });
      } else {
        // split K inside a cluster: stage this CTA's fp32 partial rows in its own
        // shared memory (the stage ring is idle once the accumulator is complete)
        float* rrow = reinterpret_cast<float*>(smem) + (size_t)r_in_tile * (BN + 4);
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          float v[32];
          tmem_ld_32x32b_x32(t_row + c, v);
          float4* dst = reinterpret_cast<float4*>(rrow + c);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (p.splits > 1) {
    // The S CTAs of a cluster computed the S K-slices of one tile.  After the
    // first cluster barrier every partial is staged; CTA `rank` sums rows
    // [rank*SR, rank*SR + SR) of all S partials over distributed shared memory
    // (in split order, so the result does not depend on timing) and runs the
    // fused epilogue on them.  The second barrier keeps every CTA (and its
    // staged partial) alive until all reads are done.
    cluster_sync_all();
    if (warp >= 2 && (int)blockIdx.x < n_units) {
      int m, n, s;
      decode_unit(blockIdx.x, m_tiles, p.tiles_n, p.splits, m, n, s, p.raster_g);
      const int S = p.splits;
      const int rank = (int)cluster_ctarank();
      const int SR = (BM + S - 1) / S;
      const int r0 = rank * SR;
      const int valid = min(BM, M - m * BM);
      const int nrow = max(0, min(min(BM, r0 + SR), valid) - r0);
      const int t = threadIdx.x - 64;
      float* R = reinterpret_cast<float*>(smem);
      constexpr int Q4 = BN / 4;
      for (int e = t; e < nrow * Q4; e += EPI_THREADS) {
        const int rr = r0 + e / Q4, c4 = e - (e / Q4) * Q4;
        float* mine = R + (size_t)rr * (BN + 4) + c4 * 4;
        const uint32_t la = smem_u32(mine);
        float4 part[8];
#pragma unroll
        for (int sp = 0; sp < 8; ++sp)
          if (sp < S) part[sp] = ld_dsmem_f4(mapa_rank(la, (uint32_t)sp));
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int sp = 0; sp < 8; ++sp)
          if (sp < S) {
            a.x += part[sp].x;
            a.y += part[sp].y;
            a.z += part[sp].z;
            a.w += part[sp].w;
          }
        *reinterpret_cast<float4*>(mine) = a;  // only this CTA reads its own slice rows
      }
      named_bar_sync(1, EPI_THREADS);
      if (t < nrow) {
        const int rl = r0 + t;
        const int row = m * BM + rl;
        const float* yrow = R + (size_t)rl * (BN + 4);
        epilogue_tile<BN, EPI>(p, row, row < M, m, n, [&](int c, float* v) {
          const float4* src = reinterpret_cast<const float4*>(yrow + c);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 x = src[i];
            v[4 * i] = x.x;
            v[4 * i + 1] = x.y;
            v[4 * i + 2] = x.z;
            v[4 * i + 3] = x.w;
          }
        });
      }
    }
    cluster_sync_all();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- CTA-pair kernel
// Plain, residual and QKV GEMMs with at least two row tiles, 256-wide tiles and
// no K split (the tensor-bound shapes, and 129-255-row weight streaming): the
// two CTAs of a cluster compute one 256 x 256 tile with tcgen05.mma.cta_group::2
// issued by CTA 0.  CTA r stages rows [128 r, 128 r + 128) of the A tile and
// columns [128 r, 128 r + 128) of the B tile (32 KB per 64-deep k-block instead
// of 48 KB, so the ring holds 7 k-blocks), and its TMEM receives its 128 rows
// of the accumulator over all 256 columns.  Each CTA's TMA loads complete on its
// own barriers; CTA 1's issuer thread forwards each landed stage to CTA 0
// (remote mbarrier arrive), CTA 0's commits arrive on both CTAs' barriers
// (multicast commit), and CTA 1's epilogue warps release accumulators to CTA 0
// by remote arrive.  No TMA multicast.

constexpr int PAIR_BN = 256;
constexpr int PAIR_STAGES = 7;
constexpr size_t PAIR_SMEM = (size_t)PAIR_STAGES * (BM * BK * 2 + (PAIR_BN / 2) * BK * 2) + 1024 + 256;

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D (+)= A * B^T over the CTA pair: M = 256 (128 rows per CTA), N = 256
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on the barrier at this offset in both CTAs of the pair once the pair's
// earlier tcgen05 ops issued by this thread complete
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
// the same, on this CTA's barrier only
__device__ __forceinline__ void tc_commit_pair_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// arrive on a barrier of another CTA of the cluster (address from mapa).  The
// cross-CTA barriers use the default (CTA-scope) semantics of arrive and
// try_wait: the data they guard is read by the tensor core or by tcgen05.ld
// after tcgen05 fences, not through the generic proxy.  Cluster-scope acquire in
// the waits cost the pair ring about half its throughput (QKV shape 684 against
// 1340 TFLOP/s).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                     const __grid_constant__ CUtensorMap tmB1,
                     const __grid_constant__ CUtensorMap tmB2, const Params p) {
  constexpr int BN = PAIR_BN, BNH = PAIR_BN / 2, STAGES = PAIR_STAGES;
  constexpr int A_BYTES = BM * BK * 2;
  constexpr int B_BYTES = BNH * BK * 2;  // this CTA's half of the B tile
  constexpr uint32_t TMEM_COLS = 2 * BN;
  constexpr int EPI_WARPS = EPI_THREADS / 32;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES);
  // bars: full[S], empty[S], pfull[S], tfull[2], tempty[2], drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 issues the MMAs, 1 is its peer
  const int pair_id = (int)blockIdx.x >> 1;
  const int n_pairs = (int)gridDim.x >> 1;

  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[STAGES + s]); };
  auto pfull_bar = [&](int s) { return smem_u32(&bars[2 * STAGES + s]); };  // CTA 0: peer landed
  auto tfull_bar = [&](int a) { return smem_u32(&bars[3 * STAGES + a]); };
  auto tempty_bar = [&](int a) { return smem_u32(&bars[3 * STAGES + 2 + a]); };
  const uint32_t drain_bar = smem_u32(&bars[3 * STAGES + 4]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
      mbar_init(pfull_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * EPI_WARPS);  // the epilogue warps of both CTAs
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (EPI == EPI_QKV) {
      tma_prefetch_desc(&tmB1);
      tma_prefetch_desc(&tmB2);
    }
  }
  tc_fence_before();
  __syncthreads();
  // both CTAs' barriers exist before either CTA signals the other's
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();

  // this CTA's half (columns [n*BN + rank*BNH, +BNH)) of the B tile of k-block kb
  // (plain, residual and QKV epilogues; the planner keeps SwiGLU and the LM head
  // on single CTAs)
  static_assert(EPI != EPI_SWIGLU && EPI != EPI_LMHEAD, "not run on CTA pairs");
  auto load_b_half = [&](uint32_t b_dst, uint32_t bar, int kb, int n) {
    if constexpr (EPI == EPI_QKV) {
      const int n0 = n * BN + (int)rank * BNH;  // segments are multiples of BN
      if (n0 < p.seg0)
        tma_load_2d(b_dst, &tmB0, bar, kb * BK, n0);
      else if (n0 < p.seg1)
        tma_load_2d(b_dst, &tmB1, bar, kb * BK, n0 - p.seg0);
      else
        tma_load_2d(b_dst, &tmB2, bar, kb * BK, n0 - p.seg1);
    } else {
      tma_load_2d(b_dst, &tmB0, bar, kb * BK, n * BN + (int)rank * BNH);
    }
  };

  griddep_wait();
  int M = p.M_cap;
  if (p.M_dev) {
    M = *p.M_dev;
    if (M > p.M_cap || M < 0) {
      if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(p.status, DEV_BAD_SHAPE);
      M = M < 0 ? 0 : p.M_cap;
    }
  }
  const int m_pairs = (M + 2 * BM - 1) / (2 * BM);
  const int n_units = m_pairs * p.tiles_n;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issue_phase = 0;
      bool ok = true;
      for (int u = pair_id; u < n_units && ok; u += n_pairs) {
        int mp, n, s;
        decode_unit(u, m_pairs, p.tiles_n, 1, mp, n, s, p.raster_g);
        for (int i = 0; i < p.kb_total; ++i) {
          const int kb = kb_at(i, 0, p.kb_total, n, p.krot);
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(stage), (uint32_t)(A_BYTES + B_BYTES));
          tma_load_2d(smem_u32(sA + stage * A_BYTES), &tmA, full_bar(stage), kb * BK,
                      mp * 2 * BM + (int)rank * BM);
          load_b_half(smem_u32(sB + stage * B_BYTES), full_bar(stage), kb, n);
          issued |= 1u << stage;
          if (phase) issue_phase |= 1u << stage; else issue_phase &= ~(1u << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (ok) {
        // every stage's last release (a commit of CTA 0 arriving here) has landed
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s)) mbar_wait_drain(empty_bar(s), (issue_phase >> s) & 1u, p.status);
      } else {
        // every load this thread issued lands before the block exits
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s)) mbar_wait_drain(full_bar(s), (issue_phase >> s) & 1u, p.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 1) {
      // ------------------------------------------------ CTA 1: forward landed stages
      const uint32_t peer_pfull0 = mapa_rank(pfull_bar(0), 0u);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = pair_id; u < n_units && ok; u += n_pairs) {
        for (int kb = 0; kb < p.kb_total; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          if (!(p.stall_test && kb == 0 && u == pair_id))
            mbar_arrive_remote(peer_pfull0 + (uint32_t)(stage * 8));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    } else if (lane == 0) {
      // ------------------------------------------------ CTA 0: MMA issuer for the pair
      constexpr uint32_t idesc = umma_idesc_bf16(2 * BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued_any = false;
      for (int u = pair_id; u < n_units && ok; u += n_pairs) {
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < p.kb_total; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, p.status) ||
              !mbar_wait(pfull_bar(stage), phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            tc_mma_bf16_pair(d_tmem, umma_desc_k_sw128(a_base + k * 32),
                             umma_desc_k_sw128(b_base + k * 32), idesc,
                             (kb > 0 || k > 0) ? 1u : 0u);
          }
          issued_any = true;
          tc_commit_pair_both(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_both(tfull_bar(acc));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok && issued_any) {
        tc_commit_pair_local(drain_bar);
        mbar_wait_drain(drain_bar, 0, p.status);
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5, both CTAs)
    const int quad = warp & 3;  // TMEM lanes [32*quad, 32*quad+32)
    const int r_in_tile = quad * 32 + lane;
    const uint32_t tempty0 = rank == 0 ? 0u : mapa_rank(tempty_bar(0), 0u);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = pair_id; u < n_units; u += n_pairs) {
      int mp, n, s;
      decode_unit(u, m_pairs, p.tiles_n, 1, mp, n, s, p.raster_g);
      const bool ok = __all_sync(0xffffffffu,
                                 mbar_wait(tfull_bar(acc), acc_phase, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      const int row = mp * 2 * BM + (int)rank * BM + r_in_tile;
      const uint32_t t_row = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
      epilogue_tile<BN, EPI>(p, row, row < M, mp * 2 + (int)rank, n,
                             [&](int c, float* v) { tmem_ld_32x32b_x32(t_row + c, v); });
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(tempty_bar(acc));
        else
          mbar_arrive_remote(tempty0 + (uint32_t)(acc * 8));
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA leaves (or frees TMEM) while the other may still signal it
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

// [rows, cols] bf16 row-major, box (64 cols, box_rows rows), 128-byte swizzle
bool make_map(CUtensorMap* m, const void* ptr, int rows, int cols, int box_rows) {
  if (rows <= 0 || cols <= 0) return false;
  return tmap_bf16_2d(m, ptr, (uint64_t)rows, (uint64_t)cols, (uint32_t)box_rows);
}

template <int BN, int EPI>
cudaError_t launch_t(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                     const CUtensorMap& b2, const Params& p, int grid, cudaStream_t s) {
  constexpr size_t smem = smem_bytes_for(BN);
  const cudaError_t ea = ensure_smem_attr<gemm_tc_kernel<BN, EPI>>((int)smem);
  if (ea != cudaSuccess) return ea;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  if (p.splits > 1) {
    // split K: one unit per CTA, the `splits` CTAs of a tile in one cluster
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)p.splits;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl_enabled()) {
    // may start while the previous kernel finishes; the kernel waits for it
    // (griddepcontrol.wait) before reading anything that kernel writes
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, EPI>, a, b0, b1, b2, p);
}

template <int EPI>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const CUtensorMap& b2, const Params& p, int grid, cudaStream_t s) {
  const cudaError_t ea = ensure_smem_attr<gemm_pair_kernel<EPI>>((int)PAIR_SMEM);
  if (ea != cudaSuccess) return ea;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = PAIR_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = 2;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = 1;
  ++na;
  if (pdl_enabled()) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, gemm_pair_kernel<EPI>, a, b0, b1, b2, p);
}

template <int EPI>
cudaError_t launch_bn(int bn, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                      const CUtensorMap& b2, const Params& p, int grid, cudaStream_t s) {
  switch (bn) {
    case 256: return launch_t<256, EPI>(a, b0, b1, b2, p, grid, s);
    case 128: return launch_t<128, EPI>(a, b0, b1, b2, p, grid, s);
    default: return launch_t<64, EPI>(a, b0, b1, b2, p, grid, s);
  }
}

}  // namespace

// CTA-pair GEMM for tensor-bound shapes; a build with -DDLLM_BUILD_NO_PAIR keeps
// single-CTA tiles (an experiment switch of the build, not a run-time one)
#ifdef DLLM_BUILD_NO_PAIR
constexpr bool pair_enabled() { return false; }
#else
constexpr bool pair_enabled() { return true; }
#endif

int gemm_total_cols(const GemmSpec& g) {
  int n = 0;
  for (int i = 0; i < g.n_seg; ++i) n += g.seg_cols[i];
  return n;
}

GemmPlan gemm_plan(const GemmSpec& g) {
  GemmPlan pl{};
  const int N = gemm_total_cols(g);
  const int kb_total = (g.K + BK - 1) / BK;
  pl.m_tiles_cap = (g.M_cap + BM - 1) / BM;
  const int sms = num_sms();
  // candidate tile widths: every B segment (and, for QKV, every head) must tile evenly
  auto bn_ok = [&](int bn) {
    if (g.epi == EPI_SWIGLU) return (g.seg_cols[0] % (bn / 2)) == 0;
    if (g.epi == EPI_QKV) {
      for (int i = 0; i < g.n_seg; ++i)
        if (g.seg_cols[i] % bn) return false;
      return bn % g.hd == 0;
    }
    return true;
  };
  int bn = g.force_bn;
  int splits = g.force_splits;
  auto tiles_for = [&](int c) {
    const int cols = g.epi == EPI_SWIGLU ? N / 2 : N;
    const int w = g.epi == EPI_SWIGLU ? c / 2 : c;
    return pl.m_tiles_cap * ((cols + w - 1) / w);
  };
  const bool weight_bound = g.M_cap < 256;
  if (!bn && weight_bound) {
    // Weight streaming (fewer than 256 rows): a CTA streams its weight boxes at
    // roughly 40-60 GB/s, so the GEMM wants ~96-148 streaming CTAs in one wave,
    // with as few K splits as reach that (each split adds a cluster reduction)
    // and at least 16 k-blocks per split.  Measured with cold weights at 77 and
    // 192 rows of the 8B projections (us): QKV 12288x4096 tile 128 unsplit 24.5
    // (tile 256: 32.7, 2 splits 31.7); O 4096x4096 tile 128 x 4 splits 13.6
    // (tile 256 x 4: 17.6); down 4096x12288 tile 128 x 4 splits 24.7 (tile 256
    // x 4: 31.7); gate/up 24576x4096 tile 256 unsplit 39.8 (tile 128: 47.6); at
    // 192 rows QKV tile 256 unsplit 35.0 and down tile 256 x 4 splits 33.7.
    // A single row tile prefers 128-wide tiles (more CTAs), two row tiles 256.
    const int order1[2] = {128, 256}, order2[2] = {256, 128};
    const int* order = pl.m_tiles_cap == 1 ? order1 : order2;
    for (int i = 0; i < 2 && !bn; ++i) {
      const int c = order[i];
      if (!bn_ok(c)) continue;
      const int t1 = tiles_for(c);
      if (t1 > sms) continue;
      int sp = 1;
      if (t1 < 96 && g.epi != EPI_LMHEAD)
        while (sp < 8 && t1 * (sp + 1) <= sms && kb_total / (sp + 1) >= 16) ++sp;
      bn = c;
      if (!splits) splits = sp;
    }
    if (!bn) {
      // more tiles than SMs even at 256 columns: persistent CTAs, no split
      for (int c : {256, 128, 64}) {
        if (bn_ok(c)) {
          bn = c;
          break;
        }
      }
      if (!bn) bn = 64;
    }
  } else if (!bn) {
    // Tensor-bound: time ~ waves x main loop of a tile; no split.
    const int cands[3] = {256, 128, 64};
    double best = 1e30;
    for (int c : cands) {
      if (!bn_ok(c)) continue;
      if (g.epi == EPI_LMHEAD && c < 128) continue;  // stats buffers are sized for >= 128
      const int units = tiles_for(c);
      const int waves = (units + sms - 1) / sms;
      // one 64-deep k-block of an M=128 x N=c tile: 2c tensor cycles, plus a
      // fixed per-unit cost (prologue, epilogue drain); narrow tiles move more
      // operand bytes per FMA through shared memory, charged in proportion
      const double smem_ratio = ((128.0 + c) / (128.0 * c)) / ((128.0 + 256) / (128.0 * 256));
      const double per_kb = 2.0 * c * std::max(1.0, smem_ratio);
      const double t = waves * (kb_total * per_kb + 1500.0);
      if (t < best * 0.999) {
        best = t;
        bn = c;
      }
    }
    if (!bn) bn = 64;
  }
  if (!splits) splits = 1;
  if (splits > kb_total) splits = kb_total;
  {
    // no split may be empty: an empty split would publish a stale accumulator
    const int per = (kb_total + splits - 1) / splits;
    splits = (kb_total + per - 1) / per;
  }
  pl.bn = bn;
  pl.splits = splits;
  pl.tiles_n = (g.epi == EPI_SWIGLU) ? (N / 2 + bn / 2 - 1) / (bn / 2) : (N + bn - 1) / bn;
  pl.units_cap = pl.m_tiles_cap * pl.tiles_n * pl.splits;
  // split K runs one unit per CTA (clusters of `splits`); otherwise persistent CTAs
  pl.grid = splits > 1 ? pl.units_cap : std::max(1, std::min(pl.units_cap, sms));
  // at least two row tiles, 256-wide tiles, no split: persistent CTA pairs, each
  // pair one 256-row tile at a time.  Inside the power-capped 8B step (32 x 308
  // rows) the pairs made the QKV GEMM 2% and the O/down GEMMs 3.5% faster, but
  // the gate/up (SwiGLU) GEMM 5% and the LM head 9% slower (both read ~30% more
  // DRAM), so those two keep single-CTA tiles.
  // With two row tiles and no split (129-255 rows, e.g. the QKV GEMM of one
  // sequence at 192 rows) a pair also halves the weight bytes each SM streams.
  pl.pair = (pair_enabled() && splits == 1 && bn == PAIR_BN && pl.m_tiles_cap >= 2 && sms >= 2 &&
             g.epi != EPI_SWIGLU && g.epi != EPI_LMHEAD)
                ? 1 : 0;
  if (pl.pair) {
    const int units = ((pl.m_tiles_cap + 1) / 2) * pl.tiles_n;
    pl.grid = 2 * std::max(1, std::min(units, sms / 2));
  }
  return pl;
}

cudaError_t gemm_launch(GemmSpec g, cudaStream_t s) {
  if (g.M_cap <= 0) return cudaSuccess;
  const GemmPlan pl = gemm_plan(g);
  const int N = gemm_total_cols(g);
  Params p{};
  p.M_cap = g.M_cap;
  p.M_dev = g.M_dev;
  p.N = N;
  p.K = g.K;
  p.tiles_n = pl.tiles_n;
  p.splits = pl.splits;
  p.kb_total = (g.K + BK - 1) / BK;
  p.kb_per_split = (p.kb_total + pl.splits - 1) / pl.splits;
  p.seg0 = g.seg_cols[0];
  p.seg1 = g.seg_cols[0] + (g.n_seg > 1 ? g.seg_cols[1] : 0);
  p.out = g.out;
  p.ldo = g.ldo;
  p.kc = g.kc;
  p.vc = g.vc;
  p.row_pos = g.row_pos;
  p.row_seq = g.row_seq;
  p.Nseq = g.Nseq;
  p.q_cols = g.seg_cols[0];
  p.kv_cols = g.n_seg > 1 ? g.seg_cols[1] : 0;
  p.hd = g.hd;
  p.rope = g.rope;
  p.lm_part = g.lm_part;
  p.V = N;
  p.status = g.status;
  p.stall_test = g.stall_test;
  if (g.stall_test && !pl.pair) return cudaErrorInvalidValue;
  // weight-streaming shapes (fewer than 256 rows): rotated k walks
  p.krot = g.M_cap < 256 ? 1 : 0;

  CUtensorMap ta, tb0, tb1, tb2;
  // with fewer than 128 rows the A box covers only them (rounded to 16): the MMA still
  // reads 128 smem rows, but rows >= M_cap only feed output rows that are never stored
  const int a_rows = g.M_cap < BM ? ((g.M_cap + 15) / 16) * 16 : BM;
  p.a_tx = a_rows * BK * 2;
  p.prefetch_b = (g.M_cap <= BM && pdl_enabled()) ? 1 : 0;
  // m-major raster groups; the A rows of a group (256 per pair) stay within ~32 MB of
  // L2 (groups of 48, 64 and 96 MB, and column-tile groups chosen by a traffic model,
  // were measured: no faster, and the larger ones read far more DRAM)
  p.raster_g = pl.pair ? std::max(2, std::min(16, (int)((32u << 20) / ((size_t)2 * BM * g.K * 2))))
                       : 32;
  if (!make_map(&ta, g.A, g.M_cap, g.K, a_rows)) return cudaErrorInvalidValue;
  // a CTA pair stages half of each 256-wide B tile per CTA
  const int bbox = (g.epi == EPI_SWIGLU || pl.pair) ? pl.bn / 2 : pl.bn;
  if (!make_map(&tb0, g.B[0], g.seg_cols[0], g.K, bbox)) return cudaErrorInvalidValue;
  tb1 = tb0;
  tb2 = tb0;
  if (g.n_seg > 1 && !make_map(&tb1, g.B[1], g.seg_cols[1], g.K, bbox)) return cudaErrorInvalidValue;
  if (g.n_seg > 2 && !make_map(&tb2, g.B[2], g.seg_cols[2], g.K, bbox)) return cudaErrorInvalidValue;

  static const char* names[5] = {"gemm_store", "gemm_resid", "gemm_swiglu", "gemm_qkv",
                                 "gemm_lmhead"};
  ProfScope prof(names[g.epi], s);
  if (pl.pair) {
    switch (g.epi) {
      case EPI_STORE: return launch_pair<EPI_STORE>(ta, tb0, tb1, tb2, p, pl.grid, s);
      case EPI_RESID: return launch_pair<EPI_RESID>(ta, tb0, tb1, tb2, p, pl.grid, s);
      case EPI_QKV: return launch_pair<EPI_QKV>(ta, tb0, tb1, tb2, p, pl.grid, s);
      default: return cudaErrorInvalidValue;  // the planner pairs no other epilogue
    }
  }
  switch (g.epi) {
    case EPI_STORE: return launch_bn<EPI_STORE>(pl.bn, ta, tb0, tb1, tb2, p, pl.grid, s);
    case EPI_RESID: return launch_bn<EPI_RESID>(pl.bn, ta, tb0, tb1, tb2, p, pl.grid, s);
    case EPI_SWIGLU: return launch_bn<EPI_SWIGLU>(pl.bn, ta, tb0, tb1, tb2, p, pl.grid, s);
    case EPI_QKV: return launch_bn<EPI_QKV>(pl.bn, ta, tb0, tb1, tb2, p, pl.grid, s);
    case EPI_LMHEAD: return launch_bn<EPI_LMHEAD>(pl.bn, ta, tb0, tb1, tb2, p, pl.grid, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dllm
