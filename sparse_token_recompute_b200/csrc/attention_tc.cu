// Partial attention on the 5th-generation tensor cores (sm_100a).
//
// The selected query rows of each sequence attend to all N cached keys of
// that sequence, bidirectionally: O = softmax(Q K^T / sqrt(hd)) V.
//
// One CTA = one (sequence, query head, tile of 128 compact query rows).
// Warp roles (192 threads):
//   warp 0  TMA producer: the Q tile once, then K and V tiles of 128 keys
//           into a two-stage ring (128-byte-swizzled 64-column boxes);
//   warp 1  TMEM owner and tcgen05.mma issuer: S_j = Q K_j^T into one of two
//           TMEM S buffers, then O += P_{j-1} V_{j-1} into the TMEM O buffer;
//   warps 2-5  softmax, one query row per thread (its TMEM lane): read S_j,
//           exponentiate against a per-row reference maximum, write P_j
//           (bf16) into shared memory in the swizzled K-major layout the MMA
//           reads, and finally normalise O and store it.
// The reference maximum is only raised (and O rescaled in TMEM) when a tile
// exceeds it by more than 2^8 in the exp2 domain, so P stays <= 256 and the
// result is the same softmax; the running sum uses the same reference.
// Every mbarrier wait is bounded; a timeout sets DLLM_DEV_TIMEOUT, drains the
// block's outstanding copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace dllm {

namespace {

constexpr int BQ = 128;       // query rows per CTA
constexpr int BKV = 128;      // keys per tile
constexpr int NTHREADS = 192;
constexpr uint32_t TMEM_COLS = 512;  // S0 [0,128), S1 [128,256), O [256, 256+hd)
constexpr float kRescaleLog2 = 8.0f;

template <int HD>
struct Smem {
  static constexpr int BLK = 64;                       // columns per swizzled box
  static constexpr int Q_BYTES = BQ * HD * 2;          // HD/64 boxes of 128 rows x 128 B
  static constexpr int KV_BYTES = BKV * HD * 2;
  static constexpr int P_BYTES = BQ * BKV * 2;         // 2 boxes of 128 rows x 64 keys
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + Q_BYTES;
  static constexpr int V_OFF = K_OFF + 2 * KV_BYTES;
  static constexpr int P_OFF = V_OFF + 2 * KV_BYTES;
  static constexpr int BAR_OFF = P_OFF + 2 * P_BYTES;
  static constexpr int TOTAL = BAR_OFF + 256 + 1024;   // + barriers + alignment slack
};

struct AttnParams {
  const int* row_off;
  __nv_bfloat16* O;
  int Nseq, Hq, Hkv, ldo;
  float scale_log2;
  int* status;
};

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) { tmem_ld_32x32b_x32(taddr, v); }

// 32 columns without the trailing wait: several loads can be in flight before
// one tcgen05.wait::ld
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
}

// B operand stored MN-major (hd contiguous, one 128-byte row per key) with the
// 128-byte swizzle: 8-key groups 1024 B apart (SBO), 64-column halves LBO apart.
__device__ __forceinline__ uint64_t umma_desc_mn_sw128(uint32_t saddr, uint32_t lbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

template <int HD>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using L = Smem<HD>;
  constexpr int NB = HD / 64;  // 64-column boxes per row of Q/K/V
  const int b = blockIdx.z, h = blockIdx.y;
  const int off = p.row_off[b];
  const int cnt = p.row_off[b + 1] - off;
  const int q0 = blockIdx.x * BQ;
  if (q0 >= cnt) return;
  const int g = (h * p.Hkv) / p.Hq;
  const int T = (p.Nseq + BKV - 1) / BKV;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR_OFF);
  // q_full, k_full[2], v_full[2], k_empty[2], v_empty[2], s_full[2], s_free[2], p_full[2],
  // pv_done[2], drain
  const uint32_t q_full = smem_u32(&bars[0]);
  auto k_full = [&](int i) { return smem_u32(&bars[1 + i]); };
  auto v_full = [&](int i) { return smem_u32(&bars[3 + i]); };
  auto k_empty = [&](int i) { return smem_u32(&bars[5 + i]); };
  auto v_empty = [&](int i) { return smem_u32(&bars[7 + i]); };
  auto s_full = [&](int i) { return smem_u32(&bars[9 + i]); };
  auto s_free = [&](int i) { return smem_u32(&bars[11 + i]); };
  auto p_full = [&](int i) { return smem_u32(&bars[13 + i]); };
  auto pv_done = [&](int i) { return smem_u32(&bars[15 + i]); };
  const uint32_t drain_bar = smem_u32(&bars[17]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[18]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sQ = smem_u32(sm + L::Q_OFF);
  const uint32_t sK = smem_u32(sm + L::K_OFF);
  const uint32_t sV = smem_u32(sm + L::V_OFF);
  const uint32_t sP = smem_u32(sm + L::P_OFF);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(v_full(i), 1);
      mbar_init(k_empty(i), 1);
      mbar_init(v_empty(i), 1);
      mbar_init(s_full(i), 1);
      mbar_init(s_free(i), 128);
      mbar_init(p_full(i), 128);
      mbar_init(pv_done(i), 1);
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
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;            // two S buffers of 128 columns
  const uint32_t tO = tmem + 2 * BKV;  // O buffer of HD columns

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      const int krow0 = b * p.Nseq;
      uint32_t issued = 0, issue_par = 0;  // bit i: K stage i (0,1), V stage i (2,3)
      bool ok = true;
      mbar_arrive_expect_tx(q_full, L::Q_BYTES);
      for (int c = 0; c < NB; ++c)
        tma_load_2d(sQ + c * BQ * 128, &tmQ, q_full, h * HD + c * 64, off + q0);
      for (int j = 0; j < T && ok; ++j) {
        const int st = j & 1;
        const uint32_t par = ((j >> 1) & 1) ^ 1u;
        if (!mbar_wait(k_empty(st), par, abort_flag, p.status)) { ok = false; break; }
        mbar_arrive_expect_tx(k_full(st), L::KV_BYTES);
        for (int c = 0; c < NB; ++c)
          tma_load_2d(sK + st * L::KV_BYTES + c * BKV * 128, &tmK, k_full(st), g * HD + c * 64,
                      krow0 + j * BKV);
        issued |= 1u << st;
        issue_par = (issue_par & ~(1u << st)) | (((uint32_t)(j >> 1) & 1u) << st);
        if (!mbar_wait(v_empty(st), par, abort_flag, p.status)) { ok = false; break; }
        mbar_arrive_expect_tx(v_full(st), L::KV_BYTES);
        for (int c = 0; c < NB; ++c)
          tma_load_2d(sV + st * L::KV_BYTES + c * BKV * 128, &tmV, v_full(st), g * HD + c * 64,
                      krow0 + j * BKV);
        issued |= 1u << (2 + st);
        issue_par = (issue_par & ~(1u << (2 + st))) | (((uint32_t)(j >> 1) & 1u) << (2 + st));
      }
      if (!ok) {
        wait_drain(q_full, 0);
        for (int st = 0; st < 2; ++st) {
          if (issued & (1u << st)) wait_drain(k_full(st), (issue_par >> st) & 1u);
          if (issued & (1u << (2 + st))) wait_drain(v_full(st), (issue_par >> (2 + st)) & 1u);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_qk = umma_idesc_bf16(BQ, BKV);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(BQ, HD) | (1u << 16);  // B (V) MN-major
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
      bool any = false;
      auto do_pv = [&](int j) -> bool {
        const int st = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (!mbar_wait(p_full(st), par, abort_flag, p.status)) return false;
        if (!mbar_wait(v_full(st), par, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t pb = sP + st * L::P_BYTES;
        const uint32_t vb = sV + st * L::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint64_t da = umma_desc_k_sw128(pb + (kk >> 2) * (BQ * 128) + (kk & 3) * 32);
          const uint64_t db = umma_desc_mn_sw128(vb + kk * 2048, BKV * 128);
          tc_mma_bf16(tO, da, db, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        any = true;
        tc_commit(pv_done(st));
        tc_commit(v_empty(st));
        return true;
      };
      for (int j = 0; j < T && ok; ++j) {
        const int st = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (!mbar_wait(k_full(st), par, abort_flag, p.status)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(s_free(st), par ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kb = sK + st * L::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t da = umma_desc_k_sw128(sQ + (kk >> 2) * (BQ * 128) + (kk & 3) * 32);
          const uint64_t db = umma_desc_k_sw128(kb + (kk >> 2) * (BKV * 128) + (kk & 3) * 32);
          tc_mma_bf16(tS + st * BKV, da, db, idesc_qk, kk > 0 ? 1u : 0u);
        }
        any = true;
        tc_commit(s_full(st));
        tc_commit(k_empty(st));
        if (j >= 1 && !do_pv(j - 1)) { ok = false; break; }
      }
      if (ok) ok = do_pv(T - 1);
      if (!ok && any) {
        tc_commit(drain_bar);
        wait_drain(drain_bar, 0);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // query row in the tile (= TMEM lane)
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    float m_ref = -INFINITY, lsum = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int st = j & 1;
      const uint32_t par = (j >> 1) & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(s_full(st), par, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      float s[BKV];
#pragma unroll
      for (int c = 0; c < BKV; c += 32) tmem_ld32_nowait(tS + st * BKV + lane_off + c, s + c);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(s_free(st));
      const int kbase = j * BKV;
      // 8 independent max chains instead of one 128-long dependency
      float mxv[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) mxv[t] = -INFINITY;
      if (kbase + BKV <= p.Nseq) {
#pragma unroll
        for (int i = 0; i < BKV; ++i) {
          s[i] *= p.scale_log2;
          mxv[i & 7] = fmaxf(mxv[i & 7], s[i]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < BKV; ++i) {
          s[i] = (kbase + i < p.Nseq) ? s[i] * p.scale_log2 : -INFINITY;
          mxv[i & 7] = fmaxf(mxv[i & 7], s[i]);
        }
      }
      const float mx = fmaxf(fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3])),
                             fmaxf(fmaxf(mxv[4], mxv[5]), fmaxf(mxv[6], mxv[7])));
      // raise the reference maximum only when this tile exceeds it by > 2^8
      const bool need = (j == 0) || (mx > m_ref + kRescaleLog2);
      const bool rescale_o = __any_sync(0xffffffffu, need && j > 0);
      float alpha = 1.f;
      if (need) {
        alpha = (j == 0) ? 0.f : exp2f(m_ref - mx);
        m_ref = mx;
      }
      lsum *= (j == 0) ? 0.f : alpha;
      // P buffer st was last read by PV_{j-2}
      if (j >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(pv_done(st), par ^ 1u, abort_flag, p.status));
        if (!ok) break;
      }
      if (rescale_o) {
        const int pj = j - 1;
        ok = __all_sync(0xffffffffu,
                        mbar_wait(pv_done(pj & 1), (pj >> 1) & 1, abort_flag, p.status));
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < HD; c += 32) {
          float o[32];
          tmem_ld32(tO + lane_off + c, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st_32x32b_x32(tO + lane_off + c, o);
        }
        tmem_wait_st();
      }
      float rsv[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) rsv[t] = 0.f;
      const uint32_t prow = sP + st * L::P_BYTES + r * 128;
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          float e[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            e[i] = exp2f(s[blk * 64 + ch * 8 + i] - m_ref);
            rsv[i] += e[i];
          }
          const uint4 v = pack8(e);
          const uint32_t addr = prow + blk * (BQ * 128) + ((ch ^ (r & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                       "r"(v.z), "r"(v.w)
                       : "memory");
        }
      }
      lsum += ((rsv[0] + rsv[1]) + (rsv[2] + rsv[3])) + ((rsv[4] + rsv[5]) + (rsv[6] + rsv[7]));
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full(st));
    }
    if (ok) {
      const int jl = T - 1;
      ok = __all_sync(0xffffffffu, mbar_wait(pv_done(jl & 1), (jl >> 1) & 1, abort_flag, p.status));
    }
    if (ok) {
      tc_fence_after();
      const int row = q0 + r;
      const float inv = 1.0f / lsum;
#pragma unroll 1
      for (int c = 0; c < HD; c += 32) {
        float o[32];
        tmem_ld32(tO + lane_off + c, o);
        if (row < cnt) {
          __nv_bfloat16* dst = p.O + (size_t)(off + row) * p.ldo + h * HD + c;
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            float f[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) f[t] = o[i + t] * inv;
            *reinterpret_cast<uint4*>(dst + i) = pack8(f);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

bool map2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return tmap_bf16_2d(m, ptr, rows, cols, box_rows);
}

template <int HD>
cudaError_t launch_hd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                      const AttnParams& p, dim3 grid, cudaStream_t s) {
  constexpr int smem = Smem<HD>::TOTAL;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<HD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  attn_tc_kernel<HD><<<grid, NTHREADS, smem, s>>>(q, k, v, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_tc(const __nv_bfloat16* q, int M_cap, const __nv_bfloat16* kc,
                                const __nv_bfloat16* vc, __nv_bfloat16* o, const int* row_off,
                                int B, int k_cap, int Nseq, int Hq, int Hkv, int hd, int* status,
                                cudaStream_t s) {
  if (B <= 0 || k_cap <= 0 || M_cap <= 0) return cudaSuccess;
  if (hd != 64 && hd != 128) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv;
  if (!map2d(&tq, q, (uint64_t)M_cap, (uint64_t)Hq * hd, BQ)) return cudaErrorInvalidValue;
  if (!map2d(&tk, kc, (uint64_t)B * Nseq, (uint64_t)Hkv * hd, BKV)) return cudaErrorInvalidValue;
  if (!map2d(&tv, vc, (uint64_t)B * Nseq, (uint64_t)Hkv * hd, BKV)) return cudaErrorInvalidValue;
  AttnParams p{row_off, o, Nseq, Hq, Hkv, Hq * hd, 1.4426950408889634f / sqrtf((float)hd), status};
  dim3 grid((k_cap + BQ - 1) / BQ, Hq, B);
  ProfScope prof("attention", s);
  return hd == 128 ? launch_hd<128>(tq, tk, tv, p, grid, s) : launch_hd<64>(tq, tk, tv, p, grid, s);
}

}  // namespace dllm
