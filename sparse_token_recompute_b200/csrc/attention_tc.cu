// Partial attention on the 5th-generation tensor cores (sm_100a).
//
// The selected query rows of each sequence attend to all N cached keys of
// that sequence, bidirectionally: O = softmax(Q K^T / sqrt(hd)) V.
//
// One CTA = one (sequence, query head) and up to NT = 2 tiles of 128 compact
// query rows (A and B) that share every K/V tile.  Warp roles (320 threads):
//   warp 0     TMA producer: both Q tiles once, then K and V tiles of 128 keys
//              through one ring of shared-memory slots (128-byte-swizzled
//              64-column boxes);
//   warp 1     TMEM owner and tcgen05.mma issuer;
//   warps 2-5  softmax of tile A, warps 6-9 softmax of tile B: one query row
//              per thread (its TMEM lane).
// With NT = 1 a CTA holds one tile (192 threads, 256 TMEM columns, under half
// the shared memory) and two CTAs share each SM: their MMAs and softmax
// interleave as the two groups of a pair do, and one CTA's start-up and
// epilogue overlap the other's main loop.
// TMEM holds S_A, S_B (fp32, 128 columns each) and O_A, O_B.  Each softmax
// group reads S_X, exponentiates against a per-row reference maximum and
// writes P_X back over the first 64 columns of S_X as packed bf16 pairs; the
// P V product reads its A operand straight from TMEM.  The issuer alternates
// the groups -- ... PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1) ... -- so one
// group's softmax overlaps the other group's MMAs.  tcgen05 operations from
// one thread complete in issue order, so QK_X(j+1) cannot overwrite P_X(j)
// before PV_X(j) has read it, and once S_X(j) is reported complete PV_X(j-1)
// is complete too (O_X may then be rescaled in place).
// The reference maximum is only raised (and O rescaled) when a tile exceeds
// it by more than 2^8 in the exp2 domain, so P stays <= 256 and the result is
// the same softmax; the running sum uses the same reference.
// Every mbarrier wait is bounded; a timeout sets DLLM_DEV_TIMEOUT, drains the
// block's outstanding copies and MMAs, frees TMEM and returns.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace dllm {

namespace {

constexpr int BT = 128;       // query rows per tile (= TMEM lanes)
constexpr int BKV = 128;      // keys per K/V tile
constexpr float kRescaleLog2 = 8.0f;
constexpr int kSmemMax = 227 * 1024;  // dynamic shared memory a block may opt in to
constexpr int kMaxShares = 8;         // key shares of a split exact attention, at most

// NT query tiles per CTA: 2 (a pair sharing every K/V tile, one CTA per SM
// holding all 512 TMEM columns) or 1 (one tile, 256 TMEM columns and under
// half the shared memory, two CTAs per SM)
template <int NT>
constexpr int nthreads() { return 64 + NT * 128; }
template <int NT>
constexpr uint32_t tmem_cols() { return NT * 256u; }  // S_X at 128 x, O_X at 128 (NT + x)

template <int HD, int NT>
struct Smem {
  static constexpr int Q_TILE = BT * HD * 2;     // HD/64 boxes of 128 rows x 128 B
  static constexpr int KV_BYTES = BKV * HD * 2;
  // K and V tiles share one ring of slots in consumption order K0 V0 K1 V1 ...,
  // as many as fit next to the Q tiles (at most 8) in this CTA's share of the SM
  static constexpr int BUDGET = NT == 2 ? kSmemMax : 112 * 1024;
  static constexpr int SLOTS_FIT = (BUDGET - 2304 - 1024 - NT * Q_TILE) / KV_BYTES;
  static constexpr int SLOTS = SLOTS_FIT < 8 ? SLOTS_FIT : 8;
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = Q_OFF + NT * Q_TILE;
  static constexpr int BAR_OFF = RING_OFF + SLOTS * KV_BYTES;
  static constexpr int STAT_OFF = BAR_OFF + 256;  // 2 x 128 floats for the key-split merge
  // + barriers + alignment slack; a pair CTA takes at least 116 KB so that one
  // CTA (which holds all 512 TMEM columns) is resident per SM
  static constexpr int NEED = STAT_OFF + 1024 + 1024;
  static constexpr int TOTAL = (NT == 1 || NEED > 116 * 1024) ? NEED : 116 * 1024;
  static_assert(NT == 2 || 2 * (TOTAL + 1024) <= 228 * 1024, "two one-tile CTAs per SM");
};

struct AttnParams {
  const int* row_off;
  __nv_bfloat16* O;
  int Nseq, Hq, Hkv, ldo;
  float scale_log2;
  int* status;
  // per query row and head, natural-log units: m = max score, l = sum exp(s - m);
  // written by the attention when non-null, read and updated by the update mode
  float* st_m;
  float* st_l;
  const int* a_off;  // update mode: changed keys of sequence b at rows a_off[b]..a_off[b+1]
  int ppc;           // pairs of query tiles per CTA (consecutive; > 1 only without key splits)
  // keys split over kv_split CTAs per pair (exact mode, few query tiles): each
  // writes its normalised partial output and (m, l) for a merge kernel
  int kv_split;
  int part_rows;     // row capacity of the partial buffers
  float* part_o;     // [kv_split, part_rows, Hq, HD]
  float* part_ml;    // [kv_split, part_rows, Hq, 2] (m in the exp2 domain, l)
  // update mode: rows r with skip[r] != 0 (r = row_off[b] + row) keep o, m, l untouched
  const uint8_t* skip;
};

// 32 columns without the trailing wait: several loads in flight before one wait
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
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 2^x with the hardware approximation (relative error about 2^-22); subnormal
// results flush to zero, which only drops probabilities below 2^-126
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max of three values in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// barrier `id` over `count` threads (a multiple of 32) of the block
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
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

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16, fp32 accumulate: A (M=128 lanes x K=16)
// occupies 8 consecutive 32-bit columns, two bf16 per column (lower index low)
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// UPD = false: attention of the selected rows over the sequence's N cached keys.
// UPD = true: the incremental update of stable rows [DyLLM 2.B]: the "keys"
// are the sequence's changed keys, first with their new values (tmK, tmV), then
// with their old values (tmK2, tmV2) entering the sums with a negative sign; the
// reference maximum starts at the row's cached m, and the epilogue merges the
// sums into the cached (m, l, o).
template <int HD, bool UPD, int NT>
__global__ void __launch_bounds__(nthreads<NT>(), NT == 1 ? 2 : 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK2,
                   const __grid_constant__ CUtensorMap tmV2, const AttnParams p) {
  using L = Smem<HD, NT>;
  constexpr int NB = HD / 64;  // 64-column boxes per row of Q/K/V
  constexpr float kLog2e = 1.4426950408889634f;
  griddep_wait();  // everything below reads what earlier kernels wrote
  const int b = blockIdx.z, h = blockIdx.y;
  const int off = p.row_off[b];
  const int cnt = p.row_off[b + 1] - off;
  griddep_launch_dependents();  // the next GEMM may start streaming its weights
  // this CTA's pairs of query tiles: pair i starts at row pair_q0(i) of the sequence
  // (several pairs per CTA only in the update mode, whose key streams are short)
  constexpr bool multi = UPD;
  const int ppc = UPD ? p.ppc : 1;
  const int S_kv = UPD ? 1 : p.kv_split;           // CTAs sharing a pair's keys
  const int s_kv = UPD ? 0 : (int)blockIdx.x % S_kv;  // this CTA's share
  const int pair0 = (UPD ? blockIdx.x : blockIdx.x / S_kv) * ppc;
  auto pair_q0 = [&](int i) { return (pair0 + i) * (NT * BT); };
  const int npairs = UPD ? min(ppc, (cnt - pair_q0(0) + NT * BT - 1) / (NT * BT))
                         : (pair_q0(0) < cnt ? 1 : 0);
  if (npairs <= 0) return;
  const int q0 = pair_q0(0);
  // update mode: a_cnt changed keys -> TH tiles of new values, then TH of old
  const int a_base = UPD ? p.a_off[b] : 0;
  const int a_cnt = UPD ? p.a_off[b + 1] - a_base : 0;
  const int TH = UPD ? (a_cnt + BKV - 1) / BKV : 0;
  // exact mode: this CTA's K/V tiles [k_lo, k_lo + T) of the sequence's T_all
  const int T_all = (p.Nseq + BKV - 1) / BKV;
  const int TS = (T_all + S_kv - 1) / S_kv;
  const int k_lo = UPD ? 0 : s_kv * TS;
  const int T = UPD ? 2 * TH : max(0, min(T_all, k_lo + TS) - k_lo);
  if (T == 0) return;  // no changed key: the cached statistics stand
  // keys of K/V tile t that exist (the rest score -inf)
  auto tile_keys = [&](int t) {
    return UPD ? min(BKV, a_cnt - (t % TH) * BKV) : min(BKV, p.Nseq - (k_lo + t) * BKV);
  };
  auto pair_nq = [&](int i) { return (NT == 2 && cnt - pair_q0(i) > BT) ? 2 : 1; };
  const int nq = pair_nq(0);
  // A lone query tile splits the keys instead (one pair per CTA only): group A
  // takes K/V tiles [0, TA), group B [TA, T), and the two partial softmax
  // results are merged at the end.
  const bool split = NT == 2 && !UPD && !multi && nq == 1 && T >= 2;
  const int TA = split ? (T + 1) / 2 : T;
  const int TB = split ? T - TA : T;
  const int ngroups = (nq == 2 || split) ? 2 : 1;
  auto ntiles = [&](int x) { return x == 0 ? TA : TB; };         // K/V tiles of group x
  auto kv_first = [&](int x) { return (split && x == 1) ? TA : 0; };
  auto qtile = [&](int x) { return split ? 0 : x; };             // query tile of group x
  // softmax warps of group x that hold at least one selected row in pair i
  auto live_warps_in = [&](int i, int x) {
    const int rows = min(BT, cnt - pair_q0(i) - qtile(x) * BT);
    return rows > 0 ? (rows + 31) / 32 : 1;
  };
  auto live_warps = [&](int x) { return live_warps_in(0, x); };
  const int g = (h * p.Hkv) / p.Hq;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR_OFF);
  float* stat = reinterpret_cast<float*>(sm + L::STAT_OFF);  // group B's (m, l) per row
  // s_full[X], p_full[X], pv_done[X], q_full, drain, full[slot], empty[slot],
  // q_empty, o_free[X]
  constexpr int NS = L::SLOTS;
  static_assert(NS >= 2 && 11 + 2 * NS + 1 <= 32, "barrier area holds 32 words");
  auto s_full = [&](int x) { return smem_u32(&bars[0 + x]); };
  auto p_full = [&](int x) { return smem_u32(&bars[2 + x]); };
  auto pv_done = [&](int x) { return smem_u32(&bars[4 + x]); };
  const uint32_t q_full = smem_u32(&bars[6]);
  const uint32_t drain_bar = smem_u32(&bars[7]);
  auto full = [&](int i) { return smem_u32(&bars[8 + i]); };
  auto empty = [&](int i) { return smem_u32(&bars[8 + NS + i]); };
  const uint32_t q_empty = smem_u32(&bars[8 + 2 * NS]);  // Q tiles read (multi-pair)
  auto o_free = [&](int x) { return smem_u32(&bars[9 + 2 * NS + x]); };  // O_X read out
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[11 + 2 * NS]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sQ = smem_u32(sm + L::Q_OFF);
  const uint32_t sRing = smem_u32(sm + L::RING_OFF);
  // The n-th K or V tile through the ring occupies slot n % NS for its (n / NS)-th use.
  // Producer and issuer walk the same sequence of tiles:
  //   two query tiles:  K0, V0, K1, V1, ...              (each read by both groups)
  //   split keys:       K0, K_TA, then per j: V_j, K_{j+1}, V_{TA+j}, K_{TA+j+1}
  auto slot_of = [&](int n) { return n % NS; };
  auto use_par = [&](int n) { return (uint32_t)((n / NS) & 1); };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(full(i), 1);
      mbar_init(empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      // one pair: the warps with rows; several: every warp of the group, every pair
      mbar_init(p_full(i), multi ? 128 : 32 * live_warps(i));
      mbar_init(pv_done(i), 1);
      mbar_init(o_free(i), 128);
    }
    mbar_init(q_empty, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols<NT>());
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (UPD) {
      tma_prefetch_desc(&tmK2);
      tma_prefetch_desc(&tmV2);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto tS = [&](int x) { return tmem + (uint32_t)(x * 128); };
  auto tO = [&](int x) { return tmem + (uint32_t)(NT * 128 + x * 128); };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      const int krow0 = b * p.Nseq;
      uint32_t issued = 0, issue_par = 0;  // per slot: a load in flight, its parity
      int n = 0;
      auto load = [&](bool is_v, int tile) -> bool {
        const int sl = slot_of(n);
        const uint32_t u = use_par(n);
        if (!mbar_wait(empty(sl), u ^ 1u, abort_flag, p.status)) return false;
        mbar_arrive_expect_tx(full(sl), L::KV_BYTES);
        const bool old = UPD && tile >= TH;
        const CUtensorMap* tm = is_v ? (old ? &tmV2 : &tmV) : (old ? &tmK2 : &tmK);
        const int row = UPD ? a_base + (tile - (old ? TH : 0)) * BKV : krow0 + (k_lo + tile) * BKV;
        for (int c = 0; c < NB; ++c)
          tma_load_2d(sRing + sl * L::KV_BYTES + c * BKV * 128, tm, full(sl), g * HD + c * 64,
                      row);
        issued |= 1u << sl;
        issue_par = (issue_par & ~(1u << sl)) | (u << sl);
        ++n;
        return true;
      };
      bool ok = true;
      int q_issued = 0;  // pairs whose Q tiles were requested
      if (!split) {
        for (int i = 0; i < npairs && ok; ++i) {
          // a later pair's first K tile enters the ring before its Q tiles wait for the
          // previous pair's last Q.K^T to run
          if (i > 0 && !(ok = load(false, 0))) break;
          if (i > 0 && !(ok = mbar_wait(q_empty, (i - 1) & 1, abort_flag, p.status))) break;
          const int nqi = pair_nq(i);
          mbar_arrive_expect_tx(q_full, nqi * L::Q_TILE);
          for (int x = 0; x < nqi; ++x)
            for (int c = 0; c < NB; ++c)
              tma_load_2d(sQ + x * L::Q_TILE + c * BT * 128, &tmQ, q_full, h * HD + c * 64,
                          off + pair_q0(i) + x * BT);
          ++q_issued;
          if (i == 0) ok = load(false, 0);
          for (int j = 0; j < T && ok; ++j) {
            ok = load(true, j);
            if (ok && j + 1 < T) ok = load(false, j + 1);
          }
        }
      } else {
        mbar_arrive_expect_tx(q_full, nq * L::Q_TILE);
        for (int c = 0; c < NB; ++c)
          tma_load_2d(sQ + c * BT * 128, &tmQ, q_full, h * HD + c * 64, off + q0);
        q_issued = 1;
        ok = load(false, 0) && load(false, TA);
        for (int j = 0; j < TA && ok; ++j) {
          ok = load(true, j);
          if (ok && j + 1 < TA) ok = load(false, j + 1);
          if (ok && j < TB) ok = load(true, TA + j);
          if (ok && j + 1 < TB) ok = load(false, TA + j + 1);
        }
      }
      if (!ok) {
        if (q_issued > 0) mbar_wait_drain(q_full, (q_issued - 1) & 1, p.status);
        for (int sl = 0; sl < NS; ++sl)
          if (issued & (1u << sl)) mbar_wait_drain(full(sl), (issue_par >> sl) & 1u, p.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_qk = umma_idesc_bf16(BT, BKV);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(BT, HD) | (1u << 16);  // B (V) MN-major
      bool ok = true;
      bool any = false;
      int m = 0;  // ring tiles consumed
      int jx[2] = {0, 0};  // K/V tiles group x has been through (barrier phases)
      int px[2] = {0, 0};  // pairs group x has finished
      auto take = [&]() -> int {  // slot of the next ring tile, once it has landed
        const int sl = slot_of(m);
        if (!mbar_wait(full(sl), use_par(m), abort_flag, p.status)) return -1;
        tc_fence_after();
        ++m;
        return sl;
      };
      auto give = [&](int sl) { tc_commit(empty(sl)); };
      auto qk = [&](int x, int sl) {
        const uint32_t kb = sRing + sl * L::KV_BYTES;
        const uint32_t qb = sQ + qtile(x) * L::Q_TILE;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t da = umma_desc_k_sw128(qb + (kk >> 2) * (BT * 128) + (kk & 3) * 32);
          const uint64_t db = umma_desc_k_sw128(kb + (kk >> 2) * (BKV * 128) + (kk & 3) * 32);
          tc_mma_bf16(tS(x), da, db, idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full(x));
        any = true;
      };
      auto pv = [&](int x, int j, int sl) -> bool {
        // a later pair's first P.V overwrites O_X: the group must have read it out
        if (j == 0 && px[x] > 0 &&
            !mbar_wait(o_free(x), (px[x] - 1) & 1, abort_flag, p.status))
          return false;
        if (!mbar_wait(p_full(x), jx[x] & 1, abort_flag, p.status)) return false;
        ++jx[x];
        tc_fence_after();
        const uint32_t vb = sRing + sl * L::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint64_t db = umma_desc_mn_sw128(vb + kk * 2048, BKV * 128);
          tc_mma_ts(tO(x), tS(x) + (uint32_t)(kk * 8), db, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        if (j == ntiles(x) - 1) {  // O_X of this pair is final
          tc_commit(pv_done(x));
          ++px[x];
        }
        return true;
      };
      if (!split) {
        for (int i = 0; i < npairs && ok; ++i) {
          if (!(ok = mbar_wait(q_full, i & 1, abort_flag, p.status))) break;
          const int nqi = pair_nq(i);
          const int sk = take();
          if (!(ok = sk >= 0)) break;
          for (int x = 0; x < nqi; ++x) qk(x, sk);
          give(sk);
          // once the pair's last Q.K^T has run, the next pair's Q tiles may load
          if (T == 1) tc_commit(q_empty);
          for (int j = 0; j < T && ok; ++j) {
            const int sv = take();
            if (!(ok = sv >= 0 && pv(0, j, sv))) break;
            int sk1 = -1;
            if (j + 1 < T) {
              if (!(ok = (sk1 = take()) >= 0)) break;
              qk(0, sk1);
            }
            if (nqi == 2) {
              if (!(ok = pv(1, j, sv))) break;
              if (sk1 >= 0) qk(1, sk1);
            }
            if (j + 2 == T) tc_commit(q_empty);
            give(sv);
            if (sk1 >= 0) give(sk1);
          }
        }
      } else if ((ok = mbar_wait(q_full, 0, abort_flag, p.status))) {
        for (int x = 0; x < 2 && ok; ++x) {
          const int sk = take();
          if ((ok = sk >= 0)) {
            qk(x, sk);
            give(sk);
          }
        }
        for (int j = 0; j < TA && ok; ++j) {
          int sl;
          if (!(ok = (sl = take()) >= 0 && pv(0, j, sl))) break;
          give(sl);
          if (j + 1 < TA) {
            if (!(ok = (sl = take()) >= 0)) break;
            qk(0, sl);
            give(sl);
          }
          if (j < TB) {
            if (!(ok = (sl = take()) >= 0 && pv(1, j, sl))) break;
            give(sl);
          }
          if (j + 1 < TB) {
            if (!(ok = (sl = take()) >= 0)) break;
            qk(1, sl);
            give(sl);
          }
        }
      }
      if (!ok && any) {
        tc_commit(drain_bar);
        mbar_wait_drain(drain_bar, 0, p.status);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax groups
    const int x = (warp - 2) >> 2;        // group: 0 = A (warps 2-5), 1 = B (warps 6-9)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;       // query row in the tile (= TMEM lane)
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    int jcnt = 0, pcnt = 0;  // this group's K/V tiles and pairs so far (barrier phases)
    for (int pi = 0; pi < npairs; ++pi) {
      if (x >= (multi ? pair_nq(pi) : ngroups)) continue;
      const bool live = quad < (multi ? live_warps_in(pi, x) : live_warps(x));
      // one pair: a warp whose 32 rows are all past the sequence's rows takes no part;
      // several pairs: it keeps the barrier counts (waits for each S tile, arrives)
      if (!multi && !live) continue;
      const float sc = p.scale_log2;
      float m_ref = -INFINITY, lsum = 0.f;  // reference maximum in the exp2 domain
      const int row_x = pair_q0(pi) + qtile(x) * BT + r;  // this thread's row in the sequence
      const size_t st_i = (size_t)(off + row_x) * p.Hq + h;
      if (UPD) m_ref = row_x < cnt ? p.st_m[st_i] * kLog2e : 0.f;  // the cached maximum
      bool ok = true;
      const int nj = ntiles(x);
      for (int j = 0; j < nj; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(s_full(x), jcnt & 1, abort_flag, p.status));
        ++jcnt;
        if (!ok) break;
        if (!live) {  // rows past the sequence: keep the count of P arrivals only
          mbar_arrive(p_full(x));
          continue;
        }
        tc_fence_after();
        float s[BKV];
#pragma unroll
        for (int c = 0; c < BKV; c += 32) tmem_ld32_nowait(tS(x) + lane_off + c, s + c);
        tmem_wait_ld();
        const int nkeys = tile_keys(kv_first(x) + j);
        if (nkeys < BKV) {
#pragma unroll
          for (int i = 0; i < BKV; ++i) s[i] = (i < nkeys) ? s[i] : -INFINITY;
        }
        // the maximum of the raw scores (the scale is positive)
        float mxv[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) mxv[t] = -INFINITY;
#pragma unroll
        for (int i = 0; i < BKV; i += 2) mxv[(i >> 1) & 3] = fmax3(mxv[(i >> 1) & 3], s[i], s[i + 1]);
        const float mx = fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3])) * sc;
        // raise the reference maximum only when this tile exceeds it by > 2^8
        // (the update mode starts from the cached maximum, not from tile 0)
        const bool first = !UPD && j == 0;
        const bool need = first || (mx > m_ref + kRescaleLog2);
        const bool rescale_o = __any_sync(0xffffffffu, need && j > 0);
        float alpha = 1.f;
        if (need) {
          alpha = first ? 0.f : ex2_approx(m_ref - mx);
          m_ref = mx;
        }
        lsum *= first ? 0.f : alpha;
        const float neg_m = -m_ref;
        float rsv[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) rsv[t] = 0.f;
        uint32_t pk[BKV / 2];
#pragma unroll
        for (int i = 0; i < BKV; i += 2) {
          const float x0 = fmaf(s[i], sc, neg_m), x1 = fmaf(s[i + 1], sc, neg_m);
          float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
          if (UPD && j >= TH) {  // an old key's term leaves the sums
            e0 = -e0;
            e1 = -e1;
          }
          rsv[i & 7] += e0;
          rsv[(i + 1) & 7] += e1;
          pk[i >> 1] = pack_bf2(e0, e1);
        }
        lsum += ((rsv[0] + rsv[1]) + (rsv[2] + rsv[3])) + ((rsv[4] + rsv[5]) + (rsv[6] + rsv[7]));
        // P_X over the first 64 columns of S_X (S_X has been read into registers)
        tmem_st32(tS(x) + lane_off, pk);
        tmem_st32(tS(x) + lane_off + 32, pk + 32);
        if (rescale_o) {
          // S_X(j) complete implies PV_X(j-1) complete: O_X is stable until P_X(j) is
          // ready (rescaled once the scores are out of the registers)
#pragma unroll 1
          for (int c = 0; c < HD; c += 32) {
            float o[32];
            tmem_ld32_nowait(tO(x) + lane_off + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tO(x) + lane_off + c, reinterpret_cast<const uint32_t*>(o));
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full(x));
      }
      if (ok && live)
        ok = __all_sync(0xffffffffu, mbar_wait(pv_done(x), pcnt & 1, abort_flag, p.status));
      ++pcnt;
      if (split) {
        // group B hands its (m, l) to group A, which merges O_B into O_A
        if (x == 1) {
          stat[r] = m_ref;
          stat[BT + r] = lsum;
        }
        tc_fence_before();
        named_bar_sync(1, 2 * 32 * live_warps(0));
        tc_fence_after();
      }
      if (ok && live && (x == 0 || !split)) {
        const int row = row_x;
        // update mode: rows the caller recomputes exactly keep their cached values (the
        // TMEM loads below stay warp-wide; only this lane's stores are skipped)
        const bool keep = UPD && p.skip && row < cnt && p.skip[off + row] != 0;
        float wa = 1.f, wb = 0.f, m_out = m_ref, w_old = 0.f;
        if (split) {
          const float mb = stat[r], lb = stat[BT + r];
          const float mm = fmaxf(m_ref, mb);
          wa = ex2_approx(m_ref - mm);
          wb = ex2_approx(mb - mm);
          lsum = lsum * wa + lb * wb;
          m_out = mm;
        }
        if (UPD && row < cnt) {
          // the cached sum and output, brought to the final reference
          w_old = p.st_l[st_i] * ex2_approx(p.st_m[st_i] * kLog2e - m_ref);
          lsum += w_old;
        }
        const float inv = 1.0f / lsum;
        wa *= inv;
        wb *= inv;
        w_old *= inv;
        const bool partial = !UPD && S_kv > 1;  // a share of the keys: fp32 partial out
#pragma unroll 1
        for (int c = 0; c < HD; c += 32) {
          float o[32], ob[32];
          tmem_ld32_nowait(tO(x) + lane_off + c, o);
          if (split) tmem_ld32_nowait(tO(1) + lane_off + c, ob);
          tmem_wait_ld();
          if (keep) {
          } else if (row < cnt && partial) {
            float* dst = p.part_o + (((size_t)s_kv * p.part_rows + off + row) * p.Hq + h) * HD + c;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dst + i) =
                  split ? make_float4(o[i] * wa + ob[i] * wb, o[i + 1] * wa + ob[i + 1] * wb,
                                      o[i + 2] * wa + ob[i + 2] * wb, o[i + 3] * wa + ob[i + 3] * wb)
                        : make_float4(o[i] * wa, o[i + 1] * wa, o[i + 2] * wa, o[i + 3] * wa);
          } else if (row < cnt) {
            __nv_bfloat16* dst = p.O + (size_t)(off + row) * p.ldo + h * HD + c;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              float f[8];
#pragma unroll
              for (int t = 0; t < 8; ++t) f[t] = split ? o[i + t] * wa + ob[i + t] * wb : o[i + t] * wa;
              if (UPD) {
                float prev[8];
                unpack8(*reinterpret_cast<const uint4*>(dst + i), prev);
#pragma unroll
                for (int t = 0; t < 8; ++t) f[t] = fmaf(w_old, prev[t], f[t]);
              }
              *reinterpret_cast<uint4*>(dst + i) = pack8(f);
            }
          }
        }
        if (keep) {
        } else if (row < cnt && partial) {
          float* ml = p.part_ml + (((size_t)s_kv * p.part_rows + off + row) * p.Hq + h) * 2;
          ml[0] = m_out;
          ml[1] = lsum;
        } else if (row < cnt && p.st_m) {
          p.st_m[st_i] = m_out / kLog2e;
          p.st_l[st_i] = lsum;
        }
      }
      if (multi) {  // O_X has been read out: the next pair's first P.V may overwrite it
        tc_fence_before();
        mbar_arrive(o_free(x));
      }
      if (!ok) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols<NT>());
  }
}

// Merge of the key shares of the split exact attention: one warp per (row,
// head): M = max m_s, w_s = l_s 2^(m_s - M), O = sum w_s o_s / sum w_s (o_s are
// the shares' normalised outputs), in share order.
template <int HD>
__global__ void __launch_bounds__(256) attn_merge_kernel(const float* __restrict__ part_o,
                                                         const float* __restrict__ part_ml,
                                                         int S, int part_rows,
                                                         const int* __restrict__ M_dev, int Hq,
                                                         __nv_bfloat16* __restrict__ O, int ldo,
                                                         float* __restrict__ st_m,
                                                         float* __restrict__ st_l) {
  constexpr int PER = HD / 32;  // floats per lane
  griddep_wait();               // the shares are written by the attention launch before
  griddep_launch_dependents();  // the O projection may start streaming its weights
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int h = blockIdx.y, lane = threadIdx.x & 31;
  if (r >= min(*M_dev, part_rows)) return;
  // every share's (m, l) and output slice in flight at once (at most 8 shares)
  float2 ml[kMaxShares];
  float o[kMaxShares][PER];
#pragma unroll
  for (int sh = 0; sh < kMaxShares; ++sh) {
    if (sh < S) {
      const size_t base = ((size_t)sh * part_rows + r) * Hq + h;
      ml[sh] = *reinterpret_cast<const float2*>(part_ml + base * 2);
      const float* src = part_o + base * HD + lane * PER;
#pragma unroll
      for (int i = 0; i < PER; ++i) o[sh][i] = src[i];
    }
  }
  float mx = -INFINITY;
#pragma unroll
  for (int sh = 0; sh < kMaxShares; ++sh)
    if (sh < S) mx = fmaxf(mx, ml[sh].x);
  float acc[PER], L = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
#pragma unroll
  for (int sh = 0; sh < kMaxShares; ++sh) {
    if (sh < S) {
      const float w = ml[sh].y * ex2_approx(ml[sh].x - mx);
      L += w;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, o[sh][i], acc[i]);
    }
  }
  const float inv = 1.0f / L;
  __nv_bfloat16* dst = O + (size_t)r * ldo + h * HD + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; i += 2) {
    __nv_bfloat162 t = __floats2bfloat162_rn(acc[i] * inv, acc[i + 1] * inv);
    *reinterpret_cast<__nv_bfloat162*>(dst + i) = t;
  }
  if (st_m && lane == 0) {
    st_m[(size_t)r * Hq + h] = mx / 1.4426950408889634f;
    st_l[(size_t)r * Hq + h] = L;
  }
}

template <int HD, bool UPD, int NT>
cudaError_t launch_hd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                      const CUtensorMap& k2, const CUtensorMap& v2, const AttnParams& p, dim3 grid,
                      cudaStream_t s) {
  constexpr int smem = Smem<HD, NT>::TOTAL;
  const cudaError_t ea = ensure_smem_attr<attn_tc_kernel<HD, UPD, NT>>(smem);
  if (ea != cudaSuccess) return ea;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(nthreads<NT>());
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  la[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = la;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, attn_tc_kernel<HD, UPD, NT>, q, k, v, k2, v2, p);
}

}  // namespace

int attention_kv_split(int B, int k_cap, int Nseq, int Hq, int NT) {
  // few CTAs leave most SMs idle: share each CTA's keys among up to 8 CTAs (one
  // CTA per SM with pairs of query tiles, whose two groups split a lone tile's
  // keys again, so at least two K/V tiles per share; two per SM with one tile)
  const int T = (Nseq + BKV - 1) / BKV;
  const int ctas = ((k_cap + NT * BT - 1) / (NT * BT)) * Hq * B;
  const int slots = (NT == 1 ? 2 : 1) * num_sms();  // resident CTAs
  const int min_tiles = NT == 1 ? 1 : 2;
  if (ctas <= 0 || 2 * ctas > slots || T < 2 * min_tiles) return 1;
  int S = std::max(1, std::min(std::min(kMaxShares, T / min_tiles), slots / ctas));
  while (S > 1 && (S - 1) * ((T + S - 1) / S) >= T) --S;  // every share holds keys
  return S;
}

size_t attention_part_bytes_bound(int cap, int Hq, int hd) {
  // a split launch has S * rows <= SMs * (rows of a pair) for any batch shape
  // (S x CTAs <= resident CTAs: SMs x 2 tiles of 128 rows either way)
  const size_t rows = std::min((size_t)kMaxShares * cap * Hq, (size_t)num_sms() * 2 * BT);
  return rows * (hd + 2) * sizeof(float);
}

size_t attention_part_bytes(int S, int M_cap, int Hq, int hd) {
  return S > 1 ? (size_t)S * M_cap * Hq * (hd + 2) * sizeof(float) : 0;
}

AttnPlan attention_plan(int B, int k_cap, int Nseq, int Hq, int hd, int M_cap,
                        size_t part_bytes) {
  // Query tiles per CTA.  A pair of tiles shares each K/V tile, but an odd tile
  // count leaves a lone last tile whose CTA streams the keys again at half the
  // work; one tile per CTA with two CTAs per SM avoids it (32 sequences, 1536
  // keys: 308 rows 0.426 -> 0.367 ms, 1152 rows 1.047 -> 1.029, 1664 rows
  // 1.475 -> 1.455), at a cost where the tiles pair up evenly (256 rows: 0.244
  // ms in pairs, 0.259 ms singly).  With few tiles in all, one-tile CTAs also
  // split the keys among twice as many CTAs (given scratch for the shares), and
  // fit one wave where pairs would need two (8 sequences x 28 heads, one tile
  // each, 2048 keys: 0.057 -> 0.052 ms).
  AttnPlan pl{};
  const int tiles = (k_cap + BT - 1) / BT;
  const int S1 = part_bytes ? attention_kv_split(B, k_cap, Nseq, Hq, 1) : 1;
  const long long ctas2 = (long long)((tiles + 1) / 2) * Hq * B;  // pairs, one per SM
  const long long ctas1 = (long long)tiles * Hq * B;              // one tile, two per SM
  const bool one_wave = ctas2 > num_sms() && ctas1 <= 2LL * num_sms();
  pl.nt = (S1 > 1 || (tiles % 2 == 1 && tiles >= 3) || one_wave) ? 1 : 2;
  pl.shares = pl.nt == 1 ? S1 : (part_bytes ? attention_kv_split(B, k_cap, Nseq, Hq, 2) : 1);
  if (pl.shares > 1 && attention_part_bytes(pl.shares, M_cap, Hq, hd) > part_bytes)
    pl.shares = 1;
  pl.ctas = ((k_cap + pl.nt * BT - 1) / (pl.nt * BT)) * pl.shares * Hq * B;
  return pl;
}

cudaError_t launch_attention_tc(const __nv_bfloat16* q, int M_cap, const __nv_bfloat16* kc,
                                const __nv_bfloat16* vc, __nv_bfloat16* o, const int* row_off,
                                int B, int k_cap, int Nseq, int Hq, int Hkv, int hd, int* status,
                                cudaStream_t s, float* st_m, float* st_l, float* part,
                                size_t part_bytes) {
  if (B <= 0 || k_cap <= 0 || M_cap <= 0) return cudaSuccess;
  if (hd != 64 && hd != 128) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv;
  if (!tmap_bf16_2d(&tq, q, (uint64_t)M_cap, (uint64_t)Hq * hd, BT)) return cudaErrorInvalidValue;
  if (!tmap_bf16_2d(&tk, kc, (uint64_t)B * Nseq, (uint64_t)Hkv * hd, BKV))
    return cudaErrorInvalidValue;
  if (!tmap_bf16_2d(&tv, vc, (uint64_t)B * Nseq, (uint64_t)Hkv * hd, BKV))
    return cudaErrorInvalidValue;
  const AttnPlan pl = attention_plan(B, k_cap, Nseq, Hq, hd, M_cap, part ? part_bytes : 0);
  const int NT = pl.nt, S = pl.shares;
  float* part_o = S > 1 ? part : nullptr;
  float* part_ml = S > 1 ? part + (size_t)S * M_cap * Hq * hd : nullptr;
  AttnParams p{row_off, o,      Nseq, Hq,      Hkv,    Hq * hd, 1.4426950408889634f / sqrtf((float)hd),
               status,  st_m,   st_l, nullptr, 1,      S,       M_cap,
               part_o,  part_ml, nullptr};
  dim3 grid(((k_cap + NT * BT - 1) / (NT * BT)) * S, Hq, B);
  ProfScope prof("attention", s);
  cudaError_t e;
  if (NT == 1)
    e = hd == 128 ? launch_hd<128, false, 1>(tq, tk, tv, tk, tv, p, grid, s)
                  : launch_hd<64, false, 1>(tq, tk, tv, tk, tv, p, grid, s);
  else
    e = hd == 128 ? launch_hd<128, false, 2>(tq, tk, tv, tk, tv, p, grid, s)
                  : launch_hd<64, false, 2>(tq, tk, tv, tk, tv, p, grid, s);
  if (e != cudaSuccess || S == 1) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((M_cap + 7) / 8, Hq);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  la[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = la;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return hd == 128 ? cudaLaunchKernelEx(&cfg, attn_merge_kernel<128>, (const float*)part_o,
                                        (const float*)part_ml, S, M_cap, row_off + B, Hq, o,
                                        Hq * hd, st_m, st_l)
                   : cudaLaunchKernelEx(&cfg, attn_merge_kernel<64>, (const float*)part_o,
                                        (const float*)part_ml, S, M_cap, row_off + B, Hq, o,
                                        Hq * hd, st_m, st_l);
}

cudaError_t launch_attention_update(const __nv_bfloat16* q, int R_cap, __nv_bfloat16* o,
                                    float* st_m, float* st_l, const int* r_off, int r_cap,
                                    const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                                    const __nv_bfloat16* k_old, const __nv_bfloat16* v_old,
                                    const int* a_off, int A_cap, int B, int Hq, int Hkv, int hd,
                                    int* status, cudaStream_t s, const uint8_t* skip) {
  if (B <= 0 || r_cap <= 0 || R_cap <= 0 || A_cap <= 0) return cudaSuccess;
  if (hd != 64 && hd != 128) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv, tk2, tv2;
  const uint64_t cols = (uint64_t)Hkv * hd;
  if (!tmap_bf16_2d(&tq, q, (uint64_t)R_cap, (uint64_t)Hq * hd, BT) ||
      !tmap_bf16_2d(&tk, k_new, (uint64_t)A_cap, cols, BKV) ||
      !tmap_bf16_2d(&tv, v_new, (uint64_t)A_cap, cols, BKV) ||
      !tmap_bf16_2d(&tk2, k_old, (uint64_t)A_cap, cols, BKV) ||
      !tmap_bf16_2d(&tv2, v_old, (uint64_t)A_cap, cols, BKV))
    return cudaErrorInvalidValue;
  // few changed keys make short key streams: a CTA takes several pairs of query
  // tiles of its (sequence, head) in turn, keeping about two CTAs per SM in flight
  const int pairs = (r_cap + 2 * BT - 1) / (2 * BT);
  const int min_x = std::max(1, (2 * num_sms() + B * Hq - 1) / (B * Hq));
  const int ppc = std::max(1, (pairs + min_x - 1) / min_x);
  AttnParams p{r_off, o,    0,    Hq,   Hkv,   Hq * hd, 1.4426950408889634f / sqrtf((float)hd),
               status, st_m, st_l, a_off, ppc,   1,       0,
               nullptr, nullptr, skip};
  dim3 grid((pairs + ppc - 1) / ppc, Hq, B);
  ProfScope prof("attention_update", s);
  return hd == 128 ? launch_hd<128, true, 2>(tq, tk, tv, tk2, tv2, p, grid, s)
                   : launch_hd<64, true, 2>(tq, tk, tv, tk2, tv2, p, grid, s);
}

}  // namespace dllm
