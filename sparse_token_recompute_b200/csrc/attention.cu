// Partial attention: the selected query rows of each sequence attend to all
// N cached keys of that sequence (bidirectional, no mask), flash-style with
// an online softmax, bf16 operands and fp32 accumulation.
//
// Grid (query tiles of 64 rows, query head, sequence).  A CTA of 4 warps
// owns 64 compact query rows of one (sequence, head); K/V tiles of 64 keys
// stream through a double-buffered shared-memory ring (cp.async, 16-byte
// chunks XOR-swizzled by row to keep ldmatrix conflict-free).  S = Q K^T and
// O += P V use the warp-level bf16 MMA (m16n8k16); P stays in registers.
#include "common.cuh"
#include "internal.h"

namespace dllm {

namespace {

constexpr int BQ = 64;
constexpr int BKV = 64;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

// byte offset of 16-byte chunk c of row r in a [rows, HD] bf16 tile
template <int HD>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(r * HD * 2 + ((c ^ (r & 7)) << 4));
}

template <int HD>
__global__ void __launch_bounds__(128) attn_bf16_kernel(const __nv_bfloat16* __restrict__ Q,
                                                        const __nv_bfloat16* __restrict__ Kc,
                                                        const __nv_bfloat16* __restrict__ Vc,
                                                        __nv_bfloat16* __restrict__ O,
                                                        const int* __restrict__ row_off, int Nseq,
                                                        int Hq, int Hkv, float scale_log2) {
  constexpr int CH = HD / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + BQ * HD * 2;
  const uint32_t sV = sK + 2 * BKV * HD * 2;

  const int b = blockIdx.z, h = blockIdx.y;
  const int off = row_off[b];
  const int cnt = row_off[b + 1] - off;
  const int q0 = blockIdx.x * BQ;
  if (q0 >= cnt) return;
  const int g = (h * Hkv) / Hq;
  const size_t ldq = (size_t)Hq * HD;
  const size_t ldkv = (size_t)Hkv * HD;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int i = tid; i < BQ * CH; i += 128) {
    const int r = i / CH, c = i % CH;
    const bool ok = q0 + r < cnt;
    const __nv_bfloat16* src = Q + (size_t)(off + (ok ? q0 + r : 0)) * ldq + h * HD + c * 8;
    cp_async16(sQ + swz<HD>(r, c), src, ok);
  }
  auto load_kv = [&](int t, int buf) {
    for (int i = tid; i < BKV * CH; i += 128) {
      const int r = i / CH, c = i % CH;
      const int key = t * BKV + r;
      const bool ok = key < Nseq;
      const size_t base = (((size_t)b * Nseq + (ok ? key : 0)) * Hkv + g) * HD + c * 8;
      cp_async16(sK + buf * BKV * HD * 2 + swz<HD>(r, c), Kc + base, ok);
      cp_async16(sV + buf * BKV * HD * 2 + swz<HD>(r, c), Vc + base, ok);
    }
  };
  load_kv(0, 0);
  cp_async_commit();

  uint32_t qf[HD / 16][4];
  float o[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  const int n_tiles = (Nseq + BKV - 1) / BKV;
  for (int t = 0; t < n_tiles; ++t) {
    const int buf = t & 1;
    cp_async_wait_all();
    __syncthreads();
    if (t + 1 < n_tiles) load_kv(t + 1, buf ^ 1);
    cp_async_commit();
    if (t == 0) {
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks)
        ldsm_x4(sQ + swz<HD>(warp * 16 + (lane & 15), ks * 2 + (lane >> 4)), qf[ks]);
    }
    // S = Q K^T for 16 rows x 64 keys
    float s[BKV / 8][4];
#pragma unroll
    for (int i = 0; i < BKV / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
    const uint32_t kb = sK + buf * BKV * HD * 2;
#pragma unroll
    for (int ks = 0; ks < HD / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < BKV / 16; ++np) {
        uint32_t bf[4];
        ldsm_x4(kb + swz<HD>(np * 16 + (lane & 7) + ((lane >> 4) << 3),
                             ks * 2 + ((lane >> 3) & 1)),
                bf);
        mma_bf16(s[2 * np], qf[ks], bf[0], bf[1]);
        mma_bf16(s[2 * np + 1], qf[ks], bf[2], bf[3]);
      }
    }
    // scale into the exp2 domain, mask keys past the end
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < BKV / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = t * BKV + nt * 8 + 2 * (lane & 3) + (e & 1);
        s[nt][e] = key < Nseq ? s[nt][e] * scale_log2 : -INFINITY;
      }
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float nm0 = fmaxf(m0, mx0), nm1 = fmaxf(m1, mx1);
    const float a0 = exp2f(m0 - nm0), a1 = exp2f(m1 - nm1);
    m0 = nm0;
    m1 = nm1;
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < BKV / 8; ++nt) {
      s[nt][0] = exp2f(s[nt][0] - nm0);
      s[nt][1] = exp2f(s[nt][1] - nm0);
      s[nt][2] = exp2f(s[nt][2] - nm1);
      s[nt][3] = exp2f(s[nt][3] - nm1);
      rs0 += s[nt][0] + s[nt][1];
      rs1 += s[nt][2] + s[nt][3];
    }
    l0 = l0 * a0 + rs0;
    l1 = l1 * a1 + rs1;
#pragma unroll
    for (int i = 0; i < HD / 8; ++i) {
      o[i][0] *= a0;
      o[i][1] *= a0;
      o[i][2] *= a1;
      o[i][3] *= a1;
    }
    // O += P V
    const uint32_t vb = sV + buf * BKV * HD * 2;
#pragma unroll
    for (int kk = 0; kk < BKV / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int np = 0; np < HD / 16; ++np) {
        uint32_t bf[4];
        ldsm_x4_t(vb + swz<HD>(kk * 16 + (lane & 15), np * 2 + (lane >> 4)), bf);
        mma_bf16(o[2 * np], pa, bf[0], bf[1]);
        mma_bf16(o[2 * np + 1], pa, bf[2], bf[3]);
      }
    }
  }
  cp_async_wait_all();
  // row sums across the quad
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float i0 = 1.0f / l0, i1 = 1.0f / l1;
  const int r0 = q0 + warp * 16 + (lane >> 2);
  const int r1 = r0 + 8;
#pragma unroll
  for (int nt = 0; nt < HD / 8; ++nt) {
    const int col = h * HD + nt * 8 + 2 * (lane & 3);
    if (r0 < cnt)
      *reinterpret_cast<uint32_t*>(O + (size_t)(off + r0) * ldq + col) =
          pack_bf2(o[nt][0] * i0, o[nt][1] * i0);
    if (r1 < cnt)
      *reinterpret_cast<uint32_t*>(O + (size_t)(off + r1) * ldq + col) =
          pack_bf2(o[nt][2] * i1, o[nt][3] * i1);
  }
}

}  // namespace

void launch_attention_bf16(const __nv_bfloat16* q, const __nv_bfloat16* kc,
                           const __nv_bfloat16* vc, __nv_bfloat16* o, const int* row_off, int B,
                           int k_cap, int Nseq, int Hq, int Hkv, int hd, cudaStream_t s) {
  if (B <= 0 || k_cap <= 0) return;
  ProfScope prof("attention", s);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)hd);
  dim3 grid((k_cap + BQ - 1) / BQ, Hq, B);
  if (hd == 128) {
    constexpr size_t smem = (size_t)(BQ + 4 * BKV) * 128 * 2;
    static bool attr = false;
    if (!attr) {
      cudaFuncSetAttribute(attn_bf16_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
      attr = true;
    }
    attn_bf16_kernel<128><<<grid, 128, smem, s>>>(q, kc, vc, o, row_off, Nseq, Hq, Hkv,
                                                  scale_log2);
  } else {
    constexpr size_t smem = (size_t)(BQ + 4 * BKV) * 64 * 2;
    attn_bf16_kernel<64><<<grid, 128, smem, s>>>(q, kc, vc, o, row_off, Nseq, Hq, Hkv,
                                                 scale_log2);
  }
}

}  // namespace dllm
