// Internal launchers shared by the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace dllm {

int num_sms();
cudaError_t last_error();

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) is a per-device setting of a
// kernel: set it once for each device the kernel is launched on (one bit per
// device ordinal below 64; higher ordinals set it on every launch).
template <auto Kernel>
cudaError_t ensure_smem_attr(int bytes) {
  static std::atomic<unsigned long long> done{0ull};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// ----- kernel timing (dllm_profile_*) -----
void prof_begin(const char* name, cudaStream_t s);
void prof_end(cudaStream_t s);
struct ProfScope {
  cudaStream_t s;
  ProfScope(const char* name, cudaStream_t st) : s(st) { prof_begin(name, st); }
  ~ProfScope() { prof_end(s); }
};

// ----- TMA descriptors -----
// [rows, cols] bf16 row-major, box (64 columns, box_rows rows), 128-byte swizzle;
// cached by (address, shape, box)
bool tmap_bf16_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols,
                  uint32_t box_rows);

// ----- tcgen05 GEMM -----
enum EpiKind { EPI_STORE = 0, EPI_RESID = 1, EPI_SWIGLU = 2, EPI_QKV = 3, EPI_LMHEAD = 4 };

struct GemmSpec {
  int epi;
  // A [M_cap, K] bf16 row-major; rows >= *M_dev are ignored
  const __nv_bfloat16* A;
  int M_cap;
  const int* M_dev;  // may be null: M = M_cap
  int K;
  // B segments: columns [0, seg_cols[0]) from B[0], then B[1], then B[2]; each [cols, K].
  // SWIGLU: B[0] = gate [F, K], B[1] = up [F, K]; output width F.
  const __nv_bfloat16* B[3];
  int seg_cols[3];
  int n_seg;
  // STORE / RESID / SWIGLU output, QKV query output
  __nv_bfloat16* out;
  int ldo;
  // QKV
  __nv_bfloat16* kc;
  __nv_bfloat16* vc;
  const int* row_pos;
  const int* row_seq;
  int Nseq;
  int hd;
  const float2* rope;  // [Nseq, hd/2] (cos, sin), null: no rotation
  // LMHEAD partial softmax stats [M_cap, n_tiles] x (max, sum, argmax)
  float* lm_part;
  int lm_tiles;  // out: number of column tiles (set by plan)
  int* status;
  int force_bn;      // 0: choose
  int force_splits;  // 0: choose
  // fault injection for tests (CTA-pair plans only): CTA 1 of every pair never
  // reports its first stage, so CTA 0's bounded wait runs out (DEV_TIMEOUT)
  int stall_test;
};

// Kernels launch with programmatic stream serialization (they griddepcontrol.wait
// before reading what earlier kernels wrote).  A build with -DDLLM_BUILD_NO_PDL
// launches them plainly (an experiment switch of the build, not a run-time one).
#ifdef DLLM_BUILD_NO_PDL
constexpr bool kPdl = false;
#else
constexpr bool kPdl = true;
#endif
inline bool pdl_enabled() { return kPdl; }

struct GemmPlan {
  int bn, splits, tiles_n, m_tiles_cap, units_cap, grid;
  int pair;  // CTA pairs (tcgen05 cta_group::2) computing 256-row tiles
};

int gemm_total_cols(const GemmSpec& g);
GemmPlan gemm_plan(const GemmSpec& g);
cudaError_t gemm_launch(GemmSpec g, cudaStream_t s);

// ----- row bookkeeping, gather, norms -----
// row_off[B+1], row_pos[cap], row_seq[cap] from idx [B, k_cap] / count [B]; M_dev = row_off[B]
void launch_row_map(const int32_t* idx, const int32_t* count, int B, int k_cap, int N,
                    int* row_off, int* row_pos, int* row_seq, int* status, cudaStream_t s);
// identity map (all N rows of every sequence)
void launch_row_map_dense(int B, int N, int* row_off, int* row_pos, int* row_seq,
                          cudaStream_t s);
// x[r] = src row (b, pos) where src is [B,N,d] (or embed[tokens] when tokens != null);
// also h_ref[b,pos] = x[r] when h_ref != null
template <typename T>
void launch_gather_rows(const T* src_full, const T* embed, const int32_t* tokens,
                        const int* row_pos, const int* row_seq, const int* M_dev, int M_cap,
                        int N, int d, T* x, T* h_ref, int vocab, int* status, cudaStream_t s);
template <typename T>
void launch_rmsnorm(const T* x, const T* g, T* out, const int* M_dev, int M_cap, int d, float eps,
                    cudaStream_t s);
// final norm on the masked subset: lm_rows[j] = compact row, writes out[j]
template <typename T>
void launch_rmsnorm_rows(const T* x, const T* g, T* out, const int* rows, const int* n_rows,
                         int cap, int d, float eps, cudaStream_t s);
void launch_rope_table(float2* table, int N, int hd, float theta, cudaStream_t s);
// lm_rows: compact rows whose (b,pos) token is masked; n_lm = their count
void launch_masked_rows(const int32_t* tokens, int mask_id, const int* row_pos,
                        const int* row_seq, const int* M_dev, int M_cap, int N, int* lm_rows,
                        int* n_lm, cudaStream_t s);
void launch_lm_merge(const float* lm_part, int tiles, const int* lm_rows, const int* n_lm,
                     int cap, const int* row_pos, const int* row_seq, int N, float* conf,
                     int32_t* pred, cudaStream_t s);

// ----- fp32 (DLLM_F32) layer pieces -----
void launch_gemm_f32(const float* A, const float* B, float* C, const float* R, const int* M_dev,
                     int M_cap, int N, int K, cudaStream_t s);  // C = A B^T (+ R)
void launch_qkv_post_f32(const float* q_raw, const float* k_raw, const float* v_raw,
                         float* q_out, float* kc, float* vc, const int* row_pos,
                         const int* row_seq, const int* M_dev, int M_cap, int Nseq, int Hq,
                         int Hkv, int hd, const float2* rope, cudaStream_t s);
void launch_swiglu_f32(const float* g, const float* u, float* a, const int* M_dev, int M_cap,
                       int F, cudaStream_t s);
void launch_attention_f32(const float* q, const float* kc, const float* vc, float* o,
                          const int* row_seq, const int* M_dev, int M_cap, int Nseq, int Hq,
                          int Hkv, int hd, cudaStream_t s);
void launch_confidence_rows_f32(const float* logits, int V, const int* lm_rows, const int* n_lm,
                                int cap, const int* row_pos, const int* row_seq, int N,
                                float* conf, int32_t* pred, cudaStream_t s);

// ----- bf16 attention -----
// tcgen05 flash attention (Q compact [M_cap, Hq*hd], caches [B, N, Hkv, hd]); with st_m/st_l
// non-null also each row's softmax statistics [M_cap, Hq] (max score, sum of exp(s - max))
cudaError_t launch_attention_tc(const __nv_bfloat16* q, int M_cap, const __nv_bfloat16* kc,
                                const __nv_bfloat16* vc, __nv_bfloat16* o, const int* row_off,
                                int B, int k_cap, int Nseq, int Hq, int Hkv, int hd, int* status,
                                cudaStream_t s, float* st_m = nullptr, float* st_l = nullptr,
                                float* part = nullptr, size_t part_bytes = 0);
// key shares per CTA of NT query tiles the attention uses for this shape (1: none), and
// the partial-output scratch (fp32) that launch_attention_tc then needs in `part`
int attention_kv_split(int B, int k_cap, int Nseq, int Hq, int NT);
// the exact attention's launch plan: query tiles per CTA (1: two CTAs per SM, 2:
// a pair sharing each K/V tile), key shares per CTA's rows (needs part scratch of
// part_bytes), CTAs launched
struct AttnPlan {
  int nt, shares, ctas;
};
AttnPlan attention_plan(int B, int k_cap, int Nseq, int Hq, int hd, int M_cap,
                        size_t part_bytes);
size_t attention_part_bytes(int S, int M_cap, int Hq, int hd);
// scratch that covers the split of any launch over at most `cap` rows
size_t attention_part_bytes_bound(int cap, int Hq, int hd);
// incremental attention of stable rows: q [R_cap, Hq*hd] with cached o, st_m, st_l (in/out),
// rows of sequence b at r_off[b].. (at most r_cap); changed keys' new and old K/V
// [A_cap, Hkv*hd] compact, sequence b at rows a_off[b]..a_off[b+1]
cudaError_t launch_attention_update(const __nv_bfloat16* q, int R_cap, __nv_bfloat16* o,
                                    float* st_m, float* st_l, const int* r_off, int r_cap,
                                    const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                                    const __nv_bfloat16* k_old, const __nv_bfloat16* v_old,
                                    const int* a_off, int A_cap, int B, int Hq, int Hkv, int hd,
                                    int* status, cudaStream_t s, const uint8_t* skip = nullptr);

// ----- score / select / unmask -----
template <typename T>
void launch_confidence(const T* logits, const int32_t* logit_pos, int B, int Mm, int V, int N,
                       float* conf, int32_t* pred, cudaStream_t s);
// h row i = tokens ? embed[tokens[i]] : h_cur[i]; masked flag from `masked` or, when that
// is null, from mask_tokens[i] == mask_id (no flag when both are null)
template <typename T>
void launch_score(const T* h_cur, const T* embed, const int32_t* tokens, const T* h_ref, int B,
                  int N, int d, const float* conf, const uint8_t* masked,
                  const int32_t* mask_tokens, int mask_id, float alpha, int kind, float* scores,
                  int vocab, int lo, int* status, cudaStream_t s);
// positions < lo (and >= lens[b] when lens is given) are never candidates
void launch_select(const float* scores, int B, int N, int lo, int mode, int k, float tau,
                   int32_t* idx, int32_t* count, int k_cap, int* status, cudaStream_t s,
                   const int* lens = nullptr);
// second skip point: scores of the compact rows into [B, k_cap] segments
template <typename T>
void launch_score_rows(const T* x, const T* h_ref, const int* row_off, const int* row_pos,
                       const int* row_seq, const int* M, int cap, int N, int d, int k_cap,
                       const float* conf, const int32_t* tokens, int mask_id, float alpha,
                       int kind, float* scores, cudaStream_t s);
// positions of the kept rows from their indices within each sequence's segment
void launch_seg_positions(const int32_t* seg_idx, const int32_t* count, const int* row_off,
                          const int* row_pos, int B, int k2_cap, int32_t* pos, cudaStream_t s);
// narrowed compact rows (and their h_ref2 refresh) from the previous compact rows
template <typename T>
void launch_gather_narrow(const T* x, const int* row_off, const int* row_pos,
                          const int* row_off2, const int* row_pos2, const int* row_seq2,
                          const int* M2, int cap2, int N, int d, T* x2, T* h_ref2, int* status,
                          cudaStream_t s);
void launch_unmask(const float* conf, const int32_t* pred, int32_t* tokens, int B, int N,
                   int mask_id, int gen_start, int block_len, int n_unmask, float tau,
                   int pos_cap, int32_t* pos_out, const int32_t* forced, cudaStream_t s);
void launch_block_start(const int32_t* tokens, int B, int N, int mask_id, int gen_start,
                        int block_len, int32_t* out, cudaStream_t s);
// DyLLM FFN gate: flag rows whose attention output moved (1 - cos > tau, or all rows,
// or forced[r] != 0 when forced is given), refresh the context cache, compact the
// salient rows (list, inverse map, count)
template <typename T>
void launch_ffn_gate(const T* o, T* ctx, const int* row_pos, const int* row_seq,
                     const int* M_dev, int M_cap, int N, int q, float tau, int all_rows,
                     const uint8_t* forced, int* flag, int* list, int* inv, int* n_sal,
                     cudaStream_t s);
// x[r] += FFN output: the new one of a salient row (cached too) or the cached one
template <typename T>
void launch_ffn_combine(T* x, const T* f_new, T* f_cache, const int* inv, const int* row_pos,
                        const int* row_seq, const int* M_dev, int M_cap, int N, int d,
                        cudaStream_t s);
// DyLLM approximate attention bookkeeping.  Compact rows r < M (row_bytes per row, a
// multiple of 4) to / from a per-row cache [B, N, row_bytes]:
void launch_row_words(void* cache, void* compact, const int* row_pos, const int* row_seq,
                      const int* M_dev, int M_cap, int N, int row_bytes, bool to_cache,
                      cudaStream_t s);
// flags [B, N] uint8: 1 at the compact rows' positions, 0 elsewhere
void launch_mark_rows(const int* row_pos, const int* row_seq, const int* M_dev, int M_cap, int B,
                      int N, uint8_t* flags, cudaStream_t s);
// off[b] = b * N, b = 0..B (every row of every sequence in cache order)
void launch_seq_offsets(int B, int N, int* off, cudaStream_t s);
void launch_copy_idx(const int32_t* src_idx, const int32_t* src_count, int32_t* dst_idx,
                     int32_t* dst_count, int B, int k_cap, cudaStream_t s);

}  // namespace dllm
