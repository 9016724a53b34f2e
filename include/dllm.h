/*
 * dllm.h - C ABI of the selected-token denoising step for masked-diffusion
 * language models, sm_100a (NVIDIA B200).
 *
 * One denoising step scores every token by how far its hidden state moved
 * since the row was last recomputed and by its cached confidence, keeps the
 * top-k (or over-threshold) positions, recomputes only those rows through
 * the transformer layers (their queries attend to the full cached K/V), and
 * writes the new K/V / hidden / confidence rows back into the caches.
 *
 * Sources, cited by page title and section:
 *   [ES-de]  "ES-dLLM: Efficient Inference for Diffusion Large Language
 *            Models by Early-Skipping", German technical summary: section 2.A
 *            (importance score I = alpha*c + (1-alpha)*variation, alpha 0.5),
 *            section 2.B (top-k rows processed, K/V/hidden caches updated for
 *            selected rows in place, skipped rows reuse cached values).
 *   [DyLLM]  "DyLLM: Efficient Diffusion LLM Inference via Saliency-based
 *            Token Selection and Partial Attention", French technical
 *            summary: section 1 (bidirectional attention over the whole
 *            sequence each step), section 2.A (cosine similarity against the
 *            previous step, salient if below a threshold tau), section 2.B
 *            (rows of salient tokens recomputed exactly).
 *   [SF-de]  "Accelerating Diffusion Large Language Models with SlowFast
 *            Sampling", German technical summary, section 2 (the most
 *            confident masked tokens of a window are revealed each step).
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is device memory owned by the caller unless the
 *     argument is documented as host memory.  The library never allocates
 *     device memory: scratch comes from a caller buffer of at least the size
 *     the matching *_workspace_size() call returns (256-byte aligned).
 *   - Every call is asynchronous on the given CUDA stream (NULL: the legacy
 *     default stream) and returns before the GPU work finishes.
 *   - Arguments are validated before anything is launched; on an error
 *     nothing is launched and outputs are untouched.
 *   - Faults the GPU detects (a wait that ran past its limit, more candidates
 *     than an index list holds) set bits in a status word inside the
 *     workspace; dllm_get_device_status() reads and clears it.
 *   - Tensors are dense row-major; weights are [out, in] (y = x W^T).
 *   - Storage dtype DLLM_BF16 computes with fp32 accumulation and stores
 *     bf16; DLLM_F32 stores fp32 (small models, exact-arithmetic checks).
 *   - No C++ exception crosses this boundary.
 *   - One kernel path per operation: no environment variable or run-time
 *     switch selects another implementation.
 */
#ifndef DLLM_H
#define DLLM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st* dllm_stream_t;

typedef enum {
  DLLM_OK = 0,
  DLLM_ERR_INVALID_ARG = 1,      /* null pointer, negative size, bad enum      */
  DLLM_ERR_UNSUPPORTED_SHAPE = 2,/* a size this build cannot run (see below)   */
  DLLM_ERR_WORKSPACE = 3,        /* workspace missing, misaligned or too small */
  DLLM_ERR_CUDA = 4,             /* a CUDA runtime call failed                 */
  DLLM_ERR_CAPACITY = 5,         /* more rows than the index capacity          */
  DLLM_ERR_DEVICE = 6            /* the device status word is non-zero         */
} dllm_status;

typedef enum { DLLM_F32 = 0, DLLM_BF16 = 1 } dllm_dtype;

/* variation measure: 1 - cos(h, h_ref) [DyLLM 2.A] or
 * ||h - h_ref||_1 / (sqrt(d) ||h_ref||_2) [ES-de 2.A] */
typedef enum { DLLM_SCORE_COS = 0, DLLM_SCORE_ES_L1 = 1 } dllm_score_kind;

/* top-k [ES-de 2.B] or every score strictly above tau [DyLLM 2.A] */
typedef enum { DLLM_SELECT_TOPK = 0, DLLM_SELECT_THRESH = 1 } dllm_select_mode;

/* device status word bits */
#define DLLM_DEV_TIMEOUT 1
#define DLLM_DEV_CAPACITY 2
#define DLLM_DEV_BAD_INDEX 4
#define DLLM_DEV_BAD_SHAPE 8

typedef struct {
  int n_layers;
  int d;            /* model width                                  */
  int n_heads;      /* query heads                                  */
  int n_kv_heads;   /* key/value heads (divides n_heads)            */
  int head_dim;     /* 64 or 128                                    */
  int ffn;          /* SwiGLU hidden width                          */
  int vocab;
  float rope_theta; /* 0 disables the rotary embedding              */
  float rms_eps;
  int mask_id;      /* token id of [MASK]                           */
  int dtype;        /* dllm_dtype of weights, caches and activations */
} dllm_model_cfg;

/* One pre-RMSNorm transformer block.  Device pointers, dtype of the model. */
typedef struct {
  const void* attn_norm; /* [d]                    */
  const void* wq;        /* [n_heads*head_dim, d]  */
  const void* wk;        /* [n_kv_heads*head_dim, d] */
  const void* wv;        /* [n_kv_heads*head_dim, d] */
  const void* wo;        /* [d, n_heads*head_dim]  */
  const void* ffn_norm;  /* [d]                    */
  const void* w_gate;    /* [ffn, d]               */
  const void* w_up;      /* [ffn, d]               */
  const void* w_down;    /* [d, ffn]               */
} dllm_layer_w;

typedef struct {
  const void* embed;            /* [vocab, d] device                      */
  const dllm_layer_w* layers;   /* HOST array [n_layers] of device pointers */
  const void* final_norm;       /* [d] device                             */
  const void* lm_head;          /* [vocab, d] device                      */
} dllm_model_w;

/* The state kept between steps.  k/v are HOST arrays of n_layers device
 * pointers, each cache [B, N, n_kv_heads, head_dim] (K stored after RoPE).
 * h_ref [B, N, d]: each row's score-layer hidden at its last recompute.
 * conf [B, N] f32 / pred [B, N] int32: confidence and argmax of each
 * position's last LM-head evaluation (c^(t-1) of [ES-de 2.A]). */
typedef struct {
  void* const* k;
  void* const* v;
  void* h_ref;
  float* conf;
  int32_t* pred;
  void* h_ref2;  /* [B, N, d]: each row's input of policy.score_layer2 at its last pass
                  * through that layer; NULL unless the policy has a second skip point */
  /* DyLLM FFN gate (policy.ffn_gate); HOST arrays of n_layers device pointers,
   * NULL when the gate is off: */
  void* const* ctx;  /* [B, N, n_heads*head_dim] each row's attention output at its
                      * last pass through the layer */
  void* const* ffn;  /* [B, N, d] each row's FFN output at its last salient pass */
  /* DyLLM approximate attention (policy.attn_update); HOST arrays of n_layers device
   * pointers, NULL when off: */
  void* const* q;       /* [B, N, n_heads*head_dim] each row's query (after RoPE) at its
                         * last exact pass through the layer */
  float* const* att_m;  /* [B, N, n_heads] f32: softmax statistics of each row's attention */
  float* const* att_l;  /* [B, N, n_heads] f32: (reference max and sum, natural log units,
                         * as dllm_attention_stats_bf16), kept up to date by the updates */
} dllm_cache;

typedef struct {
  int score_layer;   /* layers below it run on every row; the score is taken on its input */
  float alpha;       /* I = alpha * c + (1 - alpha) * v                 */
  int kind;          /* dllm_score_kind                                 */
  int mode;          /* dllm_select_mode                                */
  int k;             /* TOPK: rows per sequence; THRESH: capacity       */
  float tau;         /* THRESH: keep scores > tau                       */
  int n_unmask;      /* positions revealed per sequence and step        */
  int gen_start;     /* first generated position                        */
  int block_len;     /* generation block length                         */
  /* Step variants (0 disables each):                                     */
  int select_from;   /* partial steps never select positions below it:   */
                     /* response-only steps [DyLLM 2.C] use gen_start    */
  float unmask_tau;  /* > 0: also reveal every masked position of the    */
                     /* block with conf > unmask_tau [SF-de 2, fast phase]*/
  int refresh_every; /* dllm_generate: dense step every R steps [ES-nl 3] */
  int refresh_on_block; /* dllm_generate: dense step when a block changes */
  /* Second skip point [ES-de 2.B, "layers 1/8 and 1/4"]: when            */
  /* score_layer < score_layer2 < n_layers, the rows selected at           */
  /* score_layer are scored again on their input of score_layer2 (against */
  /* cache.h_ref2) and each sequence keeps its top-k2 of them from there.  */
  int score_layer2;  /* 0: no second skip point                         */
  int k2;            /* rows per sequence kept at the second skip point  */
  /* FFN gate [DyLLM 2.A]: a recomputed row runs a layer's FFN only when its */
  /* attention output moved since its last pass, 1 - cos > ffn_tau; else it  */
  /* adds the FFN output cached at its last salient pass (cache.ctx/ffn).    */
  /* Dense steps run every FFN and fill both caches.                         */
  int ffn_gate;      /* 0: off                                           */
  float ffn_tau;
  /* Approximate attention of stable rows [DyLLM 2.B] (needs ffn_gate and      */
  /* DLLM_BF16): in every layer a partial step recomputes, each row it does    */
  /* not recompute keeps the query and softmax statistics of its last exact    */
  /* attention (cache.q/att_m/att_l) and its output (cache.ctx) and takes in   */
  /* only the keys the step changed in that layer: their old terms leave the   */
  /* sums, their new terms enter (dllm_attention_update_bf16).  The result is  */
  /* the row's attention context, the FFN gate's reference at its next pass.   */
  /* Recomputed rows store their query and exact statistics; a dense step     */
  /* stores them for every row.  Layers below score_layer keep no such state.  */
  int attn_update;   /* 0: off                                           */
} dllm_policy;

/* Supported shapes for DLLM_BF16 layer work: d, n_heads*head_dim,
 * n_kv_heads*head_dim and ffn multiples of 128; head_dim 64 or 128;
 * vocab a multiple of 8.  DLLM_F32: any d, ffn; head_dim <= 128 even.
 * Sequence length N <= 16384 for selection and unmasking; block_len <= 1024. */

const char* dllm_status_string(int status);
int dllm_version(void);

/*
 * dllm_score - importance score of every row [ES-de 2.A; DyLLM 2.A].
 *
 * When logits != NULL, first refreshes the cached confidence of the rows
 * the logits belong to: for b < B, j < Mm, row logit_pos[b*Mm+j] of
 * sequence b gets conf = max softmax of logits[b, j, :] (in fp32) and
 * pred = its argmax (lowest id on ties).  Then for every row i:
 *   v_i = variation(h_cur[b,i,:], h_ref[b,i,:], kind)   (0 when bitwise equal)
 *   c_i = masked[b,i] ? conf[b,i] : 0
 *   scores[b,i] = alpha * c_i + (1 - alpha) * v_i       (fp32)
 * h_cur, h_ref: [B, N, d] of dtype; logits [B, Mm, V] of dtype;
 * logit_pos [B, Mm] int32 in [0, N); conf [B, N] f32 in/out;
 * pred [B, N] int32 out (may be NULL); masked [B, N] uint8; scores [B, N] f32 out.
 * d must be a multiple of 8 (bf16) or 4 (f32); V a multiple of 8 (bf16) or 4.
 */
dllm_status dllm_score(const void* h_cur, const void* h_ref, int B, int N, int d, int dtype,
                       const void* logits, const int32_t* logit_pos, int Mm, int V, float* conf,
                       int32_t* pred, const uint8_t* masked, float alpha, int kind,
                       float* scores, dllm_stream_t stream);

/*
 * dllm_select - per-sequence compaction of the rows to recompute [ES-de 2.B].
 *
 * TOPK: the min(k, N) highest scores of each sequence under the order
 * (score descending, position ascending; -0 equals +0; NaN below all).
 * THRESH: every position with score > tau, capped at k_cap by that order.
 * idx [B, k_cap] int32 receives each sequence's positions in ascending order
 * (entries past count[b] are left untouched); count [B] int32.
 * ws: at least dllm_select_workspace_size() bytes, or NULL; when given, a
 * THRESH selection clipped by k_cap sets DLLM_DEV_CAPACITY in its status word.
 * Bit-exact and deterministic.  N <= 16384; k_cap >= 1 (TOPK needs k <= k_cap).
 */
size_t dllm_select_workspace_size(int B, int N);
dllm_status dllm_select(const float* scores, int B, int N, int mode, int k, float tau,
                        int32_t* idx, int32_t* count, int k_cap, void* ws, size_t ws_bytes,
                        dllm_stream_t stream);

/*
 * dllm_select_range - dllm_select over the positions lo .. N-1 only: the
 * selection of a response-only step [DyLLM 2.C], whose prompt rows keep
 * their cached K/V until a dense step brings the prompt in again.  TOPK
 * takes min(k, N - lo) positions; 0 <= lo <= N.  Same outputs and errors
 * as dllm_select; lo = 0 is dllm_select.
 */
dllm_status dllm_select_range(const float* scores, int B, int N, int lo, int mode, int k,
                              float tau, int32_t* idx, int32_t* count, int k_cap, void* ws,
                              size_t ws_bytes, dllm_stream_t stream);

/*
 * dllm_unmask - reveal the most confident masked positions [SF-de 2].
 *
 * For each sequence: the current block is [s, min(s + block_len, N)) with
 * s = gen_start + floor((p - gen_start) / block_len) * block_len and p the
 * first masked position >= gen_start.  Among its masked positions the
 * n_unmask with the highest conf (ties: lower position) get
 * tokens[b, p] = pred[b, p].  pos_out [B, n_unmask] int32 receives the
 * revealed positions in ascending order, padded with -1.
 * Bit-exact.  block_len <= 1024, N <= 16384.
 */
dllm_status dllm_unmask(const float* conf, const int32_t* pred, int32_t* tokens, int B, int N,
                        int mask_id, int gen_start, int block_len, int n_unmask,
                        int32_t* pos_out, dllm_stream_t stream);

/*
 * dllm_unmask_tau - dllm_unmask with the over-threshold rule of the fast
 * phase [SF-de 2]: with tau > 0, every masked position of the current block
 * whose conf > tau (strict, fp32) is revealed, and when fewer than n_unmask
 * are above tau the n_unmask most confident ones are (the top-n fallback) -
 * together, the max(n_unmask, #above) most confident masked positions of the
 * block, at most pos_cap.  tau <= 0 is dllm_unmask.  pos_out [B, pos_cap]
 * (pos_cap >= n_unmask; block_len suffices for any tau), ascending, -1 padded.
 * Bit-exact.  The pages fix no threshold value; the "stable region" of the
 * fast phase is read as the current block.
 */
dllm_status dllm_unmask_tau(const float* conf, const int32_t* pred, int32_t* tokens, int B, int N,
                            int mask_id, int gen_start, int block_len, int n_unmask, float tau,
                            int32_t* pos_out, int pos_cap, dllm_stream_t stream);

/* Entries per sequence of pos_out / forced_unmask_pos under a policy:
 * n_unmask, or max(n_unmask, block_len) when unmask_tau > 0. */
int dllm_unmask_capacity(const dllm_policy* policy);

/*
 * dllm_partial_layer - one transformer layer on the selected rows only
 * [ES-de 2.B; DyLLM 2.B].
 *
 * Rows: sequence b contributes count[b] rows, positions idx[b*k_cap + j]
 * (ascending, j < count[b]).  They are packed by sequence: compact row r of
 * sequence b is r = sum_{b'<b} count[b'] + j.
 * x_in: x_in_is_full = 1 -> [B, N, d], row (b, idx) is gathered;
 *       x_in_is_full = 0 -> compact [B*k_cap, d].
 * x_out: compact [B*k_cap, d] (may equal x_in when compact).
 * Order inside the layer: RMSNorm -> Q,K,V of all selected rows (RoPE at the
 * row's position) -> their K/V rows overwrite k_cache/v_cache
 * [B, N, n_kv_heads, head_dim] -> each selected query attends to all N keys
 * of its sequence (no mask, scale 1/sqrt(head_dim)) -> O projection +
 * residual -> RMSNorm -> SwiGLU FFN + residual.
 * Rows that are not selected keep their cached K/V untouched.
 */
size_t dllm_partial_layer_workspace_size(const dllm_model_cfg* cfg, int B, int N, int k_cap);
dllm_status dllm_partial_layer(const dllm_model_cfg* cfg, const dllm_layer_w* w,
                               const void* x_in, int x_in_is_full, void* x_out,
                               const int32_t* idx, const int32_t* count, int k_cap, int B,
                               int N, void* k_cache, void* v_cache, void* ws, size_t ws_bytes,
                               dllm_stream_t stream);

/*
 * dllm_step - one whole denoising step [ES-de 2.A-2.B; DyLLM 2; SF-de 2].
 *
 * tokens [B, N] int32 in/out.  With dense = 1 every row is recomputed
 * (first step, or a full refresh).  Otherwise:
 *  1. h = embedding of tokens; layers below policy.score_layer run on every row;
 *  2. scores as dllm_score with c = cache.conf, alpha/kind from policy;
 *  3. selection as dllm_select (k_cap = min(policy.k, N));
 *  4. cache.h_ref rows of the selection <- their score-layer hidden;
 *  5. dllm_partial_layer for layers score_layer .. n_layers-1;
 *  6. for selected rows whose token is [MASK]: final RMSNorm, LM head,
 *     cache.conf <- max softmax, cache.pred <- argmax (logits never stored);
 *  7. dllm_unmask_tau with policy.n_unmask / unmask_tau / gen_start / block_len.
 * policy.select_from > 0 (response-only steps [DyLLM 2.C]): steps 2-3 only
 * consider positions >= select_from; the scores of the others are -inf.
 * forced_idx [B, k_cap] + forced_count [B] replace steps 2-3 when non-NULL;
 * forced_unmask_pos [B, cap] (-1 padded) replaces step 7's choice, with
 * cap = dllm_unmask_capacity(policy).
 * Outputs (each may be NULL): idx_out [B, k_cap], count_out [B],
 * pos_out [B, cap], scores_out [B, N].
 * The workspace size covers both dense and partial steps of this shape.
 */
size_t dllm_step_workspace_size(const dllm_model_cfg* cfg, int B, int N,
                                const dllm_policy* policy);

/* Optional inputs and outputs of dllm_step_ex; every pointer may be NULL.
 * The first eight mean what the dllm_step arguments of the same names mean.
 * forced_idx2 [B, k2_cap] + forced_count2 [B] (positions, a subset of each
 * sequence's first selection) replace the choice at the second skip point;
 * idx2_out [B, k2_cap] / count2_out [B] receive it, with k2_cap =
 * max(1, min(policy.k2, k_cap)); scores2_out [B, k_cap] receives the second
 * scores of each sequence's rows in the order of its first selection. */
typedef struct {
  const int32_t* forced_idx;
  const int32_t* forced_count;
  const int32_t* forced_unmask_pos;
  int32_t* idx_out;
  int32_t* count_out;
  int32_t* pos_out;
  float* scores_out;
  const int32_t* forced_idx2;
  const int32_t* forced_count2;
  int32_t* idx2_out;
  int32_t* count2_out;
  float* scores2_out;
  int32_t* ffn_rows_out;  /* [n_layers] device: rows that ran each layer's FFN under the
                           * FFN gate (layers the step did not run are left untouched) */
  const uint8_t* forced_ffn; /* [n_layers, B*k_cap] device: replaces the FFN gate's rule in a
                              * partial step; entry l*B*k_cap + r != 0 makes compact row r
                              * (rows packed by sequence in ascending position, after a
                              * second skip point the kept rows) salient in layer l */
} dllm_step_io;

/*
 * dllm_step_ex - dllm_step with the second skip point of [ES-de 2.B]: after
 * layers score_layer .. score_layer2-1 on the rows of the first selection,
 *  a. each of them is scored as in dllm_score on its input of layer
 *     score_layer2 against cache.h_ref2 (c = cache.conf of masked rows);
 *  b. each sequence keeps the top-k2 of its rows (dllm_select order);
 *  c. cache.h_ref2 rows of the kept rows <- that input;
 *  d. layers score_layer2 .. n_layers-1 and the LM head run on the kept rows.
 * Dropped rows keep their new K/V below score_layer2 and their cached K/V
 * from there on.  A dense step writes cache.h_ref2 for every row.  io may be
 * NULL.  Same workspace as dllm_step for the same policy.
 */
dllm_status dllm_step_ex(const dllm_model_cfg* cfg, const dllm_model_w* w,
                         const dllm_cache* cache, int32_t* tokens, int B, int N,
                         const dllm_policy* policy, int dense, const dllm_step_io* io, void* ws,
                         size_t ws_bytes, dllm_stream_t stream);
dllm_status dllm_step(const dllm_model_cfg* cfg, const dllm_model_w* w, const dllm_cache* cache,
                      int32_t* tokens, int B, int N, const dllm_policy* policy, int dense,
                      const int32_t* forced_idx, const int32_t* forced_count,
                      const int32_t* forced_unmask_pos, int32_t* idx_out, int32_t* count_out,
                      int32_t* pos_out, float* scores_out, void* ws, size_t ws_bytes,
                      dllm_stream_t stream);

/*
 * dllm_generate - n_steps denoising steps with the periodic cache refresh of
 * [ES-nl Methodologie 3]: step t is dense (every row recomputed, every cache
 * rewritten) when t = 0, when policy.refresh_every > 0 divides t, or - with
 * policy.refresh_on_block - when any sequence's current block (the block of
 * its first masked position) differs from the one it had at step t-1; every
 * other step is a partial step of dllm_step.  With refresh_every = 1 this is
 * the vanilla (dense every step) generation; with select_from = gen_start
 * and refresh_every = R it is DyLLM's response-only decoding with the prompt
 * injected every R steps [DyLLM 2.C].
 * pos_log: device [n_steps, B, dllm_unmask_capacity(policy)] int32 or NULL,
 * the positions revealed at each step.  dense_log: HOST [n_steps] uint8 or
 * NULL, 1 where the step was dense.  Steps are launched on `stream` from the
 * host without synchronising, except that refresh_on_block reads the B block
 * starts back once per step (one small device-to-host copy, which waits for
 * the previous step).  ws: dllm_generate_workspace_size() bytes.
 */
size_t dllm_generate_workspace_size(const dllm_model_cfg* cfg, int B, int N,
                                    const dllm_policy* policy);
dllm_status dllm_generate(const dllm_model_cfg* cfg, const dllm_model_w* w,
                          const dllm_cache* cache, int32_t* tokens, int B, int N,
                          const dllm_policy* policy, int n_steps, int32_t* pos_log,
                          uint8_t* dense_log, void* ws, size_t ws_bytes, dllm_stream_t stream);

/*
 * dllm_step_host - one dllm_step whose token state lives in HOST memory, for
 * callers that keep tokens on the host between steps: copies tokens_host
 * [B, N] int32 (HOST, in/out) into the workspace, runs the step there, and
 * copies the updated tokens back into tokens_host and, when pos_host is not
 * NULL, the revealed positions into pos_host [B, dllm_unmask_capacity(policy)]
 * (HOST, -1 padded).  Everything is enqueued on `stream`; the host buffers are
 * read and written by the copies in stream order, so they hold the results
 * once the stream has been synchronised (page-locked host memory keeps the
 * copies asynchronous).  ws: dllm_step_host_workspace_size() bytes.
 */
size_t dllm_step_host_workspace_size(const dllm_model_cfg* cfg, int B, int N,
                                     const dllm_policy* policy);
dllm_status dllm_step_host(const dllm_model_cfg* cfg, const dllm_model_w* w,
                           const dllm_cache* cache, int32_t* tokens_host, int B, int N,
                           const dllm_policy* policy, int dense, int32_t* pos_host, void* ws,
                           size_t ws_bytes, dllm_stream_t stream);

/*
 * dllm_attention_bf16 - the partial attention of one layer on its own
 * [DyLLM 1, 2.B]: the selected query rows attend to all N cached keys of
 * their sequence, no mask, scale 1/sqrt(head_dim), query head h reading KV
 * head floor(h * n_kv_heads / n_heads).
 * q: compact rows [B*k_cap, n_heads*head_dim] bf16, packed by sequence as in
 * dllm_partial_layer (count[b] rows for sequence b); k_cache, v_cache
 * [B, N, n_kv_heads, head_dim] bf16; o: compact [B*k_cap, n_heads*head_dim].
 * head_dim 64 or 128.  ws: dllm_attention_workspace_size(B) bytes.
 */
size_t dllm_attention_workspace_size(int B);
dllm_status dllm_attention_bf16(const void* q, const void* k_cache, const void* v_cache, void* o,
                                const int32_t* count, int B, int k_cap, int N, int n_heads,
                                int n_kv_heads, int head_dim, void* ws, size_t ws_bytes,
                                dllm_stream_t stream);

/*
 * dllm_attention_stats_bf16 - dllm_attention_bf16 that also returns each
 * row's softmax statistics per query head, in natural-log units: a reference
 * m and l = sum_j exp(q.k_j / sqrt(head_dim) - m), so that m + log(l) is the
 * log-sum-exp of the row's scores.  m is the largest score up to the kernel's
 * lazy raise (it can sit below the maximum by at most 8 ln 2, which keeps
 * every exp(s - m) <= 256).  m, l: [B*k_cap, n_heads] f32, rows packed like q
 * and o.  They are what dllm_attention_update_bf16 keeps up to date for rows
 * that are not recomputed.
 */
dllm_status dllm_attention_stats_bf16(const void* q, const void* k_cache, const void* v_cache,
                                      void* o, float* m, float* l, const int32_t* count, int B,
                                      int k_cap, int N, int n_heads, int n_kv_heads, int head_dim,
                                      void* ws, size_t ws_bytes, dllm_stream_t stream);

/*
 * dllm_attention_update_bf16 - the approximate attention of rows that are not
 * recomputed [DyLLM 2.B]: such a row keeps its query and the statistics
 * (m, l, o) of its last exact attention; when some of its sequence's keys
 * change, only those keys are visited: each one's old term leaves the softmax
 * sums and its new term enters them (reference maximum raised to cover the
 * new scores).  With the row's current query this equals the attention over
 * the updated keys; with a stale one it is DyLLM's reuse of the unchanged
 * keys' weights.  Cost O(rows x changed keys) instead of O(rows x N).
 * q: [B*r_cap, n_heads*head_dim] bf16, the stable rows' cached queries packed
 *    by sequence (r_count[b] rows for sequence b, as in dllm_attention_bf16);
 * o: same layout, in/out (the cached outputs, then the updated ones);
 * m, l: [B*r_cap, n_heads] f32 in/out, natural-log units as above;
 * k_new, v_new, k_old, v_old: [B*a_cap, n_kv_heads, head_dim] bf16, the changed
 *    keys' values after and before the change, packed by sequence
 *    (a_count[b] keys for sequence b).
 * Rows of a sequence with no changed key are left untouched.  head_dim 64 or
 * 128.  ws: dllm_attention_update_workspace_size(B) bytes.
 */
size_t dllm_attention_update_workspace_size(int B);
dllm_status dllm_attention_update_bf16(const void* q, void* o, float* m, float* l,
                                       const int32_t* r_count, int B, int r_cap,
                                       const void* k_new, const void* v_new, const void* k_old,
                                       const void* v_old, const int32_t* a_count, int a_cap,
                                       int n_heads, int n_kv_heads, int head_dim, void* ws,
                                       size_t ws_bytes, dllm_stream_t stream);

/*
 * dllm_attention_bf16_noalloc - dllm_attention_bf16 without a workspace, for
 * callers that cannot allocate device memory: servers that split all device
 * memory into fixed pools before serving (nothing may allocate on the request
 * path, and cudaMalloc can synchronise the device), and plugins or operators
 * that are handed only the tensors they compute on.  The pages have no
 * counterpart; this is an integration convenience.
 * Same arguments and result as dllm_attention_bf16 minus ws/ws_bytes.  Its
 * scratch (a status word and B + 1 row offsets) is a fixed array in the
 * library's device memory, sized for at most DLLM_NOALLOC_MAX_SEQS sequences
 * (larger B returns DLLM_ERR_CAPACITY before anything is launched); every GPU
 * that loads the library holds it until the process exits.  The first call in
 * each device context (per device, and again after the context changes, e.g.
 * after cudaDeviceReset) looks up the array's device address with a runtime
 * call on the host (cudaGetSymbolAddress).  All calls share the array: calls that may overlap on
 * the GPU (other streams, other host threads on the same device) race and
 * must be ordered by the caller.  Device-side faults are recorded in the
 * shared status word, which this entry point clears at the start of each call
 * and does not report.  Like dllm_attention_bf16, it never splits one
 * sequence's keys among several CTAs (that needs a partial-output scratch far
 * larger than the fixed array); the attention inside dllm_step and
 * dllm_partial_layer does, so with few query tiles (one or two sequences of a
 * few hundred selected rows) it runs fewer CTAs than those and can be slower.
 */
#define DLLM_NOALLOC_MAX_SEQS 4096
dllm_status dllm_attention_bf16_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                        void* o, const int32_t* count, int B, int k_cap, int N,
                                        int n_heads, int n_kv_heads, int head_dim,
                                        dllm_stream_t stream);

/*
 * dllm_get_device_status - synchronises `stream`, copies the device status
 * word of a workspace used by dllm_select / dllm_partial_layer / dllm_step
 * into *status_out (HOST memory), and clears it.  Returns DLLM_ERR_DEVICE
 * when the word was non-zero.
 */
dllm_status dllm_get_device_status(void* ws, dllm_stream_t stream, int32_t* status_out);

/*
 * dllm_gemm_bf16 - the tensor-core GEMM the layer path runs on, exposed for
 * direct checks: C[M, N] = A[M, K] * B[N, K]^T (+ C when accumulate != 0),
 * bf16 in, fp32 accumulate, bf16 out.  K, N multiples of 8; a multiple of
 * 64 in K keeps every k-block full.  splits > 1 splits K across CTAs and
 * reduces in a fixed order (deterministic); needs ws of
 * dllm_gemm_workspace_size() bytes.
 */
size_t dllm_gemm_workspace_size(int M, int N, int K, int splits);
dllm_status dllm_gemm_bf16(const void* A, const void* Bm, void* C, int M, int N, int K,
                           int accumulate, int splits, void* ws, size_t ws_bytes,
                           dllm_stream_t stream);

/*
 * dllm_gemm_plan_info - the launch plan the library picks for one projection
 * GEMM, computed on the host (no GPU work; with no device visible the plan
 * assumes 148 SMs).  kind: 0 plain, 1 residual, 2 gate/up + SwiGLU (n_seg 2:
 * seg_cols = {F, F}), 3 QKV + RoPE (n_seg 3: {q, kv, kv} columns), 4 LM head
 * (n_seg 1, as plain otherwise).  M rows (capacity), K inner size, head_dim
 * for QKV.  out (HOST, 5 int32): column-tile width, K splits, column tiles,
 * CTAs launched, 1 when CTA pairs (256-row tiles, tcgen05 cta_group::2) run it.
 * DLLM_ERR_INVALID_ARG for an unknown kind, a segment count that does not
 * match it, or non-positive sizes.
 */
dllm_status dllm_gemm_plan_info(int kind, int M, int K, const int32_t* seg_cols, int n_seg,
                                int head_dim, int32_t* out);

/*
 * dllm_attention_plan_info - the launch plan of the exact partial attention
 * (host only; with no device visible 148 SMs are assumed).  B sequences of N
 * cached keys, at most k_cap selected query rows each, n_heads query heads of
 * head_dim (64 or 128); in_step != 0 for the plan inside a step (whose layer
 * workspace holds the key-split scratch), 0 for dllm_attention_bf16 alone.
 * out (HOST, 3 int32): query tiles of 128 rows per CTA (2: a pair sharing every
 * K/V tile, one CTA per SM; 1: two CTAs per SM, taken for an odd tile count of
 * 3 or more, when keys are split, and when one-tile CTAs fit one wave where
 * pairs would need two), key shares per CTA's rows (1: none), CTAs
 * launched.  DLLM_ERR_INVALID_ARG for non-positive sizes, another head_dim or
 * a null out.
 */
dllm_status dllm_attention_plan_info(int B, int k_cap, int N, int n_heads, int head_dim,
                                     int in_step, int32_t* out);

/*
 * dllm_selftest_gemm_stall - failure-path check of the CTA-pair GEMM (256-row
 * tiles, tcgen05 cta_group::2): the same launch as dllm_gemm_bf16 (M >= 256,
 * N a multiple of 256, accumulate 0, no K split) with one signal withheld:
 * the second CTA of every pair never reports its first k-block to the first,
 * so the first CTA's bounded wait runs out after its limit (2 s).  Every CTA
 * then drains its own loads and returns; the kernel ends with DLLM_DEV_TIMEOUT
 * in the workspace's device status word (read it with
 * dllm_get_device_status) and C undefined, and the CUDA context stays usable.
 * Returns DLLM_ERR_UNSUPPORTED_SHAPE for shapes that do not run on CTA pairs.  Arguments as for
 * dllm_gemm_bf16; ws of dllm_gemm_workspace_size(M, N, K, 1) bytes.
 */
dllm_status dllm_selftest_gemm_stall(const void* A, const void* Bm, void* C, int M, int N, int K,
                                     void* ws, size_t ws_bytes, dllm_stream_t stream);

/*
 * Kernel timing.  dllm_profile_enable(1) brackets every kernel the library
 * launches with CUDA events on the launch stream; dllm_profile_read()
 * synchronises the device, writes a JSON object
 * {"kernel": [launches, total_ms], ...} into buf (HOST, len bytes) and
 * returns the bytes needed; dllm_profile_reset() clears the counters.
 */
void dllm_profile_enable(int on);
void dllm_profile_reset(void);
size_t dllm_profile_read(char* buf, size_t len);

#ifdef __cplusplus
}
#endif
#endif /* DLLM_H */
