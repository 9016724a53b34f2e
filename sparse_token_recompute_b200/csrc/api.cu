// C ABI of the selected-token denoising step: argument validation, workspace
// layout, and the launch sequence of one layer / one step on the caller's
// stream.  No device memory is allocated here; scratch is carved out of the
// caller's workspace with 256-byte alignment.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/dllm.h"
#include "internal.h"

using namespace dllm;

namespace dllm {

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!cached[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

// ---------------------------------------------------------------- kernel timing

namespace {
struct ProfEntry {
  std::string name;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfEntry> g_prof_pending;
std::vector<cudaEvent_t> g_prof_free;
std::map<std::string, std::pair<long, double>> g_prof_acc;
thread_local int g_prof_open = -1;

cudaEvent_t prof_event() {
  if (!g_prof_free.empty()) {
    cudaEvent_t e = g_prof_free.back();
    g_prof_free.pop_back();
    return e;
  }
  cudaEvent_t e;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

void prof_begin(const char* name, cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on) {
    g_prof_open = -1;
    return;
  }
  ProfEntry e{name, prof_event(), prof_event()};
  cudaEventRecord(e.a, s);
  g_prof_pending.push_back(e);
  g_prof_open = (int)g_prof_pending.size() - 1;
}

void prof_end(cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (g_prof_open < 0 || g_prof_open >= (int)g_prof_pending.size()) return;
  cudaEventRecord(g_prof_pending[g_prof_open].b, s);
  g_prof_open = -1;
}

}  // namespace dllm

extern "C" void dllm_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
}

extern "C" void dllm_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  cudaDeviceSynchronize();
  for (auto& e : g_prof_pending) {
    g_prof_free.push_back(e.a);
    g_prof_free.push_back(e.b);
  }
  g_prof_pending.clear();
  g_prof_acc.clear();
}

extern "C" size_t dllm_profile_read(char* buf, size_t len) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  cudaDeviceSynchronize();
  for (auto& e : g_prof_pending) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, e.a, e.b) == cudaSuccess) {
      auto& acc = g_prof_acc[e.name];
      acc.first += 1;
      acc.second += ms;
    }
    g_prof_free.push_back(e.a);
    g_prof_free.push_back(e.b);
  }
  g_prof_pending.clear();
  std::string out = "{";
  bool first = true;
  for (auto& kv : g_prof_acc) {
    char tmp[256];
    snprintf(tmp, sizeof(tmp), "%s\"%s\": [%ld, %.6f]", first ? "" : ", ", kv.first.c_str(),
             kv.second.first, kv.second.second);
    out += tmp;
    first = false;
  }
  out += "}";
  if (buf && len) {
    const size_t n = std::min(len - 1, out.size());
    memcpy(buf, out.data(), n);
    buf[n] = 0;
  }
  return out.size() + 1;
}

// ---------------------------------------------------------------- helpers

namespace {

struct Bump {
  char* base;
  size_t off = 0;
  explicit Bump(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

constexpr size_t kHeader = 256;  // device status word lives at offset 0

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline dllm_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DLLM_OK : DLLM_ERR_CUDA; }

inline dllm_status check_launch() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DLLM_OK : DLLM_ERR_CUDA;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t esize(int dtype) { return dtype == DLLM_BF16 ? 2 : 4; }

dllm_status check_cfg(const dllm_model_cfg* c) {
  if (!c) return DLLM_ERR_INVALID_ARG;
  if (c->dtype != DLLM_F32 && c->dtype != DLLM_BF16) return DLLM_ERR_INVALID_ARG;
  if (c->n_layers < 0 || c->d <= 0 || c->n_heads <= 0 || c->n_kv_heads <= 0 ||
      c->head_dim <= 0 || c->ffn <= 0 || c->vocab <= 1)
    return DLLM_ERR_INVALID_ARG;
  if (c->n_heads % c->n_kv_heads) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (c->mask_id < 0 || c->mask_id >= c->vocab) return DLLM_ERR_INVALID_ARG;
  if (!(c->rms_eps >= 0.f) || !(c->rope_theta >= 0.f)) return DLLM_ERR_INVALID_ARG;
  if (c->d % 8 || c->vocab % 8) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (c->dtype == DLLM_BF16) {
    const int q = c->n_heads * c->head_dim, kv = c->n_kv_heads * c->head_dim;
    if (c->head_dim != 64 && c->head_dim != 128) return DLLM_ERR_UNSUPPORTED_SHAPE;
    if (c->d % 128 || q % 128 || kv % 128 || c->ffn % 128) return DLLM_ERR_UNSUPPORTED_SHAPE;
  } else {
    if (c->head_dim % 2 || c->head_dim > 256) return DLLM_ERR_UNSUPPORTED_SHAPE;
  }
  return DLLM_OK;
}

dllm_status check_layer_w(const dllm_layer_w* w) {
  if (!w || !w->attn_norm || !w->wq || !w->wk || !w->wv || !w->wo || !w->ffn_norm ||
      !w->w_gate || !w->w_up || !w->w_down)
    return DLLM_ERR_INVALID_ARG;
  const void* ps[9] = {w->attn_norm, w->wq, w->wk, w->wv, w->wo,
                       w->ffn_norm, w->w_gate, w->w_up, w->w_down};
  for (const void* p : ps)
    if (!aligned(p, 16)) return DLLM_ERR_INVALID_ARG;
  return DLLM_OK;
}

// Scratch of one layer pass over up to `cap` compact rows.
struct LayerWs {
  int* status;
  int* row_off;
  int* row_pos;
  int* row_seq;
  float2* rope;
  void* n;
  void* q;
  void* o;
  void* act;
  float* qraw;
  float* kraw;
  float* vraw;
  float* graw;
  float* uraw;
  float* part;  // partial outputs of the key-split attention
  size_t part_bytes;
};

// scratch of a layer pass over up to `cap` compact rows
void layout_layer(Bump& bp, const dllm_model_cfg* c, int B, int N, int cap, LayerWs& w) {
  const size_t es = esize(c->dtype);
  const int q = c->n_heads * c->head_dim, kv = c->n_kv_heads * c->head_dim;
  w.row_off = bp.take<int>(B + 1);
  w.row_pos = bp.take<int>(std::max(cap, 1));
  w.row_seq = bp.take<int>(std::max(cap, 1));
  w.rope = bp.take<float2>((size_t)N * (c->head_dim / 2));
  w.n = bp.take<char>((size_t)cap * c->d * es);
  w.q = bp.take<char>((size_t)cap * q * es);
  w.o = bp.take<char>((size_t)cap * q * es);
  w.act = bp.take<char>((size_t)cap * c->ffn * es);
  w.qraw = w.kraw = w.vraw = w.graw = w.uraw = nullptr;
  w.part = nullptr;
  w.part_bytes = 0;
  if (c->dtype == DLLM_BF16) {
    w.part_bytes = attention_part_bytes_bound(cap, c->n_heads, c->head_dim);
    w.part = bp.take<float>(w.part_bytes / sizeof(float));
  }
  if (c->dtype == DLLM_F32) {
    w.qraw = bp.take<float>((size_t)cap * q);
    w.kraw = bp.take<float>((size_t)cap * kv);
    w.vraw = bp.take<float>((size_t)cap * kv);
    w.graw = bp.take<float>((size_t)cap * c->ffn);
    w.uraw = bp.take<float>((size_t)cap * c->ffn);
  }
}

// One transformer layer over the compact rows in x (in place).
// DyLLM FFN gate of one layer (see launch_ffn_gate)
struct LayerGate {
  void* ctx;          // [B, N, n_heads*head_dim] attention outputs at each row's last pass
  void* ffn;          // [B, N, d] FFN outputs at each row's last salient pass
  float tau;          // salient when 1 - cos > tau
  int all_rows;       // every row salient (dense steps)
  const uint8_t* forced;  // [cap] decisions replacing the rule, or null
  int* flag;          // [cap] scratch
  int* list;          // [cap] salient rows
  int* inv;           // [cap] row -> place in the list, or -1
  int* n_sal;         // [1] salient rows
  void* f_new;        // [cap, d] FFN outputs of the salient rows
  int32_t* rows_out;  // this layer's salient-row count (device), or null
};

// DyLLM approximate attention of one layer (dllm_policy.attn_update): caches of the
// rows' queries and softmax statistics, and the scratch of the stable-row update
struct LayerUpd {
  void* q_cache;   // [B, N, q] query of each row's last exact pass
  float* m_cache;  // [B, N, Hq] softmax statistics (natural log units)
  float* l_cache;
  bool partial;    // partial step: stable rows take in the changed keys
  float* m_c;      // [cap, Hq] exact statistics of the recomputed rows
  float* l_c;
  void* k_old;     // [cap, kv] the recomputed rows' K/V before and after the layer
  void* v_old;
  void* k_new;
  void* v_new;
  uint8_t* skip;   // [B, N] 1 at the recomputed rows
  int* seq_off;    // [B + 1] b * N
};

dllm_status layer_forward(const dllm_model_cfg* c, const dllm_layer_w* lw, void* x, int M_cap,
                          const int* M_dev, const LayerWs& w, int B, int N, int k_cap,
                          void* k_cache, void* v_cache, bool use_rope, cudaStream_t s,
                          const LayerGate* gate = nullptr, const LayerUpd* upd = nullptr) {
  const int d = c->d, q = c->n_heads * c->head_dim, kv = c->n_kv_heads * c->head_dim;
  const int F = c->ffn, hd = c->head_dim;
  const float2* rope = use_rope ? w.rope : nullptr;
  if (M_cap <= 0) return DLLM_OK;
  if (c->dtype == DLLM_BF16) {
    using bf = __nv_bfloat16;
    bf* xb = static_cast<bf*>(x);
    bf* nb = static_cast<bf*>(w.n);
    if (upd && upd->partial) {  // the recomputed rows' K/V before this layer rewrites them
      launch_row_words(k_cache, upd->k_old, w.row_pos, w.row_seq, M_dev, M_cap, N, kv * 2, false,
                       s);
      launch_row_words(v_cache, upd->v_old, w.row_pos, w.row_seq, M_dev, M_cap, N, kv * 2, false,
                       s);
    }
    launch_rmsnorm<bf>(xb, static_cast<const bf*>(lw->attn_norm), nb, M_dev, M_cap, d,
                       c->rms_eps, s);
    GemmSpec g{};
    g.A = nb;
    g.M_cap = M_cap;
    g.M_dev = M_dev;
    g.K = d;
    g.status = w.status;
    g.epi = EPI_QKV;
    g.B[0] = static_cast<const bf*>(lw->wq);
    g.B[1] = static_cast<const bf*>(lw->wk);
    g.B[2] = static_cast<const bf*>(lw->wv);
    g.seg_cols[0] = q;
    g.seg_cols[1] = kv;
    g.seg_cols[2] = kv;
    g.n_seg = 3;
    g.out = static_cast<bf*>(w.q);
    g.ldo = q;
    g.kc = static_cast<bf*>(k_cache);
    g.vc = static_cast<bf*>(v_cache);
    g.row_pos = w.row_pos;
    g.row_seq = w.row_seq;
    g.Nseq = N;
    g.hd = hd;
    g.rope = rope;
    if (gemm_launch(g, s) != cudaSuccess) return DLLM_ERR_CUDA;
    if (launch_attention_tc(static_cast<const bf*>(w.q), M_cap,
                                   static_cast<const bf*>(k_cache),
                                   static_cast<const bf*>(v_cache), static_cast<bf*>(w.o),
                                   w.row_off, B, k_cap, N, c->n_heads, c->n_kv_heads, hd,
                                   w.status, s, upd ? upd->m_c : nullptr,
                                   upd ? upd->l_c : nullptr, w.part,
                                   w.part_bytes) != cudaSuccess) {
      return DLLM_ERR_CUDA;
    }
    if (upd) {
      // DyLLM 2.B: the recomputed rows' query and exact statistics are cached; in a
      // partial step every other row of a sequence with changed keys takes in only
      // those keys (old terms out, new terms in) and its context is updated in place
      const int Hq = c->n_heads;
      launch_row_words(upd->q_cache, w.q, w.row_pos, w.row_seq, M_dev, M_cap, N, q * 2, true, s);
      launch_row_words(upd->m_cache, upd->m_c, w.row_pos, w.row_seq, M_dev, M_cap, N, Hq * 4,
                       true, s);
      launch_row_words(upd->l_cache, upd->l_c, w.row_pos, w.row_seq, M_dev, M_cap, N, Hq * 4,
                       true, s);
      if (upd->partial) {
        launch_row_words(k_cache, upd->k_new, w.row_pos, w.row_seq, M_dev, M_cap, N, kv * 2,
                         false, s);
        launch_row_words(v_cache, upd->v_new, w.row_pos, w.row_seq, M_dev, M_cap, N, kv * 2,
                         false, s);
        launch_mark_rows(w.row_pos, w.row_seq, M_dev, M_cap, B, N, upd->skip, s);
        launch_seq_offsets(B, N, upd->seq_off, s);
        if (launch_attention_update(static_cast<const bf*>(upd->q_cache), B * N,
                                    static_cast<bf*>(gate->ctx), upd->m_cache, upd->l_cache,
                                    upd->seq_off, N, static_cast<const bf*>(upd->k_new),
                                    static_cast<const bf*>(upd->v_new),
                                    static_cast<const bf*>(upd->k_old),
                                    static_cast<const bf*>(upd->v_old), w.row_off, M_cap, B, Hq,
                                    c->n_kv_heads, hd, w.status, s, upd->skip) != cudaSuccess)
          return DLLM_ERR_CUDA;
      }
    }
    GemmSpec go = g;
    go.epi = EPI_RESID;
    go.A = static_cast<const bf*>(w.o);
    go.K = q;
    go.B[0] = static_cast<const bf*>(lw->wo);
    go.seg_cols[0] = d;
    go.n_seg = 1;
    go.out = xb;
    go.ldo = d;
    if (gemm_launch(go, s) != cudaSuccess) return DLLM_ERR_CUDA;
    if (gate) {
      // DyLLM: the FFN only on rows whose attention output moved, the rest reuse it
      launch_ffn_gate<bf>(static_cast<const bf*>(w.o), static_cast<bf*>(gate->ctx), w.row_pos,
                          w.row_seq, M_dev, M_cap, N, q, gate->tau, gate->all_rows,
                          gate->forced, gate->flag, gate->list, gate->inv, gate->n_sal, s);
      launch_rmsnorm_rows<bf>(xb, static_cast<const bf*>(lw->ffn_norm), nb, gate->list,
                              gate->n_sal, M_cap, d, c->rms_eps, s);
      GemmSpec gu = g;
      gu.epi = EPI_SWIGLU;
      gu.A = nb;
      gu.M_dev = gate->n_sal;
      gu.K = d;
      gu.B[0] = static_cast<const bf*>(lw->w_gate);
      gu.B[1] = static_cast<const bf*>(lw->w_up);
      gu.seg_cols[0] = F;
      gu.seg_cols[1] = F;
      gu.n_seg = 2;
      gu.out = static_cast<bf*>(w.act);
      gu.ldo = F;
      if (gemm_launch(gu, s) != cudaSuccess) return DLLM_ERR_CUDA;
      GemmSpec gd = gu;
      gd.epi = EPI_STORE;
      gd.A = static_cast<const bf*>(w.act);
      gd.K = F;
      gd.B[0] = static_cast<const bf*>(lw->w_down);
      gd.seg_cols[0] = d;
      gd.n_seg = 1;
      gd.out = static_cast<bf*>(gate->f_new);
      gd.ldo = d;
      if (gemm_launch(gd, s) != cudaSuccess) return DLLM_ERR_CUDA;
      launch_ffn_combine<bf>(xb, static_cast<const bf*>(gate->f_new), static_cast<bf*>(gate->ffn),
                             gate->inv, w.row_pos, w.row_seq, M_dev, M_cap, N, d, s);
      if (gate->rows_out && cudaMemcpyAsync(gate->rows_out, gate->n_sal, sizeof(int32_t),
                                            cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return DLLM_ERR_CUDA;
      return check_launch();
    }
    launch_rmsnorm<bf>(xb, static_cast<const bf*>(lw->ffn_norm), nb, M_dev, M_cap, d, c->rms_eps,
                       s);
    GemmSpec gu = g;
    gu.epi = EPI_SWIGLU;
    gu.A = nb;
    gu.K = d;
    gu.B[0] = static_cast<const bf*>(lw->w_gate);
    gu.B[1] = static_cast<const bf*>(lw->w_up);
    gu.seg_cols[0] = F;
    gu.seg_cols[1] = F;
    gu.n_seg = 2;
    gu.out = static_cast<bf*>(w.act);
    gu.ldo = F;
    if (gemm_launch(gu, s) != cudaSuccess) return DLLM_ERR_CUDA;
    GemmSpec gd = g;
    gd.epi = EPI_RESID;
    gd.A = static_cast<const bf*>(w.act);
    gd.K = F;
    gd.B[0] = static_cast<const bf*>(lw->w_down);
    gd.seg_cols[0] = d;
    gd.n_seg = 1;
    gd.out = xb;
    gd.ldo = d;
    if (gemm_launch(gd, s) != cudaSuccess) return DLLM_ERR_CUDA;
  } else {
    float* xf = static_cast<float*>(x);
    float* nf = static_cast<float*>(w.n);
    launch_rmsnorm<float>(xf, static_cast<const float*>(lw->attn_norm), nf, M_dev, M_cap, d,
                          c->rms_eps, s);
    launch_gemm_f32(nf, static_cast<const float*>(lw->wq), w.qraw, nullptr, M_dev, M_cap, q, d, s);
    launch_gemm_f32(nf, static_cast<const float*>(lw->wk), w.kraw, nullptr, M_dev, M_cap, kv, d,
                    s);
    launch_gemm_f32(nf, static_cast<const float*>(lw->wv), w.vraw, nullptr, M_dev, M_cap, kv, d,
                    s);
    launch_qkv_post_f32(w.qraw, w.kraw, w.vraw, static_cast<float*>(w.q),
                        static_cast<float*>(k_cache), static_cast<float*>(v_cache), w.row_pos,
                        w.row_seq, M_dev, M_cap, N, c->n_heads, c->n_kv_heads, hd, rope, s);
    launch_attention_f32(static_cast<const float*>(w.q), static_cast<const float*>(k_cache),
                         static_cast<const float*>(v_cache), static_cast<float*>(w.o), w.row_seq,
                         M_dev, M_cap, N, c->n_heads, c->n_kv_heads, hd, s);
    launch_gemm_f32(static_cast<const float*>(w.o), static_cast<const float*>(lw->wo), xf, xf,
                    M_dev, M_cap, d, q, s);
    if (gate) {
      launch_ffn_gate<float>(static_cast<const float*>(w.o), static_cast<float*>(gate->ctx),
                             w.row_pos, w.row_seq, M_dev, M_cap, N, q, gate->tau, gate->all_rows,
                             gate->forced, gate->flag, gate->list, gate->inv, gate->n_sal, s);
      launch_rmsnorm_rows<float>(xf, static_cast<const float*>(lw->ffn_norm), nf, gate->list,
                                 gate->n_sal, M_cap, d, c->rms_eps, s);
      launch_gemm_f32(nf, static_cast<const float*>(lw->w_gate), w.graw, nullptr, gate->n_sal,
                      M_cap, F, d, s);
      launch_gemm_f32(nf, static_cast<const float*>(lw->w_up), w.uraw, nullptr, gate->n_sal,
                      M_cap, F, d, s);
      launch_swiglu_f32(w.graw, w.uraw, static_cast<float*>(w.act), gate->n_sal, M_cap, F, s);
      launch_gemm_f32(static_cast<const float*>(w.act), static_cast<const float*>(lw->w_down),
                      static_cast<float*>(gate->f_new), nullptr, gate->n_sal, M_cap, d, F, s);
      launch_ffn_combine<float>(xf, static_cast<const float*>(gate->f_new),
                                static_cast<float*>(gate->ffn), gate->inv, w.row_pos, w.row_seq,
                                M_dev, M_cap, N, d, s);
      if (gate->rows_out && cudaMemcpyAsync(gate->rows_out, gate->n_sal, sizeof(int32_t),
                                            cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return DLLM_ERR_CUDA;
      return check_launch();
    }
    launch_rmsnorm<float>(xf, static_cast<const float*>(lw->ffn_norm), nf, M_dev, M_cap, d,
                          c->rms_eps, s);
    launch_gemm_f32(nf, static_cast<const float*>(lw->w_gate), w.graw, nullptr, M_dev, M_cap, F,
                    d, s);
    launch_gemm_f32(nf, static_cast<const float*>(lw->w_up), w.uraw, nullptr, M_dev, M_cap, F, d,
                    s);
    launch_swiglu_f32(w.graw, w.uraw, static_cast<float*>(w.act), M_dev, M_cap, F, s);
    launch_gemm_f32(static_cast<const float*>(w.act), static_cast<const float*>(lw->w_down), xf,
                    xf, M_dev, M_cap, d, F, s);
  }
  return check_launch();
}

}  // namespace

// ---------------------------------------------------------------- simple entry points

extern "C" const char* dllm_status_string(int st) {
  switch (st) {
    case DLLM_OK: return "ok";
    case DLLM_ERR_INVALID_ARG: return "invalid argument";
    case DLLM_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case DLLM_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case DLLM_ERR_CUDA: return "CUDA runtime error";
    case DLLM_ERR_CAPACITY: return "index capacity exceeded";
    case DLLM_ERR_DEVICE: return "device reported a fault (see the device status word)";
  }
  return "unknown status";
}

extern "C" int dllm_version(void) { return 100; }

extern "C" dllm_status dllm_score(const void* h_cur, const void* h_ref, int B, int N, int d,
                                  int dtype, const void* logits, const int32_t* logit_pos, int Mm,
                                  int V, float* conf, int32_t* pred, const uint8_t* masked,
                                  float alpha, int kind, float* scores, dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (B < 0 || N < 0 || d <= 0) return DLLM_ERR_INVALID_ARG;
  if (dtype != DLLM_F32 && dtype != DLLM_BF16) return DLLM_ERR_INVALID_ARG;
  if (kind != DLLM_SCORE_COS && kind != DLLM_SCORE_ES_L1) return DLLM_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return DLLM_OK;
  if (!h_cur || !h_ref || !conf || !masked || !scores) return DLLM_ERR_INVALID_ARG;
  if (d % 8) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(h_cur, 16) || !aligned(h_ref, 16)) return DLLM_ERR_INVALID_ARG;
  if (logits) {
    if (!logit_pos || Mm < 0 || V <= 0) return DLLM_ERR_INVALID_ARG;
    if (V % 8) return DLLM_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(logits, 16)) return DLLM_ERR_INVALID_ARG;
    if (dtype == DLLM_BF16)
      launch_confidence<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(logits), logit_pos, B, Mm,
                                       V, N, conf, pred, s);
    else
      launch_confidence<float>(static_cast<const float*>(logits), logit_pos, B, Mm, V, N, conf,
                               pred, s);
  }
  if (dtype == DLLM_BF16)
    launch_score<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(h_cur), nullptr, nullptr,
                                static_cast<const __nv_bfloat16*>(h_ref), B, N, d, conf, masked,
                                nullptr, -1, alpha, kind, scores, 0, 0, nullptr, s);
  else
    launch_score<float>(static_cast<const float*>(h_cur), nullptr, nullptr,
                        static_cast<const float*>(h_ref), B, N, d, conf, masked, nullptr, -1,
                        alpha, kind, scores, 0, 0, nullptr, s);
  return check_launch();
}

extern "C" size_t dllm_select_workspace_size(int, int) { return kHeader; }

extern "C" dllm_status dllm_select_range(const float* scores, int B, int N, int lo, int mode,
                                         int k, float tau, int32_t* idx, int32_t* count,
                                         int k_cap, void* ws, size_t ws_bytes,
                                         dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (B < 0 || N < 0 || k < 0 || k_cap < 1 || lo < 0 || lo > N) return DLLM_ERR_INVALID_ARG;
  if (mode != DLLM_SELECT_TOPK && mode != DLLM_SELECT_THRESH) return DLLM_ERR_INVALID_ARG;
  if (mode == DLLM_SELECT_TOPK && std::min(k, N - lo) > k_cap) return DLLM_ERR_CAPACITY;
  if (N > 16384) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return DLLM_OK;
  if (!scores || !idx || !count) return DLLM_ERR_INVALID_ARG;
  if (ws && ws_bytes < kHeader) return DLLM_ERR_WORKSPACE;
  if (ws && !aligned(ws, 256)) return DLLM_ERR_WORKSPACE;
  launch_select(scores, B, N, lo, mode, k, tau, idx, count, k_cap, static_cast<int*>(ws), s);
  return check_launch();
}

extern "C" dllm_status dllm_select(const float* scores, int B, int N, int mode, int k, float tau,
                                   int32_t* idx, int32_t* count, int k_cap, void* ws,
                                   size_t ws_bytes, dllm_stream_t stream) {
  return dllm_select_range(scores, B, N, 0, mode, k, tau, idx, count, k_cap, ws, ws_bytes,
                           stream);
}

extern "C" int dllm_unmask_capacity(const dllm_policy* pol) {
  if (!pol) return 0;
  const int n = std::max(pol->n_unmask, 0);
  return pol->unmask_tau > 0.f ? std::max(n, pol->block_len) : n;
}

extern "C" dllm_status dllm_unmask_tau(const float* conf, const int32_t* pred, int32_t* tokens,
                                       int B, int N, int mask_id, int gen_start, int block_len,
                                       int n_unmask, float tau, int32_t* pos_out, int pos_cap,
                                       dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (B < 0 || N < 0 || n_unmask < 0 || gen_start < 0 || block_len < 1 || pos_cap < n_unmask)
    return DLLM_ERR_INVALID_ARG;
  if (!(tau == tau) || tau == INFINITY) return DLLM_ERR_INVALID_ARG;  // NaN / +inf
  if (block_len > 1024 || N > 16384) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || N == 0) return DLLM_OK;
  if (!conf || !pred || !tokens) return DLLM_ERR_INVALID_ARG;
  if (gen_start > N) return DLLM_ERR_INVALID_ARG;
  launch_unmask(conf, pred, tokens, B, N, mask_id, gen_start, block_len, n_unmask, tau, pos_cap,
                pos_out, nullptr, s);
  return check_launch();
}

extern "C" dllm_status dllm_unmask(const float* conf, const int32_t* pred, int32_t* tokens, int B,
                                   int N, int mask_id, int gen_start, int block_len, int n_unmask,
                                   int32_t* pos_out, dllm_stream_t stream) {
  return dllm_unmask_tau(conf, pred, tokens, B, N, mask_id, gen_start, block_len, n_unmask, 0.f,
                         pos_out, std::max(n_unmask, 0), stream);
}

extern "C" dllm_status dllm_get_device_status(void* ws, dllm_stream_t stream, int32_t* out) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!ws || !out) return DLLM_ERR_INVALID_ARG;
  int32_t v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DLLM_ERR_CUDA;
  if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return DLLM_ERR_CUDA;
  const int32_t zero = 0;
  if (cudaMemcpy(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
    return DLLM_ERR_CUDA;
  *out = v;
  return v ? DLLM_ERR_DEVICE : DLLM_OK;
}

// ---------------------------------------------------------------- GEMM entry point

extern "C" size_t dllm_gemm_workspace_size(int M, int N, int K, int splits) {
  if (M <= 0 || N <= 0 || K <= 0) return kHeader;
  GemmSpec g{};
  g.epi = EPI_STORE;
  g.M_cap = M;
  g.K = K;
  g.n_seg = 1;
  g.seg_cols[0] = N;
  g.force_splits = splits;
  GemmPlan p = gemm_plan(g);
  Bump bp(nullptr);
  bp.take<char>(kHeader);
  return bp.off;
}

extern "C" dllm_status dllm_gemm_bf16(const void* A, const void* Bm, void* C, int M, int N, int K,
                                      int accumulate, int splits, void* ws, size_t ws_bytes,
                                      dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (M < 0 || N <= 0 || K <= 0 || splits < 0) return DLLM_ERR_INVALID_ARG;
  if (M == 0) return DLLM_OK;
  if (!A || !Bm || !C) return DLLM_ERR_INVALID_ARG;
  if (N % 8 || K % 8) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(A, 16) || !aligned(Bm, 16) || !aligned(C, 16)) return DLLM_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < dllm_gemm_workspace_size(M, N, K, splits))
    return DLLM_ERR_WORKSPACE;
  GemmSpec g{};
  g.epi = accumulate ? EPI_RESID : EPI_STORE;
  g.A = static_cast<const __nv_bfloat16*>(A);
  g.M_cap = M;
  g.K = K;
  g.B[0] = static_cast<const __nv_bfloat16*>(Bm);
  g.seg_cols[0] = N;
  g.n_seg = 1;
  g.out = static_cast<__nv_bfloat16*>(C);
  g.ldo = N;
  g.force_splits = splits;
  GemmPlan p = gemm_plan(g);
  Bump bp(ws);
  g.status = bp.take<int>(kHeader / sizeof(int));
  return cuda_status(gemm_launch(g, s));
}

extern "C" dllm_status dllm_gemm_plan_info(int kind, int M, int K, const int32_t* seg_cols,
                                           int n_seg, int head_dim, int32_t* out) {
  if (kind < EPI_STORE || kind > EPI_LMHEAD || M <= 0 || K <= 0 || !seg_cols || !out ||
      n_seg < 1 || n_seg > 3)
    return DLLM_ERR_INVALID_ARG;
  if ((kind == EPI_QKV) != (n_seg == 3) || (kind == EPI_SWIGLU) != (n_seg == 2))
    return DLLM_ERR_INVALID_ARG;
  GemmSpec g{};
  g.epi = kind;
  g.M_cap = M;
  g.K = K;
  g.n_seg = n_seg;
  for (int i = 0; i < n_seg; ++i) {
    if (seg_cols[i] <= 0) return DLLM_ERR_INVALID_ARG;
    g.seg_cols[i] = seg_cols[i];
  }
  g.hd = head_dim;
  const GemmPlan pl = gemm_plan(g);
  out[0] = pl.bn;
  out[1] = pl.splits;
  out[2] = pl.tiles_n;
  out[3] = pl.grid;
  out[4] = pl.pair;
  return DLLM_OK;
}

extern "C" dllm_status dllm_attention_plan_info(int B, int k_cap, int N, int n_heads,
                                                int head_dim, int in_step, int32_t* out) {
  if (B <= 0 || k_cap <= 0 || N <= 0 || n_heads <= 0 || !out ||
      (head_dim != 64 && head_dim != 128))
    return DLLM_ERR_INVALID_ARG;
  // in a step the layer workspace carries the key-split scratch; the attention
  // entry points alone have none
  const size_t part = in_step ? attention_part_bytes_bound(B * N, n_heads, head_dim) : 0;
  const AttnPlan pl = attention_plan(B, k_cap, N, n_heads, head_dim, B * k_cap, part);
  out[0] = pl.nt;
  out[1] = pl.shares;
  out[2] = pl.ctas;
  return DLLM_OK;
}

extern "C" dllm_status dllm_selftest_gemm_stall(const void* A, const void* Bm, void* C, int M,
                                                int N, int K, void* ws, size_t ws_bytes,
                                                dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (M < 256 || N < 256 || N % 256 || K <= 0 || K % 8) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (!A || !Bm || !C) return DLLM_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(Bm, 16) || !aligned(C, 16)) return DLLM_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < dllm_gemm_workspace_size(M, N, K, 1))
    return DLLM_ERR_WORKSPACE;
  GemmSpec g{};
  g.epi = EPI_STORE;
  g.A = static_cast<const __nv_bfloat16*>(A);
  g.M_cap = M;
  g.K = K;
  g.B[0] = static_cast<const __nv_bfloat16*>(Bm);
  g.seg_cols[0] = N;
  g.n_seg = 1;
  g.out = static_cast<__nv_bfloat16*>(C);
  g.ldo = N;
  g.force_bn = 256;
  g.force_splits = 1;
  g.stall_test = 1;
  if (!gemm_plan(g).pair) return DLLM_ERR_UNSUPPORTED_SHAPE;
  Bump bp(ws);
  g.status = bp.take<int>(kHeader / sizeof(int));
  return cuda_status(gemm_launch(g, s));
}

// ---------------------------------------------------------------- attention alone

extern "C" size_t dllm_attention_workspace_size(int B) {
  Bump bp(nullptr);
  bp.take<char>(kHeader);
  bp.take<int>((size_t)std::max(B, 0) + 1);
  return bp.off;
}

extern "C" dllm_status dllm_attention_bf16(const void* q, const void* k_cache,
                                           const void* v_cache, void* o, const int32_t* count,
                                           int B, int k_cap, int N, int n_heads, int n_kv_heads,
                                           int head_dim, void* ws, size_t ws_bytes,
                                           dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (B < 0 || k_cap < 1 || N < 0 || n_heads <= 0 || n_kv_heads <= 0) return DLLM_ERR_INVALID_ARG;
  if (n_heads % n_kv_heads) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (head_dim != 64 && head_dim != 128) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || N == 0) return DLLM_OK;
  if (!q || !k_cache || !v_cache || !o || !count) return DLLM_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16))
    return DLLM_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < dllm_attention_workspace_size(B))
    return DLLM_ERR_WORKSPACE;
  Bump bp(ws);
  int* status = bp.take<int>(kHeader / sizeof(int));
  int* row_off = bp.take<int>((size_t)B + 1);
  launch_row_map(nullptr, count, B, k_cap, N, row_off, nullptr, nullptr, status, s);
  const cudaError_t e = launch_attention_tc(
      static_cast<const __nv_bfloat16*>(q), B * k_cap, static_cast<const __nv_bfloat16*>(k_cache),
      static_cast<const __nv_bfloat16*>(v_cache), static_cast<__nv_bfloat16*>(o), row_off, B,
      k_cap, N, n_heads, n_kv_heads, head_dim, status, s);
  return e == cudaSuccess ? check_launch() : DLLM_ERR_CUDA;
}

extern "C" dllm_status dllm_attention_stats_bf16(const void* q, const void* k_cache,
                                                 const void* v_cache, void* o, float* m, float* l,
                                                 const int32_t* count, int B, int k_cap, int N,
                                                 int n_heads, int n_kv_heads, int head_dim,
                                                 void* ws, size_t ws_bytes, dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (B < 0 || k_cap < 1 || N < 0 || n_heads <= 0 || n_kv_heads <= 0) return DLLM_ERR_INVALID_ARG;
  if (n_heads % n_kv_heads) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (head_dim != 64 && head_dim != 128) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || N == 0) return DLLM_OK;
  if (!q || !k_cache || !v_cache || !o || !count || !m || !l) return DLLM_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16))
    return DLLM_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < dllm_attention_workspace_size(B))
    return DLLM_ERR_WORKSPACE;
  Bump bp(ws);
  int* status = bp.take<int>(kHeader / sizeof(int));
  int* row_off = bp.take<int>((size_t)B + 1);
  launch_row_map(nullptr, count, B, k_cap, N, row_off, nullptr, nullptr, status, s);
  const cudaError_t e = launch_attention_tc(
      static_cast<const __nv_bfloat16*>(q), B * k_cap, static_cast<const __nv_bfloat16*>(k_cache),
      static_cast<const __nv_bfloat16*>(v_cache), static_cast<__nv_bfloat16*>(o), row_off, B,
      k_cap, N, n_heads, n_kv_heads, head_dim, status, s, m, l);
  return e == cudaSuccess ? check_launch() : DLLM_ERR_CUDA;
}

extern "C" size_t dllm_attention_update_workspace_size(int B) {
  Bump bp(nullptr);
  bp.take<char>(kHeader);
  bp.take<int>((size_t)std::max(B, 0) + 1);
  bp.take<int>((size_t)std::max(B, 0) + 1);
  return bp.off;
}

extern "C" dllm_status dllm_attention_update_bf16(const void* q, void* o, float* m, float* l,
                                                  const int32_t* r_count, int B, int r_cap,
                                                  const void* k_new, const void* v_new,
                                                  const void* k_old, const void* v_old,
                                                  const int32_t* a_count, int a_cap, int n_heads,
                                                  int n_kv_heads, int head_dim, void* ws,
                                                  size_t ws_bytes, dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (B < 0 || r_cap < 1 || a_cap < 1 || n_heads <= 0 || n_kv_heads <= 0)
    return DLLM_ERR_INVALID_ARG;
  if (n_heads % n_kv_heads) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (head_dim != 64 && head_dim != 128) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return DLLM_OK;
  if (!q || !o || !m || !l || !r_count || !k_new || !v_new || !k_old || !v_old || !a_count)
    return DLLM_ERR_INVALID_ARG;
  for (const void* ptr : {q, static_cast<const void*>(o), k_new, v_new, k_old, v_old})
    if (!aligned(ptr, 16)) return DLLM_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < dllm_attention_update_workspace_size(B))
    return DLLM_ERR_WORKSPACE;
  Bump bp(ws);
  int* status = bp.take<int>(kHeader / sizeof(int));
  int* r_off = bp.take<int>((size_t)B + 1);
  int* a_off = bp.take<int>((size_t)B + 1);
  launch_row_map(nullptr, r_count, B, r_cap, r_cap, r_off, nullptr, nullptr, status, s);
  launch_row_map(nullptr, a_count, B, a_cap, a_cap, a_off, nullptr, nullptr, status, s);
  const cudaError_t e = launch_attention_update(
      static_cast<const __nv_bfloat16*>(q), B * r_cap, static_cast<__nv_bfloat16*>(o), m, l,
      r_off, r_cap, static_cast<const __nv_bfloat16*>(k_new),
      static_cast<const __nv_bfloat16*>(v_new), static_cast<const __nv_bfloat16*>(k_old),
      static_cast<const __nv_bfloat16*>(v_old), a_off, B * a_cap, B, n_heads, n_kv_heads,
      head_dim, status, s);
  return e == cudaSuccess ? check_launch() : DLLM_ERR_CUDA;
}

// ---------------------------------------------------------------- partial layer

extern "C" size_t dllm_partial_layer_workspace_size(const dllm_model_cfg* c, int B, int N,
                                                    int k_cap) {
  if (check_cfg(c) != DLLM_OK || B < 0 || N < 0 || k_cap < 0) return 0;
  Bump bp(nullptr);
  bp.take<char>(kHeader);
  LayerWs w{};
  layout_layer(bp, c, B, N, B * k_cap, w);
  return bp.off;
}

extern "C" dllm_status dllm_partial_layer(const dllm_model_cfg* c, const dllm_layer_w* lw,
                                          const void* x_in, int x_in_is_full, void* x_out,
                                          const int32_t* idx, const int32_t* count, int k_cap,
                                          int B, int N, void* k_cache, void* v_cache, void* ws,
                                          size_t ws_bytes, dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  dllm_status st = check_cfg(c);
  if (st != DLLM_OK) return st;
  if ((st = check_layer_w(lw)) != DLLM_OK) return st;
  if (B < 0 || N < 0 || k_cap < 1) return DLLM_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return DLLM_OK;
  if (!x_in || !x_out || !idx || !count || !k_cache || !v_cache) return DLLM_ERR_INVALID_ARG;
  if (!aligned(x_in, 16) || !aligned(x_out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
    return DLLM_ERR_INVALID_ARG;
  if (c->dtype == DLLM_F32 && N > 16384) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if (!ws || !aligned(ws, 256) || ws_bytes < dllm_partial_layer_workspace_size(c, B, N, k_cap))
    return DLLM_ERR_WORKSPACE;
  const int cap = B * k_cap;
  Bump bp(ws);
  LayerWs w{};
  w.status = bp.take<int>(kHeader / sizeof(int));
  layout_layer(bp, c, B, N, cap, w);
  launch_row_map(idx, count, B, k_cap, N, w.row_off, w.row_pos, w.row_seq, w.status, s);
  const bool use_rope = c->rope_theta > 0.f;
  if (use_rope) launch_rope_table(w.rope, N, c->head_dim, c->rope_theta, s);
  const int* M_dev = w.row_off + B;
  if (x_in_is_full) {
    if (c->dtype == DLLM_BF16)
      launch_gather_rows<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x_in), nullptr, nullptr,
                                        w.row_pos, w.row_seq, M_dev, cap, N, c->d,
                                        static_cast<__nv_bfloat16*>(x_out), nullptr, 0,
                                        w.status, s);
    else
      launch_gather_rows<float>(static_cast<const float*>(x_in), nullptr, nullptr, w.row_pos,
                                w.row_seq, M_dev, cap, N, c->d, static_cast<float*>(x_out),
                                nullptr, 0, w.status, s);
  } else if (x_in != x_out) {
    if (cudaMemcpyAsync(x_out, x_in, (size_t)cap * c->d * esize(c->dtype),
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return DLLM_ERR_CUDA;
  }
  return layer_forward(c, lw, x_out, cap, M_dev, w, B, N, k_cap, k_cache, v_cache, use_rope, s);
}

// ---------------------------------------------------------------- step

namespace {

struct StepWs {
  int* status;
  LayerWs L;
  void* x;       // compact hidden [cap, d]
  void* h_full;  // [B, N, d] hidden at the score layer (score_layer > 0)
  float* scores;
  int32_t* idx;
  int32_t* count;
  int* lm_rows;
  int* n_lm;
  void* lmx;      // normalized LM rows [cap, d]
  float* lm_out;  // bf16: per-tile stats [cap, tiles, 3]; f32: logits [cap, V]
  int lm_tiles;
  // second skip point (k2_cap > 0)
  int k2_cap;
  float* scores2;   // [B, k_cap]
  int32_t* idx2;    // [B, k2_cap] indices within each sequence's segment
  int32_t* count2;  // [B]
  int32_t* pos2;    // [B, k2_cap] positions
  int* row_off2;    // [B + 1]
  int* row_pos2;    // [B * k2_cap]
  int* row_seq2;    // [B * k2_cap]
  void* x2;         // [B * k2_cap, d]
  // DyLLM FFN gate (policy.ffn_gate)
  int* g_flag;      // [cap]
  int* g_list;      // [cap]
  int* g_inv;       // [cap]
  int* g_n;         // [1]
  void* g_f;        // [cap, d]
  // DyLLM approximate attention (policy.attn_update)
  float* u_m;       // [cap, Hq]
  float* u_l;
  void* u_kold;     // [cap, kv] x 4
  void* u_vold;
  void* u_knew;
  void* u_vnew;
  uint8_t* u_skip;  // [B * N]
  int* u_off;       // [B + 1]
};

int k2_cap_of(const dllm_policy* pol, int N) {
  const int k_cap = std::max(1, std::min(pol->k, N));
  return pol->score_layer2 > 0 ? std::max(1, std::min(pol->k2, k_cap)) : 0;
}

// the LM-head GEMM uses column tiles of 128 or 256: size its statistics for 128
int lm_tiles_for(const dllm_model_cfg* c) { return (c->vocab + 127) / 128; }

void layout_step(Bump& bp, const dllm_model_cfg* c, int B, int N, int k_cap, int k2_cap,
                 bool gate, bool upd, StepWs& w) {
  const size_t es = esize(c->dtype);
  const int cap = B * N;  // covers the dense step
  w.status = bp.take<int>(kHeader / sizeof(int));
  layout_layer(bp, c, B, N, cap, w.L);
  w.L.status = w.status;
  w.x = bp.take<char>((size_t)cap * c->d * es);
  w.h_full = bp.take<char>((size_t)cap * c->d * es);
  w.scores = bp.take<float>((size_t)B * N);
  w.idx = bp.take<int32_t>((size_t)B * std::max(k_cap, 1));
  w.count = bp.take<int32_t>(B);
  w.lm_rows = bp.take<int>(cap);
  w.n_lm = bp.take<int>(1);
  w.lmx = bp.take<char>((size_t)cap * c->d * es);
  if (c->dtype == DLLM_BF16) {
    w.lm_tiles = lm_tiles_for(c);
    w.lm_out = bp.take<float>((size_t)cap * w.lm_tiles * 3);
  } else {
    w.lm_tiles = 0;
    w.lm_out = bp.take<float>((size_t)cap * c->vocab);
  }
  w.k2_cap = k2_cap;
  if (k2_cap > 0) {
    w.scores2 = bp.take<float>((size_t)B * k_cap);
    w.idx2 = bp.take<int32_t>((size_t)B * k2_cap);
    w.count2 = bp.take<int32_t>(B);
    w.pos2 = bp.take<int32_t>((size_t)B * k2_cap);
    w.row_off2 = bp.take<int>((size_t)B + 1);
    w.row_pos2 = bp.take<int>((size_t)B * k2_cap);
    w.row_seq2 = bp.take<int>((size_t)B * k2_cap);
    w.x2 = bp.take<char>((size_t)B * k2_cap * c->d * es);
  }
  if (gate) {
    w.g_flag = bp.take<int>(cap);
    w.g_list = bp.take<int>(cap);
    w.g_inv = bp.take<int>(cap);
    w.g_n = bp.take<int>(1);
    w.g_f = bp.take<char>((size_t)cap * c->d * es);
  }
  if (upd) {
    const size_t kvb = (size_t)cap * c->n_kv_heads * c->head_dim * es;
    w.u_m = bp.take<float>((size_t)cap * c->n_heads);
    w.u_l = bp.take<float>((size_t)cap * c->n_heads);
    w.u_kold = bp.take<char>(kvb);
    w.u_vold = bp.take<char>(kvb);
    w.u_knew = bp.take<char>(kvb);
    w.u_vnew = bp.take<char>(kvb);
    w.u_skip = bp.take<uint8_t>((size_t)B * N);
    w.u_off = bp.take<int>((size_t)B + 1);
  }
}

}  // namespace

extern "C" size_t dllm_step_workspace_size(const dllm_model_cfg* c, int B, int N,
                                           const dllm_policy* pol) {
  if (check_cfg(c) != DLLM_OK || !pol || B < 0 || N < 0) return 0;
  const int k_cap = std::max(1, std::min(pol->k, N));
  Bump bp(nullptr);
  StepWs w{};
  layout_step(bp, c, B, N, k_cap, k2_cap_of(pol, N), pol->ffn_gate != 0, pol->attn_update != 0,
              w);
  return bp.off;
}

extern "C" dllm_status dllm_step(const dllm_model_cfg* c, const dllm_model_w* mw,
                                 const dllm_cache* cache, int32_t* tokens, int B, int N,
                                 const dllm_policy* pol, int dense, const int32_t* forced_idx,
                                 const int32_t* forced_count, const int32_t* forced_unmask_pos,
                                 int32_t* idx_out, int32_t* count_out, int32_t* pos_out,
                                 float* scores_out, void* ws, size_t ws_bytes,
                                 dllm_stream_t stream) {
  dllm_step_io io{};
  io.forced_idx = forced_idx;
  io.forced_count = forced_count;
  io.forced_unmask_pos = forced_unmask_pos;
  io.idx_out = idx_out;
  io.count_out = count_out;
  io.pos_out = pos_out;
  io.scores_out = scores_out;
  return dllm_step_ex(c, mw, cache, tokens, B, N, pol, dense, &io, ws, ws_bytes, stream);
}

extern "C" dllm_status dllm_step_ex(const dllm_model_cfg* c, const dllm_model_w* mw,
                                    const dllm_cache* cache, int32_t* tokens, int B, int N,
                                    const dllm_policy* pol, int dense, const dllm_step_io* io_in,
                                    void* ws, size_t ws_bytes, dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dllm_step_io io = io_in ? *io_in : dllm_step_io{};
  const int32_t* forced_idx = io.forced_idx;
  const int32_t* forced_count = io.forced_count;
  const int32_t* forced_unmask_pos = io.forced_unmask_pos;
  int32_t* idx_out = io.idx_out;
  int32_t* count_out = io.count_out;
  int32_t* pos_out = io.pos_out;
  float* scores_out = io.scores_out;
  dllm_status st = check_cfg(c);
  if (st != DLLM_OK) return st;
  if (!mw || !cache || !pol || !tokens) return DLLM_ERR_INVALID_ARG;
  if (B < 0 || N < 0) return DLLM_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return DLLM_OK;
  if (!mw->embed || !mw->final_norm || !mw->lm_head || (c->n_layers > 0 && !mw->layers))
    return DLLM_ERR_INVALID_ARG;
  for (int l = 0; l < c->n_layers; ++l)
    if ((st = check_layer_w(&mw->layers[l])) != DLLM_OK) return st;
  if (!cache->k || !cache->v || !cache->h_ref || !cache->conf || !cache->pred)
    return DLLM_ERR_INVALID_ARG;
  for (int l = 0; l < c->n_layers; ++l)
    if (!cache->k[l] || !cache->v[l] || !aligned(cache->k[l], 16) || !aligned(cache->v[l], 16))
      return DLLM_ERR_INVALID_ARG;
  if (pol->score_layer < 0 || pol->score_layer > c->n_layers) return DLLM_ERR_INVALID_ARG;
  if (pol->kind != DLLM_SCORE_COS && pol->kind != DLLM_SCORE_ES_L1) return DLLM_ERR_INVALID_ARG;
  if (pol->mode != DLLM_SELECT_TOPK && pol->mode != DLLM_SELECT_THRESH)
    return DLLM_ERR_INVALID_ARG;
  if (pol->k < 0 || pol->n_unmask < 0 || pol->gen_start < 0 || pol->gen_start > N ||
      pol->block_len < 1)
    return DLLM_ERR_INVALID_ARG;
  if (pol->select_from < 0 || pol->select_from > N || !(pol->unmask_tau == pol->unmask_tau) ||
      pol->unmask_tau == INFINITY || pol->refresh_every < 0)
    return DLLM_ERR_INVALID_ARG;
  if (N > 16384 || pol->block_len > 1024) return DLLM_ERR_UNSUPPORTED_SHAPE;
  if ((forced_idx == nullptr) != (forced_count == nullptr)) return DLLM_ERR_INVALID_ARG;
  if ((io.forced_idx2 == nullptr) != (io.forced_count2 == nullptr)) return DLLM_ERR_INVALID_ARG;
  if (pol->ffn_gate) {
    if (!(pol->ffn_tau == pol->ffn_tau)) return DLLM_ERR_INVALID_ARG;
    if (!cache->ctx || !cache->ffn) return DLLM_ERR_INVALID_ARG;
    for (int l = 0; l < c->n_layers; ++l)
      if (!cache->ctx[l] || !cache->ffn[l] || !aligned(cache->ctx[l], 16) ||
          !aligned(cache->ffn[l], 16))
        return DLLM_ERR_INVALID_ARG;
  }
  if (pol->attn_update) {
    if (!pol->ffn_gate) return DLLM_ERR_INVALID_ARG;
    if (c->dtype != DLLM_BF16) return DLLM_ERR_UNSUPPORTED_SHAPE;
    if (!cache->q || !cache->att_m || !cache->att_l) return DLLM_ERR_INVALID_ARG;
    for (int l = 0; l < c->n_layers; ++l)
      if (!cache->q[l] || !cache->att_m[l] || !cache->att_l[l] || !aligned(cache->q[l], 16) ||
          !aligned(cache->att_m[l], 16) || !aligned(cache->att_l[l], 16))
        return DLLM_ERR_INVALID_ARG;
  }
  const int l2 = pol->score_layer2;
  if (l2 != 0) {
    if (l2 <= pol->score_layer || l2 >= c->n_layers || pol->k2 < 0) return DLLM_ERR_INVALID_ARG;
    if (!cache->h_ref2 || !aligned(cache->h_ref2, 16)) return DLLM_ERR_INVALID_ARG;
  }
  if (!ws || !aligned(ws, 256) || ws_bytes < dllm_step_workspace_size(c, B, N, pol))
    return DLLM_ERR_WORKSPACE;

  const int k_cap = std::max(1, std::min(pol->k, N));
  const int k2_cap = k2_cap_of(pol, N);
  const int d = c->d;
  Bump bp(ws);
  StepWs w{};
  layout_step(bp, c, B, N, k_cap, k2_cap, pol->ffn_gate != 0, pol->attn_update != 0, w);
  LayerWs& L = w.L;
  const bool use_rope = c->rope_theta > 0.f;
  if (use_rope) launch_rope_table(L.rope, N, c->head_dim, c->rope_theta, s);
  const bool bf = c->dtype == DLLM_BF16;
  const int ls = pol->score_layer;
  const int* M_dev = L.row_off + B;
  auto gate_of = [&](int l, bool all_rows, LayerGate& gt) -> const LayerGate* {
    if (!pol->ffn_gate) return nullptr;
    const uint8_t* forced =
        (!all_rows && io.forced_ffn) ? io.forced_ffn + (size_t)l * B * k_cap : nullptr;
    gt = LayerGate{cache->ctx[l], cache->ffn[l], pol->ffn_tau, all_rows ? 1 : 0, forced,
                   w.g_flag, w.g_list, w.g_inv, w.g_n, w.g_f,
                   io.ffn_rows_out ? io.ffn_rows_out + l : nullptr};
    return &gt;
  };

  // 1. hidden at the score layer: embeddings, then dense layers below it
  const void* h_src = nullptr;  // [B, N, d] source of the score-layer hidden, or null = embed
  if (ls > 0) {
    launch_row_map_dense(B, N, L.row_off, L.row_pos, L.row_seq, s);
    if (bf)
      launch_gather_rows<__nv_bfloat16>(nullptr, static_cast<const __nv_bfloat16*>(mw->embed),
                                        tokens, L.row_pos, L.row_seq, M_dev, B * N, N, d,
                                        static_cast<__nv_bfloat16*>(w.h_full), nullptr, c->vocab,
                                        w.status, s);
    else
      launch_gather_rows<float>(nullptr, static_cast<const float*>(mw->embed), tokens, L.row_pos,
                                L.row_seq, M_dev, B * N, N, d, static_cast<float*>(w.h_full),
                                nullptr, c->vocab, w.status, s);
    for (int l = 0; l < ls; ++l) {
      LayerGate gt;
      st = layer_forward(c, &mw->layers[l], w.h_full, B * N, M_dev, L, B, N, N, cache->k[l],
                         cache->v[l], use_rope, s, gate_of(l, true, gt));
      if (st != DLLM_OK) return st;
    }
    h_src = w.h_full;
  }

  // 2-3. rows to recompute
  int rows_per_seq;
  if (dense) {
    rows_per_seq = N;
    launch_row_map_dense(B, N, L.row_off, L.row_pos, L.row_seq, s);
  } else {
    rows_per_seq = k_cap;
    if (forced_idx) {
      launch_copy_idx(forced_idx, forced_count, w.idx, w.count, B, k_cap, s);
    } else {
      if (bf)
        launch_score<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(h_src),
                                    static_cast<const __nv_bfloat16*>(mw->embed),
                                    h_src ? nullptr : tokens,
                                    static_cast<const __nv_bfloat16*>(cache->h_ref), B, N, d,
                                    cache->conf, nullptr, tokens, c->mask_id, pol->alpha,
                                    pol->kind, w.scores, c->vocab, pol->select_from, w.status,
                                    s);
      else
        launch_score<float>(static_cast<const float*>(h_src),
                            static_cast<const float*>(mw->embed), h_src ? nullptr : tokens,
                            static_cast<const float*>(cache->h_ref), B, N, d, cache->conf,
                            nullptr, tokens, c->mask_id, pol->alpha, pol->kind, w.scores,
                            c->vocab, pol->select_from, w.status, s);
      launch_select(w.scores, B, N, pol->select_from, pol->mode, pol->k, pol->tau, w.idx, w.count,
                    k_cap, w.status, s);
    }
    launch_row_map(w.idx, w.count, B, k_cap, N, L.row_off, L.row_pos, L.row_seq, w.status, s);
  }
  const int cap = B * rows_per_seq;

  // 4. gather the selected rows (and refresh their hidden reference)
  if (bf)
    launch_gather_rows<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(h_src),
                                      static_cast<const __nv_bfloat16*>(mw->embed),
                                      h_src ? nullptr : tokens, L.row_pos, L.row_seq, M_dev, cap,
                                      N, d, static_cast<__nv_bfloat16*>(w.x),
                                      static_cast<__nv_bfloat16*>(cache->h_ref), c->vocab,
                                      w.status, s);
  else
    launch_gather_rows<float>(static_cast<const float*>(h_src),
                              static_cast<const float*>(mw->embed), h_src ? nullptr : tokens,
                              L.row_pos, L.row_seq, M_dev, cap, N, d, static_cast<float*>(w.x),
                              static_cast<float*>(cache->h_ref), c->vocab, w.status, s);

  // 5. remaining layers on the compact rows (narrowed at the second skip point)
  void* xc = w.x;
  int cap_c = cap, rps = rows_per_seq;
  const int* M_c = M_dev;
  for (int l = ls; l < c->n_layers; ++l) {
    if (l2 > 0 && l == l2) {
      if (dense) {
        if (cudaMemcpyAsync(cache->h_ref2, xc, (size_t)B * N * d * esize(c->dtype),
                            cudaMemcpyDeviceToDevice, s) != cudaSuccess)
          return DLLM_ERR_CUDA;
      } else {
        if (io.forced_idx2) {
          launch_copy_idx(io.forced_idx2, io.forced_count2, w.pos2, w.count2, B, k2_cap, s);
        } else {
          if (bf)
            launch_score_rows<__nv_bfloat16>(
                static_cast<const __nv_bfloat16*>(xc),
                static_cast<const __nv_bfloat16*>(cache->h_ref2), L.row_off, L.row_pos,
                L.row_seq, M_c, cap_c, N, d, k_cap, cache->conf, tokens, c->mask_id, pol->alpha,
                pol->kind, w.scores2, s);
          else
            launch_score_rows<float>(static_cast<const float*>(xc),
                                     static_cast<const float*>(cache->h_ref2), L.row_off,
                                     L.row_pos, L.row_seq, M_c, cap_c, N, d, k_cap, cache->conf,
                                     tokens, c->mask_id, pol->alpha, pol->kind, w.scores2, s);
          launch_select(w.scores2, B, k_cap, 0, DLLM_SELECT_TOPK, pol->k2, 0.f, w.idx2, w.count2,
                        k2_cap, w.status, s, w.count);
          launch_seg_positions(w.idx2, w.count2, L.row_off, L.row_pos, B, k2_cap, w.pos2, s);
        }
        launch_row_map(w.pos2, w.count2, B, k2_cap, N, w.row_off2, w.row_pos2, w.row_seq2,
                       w.status, s);
        const int cap2 = B * k2_cap;
        if (bf)
          launch_gather_narrow<__nv_bfloat16>(
              static_cast<const __nv_bfloat16*>(xc), L.row_off, L.row_pos, w.row_off2,
              w.row_pos2, w.row_seq2, w.row_off2 + B, cap2, N, d,
              static_cast<__nv_bfloat16*>(w.x2), static_cast<__nv_bfloat16*>(cache->h_ref2),
              w.status, s);
        else
          launch_gather_narrow<float>(static_cast<const float*>(xc), L.row_off, L.row_pos,
                                      w.row_off2, w.row_pos2, w.row_seq2, w.row_off2 + B, cap2,
                                      N, d, static_cast<float*>(w.x2),
                                      static_cast<float*>(cache->h_ref2), w.status, s);
        // the kept rows' maps replace the first selection's from here on
        L.row_off = w.row_off2;
        L.row_pos = w.row_pos2;
        L.row_seq = w.row_seq2;
        M_c = w.row_off2 + B;
        xc = w.x2;
        cap_c = cap2;
        rps = k2_cap;
      }
    }
    LayerGate gt;
    LayerUpd ut;
    const LayerUpd* upd = nullptr;
    if (pol->attn_update) {
      ut = LayerUpd{cache->q[l], cache->att_m[l], cache->att_l[l], dense == 0, w.u_m, w.u_l,
                    w.u_kold, w.u_vold, w.u_knew, w.u_vnew, w.u_skip, w.u_off};
      upd = &ut;
    }
    st = layer_forward(c, &mw->layers[l], xc, cap_c, M_c, L, B, N, rps, cache->k[l],
                       cache->v[l], use_rope, s, gate_of(l, dense != 0, gt), upd);
    if (st != DLLM_OK) return st;
  }

  // 6. LM head on selected rows that are still masked
  launch_masked_rows(tokens, c->mask_id, L.row_pos, L.row_seq, M_c, cap_c, N, w.lm_rows, w.n_lm,
                     s);
  if (bf) {
    using bfl = __nv_bfloat16;
    launch_rmsnorm_rows<bfl>(static_cast<const bfl*>(xc), static_cast<const bfl*>(mw->final_norm),
                             static_cast<bfl*>(w.lmx), w.lm_rows, w.n_lm, cap_c, d, c->rms_eps, s);
    GemmSpec g{};
    g.epi = EPI_LMHEAD;
    g.A = static_cast<const bfl*>(w.lmx);
    g.M_cap = cap_c;
    g.M_dev = w.n_lm;
    g.K = d;
    g.B[0] = static_cast<const bfl*>(mw->lm_head);
    g.seg_cols[0] = c->vocab;
    g.n_seg = 1;
    g.lm_part = w.lm_out;
    g.status = w.status;
    GemmPlan pl = gemm_plan(g);
    if (gemm_launch(g, s) != cudaSuccess) return DLLM_ERR_CUDA;
    launch_lm_merge(w.lm_out, pl.tiles_n, w.lm_rows, w.n_lm, cap_c, L.row_pos, L.row_seq, N,
                    cache->conf, cache->pred, s);
  } else {
    launch_rmsnorm_rows<float>(static_cast<const float*>(xc),
                               static_cast<const float*>(mw->final_norm),
                               static_cast<float*>(w.lmx), w.lm_rows, w.n_lm, cap_c, d, c->rms_eps,
                               s);
    launch_gemm_f32(static_cast<const float*>(w.lmx), static_cast<const float*>(mw->lm_head),
                    w.lm_out, nullptr, w.n_lm, cap_c, c->vocab, d, s);
    launch_confidence_rows_f32(w.lm_out, c->vocab, w.lm_rows, w.n_lm, cap_c, L.row_pos, L.row_seq,
                               N, cache->conf, cache->pred, s);
  }

  // 7. unmask
  launch_unmask(cache->conf, cache->pred, tokens, B, N, c->mask_id, pol->gen_start,
                pol->block_len, pol->n_unmask, pol->unmask_tau, dllm_unmask_capacity(pol), pos_out,
                forced_unmask_pos, s);

  if (!dense) {
    if (idx_out || count_out) {
      if (idx_out && count_out) {
        launch_copy_idx(w.idx, w.count, idx_out, count_out, B, k_cap, s);
      } else if (idx_out) {
        if (cudaMemcpyAsync(idx_out, w.idx, (size_t)B * k_cap * 4, cudaMemcpyDeviceToDevice, s))
          return DLLM_ERR_CUDA;
      } else {
        if (cudaMemcpyAsync(count_out, w.count, (size_t)B * 4, cudaMemcpyDeviceToDevice, s))
          return DLLM_ERR_CUDA;
      }
    }
    if (scores_out && !forced_idx &&
        cudaMemcpyAsync(scores_out, w.scores, (size_t)B * N * 4, cudaMemcpyDeviceToDevice, s))
      return DLLM_ERR_CUDA;
    if (l2 > 0) {
      if (io.idx2_out && io.count2_out)
        launch_copy_idx(w.pos2, w.count2, io.idx2_out, io.count2_out, B, k2_cap, s);
      if (io.scores2_out && !io.forced_idx2 &&
          cudaMemcpyAsync(io.scores2_out, w.scores2, (size_t)B * k_cap * 4,
                          cudaMemcpyDeviceToDevice, s))
        return DLLM_ERR_CUDA;
    }
  }
  return check_launch();
}

// ---------------------------------------------------------------- generation

extern "C" size_t dllm_generate_workspace_size(const dllm_model_cfg* c, int B, int N,
                                               const dllm_policy* pol) {
  const size_t step = dllm_step_workspace_size(c, B, N, pol);
  if (step == 0) return 0;
  return round_up(step, 256) + round_up((size_t)std::max(B, 1) * sizeof(int32_t), 256);
}

extern "C" dllm_status dllm_generate(const dllm_model_cfg* c, const dllm_model_w* mw,
                                     const dllm_cache* cache, int32_t* tokens, int B, int N,
                                     const dllm_policy* pol, int n_steps, int32_t* pos_log,
                                     uint8_t* dense_log, void* ws, size_t ws_bytes,
                                     dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!c || !pol || n_steps < 0 || B < 0 || N < 0) return DLLM_ERR_INVALID_ARG;
  if (pol->refresh_every < 0) return DLLM_ERR_INVALID_ARG;
  if (n_steps == 0 || B == 0 || N == 0) return DLLM_OK;
  const size_t step_ws = dllm_step_workspace_size(c, B, N, pol);
  if (step_ws == 0) return check_cfg(c) != DLLM_OK ? check_cfg(c) : DLLM_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < dllm_generate_workspace_size(c, B, N, pol))
    return DLLM_ERR_WORKSPACE;
  int32_t* d_blocks = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + round_up(step_ws, 256));
  const int cap = dllm_unmask_capacity(pol);
  std::vector<int32_t> prev(B), cur(B);
  for (int t = 0; t < n_steps; ++t) {
    bool dense = t == 0 || (pol->refresh_every > 0 && t % pol->refresh_every == 0);
    if (pol->refresh_on_block) {
      launch_block_start(tokens, B, N, c->mask_id, pol->gen_start, pol->block_len, d_blocks, s);
      if (cudaMemcpyAsync(cur.data(), d_blocks, (size_t)B * sizeof(int32_t),
                          cudaMemcpyDeviceToHost, s) != cudaSuccess ||
          cudaStreamSynchronize(s) != cudaSuccess)
        return DLLM_ERR_CUDA;
      if (t > 0 && cur != prev) dense = true;
      prev.swap(cur);
    }
    const dllm_status st =
        dllm_step(c, mw, cache, tokens, B, N, pol, dense ? 1 : 0, nullptr, nullptr, nullptr,
                  nullptr, nullptr, pos_log ? pos_log + (size_t)t * B * cap : nullptr, nullptr,
                  ws, step_ws, stream);
    if (st != DLLM_OK) return st;
    if (dense_log) dense_log[t] = dense ? 1 : 0;
  }
  return DLLM_OK;
}

// ---------------------------------------------------------------- host token buffers

extern "C" size_t dllm_step_host_workspace_size(const dllm_model_cfg* c, int B, int N,
                                                const dllm_policy* pol) {
  const size_t step = dllm_step_workspace_size(c, B, N, pol);
  if (step == 0) return 0;
  const size_t cap = (size_t)std::max(dllm_unmask_capacity(pol), 1);
  return round_up(step, 256) + round_up((size_t)B * N * sizeof(int32_t), 256) +
         round_up((size_t)B * cap * sizeof(int32_t), 256);
}

extern "C" dllm_status dllm_step_host(const dllm_model_cfg* c, const dllm_model_w* mw,
                                      const dllm_cache* cache, int32_t* tokens_host, int B, int N,
                                      const dllm_policy* pol, int dense, int32_t* pos_host,
                                      void* ws, size_t ws_bytes, dllm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!c || !pol || !tokens_host || B < 0 || N < 0) return DLLM_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return DLLM_OK;
  const size_t step_ws = dllm_step_workspace_size(c, B, N, pol);
  if (step_ws == 0) return check_cfg(c) != DLLM_OK ? check_cfg(c) : DLLM_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < dllm_step_host_workspace_size(c, B, N, pol))
    return DLLM_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  int32_t* d_tok = reinterpret_cast<int32_t*>(base + round_up(step_ws, 256));
  int32_t* d_pos = reinterpret_cast<int32_t*>(base + round_up(step_ws, 256) +
                                              round_up((size_t)B * N * sizeof(int32_t), 256));
  const size_t tok_bytes = (size_t)B * N * sizeof(int32_t);
  const size_t pos_bytes = (size_t)B * std::max(dllm_unmask_capacity(pol), 1) * sizeof(int32_t);
  if (cudaMemcpyAsync(d_tok, tokens_host, tok_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return DLLM_ERR_CUDA;
  const dllm_status st = dllm_step(c, mw, cache, d_tok, B, N, pol, dense, nullptr, nullptr,
                                   nullptr, nullptr, nullptr, pos_host ? d_pos : nullptr, nullptr,
                                   ws, step_ws, stream);
  if (st != DLLM_OK) return st;
  if (cudaMemcpyAsync(tokens_host, d_tok, tok_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DLLM_ERR_CUDA;
  if (pos_host &&
      cudaMemcpyAsync(pos_host, d_pos, pos_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DLLM_ERR_CUDA;
  return DLLM_OK;
}
