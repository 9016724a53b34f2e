"""Python binding of libdllm.so, the sm_100a selected-token denoising step.

Argument marshalling only: every step of the path runs in the library's
CUDA kernels.  Tensors are torch CUDA tensors (device memory and streams);
they are passed as raw pointers through ctypes.  If the shared library is
missing, importing this package raises: there is no fallback path.

The functions carry the C names (``dllm_score``, ``dllm_select``,
``dllm_unmask``, ``dllm_partial_layer``, ``dllm_step`` ...); ``Model``,
``Cache`` and ``Workspace`` hold the ctypes structs and the torch-owned
buffers the calls need.
"""
from __future__ import annotations

import ctypes as C
import json
import os
from typing import Dict, List, Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdllm.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m sparse_token_recompute_b200.build` "
        "(there is no CPU or eager fallback)")

_lib = C.CDLL(LIB_PATH)

DLLM_OK = 0
DLLM_F32, DLLM_BF16 = 0, 1
DLLM_SCORE_COS, DLLM_SCORE_ES_L1 = 0, 1
DLLM_SELECT_TOPK, DLLM_SELECT_THRESH = 0, 1
DLLM_DEV_TIMEOUT, DLLM_DEV_CAPACITY, DLLM_DEV_BAD_INDEX, DLLM_DEV_BAD_SHAPE = 1, 2, 4, 8

vp = C.c_void_p


class ModelCfg(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("d", C.c_int), ("n_heads", C.c_int),
                ("n_kv_heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int),
                ("vocab", C.c_int), ("rope_theta", C.c_float), ("rms_eps", C.c_float),
                ("mask_id", C.c_int), ("dtype", C.c_int)]


class LayerW(C.Structure):
    _fields_ = [(n, vp) for n in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate",
                                  "w_up", "w_down")]


class ModelW(C.Structure):
    _fields_ = [("embed", vp), ("layers", C.POINTER(LayerW)), ("final_norm", vp),
                ("lm_head", vp)]


class CacheS(C.Structure):
    _fields_ = [("k", C.POINTER(vp)), ("v", C.POINTER(vp)), ("h_ref", vp), ("conf", vp),
                ("pred", vp), ("h_ref2", vp), ("ctx", C.POINTER(vp)), ("ffn", C.POINTER(vp)),
                ("q", C.POINTER(vp)), ("att_m", C.POINTER(vp)), ("att_l", C.POINTER(vp))]


class Policy(C.Structure):
    _fields_ = [("score_layer", C.c_int), ("alpha", C.c_float), ("kind", C.c_int),
                ("mode", C.c_int), ("k", C.c_int), ("tau", C.c_float), ("n_unmask", C.c_int),
                ("gen_start", C.c_int), ("block_len", C.c_int), ("select_from", C.c_int),
                ("unmask_tau", C.c_float), ("refresh_every", C.c_int),
                ("refresh_on_block", C.c_int), ("score_layer2", C.c_int), ("k2", C.c_int),
                ("ffn_gate", C.c_int), ("ffn_tau", C.c_float), ("attn_update", C.c_int)]


class StepIO(C.Structure):
    _fields_ = [("forced_idx", vp), ("forced_count", vp), ("forced_unmask_pos", vp),
                ("idx_out", vp), ("count_out", vp), ("pos_out", vp), ("scores_out", vp),
                ("forced_idx2", vp), ("forced_count2", vp), ("idx2_out", vp),
                ("count2_out", vp), ("scores2_out", vp), ("ffn_rows_out", vp),
                ("forced_ffn", vp)]


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_i, _f, _sz = C.c_int, C.c_float, C.c_size_t
_status_string = _sig("dllm_status_string", C.c_char_p, [_i])
_version = _sig("dllm_version", _i, [])
_score = _sig("dllm_score", _i, [vp, vp, _i, _i, _i, _i, vp, vp, _i, _i, vp, vp, vp, _f, _i,
                                 vp, vp])
_select_ws = _sig("dllm_select_workspace_size", _sz, [_i, _i])
_select = _sig("dllm_select", _i, [vp, _i, _i, _i, _i, _f, vp, vp, _i, vp, _sz, vp])
_unmask = _sig("dllm_unmask", _i, [vp, vp, vp, _i, _i, _i, _i, _i, _i, vp, vp])
_unmask_tau = _sig("dllm_unmask_tau", _i, [vp, vp, vp, _i, _i, _i, _i, _i, _i, _f, vp, _i, vp])
_unmask_cap = _sig("dllm_unmask_capacity", _i, [C.POINTER(Policy)])
_select_range = _sig("dllm_select_range", _i, [vp, _i, _i, _i, _i, _i, _f, vp, vp, _i, vp, _sz,
                                               vp])
_layer_ws = _sig("dllm_partial_layer_workspace_size", _sz, [C.POINTER(ModelCfg), _i, _i, _i])
_layer = _sig("dllm_partial_layer", _i, [C.POINTER(ModelCfg), C.POINTER(LayerW), vp, _i, vp,
                                         vp, vp, _i, _i, _i, vp, vp, vp, _sz, vp])
_step_ws = _sig("dllm_step_workspace_size", _sz, [C.POINTER(ModelCfg), _i, _i,
                                                  C.POINTER(Policy)])
_step = _sig("dllm_step", _i, [C.POINTER(ModelCfg), C.POINTER(ModelW), C.POINTER(CacheS), vp,
                               _i, _i, C.POINTER(Policy), _i, vp, vp, vp, vp, vp, vp, vp, vp,
                               _sz, vp])
_step_ex = _sig("dllm_step_ex", _i, [C.POINTER(ModelCfg), C.POINTER(ModelW), C.POINTER(CacheS),
                                     vp, _i, _i, C.POINTER(Policy), _i, C.POINTER(StepIO), vp,
                                     _sz, vp])
_gen_ws = _sig("dllm_generate_workspace_size", _sz, [C.POINTER(ModelCfg), _i, _i,
                                                     C.POINTER(Policy)])
_gen = _sig("dllm_generate", _i, [C.POINTER(ModelCfg), C.POINTER(ModelW), C.POINTER(CacheS), vp,
                                  _i, _i, C.POINTER(Policy), _i, vp, C.POINTER(C.c_uint8), vp,
                                  _sz, vp])
_step_host_ws = _sig("dllm_step_host_workspace_size", _sz, [C.POINTER(ModelCfg), _i, _i,
                                                            C.POINTER(Policy)])
_step_host = _sig("dllm_step_host", _i, [C.POINTER(ModelCfg), C.POINTER(ModelW),
                                         C.POINTER(CacheS), vp, _i, _i, C.POINTER(Policy), _i,
                                         vp, vp, _sz, vp])
_devstat = _sig("dllm_get_device_status", _i, [vp, vp, C.POINTER(C.c_int32)])
_attn_noalloc = _sig("dllm_attention_bf16_noalloc", _i, [vp, vp, vp, vp, vp, _i, _i, _i, _i, _i,
                                                         _i, vp])
_attn_ws = _sig("dllm_attention_workspace_size", _sz, [_i])
_attn_stats = _sig("dllm_attention_stats_bf16", _i, [vp, vp, vp, vp, vp, vp, vp, _i, _i, _i, _i,
                                                     _i, _i, vp, _sz, vp])
_attn_upd_ws = _sig("dllm_attention_update_workspace_size", _sz, [_i])
_attn_upd = _sig("dllm_attention_update_bf16", _i, [vp, vp, vp, vp, vp, _i, _i, vp, vp, vp, vp,
                                                    vp, _i, _i, _i, _i, vp, _sz, vp])
_attn = _sig("dllm_attention_bf16", _i, [vp, vp, vp, vp, vp, _i, _i, _i, _i, _i, _i, vp, _sz,
                                         vp])
_gemm_ws = _sig("dllm_gemm_workspace_size", _sz, [_i, _i, _i, _i])
_gemm = _sig("dllm_gemm_bf16", _i, [vp, vp, vp, _i, _i, _i, _i, _i, vp, _sz, vp])
_gemm_stall = _sig("dllm_selftest_gemm_stall", _i, [vp, vp, vp, _i, _i, _i, vp, _sz, vp])
_gemm_plan = _sig("dllm_gemm_plan_info", _i, [_i, _i, _i, vp, _i, _i, vp])
_attn_plan = _sig("dllm_attention_plan_info", _i, [_i, _i, _i, _i, _i, _i, vp])
_prof_enable = _sig("dllm_profile_enable", None, [_i])
_prof_reset = _sig("dllm_profile_reset", None, [])
_prof_read = _sig("dllm_profile_read", _sz, [C.c_char_p, _sz])


class DllmError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def status_string(st: int) -> str:
    return _status_string(int(st)).decode()


def version() -> int:
    return int(_version())


def _check(st: int, where: str):
    if st != DLLM_OK:
        raise DllmError(st, where)


def ptr(t) -> Optional[int]:
    """Device (or host) address of a tensor; None stays NULL."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return DLLM_BF16
    if t.dtype == torch.float32:
        return DLLM_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


# ----------------------------------------------------------------- workspace

def _empty_bytes(nbytes: int, device):
    import torch
    # 256-byte alignment: torch's caching allocator returns at least 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


class Workspace:
    """A caller-owned scratch buffer (torch memory) passed to the library."""

    def __init__(self, nbytes: int, device="cuda"):
        self.buf = _empty_bytes(nbytes, device)
        self.buf[:256].zero_()
        self.nbytes = self.buf.numel()

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()

    def device_status(self, stream=None) -> int:
        v = C.c_int32(0)
        _devstat(self.ptr, _stream(stream), C.byref(v))
        return int(v.value)


# ----------------------------------------------------------------- thin calls

def dllm_score(h_cur, h_ref, conf, masked, scores, alpha: float, kind: int = DLLM_SCORE_COS,
               logits=None, logit_pos=None, pred=None, stream=None):
    B, N, d = h_cur.shape
    Mm = V = 0
    if logits is not None:
        _, Mm, V = logits.shape
    st = _score(ptr(h_cur), ptr(h_ref), B, N, d, _dtype_code(h_cur), ptr(logits), ptr(logit_pos),
                Mm, V, ptr(conf), ptr(pred), ptr(masked), float(alpha), int(kind), ptr(scores),
                _stream(stream))
    _check(st, "dllm_score")


def dllm_select(scores, idx, count, mode: int, k: int, tau: float = 0.0, ws: Workspace = None,
                stream=None):
    B, N = scores.shape
    k_cap = idx.shape[1]
    st = _select(ptr(scores), B, N, int(mode), int(k), float(tau), ptr(idx), ptr(count), k_cap,
                 ws.ptr if ws else None, ws.nbytes if ws else 0, _stream(stream))
    _check(st, "dllm_select")


def dllm_select_range(scores, idx, count, lo: int, mode: int, k: int, tau: float = 0.0,
                      ws: Workspace = None, stream=None):
    B, N = scores.shape
    k_cap = idx.shape[1]
    st = _select_range(ptr(scores), B, N, int(lo), int(mode), int(k), float(tau), ptr(idx),
                       ptr(count), k_cap, ws.ptr if ws else None, ws.nbytes if ws else 0,
                       _stream(stream))
    _check(st, "dllm_select_range")


def dllm_select_workspace_size(B: int, N: int) -> int:
    return int(_select_ws(B, N))


def dllm_unmask(conf, pred, tokens, mask_id: int, gen_start: int, block_len: int, n_unmask: int,
                pos_out=None, stream=None):
    B, N = tokens.shape
    st = _unmask(ptr(conf), ptr(pred), ptr(tokens), B, N, int(mask_id), int(gen_start),
                 int(block_len), int(n_unmask), ptr(pos_out), _stream(stream))
    _check(st, "dllm_unmask")


def dllm_unmask_tau(conf, pred, tokens, mask_id: int, gen_start: int, block_len: int,
                    n_unmask: int, tau: float, pos_out=None, stream=None):
    B, N = tokens.shape
    pos_cap = pos_out.shape[1] if pos_out is not None else max(n_unmask, block_len)
    st = _unmask_tau(ptr(conf), ptr(pred), ptr(tokens), B, N, int(mask_id), int(gen_start),
                     int(block_len), int(n_unmask), float(tau), ptr(pos_out), int(pos_cap),
                     _stream(stream))
    _check(st, "dllm_unmask_tau")


def dllm_unmask_capacity(pol: "Policy") -> int:
    return int(_unmask_cap(C.byref(pol)))


def dllm_gemm_workspace_size(M, N, K, splits=0) -> int:
    return int(_gemm_ws(M, N, K, splits))


def dllm_gemm_bf16(A, Bm, Cm, accumulate=False, splits=0, ws: Workspace = None, stream=None):
    M, K = A.shape
    N = Bm.shape[0]
    if ws is None:
        ws = Workspace(dllm_gemm_workspace_size(M, N, K, splits), A.device)
    st = _gemm(ptr(A), ptr(Bm), ptr(Cm), M, N, K, int(bool(accumulate)), int(splits), ws.ptr,
               ws.nbytes, _stream(stream))
    _check(st, "dllm_gemm_bf16")
    return ws


GEMM_KINDS = {"plain": 0, "residual": 1, "swiglu": 2, "qkv": 3, "lmhead": 4}


def dllm_gemm_plan_info(kind: str, M: int, K: int, seg_cols, head_dim: int = 0) -> Dict[str, int]:
    """The host-side launch plan of one projection GEMM (no GPU work)."""
    segs = (C.c_int32 * len(seg_cols))(*[int(c) for c in seg_cols])
    out = (C.c_int32 * 5)()
    st = _gemm_plan(GEMM_KINDS[kind], int(M), int(K), C.cast(segs, C.c_void_p), len(seg_cols),
                    int(head_dim), C.cast(out, C.c_void_p))
    _check(st, "dllm_gemm_plan_info")
    return {"bn": out[0], "splits": out[1], "tiles_n": out[2], "grid": out[3], "pair": out[4]}


def dllm_attention_plan_info(B: int, k_cap: int, N: int, n_heads: int, head_dim: int,
                             in_step: bool = True) -> Dict[str, int]:
    """The host-side launch plan of the exact partial attention (no GPU work)."""
    out = (C.c_int32 * 3)()
    st = _attn_plan(int(B), int(k_cap), int(N), int(n_heads), int(head_dim), int(bool(in_step)),
                    C.cast(out, C.c_void_p))
    _check(st, "dllm_attention_plan_info")
    return {"tiles_per_cta": out[0], "key_shares": out[1], "ctas": out[2]}


def dllm_selftest_gemm_stall(A, Bm, Cm, ws: Workspace = None, stream=None):
    """The CTA-pair GEMM with one stage signal withheld: ends with DLLM_DEV_TIMEOUT
    in ws's device status (after the 2 s wait limit); C is undefined."""
    M, K = A.shape
    N = Bm.shape[0]
    if ws is None:
        ws = Workspace(dllm_gemm_workspace_size(M, N, K, 1), A.device)
    st = _gemm_stall(ptr(A), ptr(Bm), ptr(Cm), M, N, K, ws.ptr, ws.nbytes, _stream(stream))
    _check(st, "dllm_selftest_gemm_stall")
    return ws


def dllm_attention_workspace_size(B: int) -> int:
    return int(_attn_ws(B))


def dllm_attention_bf16(q, k_cache, v_cache, o, count, k_cap: int, ws: Workspace = None,
                        stream=None):
    B, N, Hkv, hd = k_cache.shape
    Hq = q.shape[1] // hd
    if ws is None:
        ws = Workspace(dllm_attention_workspace_size(B), q.device)
    st = _attn(ptr(q), ptr(k_cache), ptr(v_cache), ptr(o), ptr(count), B, int(k_cap), N, Hq, Hkv,
               hd, ws.ptr, ws.nbytes, _stream(stream))
    _check(st, "dllm_attention_bf16")
    return ws


def dllm_attention_stats_bf16(q, k_cache, v_cache, o, m, l, count, k_cap: int,
                              ws: Workspace = None, stream=None):
    """dllm_attention_bf16 plus each row's softmax statistics m, l [B*k_cap, Hq] (f32)."""
    B, N, Hkv, hd = k_cache.shape
    Hq = q.shape[1] // hd
    if ws is None:
        ws = Workspace(dllm_attention_workspace_size(B), q.device)
    st = _attn_stats(ptr(q), ptr(k_cache), ptr(v_cache), ptr(o), ptr(m), ptr(l), ptr(count), B,
                     int(k_cap), N, Hq, Hkv, hd, ws.ptr, ws.nbytes, _stream(stream))
    _check(st, "dllm_attention_stats_bf16")
    return ws


def dllm_attention_update_bf16(q, o, m, l, r_count, r_cap: int, k_new, v_new, k_old, v_old,
                               a_count, a_cap: int, n_kv_heads: int, ws: Workspace = None,
                               stream=None):
    """Incremental attention of stable rows (see include/dllm.h); q/o [B*r_cap, Hq*hd],
    m/l [B*r_cap, Hq] updated in place; changed keys [B*a_cap, Hkv, hd]."""
    B = r_count.shape[0]
    hd = k_new.shape[-1]
    Hq = q.shape[1] // hd
    if ws is None:
        ws = Workspace(int(_attn_upd_ws(B)), q.device)
    st = _attn_upd(ptr(q), ptr(o), ptr(m), ptr(l), ptr(r_count), B, int(r_cap), ptr(k_new),
                   ptr(v_new), ptr(k_old), ptr(v_old), ptr(a_count), int(a_cap), Hq,
                   int(n_kv_heads), hd, ws.ptr, ws.nbytes, _stream(stream))
    _check(st, "dllm_attention_update_bf16")
    return ws


DLLM_NOALLOC_MAX_SEQS = 4096


def dllm_attention_bf16_noalloc(q, k_cache, v_cache, o, count, k_cap: int, stream=None):
    """Partial attention without a workspace, for callers that cannot allocate
    device memory (memory carved into fixed pools, operators handed only their
    tensors); its scratch is a fixed array inside the library shared by all calls."""
    B, N, Hkv, hd = k_cache.shape
    Hq = q.shape[1] // hd
    st = _attn_noalloc(ptr(q), ptr(k_cache), ptr(v_cache), ptr(o), ptr(count), B, int(k_cap), N,
                       Hq, Hkv, hd, _stream(stream))
    _check(st, "dllm_attention_bf16_noalloc")


def profile_enable(on: bool = True):
    _prof_enable(int(bool(on)))


def profile_reset():
    _prof_reset()


def profile_read() -> Dict[str, List[float]]:
    n = _prof_read(None, 0)
    buf = C.create_string_buffer(int(n))
    _prof_read(buf, n)
    return json.loads(buf.value.decode())


# ----------------------------------------------------------------- model / cache

def make_cfg(n_layers, d, n_heads, n_kv_heads, head_dim, ffn, vocab, rope_theta, rms_eps,
             mask_id, dtype) -> ModelCfg:
    return ModelCfg(n_layers, d, n_heads, n_kv_heads, head_dim, ffn, vocab, float(rope_theta),
                    float(rms_eps), mask_id, DLLM_BF16 if dtype == "bf16" else DLLM_F32)


def cfg_from_shape(s) -> ModelCfg:
    return make_cfg(s.n_layers, s.d, s.n_heads, s.n_kv_heads, s.head_dim, s.ffn, s.vocab,
                    s.rope_theta, s.rms_eps, s.mask_id, s.dtype)


def layer_struct(L: Dict[str, object]) -> LayerW:
    return LayerW(*(ptr(L[n]) for n in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm",
                                        "w_gate", "w_up", "w_down")))


class Model:
    """Weights (torch CUDA tensors, dict layout of ``dllm_synth.model_weights``) plus
    the ctypes structs that point at them."""

    def __init__(self, cfg: ModelCfg, W: Dict[str, object]):
        self.cfg = cfg
        self.W = W
        n = len(W["layers"])
        self._layers = (LayerW * max(n, 1))(*[layer_struct(L) for L in W["layers"]])
        self.s = ModelW(ptr(W["embed"]), self._layers, ptr(W["final_norm"]), ptr(W["lm_head"]))

    def layer(self, i: int) -> LayerW:
        return self._layers[i]


class Cache:
    """Per-layer K/V caches, hidden reference, cached confidence and argmax (torch memory)."""

    def __init__(self, cfg: ModelCfg, B: int, N: int, device="cuda", second_ref: bool = False,
                 ffn_gate: bool = False, attn_update: bool = False):
        import torch
        dt = torch.bfloat16 if cfg.dtype == DLLM_BF16 else torch.float32
        kv = (B, N, cfg.n_kv_heads, cfg.head_dim)
        self.k = [torch.zeros(kv, dtype=dt, device=device) for _ in range(cfg.n_layers)]
        self.v = [torch.zeros(kv, dtype=dt, device=device) for _ in range(cfg.n_layers)]
        self.h_ref = torch.zeros(B, N, cfg.d, dtype=dt, device=device)
        # reference of the second skip point (policies with score_layer2 > 0)
        self.h_ref2 = torch.zeros(B, N, cfg.d, dtype=dt, device=device) if second_ref else None
        # DyLLM FFN gate: per layer, attention outputs and FFN outputs of every row
        q = cfg.n_heads * cfg.head_dim
        self.ctx = [torch.zeros(B, N, q, dtype=dt, device=device)
                    for _ in range(cfg.n_layers)] if ffn_gate else None
        self.ffn = [torch.zeros(B, N, cfg.d, dtype=dt, device=device)
                    for _ in range(cfg.n_layers)] if ffn_gate else None
        # approximate attention: per layer each row's query and softmax statistics
        self.q = [torch.zeros(B, N, q, dtype=dt, device=device)
                  for _ in range(cfg.n_layers)] if attn_update else None
        self.att_m = [torch.zeros(B, N, cfg.n_heads, dtype=torch.float32, device=device)
                      for _ in range(cfg.n_layers)] if attn_update else None
        self.att_l = [torch.zeros(B, N, cfg.n_heads, dtype=torch.float32, device=device)
                      for _ in range(cfg.n_layers)] if attn_update else None
        self.conf = torch.zeros(B, N, dtype=torch.float32, device=device)
        self.pred = torch.zeros(B, N, dtype=torch.int32, device=device)
        self._refresh()

    def _refresh(self):
        L = max(len(self.k), 1)
        self._kp = (vp * L)(*[ptr(t) for t in self.k])
        self._vp = (vp * L)(*[ptr(t) for t in self.v])
        self._cp = (vp * L)(*[ptr(t) for t in self.ctx]) if self.ctx else None
        self._fp = (vp * L)(*[ptr(t) for t in self.ffn]) if self.ffn else None
        self._qp = (vp * L)(*[ptr(t) for t in self.q]) if self.q else None
        self._mp = (vp * L)(*[ptr(t) for t in self.att_m]) if self.att_m else None
        self._lp = (vp * L)(*[ptr(t) for t in self.att_l]) if self.att_l else None
        self.s = CacheS(self._kp, self._vp, ptr(self.h_ref), ptr(self.conf), ptr(self.pred),
                        ptr(self.h_ref2), self._cp, self._fp, self._qp, self._mp, self._lp)


def make_policy(score_layer=0, alpha=0.5, kind=DLLM_SCORE_COS, mode=DLLM_SELECT_TOPK, k=1,
                tau=0.0, n_unmask=1, gen_start=0, block_len=32, select_from=0, unmask_tau=0.0,
                refresh_every=0, refresh_on_block=False, score_layer2=0, k2=0, ffn_gate=False,
                ffn_tau=0.0, attn_update=False) -> Policy:
    return Policy(score_layer, float(alpha), kind, mode, k, float(tau), n_unmask, gen_start,
                  block_len, int(select_from), float(unmask_tau), int(refresh_every),
                  int(bool(refresh_on_block)), int(score_layer2), int(k2), int(bool(ffn_gate)),
                  float(ffn_tau), int(bool(attn_update)))


def dllm_partial_layer_workspace_size(cfg: ModelCfg, B: int, N: int, k_cap: int) -> int:
    return int(_layer_ws(C.byref(cfg), B, N, k_cap))


def dllm_partial_layer(cfg: ModelCfg, lw: LayerW, x_in, x_out, idx, count, k_cache, v_cache,
                       ws: Workspace, x_in_is_full: bool, stream=None):
    B, k_cap = idx.shape
    N = k_cache.shape[1]
    st = _layer(C.byref(cfg), C.byref(lw), ptr(x_in), int(bool(x_in_is_full)), ptr(x_out),
                ptr(idx), ptr(count), k_cap, B, N, ptr(k_cache), ptr(v_cache), ws.ptr, ws.nbytes,
                _stream(stream))
    _check(st, "dllm_partial_layer")


def dllm_step_workspace_size(cfg: ModelCfg, B: int, N: int, pol: Policy) -> int:
    return int(_step_ws(C.byref(cfg), B, N, C.byref(pol)))


def dllm_step(model: Model, cache: Cache, tokens, pol: Policy, dense: bool, ws: Workspace,
              forced_idx=None, forced_count=None, forced_unmask_pos=None, idx_out=None,
              count_out=None, pos_out=None, scores_out=None, stream=None):
    B, N = tokens.shape
    st = _step(C.byref(model.cfg), C.byref(model.s), C.byref(cache.s), ptr(tokens), B, N,
               C.byref(pol), int(bool(dense)), ptr(forced_idx), ptr(forced_count),
               ptr(forced_unmask_pos), ptr(idx_out), ptr(count_out), ptr(pos_out),
               ptr(scores_out), ws.ptr, ws.nbytes, _stream(stream))
    _check(st, "dllm_step")


def dllm_generate_workspace_size(cfg: ModelCfg, B: int, N: int, pol: Policy) -> int:
    return int(_gen_ws(C.byref(cfg), B, N, C.byref(pol)))


def dllm_generate(model: Model, cache: Cache, tokens, pol: Policy, n_steps: int, ws: Workspace,
                  pos_log=None, stream=None):
    """n_steps steps with the policy's refresh schedule; returns the per-step
    dense flags (host list of bool).  pos_log: device [n_steps, B, capacity]."""
    B, N = tokens.shape
    flags = (C.c_uint8 * max(int(n_steps), 1))()
    st = _gen(C.byref(model.cfg), C.byref(model.s), C.byref(cache.s), ptr(tokens), B, N,
              C.byref(pol), int(n_steps), ptr(pos_log), flags, ws.ptr, ws.nbytes,
              _stream(stream))
    _check(st, "dllm_generate")
    return [bool(flags[t]) for t in range(int(n_steps))]


def dllm_step_ex(model: Model, cache: Cache, tokens, pol: Policy, dense: bool, ws: Workspace,
                 stream=None, **io):
    """dllm_step with the second skip point; keyword tensors fill dllm_step_io
    (forced_idx, forced_count, forced_unmask_pos, idx_out, count_out, pos_out,
    scores_out, forced_idx2, forced_count2, idx2_out, count2_out, scores2_out,
    ffn_rows_out, forced_ffn)."""
    B, N = tokens.shape
    s = StepIO(*[ptr(io.get(name)) for name, _ in StepIO._fields_])
    unknown = set(io) - {name for name, _ in StepIO._fields_}
    if unknown:
        raise TypeError(f"unknown dllm_step_io fields: {sorted(unknown)}")
    st = _step_ex(C.byref(model.cfg), C.byref(model.s), C.byref(cache.s), ptr(tokens), B, N,
                  C.byref(pol), int(bool(dense)), C.byref(s), ws.ptr, ws.nbytes,
                  _stream(stream))
    _check(st, "dllm_step_ex")


def dllm_step_host_workspace_size(cfg: ModelCfg, B: int, N: int, pol: Policy) -> int:
    return int(_step_host_ws(C.byref(cfg), B, N, C.byref(pol)))


def dllm_step_host(model: Model, cache: Cache, tokens_host, pol: Policy, dense: bool,
                   ws: Workspace, pos_host=None, stream=None):
    """One step whose tokens live in HOST memory (the C entry point copies them
    in, runs the step and copies tokens and revealed positions back, all on the
    stream; the host tensors hold the results after the stream synchronises).
    tokens_host [B, N] int32 and pos_host [B, capacity] int32: CPU tensors,
    preferably pinned."""
    B, N = tokens_host.shape
    st = _step_host(C.byref(model.cfg), C.byref(model.s), C.byref(cache.s), ptr(tokens_host), B,
                    N, C.byref(pol), int(bool(dense)), ptr(pos_host), ws.ptr, ws.nbytes,
                    _stream(stream))
    _check(st, "dllm_step_host")


class StepGraph:
    """One ``dllm_step`` captured into a CUDA graph and replayed.

    Every launch of a step depends only on device data (the index lists and
    row counts are produced on the device), so a step with fixed buffers can
    be recorded once and replayed for each later step, removing the per-launch
    host cost.  Capture once after an eager call of the same step (which sets
    the kernels' shared-memory attributes); buffers must stay at the same
    addresses for the life of the graph.
    """

    def __init__(self, model: Model, cache: Cache, tokens, pol: Policy, ws: Workspace,
                 dense: bool = False, pos_out=None):
        import torch
        profile_enable(False)  # per-launch timing events cannot be read back from a graph
        self.stream = torch.cuda.Stream()
        self.graph = torch.cuda.CUDAGraph()
        self.stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(self.graph, stream=self.stream):
            dllm_step(model, cache, tokens, pol, dense, ws, pos_out=pos_out,
                      stream=self.stream)
        torch.cuda.current_stream().wait_stream(self.stream)

    def replay(self):
        self.graph.replay()


__all__ = [n for n in dir() if n.startswith(("dllm_", "DLLM_"))] + ["StepGraph",

    "Model", "Cache", "Workspace", "ModelCfg", "LayerW", "Policy", "make_cfg", "cfg_from_shape",
    "make_policy", "profile_enable", "profile_reset", "profile_read", "status_string", "version",
    "DllmError", "LIB_PATH"]
