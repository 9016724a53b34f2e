"""Single-kernel cases for profiling the library's kernels under ncu.

Each case sets up inputs larger than L2 (so DRAM counters mean something)
but a few GB at most, runs the kernel `--warmup` times untimed and then
`--iters` times, and prints the CUDA-event time per launch.

  python -m sparse_token_recompute_b200.profile_cases gemm --M 9856 --N 12288 --K 4096
  python -m sparse_token_recompute_b200.profile_cases score --B 32 --L 1024 --d 4096
  python -m sparse_token_recompute_b200.profile_cases layer --B 32 --N 1536 --k 308
  python -m sparse_token_recompute_b200.profile_cases attention --B 32 --N 1536 --k 308
  python -m sparse_token_recompute_b200.profile_cases step --B 1 --ratio 0.10
  python -m sparse_token_recompute_b200.profile_cases step_graph --B 1 --ratio 0.10
"""
from __future__ import annotations

import argparse
import json

import torch

import dllm_synth as SY
import sparse_token_recompute_b200 as S


def _time(fn, warmup, iters):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / max(iters, 1)


def case_gemm(a):
    A = SY.normal((a.M, a.K), 1.0, 1, "cuda", "bf16")
    Bm = SY.normal((a.N, a.K), 0.02, 2, "cuda", "bf16")
    Cm = torch.empty(a.M, a.N, dtype=torch.bfloat16, device="cuda")
    ws = S.Workspace(S.dllm_gemm_workspace_size(a.M, a.N, a.K, a.splits))
    ms = _time(lambda: S.dllm_gemm_bf16(A, Bm, Cm, splits=a.splits, ws=ws), a.warmup, a.iters)
    fl = 2.0 * a.M * a.N * a.K
    return {"case": "gemm", "M": a.M, "N": a.N, "K": a.K, "ms": ms, "tflops": fl / ms / 1e9,
            "bytes_min": 2 * (a.M * a.K + a.N * a.K + a.M * a.N)}


def case_score(a):
    si = SY.score_inputs(a.B, a.L, a.d, a.V, a.Mm, device="cuda")
    scores = torch.empty(a.B, a.L, dtype=torch.float32, device="cuda")
    idx = torch.empty(a.B, a.k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(a.B, dtype=torch.int32, device="cuda")
    conf = si.conf.clone()

    def run():
        S.dllm_score(si.h_cur, si.h_ref, conf, si.masked, scores, 0.5, 0, logits=si.logits,
                     logit_pos=si.logit_pos, pred=si.pred)
        S.dllm_select(scores, idx, cnt, S.DLLM_SELECT_TOPK, a.k)

    ms = _time(run, a.warmup, a.iters)
    S.profile_reset()
    S.profile_enable(True)
    _time(run, 0, a.iters)
    S.profile_enable(False)
    per = {k: round(v[1] / v[0] * 1000, 1) for k, v in S.profile_read().items()}
    nbytes = 2 * a.B * a.L * a.d * 2 + a.B * a.Mm * a.V * 2
    return {"case": "score+select", "ms": ms, "GBps": nbytes / ms / 1e6, "bytes": nbytes,
            "us_per_kernel": per}


def case_attention(a):
    """Selected-query attention of one 8B layer: B sequences x k rows, N keys, 32 heads."""
    H, hd = a.heads, 128
    q = SY.normal((a.B * a.k, H * hd), 1.0, 1, "cuda", "bf16")
    kc = SY.normal((a.B, a.N, a.kv_heads, hd), 1.0, 2, "cuda", "bf16")
    vc = SY.normal((a.B, a.N, a.kv_heads, hd), 1.0, 3, "cuda", "bf16")
    o = torch.empty_like(q)
    cnt = torch.full((a.B,), a.k, dtype=torch.int32, device="cuda")
    ws = S.Workspace(S.dllm_attention_workspace_size(a.B))
    ms = _time(lambda: S.dllm_attention_bf16(q, kc, vc, o, cnt, a.k, ws=ws), a.warmup, a.iters)
    fl = 4.0 * a.B * a.k * a.N * H * hd
    return {"case": "attention", "ms": ms, "tflops": fl / ms / 1e9,
            "kv_bytes": 2 * a.B * a.N * a.kv_heads * hd * 2}


def case_attention_update(a):
    """Incremental attention of the stable rows of one 8B layer: B sequences, N - k
    stable rows each, k changed keys each (the rows the step recomputed)."""
    H, hd, Hkv = a.heads, 128, a.kv_heads
    R = a.N - a.k
    q = SY.normal((a.B * R, H * hd), 1.0, 1, "cuda", "bf16")
    o = SY.normal((a.B * R, H * hd), 0.05, 2, "cuda", "bf16")
    m = torch.zeros(a.B * R, H, dtype=torch.float32, device="cuda")
    l = torch.full((a.B * R, H), float(a.N), dtype=torch.float32, device="cuda")
    kv = [SY.normal((a.B * a.k, Hkv, hd), 1.0, 3 + i, "cuda", "bf16") for i in range(4)]
    rc = torch.full((a.B,), R, dtype=torch.int32, device="cuda")
    ac = torch.full((a.B,), a.k, dtype=torch.int32, device="cuda")
    ws = S.Workspace(S._attn_upd_ws(a.B))
    m0, l0, o0 = m.clone(), l.clone(), o.clone()

    def run():
        m.copy_(m0), l.copy_(l0), o.copy_(o0)
        S.dllm_attention_update_bf16(q, o, m, l, rc, R, kv[0], kv[1], kv[2], kv[3], ac, a.k, Hkv,
                                     ws=ws)
    reset_ms = _time(lambda: (m.copy_(m0), l.copy_(l0), o.copy_(o0)), a.warmup, a.iters)
    ms = _time(run, a.warmup, a.iters) - reset_ms
    fl = 2.0 * 2 * (2 * a.k) * R * H * hd * a.B   # QK and PV over old + new keys
    return {"case": "attention_update", "stable_rows": R, "changed": a.k, "ms": ms,
            "tflops": fl / ms / 1e9}


def case_step(a):
    """Whole partial denoising steps of the 8B model at batch B, N tokens, ratio r:
    one dense step, `--warmup` partial steps, then `--iters` timed partial steps."""
    base = SY.DENSE8B_B1_N768 if a.B == 1 else SY.DENSE8B_B32_N1536
    shape = SY.with_(base, ratio=a.ratio)
    W = SY.model_weights(shape, seed=0, device="cuda")
    model = S.Model(S.cfg_from_shape(shape), W)
    tokens = SY.prompt_tokens(shape, seed=1, device="cuda")
    cache = S.Cache(model.cfg, shape.batch, shape.seq_len)
    pol = S.make_policy(0, shape.alpha, 0, 0, shape.k, 0.0, shape.n_unmask, shape.prompt_len,
                        shape.block_len)
    ws = S.Workspace(S.dllm_step_workspace_size(model.cfg, shape.batch, shape.seq_len, pol))
    S.dllm_step(model, cache, tokens, pol, True, ws)
    ms = _time(lambda: S.dllm_step(model, cache, tokens, pol, False, ws), a.warmup, a.iters)
    return {"case": "step", "B": shape.batch, "N": shape.seq_len, "k": shape.k, "ms": ms}


def case_step_graph(a):
    """case_step, with the timed partial steps replayed from a CUDA graph (no
    per-launch host cost), as the benchmark's batch-1 figures are."""
    base = SY.DENSE8B_B1_N768 if a.B == 1 else SY.DENSE8B_B32_N1536
    shape = SY.with_(base, ratio=a.ratio)
    W = SY.model_weights(shape, seed=0, device="cuda")
    model = S.Model(S.cfg_from_shape(shape), W)
    tokens = SY.prompt_tokens(shape, seed=1, device="cuda")
    cache = S.Cache(model.cfg, shape.batch, shape.seq_len)
    pol = S.make_policy(0, shape.alpha, 0, 0, shape.k, 0.0, shape.n_unmask, shape.prompt_len,
                        shape.block_len)
    ws = S.Workspace(S.dllm_step_workspace_size(model.cfg, shape.batch, shape.seq_len, pol))
    S.dllm_step(model, cache, tokens, pol, True, ws)
    S.dllm_step(model, cache, tokens, pol, False, ws)
    graph = S.StepGraph(model, cache, tokens, pol, ws)
    ms = _time(graph.replay, a.warmup, a.iters)
    return {"case": "step_graph", "B": shape.batch, "N": shape.seq_len, "k": shape.k, "ms": ms}


def case_layer(a):
    shape = SY.with_(SY.DENSE8B_B32_N1536, n_layers=1)
    W = SY.model_weights(shape, seed=0, device="cuda")
    cfg = S.cfg_from_shape(shape)
    lw = S.layer_struct(W["layers"][0])
    kv = (a.B, a.N, shape.n_kv_heads, shape.head_dim)
    kc = SY.normal(kv, 1.0, 3, "cuda", "bf16")
    vc = SY.normal(kv, 1.0, 4, "cuda", "bf16")
    h = SY.normal((a.B, a.N, shape.d), 1.0, 5, "cuda", "bf16")
    g = torch.Generator(device="cuda")
    g.manual_seed(6)
    idx = torch.sort(torch.rand(a.B, a.N, generator=g, device="cuda").argsort(1)[:, :a.k], 1)[0]
    idx = idx.to(torch.int32).contiguous()
    cnt = torch.full((a.B,), a.k, dtype=torch.int32, device="cuda")
    x = torch.empty(a.B * a.k, shape.d, dtype=torch.bfloat16, device="cuda")
    ws = S.Workspace(S.dllm_partial_layer_workspace_size(cfg, a.B, a.N, a.k))
    ms = _time(lambda: S.dllm_partial_layer(cfg, lw, h, x, idx, cnt, kc, vc, ws, True),
               a.warmup, a.iters)
    return {"case": "partial_layer", "ms": ms}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["gemm", "score", "layer", "attention", "attention_update",
                                     "step", "step_graph"])
    ap.add_argument("--ratio", type=float, default=0.10)
    ap.add_argument("--heads", type=int, default=32)
    ap.add_argument("--kv-heads", dest="kv_heads", type=int, default=32)
    ap.add_argument("--M", type=int, default=9856)
    ap.add_argument("--N", type=int, default=12288)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--B", type=int, default=32)
    ap.add_argument("--L", type=int, default=1024)
    ap.add_argument("--d", type=int, default=4096)
    ap.add_argument("--V", type=int, default=32768)
    ap.add_argument("--Mm", type=int, default=256)
    ap.add_argument("--k", type=int, default=None,
                    help="rows per sequence (default 256 for score, 308 for layer/attention)")
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args()
    if a.k is None:
        a.k = 308 if a.case in ("layer", "attention", "attention_update") else 256
    if a.case in ("layer", "attention", "attention_update"):
        a.N = 1536 if a.N == 12288 else a.N
    out = {"gemm": case_gemm, "score": case_score, "layer": case_layer,
           "attention": case_attention, "attention_update": case_attention_update,
           "step": case_step, "step_graph": case_step_graph}[a.case](a)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
