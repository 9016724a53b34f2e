"""Helpers shared by the tests: conversions between synthetic torch inputs
and the oracle's float64 arrays, and the error metric."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from dllm_synth import Shape


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_cfg(s: Shape) -> O.ModelCfg:
    return O.ModelCfg(s.n_layers, s.d, s.n_heads, s.n_kv_heads, s.head_dim, s.ffn, s.vocab,
                      s.rope_theta, s.rms_eps, s.mask_id, s.dtype)


def oracle_weights(W) -> O.ModelW:
    layers = [O.LayerW(**{k: f64(v) for k, v in L.items()}) for L in W["layers"]]
    return O.ModelW(f64(W["embed"]), layers, f64(W["final_norm"]), f64(W["lm_head"]))


def oracle_policy(s: Shape, **kw) -> O.Policy:
    p = O.Policy(score_layer=s.score_layer, alpha=s.alpha, kind=O.SCORE_COS,
                 mode=O.SELECT_TOPK, k=s.k, tau=0.0, n_unmask=s.n_unmask,
                 gen_start=s.prompt_len, block_len=s.block_len)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def max_abs_rel(gpu, ora) -> float:
    """max_i |gpu_i - ora_i| / max_i |ora_i| (0 when both are all zero)."""
    g = np.asarray(gpu, dtype=np.float64)
    o = np.asarray(ora, dtype=np.float64)
    den = np.max(np.abs(o)) if o.size else 0.0
    num = np.max(np.abs(g - o)) if o.size else 0.0
    if den == 0.0:
        return float(num)
    return float(num / den)


# tolerances fixed by the method statement: fp32 1e-4, bf16 2e-2 (max-abs-relative)
TOL = {"f32": 1e-4, "bf16": 2e-2}
