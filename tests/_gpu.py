"""Helpers for the GPU parity tests: build the library model from seeded
synthetic weights, mirror it for the oracle, compare argmax decisions."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import dllm_synth as SY
from _util import f64, oracle_cfg, oracle_weights


def to_dev(W, device="cuda"):
    out = {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in W.items() if k != "layers"}
    out["layers"] = [{k: v.to(device) for k, v in L.items()} for L in W["layers"]]
    return out


def build(shape, seed=0, device="cuda", weights_on_gpu=False):
    """(library Model, oracle cfg, oracle weights, host weights)."""
    import sparse_token_recompute_b200 as S
    if weights_on_gpu:
        Wd = SY.model_weights(shape, seed=seed, device=device)
        Wh = None
    else:
        Wh = SY.model_weights(shape, seed=seed, device="cpu")
        Wd = to_dev(Wh, device)
    model = S.Model(S.cfg_from_shape(shape), Wd)
    return model, oracle_cfg(shape), Wd, Wh


def oracle_w_from(Wd_or_h):
    return oracle_weights(Wd_or_h)


def argmax_ok(gpu_pred, logits_row, tol):
    """A different argmax is accepted only when the two logits are a near tie:
    within twice the logit tolerance (max-abs-relative `tol`, so each side may be
    off by tol * max|z|) of the oracle's maximum."""
    z = np.asarray(logits_row, dtype=np.float64)
    return (z.max() - z[int(gpu_pred)]) <= 2.0 * tol * np.abs(z).max()


def state_from_cache(cache, tokens) -> O.State:
    return O.State(f64(tokens).astype(np.int64), [f64(t) for t in cache.k],
                   [f64(t) for t in cache.v], f64(cache.h_ref), f64(cache.conf),
                   f64(cache.pred).astype(np.int64))
