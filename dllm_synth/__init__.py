"""Seeded synthetic inputs for the selected-token denoising step.

This module only draws random numbers and lays out shapes; it holds none
of the method's arithmetic.  Both the CUDA path (through the tests and the
benchmark) and the CPU oracle receive the bits it produces.

Generators: ``torch.Generator`` on the requested device (CPU: Mersenne
Twister; CUDA: Philox).  A tensor is a function of (seed, tensor id,
device): the same call on the same device always returns the same bits.
Large inputs are drawn on the GPU; when the oracle needs them they are
copied to the host unchanged (an input copy, never an output).
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Dict, List, Optional

import torch


@dataclass(frozen=True)
class Shape:
    """A model shape plus the workload it runs (batch, lengths, schedule)."""
    name: str
    n_layers: int
    d: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rope_theta: float
    dtype: str            # "f32" or "bf16"
    batch: int
    prompt_len: int
    gen_len: int
    block_len: int
    n_unmask: int
    ratio: float          # recompute ratio of a partial step
    alpha: float
    score_layer: int = 0
    rms_eps: float = 1e-5
    w_std: float = 0.02

    @property
    def seq_len(self) -> int:
        return self.prompt_len + self.gen_len

    @property
    def mask_id(self) -> int:
        return self.vocab - 1

    @property
    def k(self) -> int:
        """Rows recomputed per sequence: ceil(ratio * N)."""
        import math
        return int(math.ceil(self.ratio * self.seq_len - 1e-9))


# The workloads.  Names say what each is.
TINY = Shape("tiny_1L_d256_f32_B1_N128", 1, 256, 4, 4, 64, 688, 1024, 5.0e5, "f32",
             1, 64, 64, 64, 8, 0.25, 0.0)
DENSE8B_B1_N768 = Shape("8B_B1_N768", 32, 4096, 32, 32, 128, 12288, 126464, 5.0e5, "bf16",
                        1, 512, 256, 32, 8, 0.10, 0.5)
DENSE8B_B32_N1536 = Shape("8B_B32_N1536_r20", 32, 4096, 32, 32, 128, 12288, 126464, 5.0e5,
                          "bf16", 32, 512, 1024, 64, 16, 0.20, 0.5)
GQA7B_B8_N2048 = Shape("7B_GQA_B8_N2048", 28, 3584, 28, 4, 128, 18944, 152064, 5.0e5, "bf16",
                       8, 1024, 1024, 64, 16, 0.05, 0.5)

SHAPES: Dict[str, Shape] = {s.name: s for s in (TINY, DENSE8B_B1_N768, DENSE8B_B32_N1536,
                                                 GQA7B_B8_N2048)}


def with_(shape: Shape, **kw) -> Shape:
    """A copy of ``shape`` with fields replaced (fewer layers, smaller batch, ...)."""
    return replace(shape, **kw)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def _tensor_seed(seed: int, tid: int) -> int:
    # distinct, reproducible stream per tensor (plain integer mixing of two ids)
    return (seed * 1000003 + tid * 7919 + 12345) & 0x7FFFFFFF


def torch_dtype(dtype: str):
    return torch.float32 if dtype == "f32" else torch.bfloat16


def normal(shape, std: float, seed: int, device="cpu", dtype="bf16") -> torch.Tensor:
    """N(0, std^2) samples in float32, then cast to the storage dtype (RNE)."""
    g = _gen(seed, device)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch_dtype(dtype)) if dtype != "f32" else t


def model_weights(s: Shape, seed: int = 0, device="cpu") -> Dict[str, object]:
    """Random-init weights: matrices N(0, w_std^2), norm gains 1, no biases.

    Returns {"embed", "final_norm", "lm_head", "layers": [dict per layer]},
    weights row-major [out, in].
    """
    dt = s.dtype
    q_out = s.n_heads * s.head_dim
    kv_out = s.n_kv_heads * s.head_dim
    tid = 0

    def mat(rows, cols):
        nonlocal tid
        tid += 1
        return normal((rows, cols), s.w_std, _tensor_seed(seed, tid), device, dt)

    def ones(n):
        return torch.ones(n, device=device, dtype=torch_dtype(dt))

    W = {"embed": mat(s.vocab, s.d), "layers": []}
    for _ in range(s.n_layers):
        W["layers"].append({
            "attn_norm": ones(s.d), "wq": mat(q_out, s.d), "wk": mat(kv_out, s.d),
            "wv": mat(kv_out, s.d), "wo": mat(s.d, q_out), "ffn_norm": ones(s.d),
            "w_gate": mat(s.ffn, s.d), "w_up": mat(s.ffn, s.d), "w_down": mat(s.d, s.ffn),
        })
    W["final_norm"] = ones(s.d)
    W["lm_head"] = mat(s.vocab, s.d)
    return W


def prompt_tokens(s: Shape, seed: int = 1, device="cpu") -> torch.Tensor:
    """[B, N] int32: uniform prompt ids in [0, vocab-2], then gen_len [MASK] ids."""
    g = _gen(seed, device)
    B, P, N = s.batch, s.prompt_len, s.seq_len
    t = torch.full((B, N), s.mask_id, dtype=torch.int32, device=device)
    if P:
        t[:, :P] = torch.randint(0, s.vocab - 1, (B, P), generator=g, device=device,
                                 dtype=torch.int32)
    return t


@dataclass
class ScoreInputs:
    h_cur: torch.Tensor      # [B, L, d]
    h_ref: torch.Tensor      # [B, L, d]
    logits: torch.Tensor     # [B, Mm, V]
    logit_pos: torch.Tensor  # [B, Mm] int32
    masked: torch.Tensor     # [B, L] uint8
    conf: torch.Tensor       # [B, L] float32 (cached confidence before the refresh)
    pred: torch.Tensor       # [B, L] int32
    changed: torch.Tensor    # [B, L] bool (rows given the large perturbation)


def score_inputs(B=32, L=1024, d=4096, V=32768, Mm=256, p_changed=0.2, sd_changed=0.5,
                 sd_same=1e-3, logit_sd=2.0, seed: int = 1, device="cpu",
                 dtype="bf16") -> ScoreInputs:
    """Inputs of the standalone score + select workload.

    h_cur ~ N(0,1); h_ref = h_cur + N(0, sd_changed^2) on a Bernoulli(p_changed)
    subset of rows and + N(0, sd_same^2) elsewhere; logits ~ N(0, logit_sd^2)
    for the last Mm positions of each sequence (the masked ones).
    """
    g = _gen(seed, device)
    h_cur32 = torch.randn(B, L, d, generator=g, device=device)
    changed = torch.rand(B, L, generator=g, device=device) < p_changed
    noise = torch.randn(B, L, d, generator=g, device=device)
    sd = torch.where(changed, torch.tensor(sd_changed, device=device),
                     torch.tensor(sd_same, device=device))
    h_ref32 = h_cur32 + noise * sd[..., None]
    del noise
    td = torch_dtype(dtype)
    h_cur = h_cur32.to(td)
    del h_cur32
    h_ref = h_ref32.to(td)
    del h_ref32
    logits = (torch.randn(B, Mm, V, generator=g, device=device) * logit_sd).to(td)
    logit_pos = torch.arange(L - Mm, L, device=device, dtype=torch.int32).repeat(B, 1)
    masked = torch.zeros(B, L, dtype=torch.uint8, device=device)
    masked[:, L - Mm:] = 1
    conf = torch.rand(B, L, generator=g, device=device) * 0.5
    pred = torch.zeros(B, L, dtype=torch.int32, device=device)
    return ScoreInputs(h_cur.contiguous(), h_ref.contiguous(), logits.contiguous(),
                       logit_pos.contiguous(), masked, conf.contiguous(), pred, changed)


def hidden_rows(rows: int, d: int, seed: int, device="cpu", dtype="bf16", std=1.0):
    """Generic N(0, std^2) activations [rows, d]."""
    return normal((rows, d), std, seed, device, dtype)
