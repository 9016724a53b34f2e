"""Plain, slow CPU oracle of one selected-token denoising step.

TEST INFRASTRUCTURE.  This module is the yardstick the CUDA library is
checked against.  It is imported only by ``tests/``, by
``__graft_entry__.smoke()`` and by the CPU-baseline legs of ``bench.py``;
the library never calls it and it never calls the library.  It shares no
code with the CUDA path: it is numpy in float64, with an optional bf16
storage emulation (round-to-nearest-even at the points where the bf16
path stores a tensor).

Sources (web pages; cited by title and section):
  [ES-de]  "ES-dLLM: Efficient Inference for Diffusion Large Language Models
           by Early-Skipping", gist.science German technical summary.
           §1 problem statement, §2.A importance-score equation, §2.B partial
           cache update / early skip, §4 results (cache size per sample).
  [ES-nl]  same paper, gist.science Dutch technical summary, "Methodologie"
           items 1-3 (importance score, early skipping, partial cache update).
  [DyLLM]  "DyLLM: Efficient Diffusion LLM Inference via Saliency-based
           Token Selection and Partial Attention", gist.science French
           technical summary, §1 problem (bidirectional attention, FFN and
           attention dominate), §2.A saliency by cosine similarity and
           threshold tau, §2.B partial attention.
  [SF-de]  "Accelerating Diffusion Large Language Models with SlowFast
           Sampling", gist.science German technical summary, §2 (top-k
           confidence unmasking in the exploratory phase).

What the pages leave open and the reading taken here (each is listed again
in the design notes):
  * The model is a pre-RMSNorm transformer block with rotate-half RoPE,
    bidirectional (unmasked) softmax attention, grouped KV heads and a
    SwiGLU FFN; no biases; untied LM head.  [DyLLM §1] only says
    "bidirectional" and "FFN"; the shape is the 8B/7B-class layout.
  * The variation score is taken on the input of the score layer l_s,
    against that row's value at its last recompute (the hidden-reference
    cache).  Default kind is 1 - cosine [DyLLM §2.A]; the ES L1 form of
    [ES-de §2.A] is the alternative.  Rows bitwise equal to their reference
    score exactly 0.
  * Importance I = alpha*c + (1-alpha)*v [ES-de §2.A]; c is the cached
    confidence for masked positions and 0 for unmasked ones.
  * Top-k ranks by (I descending, position ascending); -0 counts as +0;
    NaN ranks below everything.  Index lists are returned in ascending
    position order.
  * Threshold selection keeps the rows whose score is strictly above tau
    (with alpha = 0 and the cosine kind this is cos < 1 - tau, the
    [DyLLM §2.A] rule), capped at k_cap by the same total order.
  * Selected rows are recomputed through layers l_s..L-1; their new K/V
    rows overwrite the cache before the layer's attention runs; every
    other row keeps its cached K/V [ES-de §2.B].
  * Confidence is the max softmax probability, 1 / sum_j exp(z_j - z_max);
    argmax ties go to the lowest token id.  Only selected rows that are
    still masked get new logits; other masked rows keep their cached
    confidence (c^(t-1) of [ES-de §2.A]).
  * Unmasking reveals, in the first generation block that still holds a
    masked position, the n masked positions of highest confidence
    (ties: lower position first) [SF-de §2].
  * Over-threshold unmasking (the fast phase of [SF-de §2]): with a
    threshold tau_u > 0, every masked position of the current block whose
    confidence is strictly above tau_u is revealed; when fewer than n are
    above it, the top-n rule applies instead.  Both cases reveal the
    max(n, #above) most confident masked positions.  The stable region of
    the fast phase is read as the current block (the pages give no rule
    for the region's end point or the variance window).
  * Response-only steps [DyLLM §2.C]: rows before select_from (the prompt)
    are never selected in a partial step; their K/V stay as cached until a
    dense step injects the prompt again.
  * Two skip points [ES-de §2.B "Strategie": layers 1/8 and 1/4]: with a
    second score layer l2 > l_s, the rows selected at l_s run layers
    l_s..l2-1; at l2 every one of them is scored again, on its input of
    layer l2 against a second reference cache h_ref2 (its value at its last
    pass through l2), with the same importance formula, and each sequence
    keeps the top-k2 of its rows for layers l2..L-1 and the LM head.  Rows
    dropped at l2 keep their fresh K/V below l2 and their cached K/V from l2
    on.  A dense step writes h_ref2 for every row.
  * FFN gating [DyLLM §2.A]: with ffn_gate on, each recomputed row compares
    its attention output of the layer (the context C_{t,l}, as stored) with
    the one cached at its last pass (1 - cos); above ffn_tau the row is
    salient and runs the FFN, else it adds the FFN output cached at its last
    salient pass.  The FFN output is a stored tensor (rounded before the
    residual add) so that both branches add the same kind of value.  Dense
    steps treat every row as salient and fill both caches.
  * Approximate attention of stable rows [DyLLM §2.B]: a row that is not
    recomputed keeps its query and the statistics (max, sum, output) of its
    last exact attention; when some keys change, their old terms are taken
    out of the softmax sums and their new terms put in (reference max raised
    to cover the new scores).  Exact when the query is current; DyLLM's
    approximation when the query is stale.
  * Approximate attention inside a step [DyLLM §2.B], with the FFN gate on:
    in every layer a partial step recomputes, the rows it does not recompute
    (stable rows) keep the query, softmax statistics and attention output of
    their last pass (per-layer caches q, m, l and the context cache) and
    receive the incremental update from the keys the step changed in that
    layer (the recomputed rows' old and new K/V).  The updated output is
    their context C_{t,l} (the FFN gate's reference for later steps); their
    hidden states and K/V stay cached.  Recomputed rows write their query and
    exact statistics into the caches; a dense step writes them for every row.
  * Periodic refresh [ES-nl Methodologie 3]: in a generation, a step is
    dense (every row recomputed, every cache rewritten) at step 0, every
    refresh_every steps, and, with refresh_on_block, at the first step at
    which any sequence's current block differs from the previous step's.

Parity pins: every public function here is pinned by tests under
``tests/test_oracle_*.py`` (closed forms, textbook/library special cases,
brute force on tiny inputs, and invariants the pages state).  The quality
of the approximate method itself (accuracy on a benchmark) is not pinned:
that needs trained weights.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

F32 = "f32"
BF16 = "bf16"

SCORE_COS = 0
SCORE_ES_L1 = 1
SELECT_TOPK = 0
SELECT_THRESH = 1


# ---------------------------------------------------------------------------
# storage precision
# ---------------------------------------------------------------------------

def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even).

    bfloat16 keeps float32's 8 exponent bits and 7 explicit mantissa bits.
    Normal numbers are rounded directly on the float64 bit pattern (52 -> 7
    mantissa bits, no intermediate float32 rounding); values below the
    smallest normal float32 are rounded on the fixed 2^-133 subnormal grid.
    Values beyond the bf16 range become +-inf; NaN stays NaN.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    bits = x.view(np.uint64)
    tiny = np.abs(x) < 2.0 ** -126
    # normal range: round mantissa bits 52 -> 7 with ties to even
    keep = np.uint64(45)
    lsb = (bits >> keep) & np.uint64(1)
    bias = (np.uint64(1) << np.uint64(44)) - np.uint64(1) + lsb
    rounded = ((bits + bias) >> keep) << keep
    out_n = rounded.view(np.float64)
    # bf16 max finite = (2 - 2^-7) * 2^127; anything that rounded past it is inf
    over = np.abs(out_n) > (2.0 - 2.0 ** -7) * 2.0 ** 127
    out_n = np.where(over, np.copysign(np.inf, x), out_n)
    out[...] = out_n
    # subnormal range of bf16: multiples of 2^-133, round half to even
    if np.any(tiny):
        q = 2.0 ** -133
        out[tiny] = np.round(x[tiny] / q) * q
    nan = np.isnan(x)
    if np.any(nan):
        out[nan] = np.nan
    return out


def store(x, dtype: str) -> np.ndarray:
    """Value of ``x`` after it is written to a tensor of the path's storage dtype."""
    if dtype == BF16:
        return bf16_round(x)
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# model definition
# ---------------------------------------------------------------------------

@dataclass
class ModelCfg:
    n_layers: int
    d: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rope_theta: float = 5.0e5
    rms_eps: float = 1.0e-5
    mask_id: int = -1          # -1 means vocab - 1
    dtype: str = BF16

    def __post_init__(self):
        if self.mask_id < 0:
            self.mask_id = self.vocab - 1


@dataclass
class LayerW:
    attn_norm: np.ndarray   # [d]
    wq: np.ndarray          # [Hq*hd, d]
    wk: np.ndarray          # [Hkv*hd, d]
    wv: np.ndarray          # [Hkv*hd, d]
    wo: np.ndarray          # [d, Hq*hd]
    ffn_norm: np.ndarray    # [d]
    w_gate: np.ndarray      # [F, d]
    w_up: np.ndarray        # [F, d]
    w_down: np.ndarray      # [d, F]


@dataclass
class ModelW:
    embed: np.ndarray       # [V, d]
    layers: List[LayerW]
    final_norm: np.ndarray  # [d]
    lm_head: np.ndarray     # [V, d]


@dataclass
class Policy:
    score_layer: int = 0
    alpha: float = 0.5
    kind: int = SCORE_COS
    mode: int = SELECT_TOPK
    k: int = 0
    tau: float = 0.0
    n_unmask: int = 1
    gen_start: int = 0
    block_len: int = 32
    score_layer2: int = 0         # > score_layer: second skip point (0: none)
    k2: int = 0                   # rows per sequence kept at the second skip point
    select_from: int = 0          # positions below it are never selected (partial steps)
    ffn_gate: bool = False        # DyLLM FFN gating on the attention context
    ffn_tau: float = 0.0          # salient when 1 - cos(context, cached context) > ffn_tau
    attn_update: bool = False     # DyLLM approximate attention of stable rows (needs ffn_gate)
    unmask_tau: float = 0.0       # > 0: over-threshold unmasking with top-n fallback
    refresh_every: int = 0        # generation: dense step every R steps (0: never)
    refresh_on_block: bool = False  # generation: dense step when a block changes


@dataclass
class State:
    """Everything that persists between denoising steps (all float64 / int64)."""
    tokens: np.ndarray                  # [B, N] int
    k: List[np.ndarray]                 # per layer [B, N, Hkv, hd]
    v: List[np.ndarray]                 # per layer [B, N, Hkv, hd]
    h_ref: np.ndarray                   # [B, N, d] hidden at the score layer, last recompute
    conf: np.ndarray                    # [B, N] cached confidence
    pred: np.ndarray                    # [B, N] cached argmax token
    h_ref2: Optional[np.ndarray] = None  # [B, N, d] hidden at the second skip point
    ctx: Optional[List[np.ndarray]] = None  # per layer [B, N, Hq*hd] attention output
    ffn: Optional[List[np.ndarray]] = None  # per layer [B, N, d] FFN output
    # approximate attention: per layer the query [B, N, Hq*hd] of each row's last exact
    # pass and its softmax statistics m, l [B, N, Hq] (natural log), kept up to date
    q: Optional[List[np.ndarray]] = None
    att_m: Optional[List[np.ndarray]] = None
    att_l: Optional[List[np.ndarray]] = None

    def copy(self) -> "State":
        cp = lambda a: None if a is None else [x.copy() for x in a]
        return State(self.tokens.copy(), [a.copy() for a in self.k],
                     [a.copy() for a in self.v], self.h_ref.copy(),
                     self.conf.copy(), self.pred.copy(),
                     None if self.h_ref2 is None else self.h_ref2.copy(), cp(self.ctx),
                     cp(self.ffn), cp(self.q), cp(self.att_m), cp(self.att_l))


def empty_state(cfg: ModelCfg, tokens: np.ndarray) -> State:
    B, N = tokens.shape
    kv = (B, N, cfg.n_kv_heads, cfg.head_dim)
    return State(np.array(tokens, dtype=np.int64).copy(),
                 [np.zeros(kv) for _ in range(cfg.n_layers)],
                 [np.zeros(kv) for _ in range(cfg.n_layers)],
                 np.zeros((B, N, cfg.d)), np.zeros((B, N)),
                 np.zeros((B, N), dtype=np.int64), np.zeros((B, N, cfg.d)),
                 [np.zeros((B, N, cfg.n_heads * cfg.head_dim)) for _ in range(cfg.n_layers)],
                 [np.zeros((B, N, cfg.d)) for _ in range(cfg.n_layers)],
                 [np.zeros((B, N, cfg.n_heads * cfg.head_dim)) for _ in range(cfg.n_layers)],
                 [np.zeros((B, N, cfg.n_heads)) for _ in range(cfg.n_layers)],
                 [np.zeros((B, N, cfg.n_heads)) for _ in range(cfg.n_layers)])


# ---------------------------------------------------------------------------
# transformer sub-blocks
# ---------------------------------------------------------------------------

def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)


def rope_inv_freq(head_dim: int, theta: float) -> np.ndarray:
    """theta^(-2j/hd) for j = 0 .. hd/2-1 (the pair (j, j+hd/2) turns at this rate)."""
    j = np.arange(head_dim // 2, dtype=np.float64)
    return theta ** (-2.0 * j / head_dim)


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding.

    ``x`` is [R, H, hd]; ``pos`` is [R] (the row's token index).  The pair
    (x_j, x_{j+hd/2}) is turned by the angle pos * theta^(-2j/hd).
    ``theta == 0`` disables the rotation.
    """
    x = np.asarray(x, dtype=np.float64)
    if theta == 0.0:
        return x.copy()
    hd = x.shape[-1]
    half = hd // 2
    ang = np.asarray(pos, dtype=np.float64)[:, None] * rope_inv_freq(hd, theta)[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def softmax_rows(s: np.ndarray) -> np.ndarray:
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """Bidirectional softmax attention of R query rows over all N keys.

    q [R, Hq, hd]; K, V [N, Hkv, hd]; query head h reads KV head
    floor(h * Hkv / Hq).  No mask: every query sees every key [DyLLM §1].
    Returns [R, Hq, hd].
    """
    R, Hq, hd = q.shape
    Hkv = K.shape[1]
    out = np.empty((R, Hq, hd))
    scale = 1.0 / math.sqrt(hd)
    for h in range(Hq):
        g = (h * Hkv) // Hq
        p = softmax_rows((q[:, h, :] @ K[:, g, :].T) * scale)
        out[:, h, :] = p @ V[:, g, :]
    return out


def attention_stats(q: np.ndarray, K: np.ndarray, V: np.ndarray):
    """attention() together with each row's softmax statistics, per query head:
    m = max_j s_j and l = sum_j exp(s_j - m), s_j = q . k_j / sqrt(hd).
    Returns (m [R, Hq], l [R, Hq], o [R, Hq, hd])."""
    R, Hq, hd = q.shape
    Hkv = K.shape[1]
    m = np.empty((R, Hq))
    l = np.empty((R, Hq))
    o = np.empty((R, Hq, hd))
    scale = 1.0 / math.sqrt(hd)
    for h in range(Hq):
        g = (h * Hkv) // Hq
        s = (q[:, h, :] @ K[:, g, :].T) * scale
        m[:, h] = np.max(s, axis=1)
        e = np.exp(s - m[:, h:h + 1])
        l[:, h] = np.sum(e, axis=1)
        o[:, h, :] = (e @ V[:, g, :]) / l[:, h:h + 1]
    return m, l, o


def attention_update(q, m, l, o, K_old, V_old, K_new, V_new):
    """Attention of stable rows after some keys changed [DyLLM §2.B].

    The rows' queries q [R, Hq, hd] and statistics (m, l, o) from their last
    exact attention are reused; only the changed keys contribute work: their
    old terms are taken out of the softmax sums and their new terms put in,
    against the reference max(m, new scores).  K_old, V_old, K_new, V_new
    [A, Hkv, hd] are the changed keys' values before and after the step.  When
    (m, l, o) are exact for the old keys and q is the row's current query, the
    result is the exact attention over the updated keys; with a stale q it is
    DyLLM's approximation (weights of unchanged keys reused).
    Returns (m', l', o')."""
    R, Hq, hd = q.shape
    Hkv = K_new.shape[1]
    scale = 1.0 / math.sqrt(hd)
    m2 = np.empty((R, Hq))
    l2 = np.empty((R, Hq))
    o2 = np.empty((R, Hq, hd))
    for h in range(Hq):
        g = (h * Hkv) // Hq
        s_old = (q[:, h, :] @ K_old[:, g, :].T) * scale
        s_new = (q[:, h, :] @ K_new[:, g, :].T) * scale
        mh = m[:, h]
        if s_new.shape[1]:
            mh = np.maximum(mh, np.max(s_new, axis=1))
        w = l[:, h] * np.exp(m[:, h] - mh)
        e_old = np.exp(s_old - mh[:, None])
        e_new = np.exp(s_new - mh[:, None])
        lh = w - e_old.sum(axis=1) + e_new.sum(axis=1)
        num = w[:, None] * o[:, h, :] - e_old @ V_old[:, g, :] + e_new @ V_new[:, g, :]
        m2[:, h] = mh
        l2[:, h] = lh
        o2[:, h, :] = num / lh[:, None]
    return m2, l2, o2


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


@dataclass
class FfnGate:
    """The DyLLM FFN gate of one layer: its context and FFN-output caches
    [B, N, .], the threshold, whether every row counts as salient (dense
    steps), and (out) the salient flags of the rows."""
    ctx: np.ndarray
    ffn: np.ndarray
    tau: float
    all_rows: bool = False
    salient: Optional[np.ndarray] = None
    # approximate attention of the layer's stable rows (None: off): the query and
    # softmax statistics caches [B, N, .] of the layer
    q: Optional[np.ndarray] = None
    att_m: Optional[np.ndarray] = None
    att_l: Optional[np.ndarray] = None


def layer_rows(cfg: ModelCfg, w: LayerW, x: np.ndarray, b_of_row: np.ndarray,
               pos_of_row: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
               gate: Optional[FfnGate] = None) -> np.ndarray:
    """One transformer layer on a set of rows; updates the layer's K/V cache.

    ``x`` [R, d] are the rows' layer inputs; row r belongs to sequence
    ``b_of_row[r]`` at position ``pos_of_row[r]``.  The rows' new K/V
    overwrite the cache before attention, so each selected query sees the
    fresh K/V of every recomputed row and the cached K/V of the rest
    [ES-de §2.B].  Returns the layer outputs [R, d] (stored precision).
    """
    dt = cfg.dtype
    Hq, Hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    R = x.shape[0]
    n = store(rms_norm(x, w.attn_norm, cfg.rms_eps), dt)
    q = rope((n @ w.wq.T).reshape(R, Hq, hd), pos_of_row, cfg.rope_theta)
    k = rope((n @ w.wk.T).reshape(R, Hkv, hd), pos_of_row, cfg.rope_theta)
    v = (n @ w.wv.T).reshape(R, Hkv, hd)
    q, k, v = store(q, dt), store(k, dt), store(v, dt)
    upd = gate is not None and gate.q is not None
    if upd:
        k_old, v_old = k_cache[b_of_row, pos_of_row], v_cache[b_of_row, pos_of_row]
    k_cache[b_of_row, pos_of_row] = k
    v_cache[b_of_row, pos_of_row] = v
    o = np.empty((R, Hq, hd))
    for b in np.unique(b_of_row):
        rows = np.nonzero(b_of_row == b)[0]
        if not upd:
            o[rows] = attention(q[rows], k_cache[b], v_cache[b])
            continue
        m_b, l_b, o[rows] = attention_stats(q[rows], k_cache[b], v_cache[b])
        # DyLLM §2.B: the sequence's stable rows reuse their attention and take in
        # only the changed keys (their old terms out, their new terms in)
        N = k_cache.shape[1]
        stable = np.setdiff1d(np.arange(N), pos_of_row[rows])
        if len(stable):
            m2, l2, o2 = attention_update(gate.q[b, stable].reshape(-1, Hq, hd),
                                          gate.att_m[b, stable], gate.att_l[b, stable],
                                          gate.ctx[b, stable].reshape(-1, Hq, hd),
                                          k_old[rows], v_old[rows], k[rows], v[rows])
            gate.att_m[b, stable], gate.att_l[b, stable] = m2, l2
            gate.ctx[b, stable] = store(o2.reshape(len(stable), Hq * hd), dt)
        # the recomputed rows' query and exact statistics, for later updates
        gate.q[b, pos_of_row[rows]] = q[rows].reshape(len(rows), Hq * hd)
        gate.att_m[b, pos_of_row[rows]], gate.att_l[b, pos_of_row[rows]] = m_b, l_b
    o = store(o.reshape(R, Hq * hd), dt)
    x = store(x + o @ w.wo.T, dt)
    n2 = store(rms_norm(x, w.ffn_norm, cfg.rms_eps), dt)
    if gate is None:
        a = store(silu(n2 @ w.w_gate.T) * (n2 @ w.w_up.T), dt)
        return store(x + a @ w.w_down.T, dt)
    # DyLLM §2.A: salient rows (context moved) run the FFN, the rest reuse it
    v = variation(o, gate.ctx[b_of_row, pos_of_row], SCORE_COS)
    sal = np.ones(R, dtype=bool) if gate.all_rows else v > gate.tau
    gate.ctx[b_of_row, pos_of_row] = o
    f = gate.ffn[b_of_row, pos_of_row].copy()
    if np.any(sal):
        a = store(silu(n2[sal] @ w.w_gate.T) * (n2[sal] @ w.w_up.T), dt)
        f[sal] = store(a @ w.w_down.T, dt)
        gate.ffn[b_of_row[sal], pos_of_row[sal]] = f[sal]
    gate.salient = sal
    return store(x + f, dt)


# ---------------------------------------------------------------------------
# scoring, confidence, selection, unmasking
# ---------------------------------------------------------------------------

def variation(h_cur: np.ndarray, h_ref: np.ndarray, kind: int) -> np.ndarray:
    """Per-row variation of the hidden state since the row's last recompute.

    kind SCORE_COS:   1 - cos(h, h_ref) [DyLLM §2.A].
    kind SCORE_ES_L1: ||h - h_ref||_1 / (sqrt(d) * ||h_ref||_2) [ES-de §2.A].
    Rows bitwise equal to their reference give exactly 0.  For the cosine a
    zero-norm row against a non-zero one gives cos = 0 (v = 1); for the L1
    form a zero reference against a different row gives +inf.
    """
    h = np.asarray(h_cur, dtype=np.float64)
    r = np.asarray(h_ref, dtype=np.float64)
    d = h.shape[-1]
    same = np.all(h == r, axis=-1)
    if kind == SCORE_COS:
        dot = np.sum(h * r, axis=-1)
        nn = np.sqrt(np.sum(h * h, axis=-1)) * np.sqrt(np.sum(r * r, axis=-1))
        with np.errstate(divide="ignore", invalid="ignore"):
            cos = np.where(nn > 0, dot / np.where(nn > 0, nn, 1.0), 0.0)
        v = 1.0 - cos
    elif kind == SCORE_ES_L1:
        l1 = np.sum(np.abs(h - r), axis=-1)
        nr = np.sqrt(np.sum(r * r, axis=-1))
        with np.errstate(divide="ignore", invalid="ignore"):
            v = np.where(nr > 0, l1 / (math.sqrt(d) * np.where(nr > 0, nr, 1.0)), np.inf)
    else:
        raise ValueError("unknown score kind")
    return np.where(same, 0.0, v)


def importance(v: np.ndarray, conf: np.ndarray, masked: np.ndarray, alpha: float) -> np.ndarray:
    """I = alpha * c + (1 - alpha) * v, with c = cached confidence on masked
    positions and 0 elsewhere [ES-de §2.A]."""
    c = np.where(np.asarray(masked, dtype=bool), np.asarray(conf, dtype=np.float64), 0.0)
    return alpha * c + (1.0 - alpha) * np.asarray(v, dtype=np.float64)


def confidence(logits: np.ndarray):
    """Max softmax probability and argmax of each row of ``logits`` [..., V].

    conf = 1 / sum_j exp(z_j - z_max); ties of the maximum go to the lowest id.
    """
    z = np.asarray(logits, dtype=np.float64)
    zmax = np.max(z, axis=-1, keepdims=True)
    conf = 1.0 / np.sum(np.exp(z - zmax), axis=-1)
    pred = np.argmax(z, axis=-1)  # first occurrence = lowest id
    return conf, pred.astype(np.int64)


def _rank_key(value: float, pos: int):
    """Total order for selection: larger value first, NaN last, lower position first."""
    v = float(value)
    if math.isnan(v):
        return (0, 0.0, -pos)
    if v == 0.0:
        v = 0.0  # -0 counts as +0
    return (1, v, -pos)


def select_topk(scores: np.ndarray, k: int) -> np.ndarray:
    """The k highest-ranked positions of one sequence, ascending by position."""
    n = len(scores)
    k = max(0, min(int(k), n))
    order = sorted(range(n), key=lambda i: _rank_key(scores[i], i), reverse=True)
    return np.array(sorted(order[:k]), dtype=np.int64)


def select_thresh(scores: np.ndarray, tau: float, k_cap: int):
    """Positions with score > tau (strict), capped at k_cap by the top-k order.

    Returns (idx ascending, number over the threshold before the cap).
    """
    over = [i for i in range(len(scores))
            if not math.isnan(float(scores[i])) and float(scores[i]) > tau]
    n_over = len(over)
    if n_over > k_cap:
        over = sorted(over, key=lambda i: _rank_key(scores[i], i), reverse=True)[:k_cap]
    return np.array(sorted(over), dtype=np.int64), n_over


def select(scores: np.ndarray, mode: int, k: int, tau: float, k_cap: int, lo: int = 0):
    """Per-sequence selection over scores [B, N] -> list of ascending index arrays.
    Only positions >= lo are candidates (response-only steps, [DyLLM §2.C])."""
    out = []
    for b in range(scores.shape[0]):
        sub = scores[b, lo:]
        if mode == SELECT_TOPK:
            out.append(lo + select_topk(sub, min(k, k_cap)))
        else:
            out.append(lo + select_thresh(sub, tau, k_cap)[0])
    return out


def current_block(tokens_b: np.ndarray, mask_id: int, gen_start: int, block_len: int):
    """[start, end) of the first generation block that still has a masked position."""
    N = len(tokens_b)
    m = np.nonzero(tokens_b[gen_start:] == mask_id)[0]
    if len(m) == 0:
        return None
    first = gen_start + int(m[0])
    start = gen_start + ((first - gen_start) // block_len) * block_len
    return start, min(start + block_len, N)


def unmask_positions(conf_b, tokens_b, mask_id: int, gen_start: int, block_len: int, n: int,
                     tau: float = 0.0):
    """Positions revealed in one sequence this step, ascending [SF-de §2].
    tau > 0: every masked position of the block with conf > tau, or the top n
    when fewer than n are above it."""
    blk = current_block(tokens_b, mask_id, gen_start, block_len)
    if blk is None or n <= 0:
        return np.zeros(0, dtype=np.int64)
    cand = [p for p in range(blk[0], blk[1]) if tokens_b[p] == mask_id]
    take = n
    if tau > 0:
        above = [p for p in cand if float(conf_b[p]) > tau]
        take = max(n, len(above))
    cand.sort(key=lambda p: _rank_key(conf_b[p], p), reverse=True)
    return np.array(sorted(cand[:take]), dtype=np.int64)


def unmask_capacity(n: int, block_len: int, tau: float) -> int:
    """Most positions one sequence can reveal in a step."""
    return max(n, block_len) if tau > 0 else n


def unmask(conf, pred, tokens, mask_id, gen_start, block_len, n, tau: float = 0.0):
    """Applies the unmask rule to every sequence in place; returns pos [B, cap] padded with -1."""
    B = tokens.shape[0]
    pos = -np.ones((B, max(unmask_capacity(n, block_len, tau), 0)), dtype=np.int64)
    for b in range(B):
        p = unmask_positions(conf[b], tokens[b], mask_id, gen_start, block_len, n, tau)
        tokens[b, p] = pred[b, p]
        pos[b, :len(p)] = p
    return pos


def apply_unmask(pred, tokens, pos):
    """Reveals given positions (-1 entries are ignored); used with forced decisions."""
    for b in range(tokens.shape[0]):
        p = pos[b][pos[b] >= 0]
        tokens[b, p] = pred[b, p]


# ---------------------------------------------------------------------------
# the standalone score call (confidence from logits, then importance)
# ---------------------------------------------------------------------------

def score_call(h_cur, h_ref, conf, pred, masked, alpha, kind,
               logits=None, logit_pos=None):
    """Confidence refresh from logits (if given) followed by importance scores.

    logits [B, Mm, V] belong to positions logit_pos [B, Mm]; their max-softmax
    confidence and argmax overwrite conf/pred there first.  Returns
    (scores [B, N], conf, pred) as new arrays.
    """
    conf = np.array(conf, dtype=np.float64)
    pred = np.array(pred, dtype=np.int64)
    if logits is not None:
        c, p = confidence(logits)
        for b in range(conf.shape[0]):
            conf[b, logit_pos[b]] = c[b]
            pred[b, logit_pos[b]] = p[b]
    v = variation(h_cur, h_ref, kind)
    return importance(v, conf, masked, alpha), conf, pred


# ---------------------------------------------------------------------------
# one denoising step
# ---------------------------------------------------------------------------

@dataclass
class StepOut:
    idx: List[np.ndarray]          # per sequence, ascending
    scores: Optional[np.ndarray]   # [B, N] or None for a dense step
    unmasked: np.ndarray           # [B, n] padded with -1
    final_rows: List[np.ndarray] = field(default_factory=list)  # per sequence [k_b, d]
    idx2: Optional[List[np.ndarray]] = None   # rows kept at the second skip point
    scores2: Optional[List[np.ndarray]] = None  # their scores, per sequence in idx order
    ffn_rows: Optional[List[int]] = None  # FFN gating: salient rows per recomputed layer
    # FFN gating: per recomputed layer, the salient flag of each compact row (rows packed
    # by sequence, ascending positions; after a second skip point, the kept rows)
    ffn_salient: Optional[List[np.ndarray]] = None


def embed(W: ModelW, tokens: np.ndarray) -> np.ndarray:
    return np.asarray(W.embed, dtype=np.float64)[tokens]


def dense_layers(cfg: ModelCfg, W: ModelW, st: State, h: np.ndarray, upto: int,
                 gate_on: bool = False) -> np.ndarray:
    """Layers 0 .. upto-1 on every row (writes every row's K/V there)."""
    B, N, d = h.shape
    b_of = np.repeat(np.arange(B), N)
    p_of = np.tile(np.arange(N), B)
    x = h.reshape(B * N, d)
    for l in range(upto):
        gate = FfnGate(st.ctx[l], st.ffn[l], 0.0, True) if gate_on else None
        x = layer_rows(cfg, W.layers[l], x, b_of, p_of, st.k[l], st.v[l], gate)
    return x.reshape(B, N, d)


def narrow(st: State, pol: Policy, masked: np.ndarray, x: np.ndarray, b_of: np.ndarray,
           p_of: np.ndarray, forced_idx2=None):
    """The second skip point: score the compact rows on their input of layer
    score_layer2 against h_ref2, keep each sequence's top-k2 (ES-de §2.A, §2.B).
    Returns (kept positions per sequence, their scores per sequence, keep mask)."""
    B = st.tokens.shape[0]
    I2 = importance(variation(x, st.h_ref2[b_of, p_of], pol.kind), st.conf[b_of, p_of],
                    masked[b_of, p_of], pol.alpha)
    idx2, sc2 = [], []
    for b in range(B):
        rows = np.nonzero(b_of == b)[0]          # ascending positions
        sc2.append(I2[rows])
        if forced_idx2 is not None:
            idx2.append(np.asarray(forced_idx2[b], dtype=np.int64))
        else:
            idx2.append(p_of[rows][select_topk(I2[rows], pol.k2)])
    keep = np.zeros(len(b_of), dtype=bool)
    for b in range(B):
        keep |= (b_of == b) & np.isin(p_of, idx2[b])
    return idx2, sc2, keep


def step(cfg: ModelCfg, W: ModelW, st: State, pol: Policy, dense: bool,
         forced_idx=None, forced_unmask=None, k_cap: Optional[int] = None,
         forced_idx2=None) -> StepOut:
    """One denoising step, in place on ``st``.

    1. embed the tokens; run layers below the score layer on every row;
    2. score every row and select (skipped when ``dense``: all rows);
    3. store the selected rows' score-layer hidden into the reference cache;
    4. recompute the selected rows through the remaining layers, updating
       their K/V rows in each layer's cache [ES-de §2.B, ES-nl Methodologie 3];
    5. logits -> confidence / argmax for selected rows that are masked;
    6. unmask in the current block [SF-de §2].
    ``forced_idx`` / ``forced_unmask`` replace the decisions of steps 2 / 6.
    """
    B, N = st.tokens.shape
    ls = pol.score_layer
    masked = st.tokens == cfg.mask_id
    h = embed(W, st.tokens)
    h = dense_layers(cfg, W, st, h, ls, pol.ffn_gate)
    scores = None
    if dense:
        idx = [np.arange(N, dtype=np.int64) for _ in range(B)]
    elif forced_idx is not None:
        idx = [np.asarray(a, dtype=np.int64) for a in forced_idx]
    else:
        v = variation(h, st.h_ref, pol.kind)
        scores = importance(v, st.conf, masked, pol.alpha)
        kc = k_cap if k_cap is not None else (pol.k if pol.mode == SELECT_TOPK else N)
        idx = select(scores, pol.mode, pol.k, pol.tau, kc, pol.select_from)
    b_of = np.concatenate([np.full(len(a), b, dtype=np.int64) for b, a in enumerate(idx)])
    p_of = np.concatenate(idx) if len(idx) else np.zeros(0, dtype=np.int64)
    x = h[b_of, p_of]
    st.h_ref[b_of, p_of] = x
    l2 = pol.score_layer2 if pol.score_layer2 > ls else -1
    idx2 = sc2 = None
    ffn_rows = [] if pol.ffn_gate else None
    ffn_sal = [] if pol.ffn_gate else None
    for l in range(ls, cfg.n_layers):
        if l == l2:
            if not dense:
                idx2, sc2, keep = narrow(st, pol, masked, x, b_of, p_of, forced_idx2)
                b_of, p_of, x = b_of[keep], p_of[keep], x[keep]
            st.h_ref2[b_of, p_of] = x
        if len(b_of):
            gate = FfnGate(st.ctx[l], st.ffn[l], pol.ffn_tau, dense) if pol.ffn_gate else None
            if gate is not None and pol.attn_update:
                gate.q, gate.att_m, gate.att_l = st.q[l], st.att_m[l], st.att_l[l]
            x = layer_rows(cfg, W.layers[l], x, b_of, p_of, st.k[l], st.v[l], gate)
            if gate is not None:
                ffn_rows.append(int(np.sum(gate.salient)))
                ffn_sal.append(gate.salient.copy())
    sel_masked = masked[b_of, p_of]
    if np.any(sel_masked):
        n = store(rms_norm(x[sel_masked], W.final_norm, cfg.rms_eps), cfg.dtype)
        c, p = confidence(n @ np.asarray(W.lm_head, dtype=np.float64).T)
        st.conf[b_of[sel_masked], p_of[sel_masked]] = c
        st.pred[b_of[sel_masked], p_of[sel_masked]] = p
    if forced_unmask is not None:
        pos = np.asarray(forced_unmask, dtype=np.int64)
        apply_unmask(st.pred, st.tokens, pos)
    else:
        pos = unmask(st.conf, st.pred, st.tokens, cfg.mask_id, pol.gen_start,
                     pol.block_len, pol.n_unmask, pol.unmask_tau)
    rows = []
    off = 0
    for a in (idx2 if idx2 is not None else idx):
        rows.append(x[off:off + len(a)].copy())
        off += len(a)
    return StepOut(idx, scores, pos, rows, idx2, sc2, ffn_rows, ffn_sal)


def block_starts(cfg: ModelCfg, pol: Policy, tokens: np.ndarray) -> List[int]:
    """Start of each sequence's current block (-1 once it has no masked position)."""
    out = []
    for b in range(tokens.shape[0]):
        blk = current_block(tokens[b], cfg.mask_id, pol.gen_start, pol.block_len)
        out.append(-1 if blk is None else blk[0])
    return out


def generate(cfg: ModelCfg, W: ModelW, st: State, pol: Policy, n_steps: int):
    """n_steps denoising steps with the periodic refresh of [ES-nl Methodologie 3]:
    a step is dense at t = 0, at every multiple of refresh_every, and (with
    refresh_on_block) when any sequence's current block differs from the one
    it had at the previous step.  Returns (dense flags, revealed positions)."""
    dense_log, pos_log = [], []
    prev = None
    for t in range(n_steps):
        blocks = block_starts(cfg, pol, st.tokens)
        dense = (t == 0 or (pol.refresh_every > 0 and t % pol.refresh_every == 0)
                 or (pol.refresh_on_block and prev is not None and blocks != prev))
        prev = blocks
        out = step(cfg, W, st, pol, dense)
        dense_log.append(bool(dense))
        pos_log.append(out.unmasked)
    return dense_log, pos_log


def dense_forward(cfg: ModelCfg, W: ModelW, tokens: np.ndarray) -> np.ndarray:
    """Full recomputation of every row through every layer (the vanilla pass);
    returns the final hidden rows [B, N, d]."""
    st = empty_state(cfg, tokens)
    return dense_layers(cfg, W, st, embed(W, st.tokens), cfg.n_layers)


def kv_cache_bytes(n_layers: int, n_tokens: int, n_kv_heads: int, head_dim: int,
                   bytes_per_elem: int = 2) -> int:
    """Bytes of the per-layer K and V caches of one sequence."""
    return 2 * n_layers * n_tokens * n_kv_heads * head_dim * bytes_per_elem
