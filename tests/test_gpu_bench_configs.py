"""GPU parity of whole denoising steps in the launch configurations the
benchmark times, at full model width and vocabulary with 2 of the layers.

* 8B, one sequence of 768 tokens (ES-dLLM, German summary §2.B, partial cache
  update): the dense first step, then partial steps at 10 %, 25 % and 50 %
  recompute (77, 192 and 384 rows).  These run the weight-streaming GEMM plans
  (K split across a thread-block cluster with the residual epilogue at
  K = 12288, the QKV epilogue on CTA pairs at 192 rows) and the attention whose
  keys are shared among three CTAs.
* 8B, 32 sequences of 1536 tokens, 308 rows each (the headline step), and 7B
  GQA, 8 sequences of 2048 tokens at 5 % and 25 %: one partial step of the
  whole batch on the GPU from a seeded cache state.  A sequence's outputs
  depend only on its own rows and caches, so the oracle computes a sample of
  the sequences and every cache row of those sequences is compared.
* 7B GQA, 2 of its 8 sequences: the dense first step and partial steps at 5 %
  and 25 %.

Decisions (index lists, revealed positions) are the oracle's, given to the
GPU through the forced arguments; the tolerance is the bf16 one.
"""
import numpy as np
import pytest
import torch

import oracle as O
import dllm_synth as SY
from _util import f64, max_abs_rel, TOL, oracle_cfg, oracle_policy
from _gpu import to_dev, oracle_w_from, argmax_ok
from test_gpu_step import Run

pytestmark = pytest.mark.gpu

_WEIGHTS = {}


def _weights(shape):
    """(host weights, oracle weights, device weights), one draw shared by the tests
    of one model shape."""
    key = (shape.name, shape.n_layers)
    if key not in _WEIGHTS:
        _WEIGHTS.clear()
        torch.cuda.empty_cache()
        Wh = SY.model_weights(shape, seed=0, device="cpu")
        _WEIGHTS[key] = (Wh, oracle_w_from(Wh), to_dev(Wh))
    return _WEIGHTS[key]


def _set_k(r, k):
    """Change the recompute count of a Run between steps (its workspace covers it)."""
    r.pol.k = k
    r.opol.k = k
    r.k_cap = max(1, min(k, r.N))


def _plan(lib, kind, M, K, segs, hd=0):
    return lib.dllm_gemm_plan_info(kind, M, K, segs, hd)


def test_8b_single_sequence_dense_then_10_25_50(lib):
    shape = SY.with_(SY.DENSE8B_B1_N768, n_layers=2, ratio=0.50)
    d, F = shape.d, shape.ffn
    # the plans these row counts run (the same as the benchmark's 32-layer steps)
    assert _plan(lib, "residual", 77, F, [d])["splits"] > 1           # cluster split-K, K 12288
    assert _plan(lib, "qkv", 192, d, [d, d, d], 128)["pair"] == 1      # QKV on CTA pairs
    r = Run(lib, shape, prebuilt=_weights(shape))   # workspace sized for the 50 % step
    k_of = {0.10: 77, 0.25: 192, 0.50: 384}
    ratios = [None, 0.10, 0.25, 0.50]
    for t, ratio in enumerate(ratios):
        if ratio is not None:
            assert SY.with_(shape, ratio=ratio).k == k_of[ratio]
            _set_k(r, k_of[ratio])
        out = O.step(r.ocfg, r.ow, r.st, r.opol, dense=(t == 0))
        r.gpu_step(t == 0, None if t == 0 else out.idx, out.unmasked)
        r.compare_tokens(r.compare_state(TOL["bf16"], out.final_rows, out.idx))


def _synthetic_state_run(lib, shape, seed):
    """A Run whose caches hold seeded synthetic values (as after earlier steps):
    K/V ~ N(0, 1), hidden references ~ N(0, 0.02^2), confidences U(0, 1),
    predictions uniform ids; tokens: the prompt, then generated positions of
    which the first block is half revealed.  Returns the Run."""
    r = Run(lib, shape, prebuilt=_weights(shape))
    B, N = r.B, r.N
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    for l in range(shape.n_layers):
        r.cache.k[l].copy_(SY.normal(r.cache.k[l].shape, 1.0, seed + 10 + l, "cuda", "bf16"))
        r.cache.v[l].copy_(SY.normal(r.cache.v[l].shape, 1.0, seed + 50 + l, "cuda", "bf16"))
    r.cache.h_ref.copy_(SY.normal(r.cache.h_ref.shape, 0.02, seed + 90, "cuda", "bf16"))
    r.cache.conf.copy_(torch.rand(B, N, generator=g, device="cuda"))
    r.cache.pred.copy_(torch.randint(0, shape.vocab - 1, (B, N), generator=g, device="cuda",
                                     dtype=torch.int32))
    P, bl = shape.prompt_len, shape.block_len
    reveal = torch.rand(B, bl, generator=g, device="cuda") < 0.5
    blk = r.tokens[:, P:P + bl]
    blk.copy_(torch.where(reveal, r.cache.pred[:, P:P + bl], blk))
    return r


def _sub_state(r, seqs):
    c = r.cache
    s = lambda t: f64(t[seqs])
    return O.State(s(r.tokens).astype(np.int64), [s(t) for t in c.k], [s(t) for t in c.v],
                   s(c.h_ref), s(c.conf), s(c.pred).astype(np.int64))


def _sampled_partial_step(lib, shape, seqs, seed):
    r = _synthetic_state_run(lib, shape, seed)
    B, N, k = r.B, r.N, shape.k
    # index lists: k positions per sequence drawn without replacement (seeded)
    g = torch.Generator().manual_seed(seed + 1)
    idx = [np.sort(torch.randperm(N, generator=g)[:k].numpy()).astype(np.int64)
           for _ in range(B)]
    st = _sub_state(r, seqs)
    out = O.step(r.ocfg, r.ow, st, r.opol, dense=False, forced_idx=[idx[b] for b in seqs])
    cap = max(lib.dllm_unmask_capacity(r.pol), 1)
    unm = np.full((B, cap), -1, dtype=np.int64)       # other sequences reveal nothing
    for j, b in enumerate(seqs):
        unm[b] = out.unmasked[j]
    r.gpu_step(False, idx, unm)
    c = r.cache
    for j, b in enumerate(seqs):
        for l in range(shape.n_layers):
            assert max_abs_rel(f64(c.k[l][b]), st.k[l][j]) < TOL["bf16"], ("k", b, l)
            assert max_abs_rel(f64(c.v[l][b]), st.v[l][j]) < TOL["bf16"], ("v", b, l)
        assert max_abs_rel(f64(c.h_ref[b]), st.h_ref[j]) < TOL["bf16"], ("h_ref", b)
        def logits(p):
            row = int(np.nonzero(idx[b] == p)[0][0])
            n = O.store(O.rms_norm(out.final_rows[j][row], r.ow.final_norm, r.ocfg.rms_eps),
                        r.ocfg.dtype)
            return n @ r.ow.lm_head.T
        cg, co = f64(c.conf[b]), st.conf[j]
        for p in np.nonzero(np.abs(cg - co) >= TOL["bf16"] * np.abs(co).max())[0]:
            # ln conf = z_max - logsumexp(z) moves by at most twice a logit error
            z = logits(p)
            assert abs(np.log(cg[p]) - np.log(co[p])) <= 2 * TOL["bf16"] * np.abs(z).max(), (b, p)
        gp = f64(c.pred[b]).astype(np.int64)
        tie = np.zeros(N, dtype=bool)
        for p in np.nonzero(gp != st.pred[j])[0]:
            # a different argmax must be a near tie of the oracle's logits
            assert argmax_ok(gp[p], logits(p), TOL["bf16"]), (b, p)
            tie[p] = True
        # revealed tokens: the forced positions took the (GPU's) prediction
        gt = f64(r.tokens[b]).astype(np.int64)
        np.testing.assert_array_equal(gt[~tie], st.tokens[j][~tie])
    return r


def test_8b_headline_batch_partial_step_sampled(lib):
    """32 x 1536 tokens, 308 rows per sequence: the GEMMs on CTA pairs with the
    QKV/residual epilogues, gate/up on single CTAs, the LM head over 126464 ids."""
    shape = SY.with_(SY.DENSE8B_B32_N1536, n_layers=2)
    assert shape.k == 308 and shape.batch == 32
    _sampled_partial_step(lib, shape, [0, 13, 31], seed=101)


@pytest.mark.parametrize("ratio,k", [(0.05, 103), (0.25, 512)])
def test_7b_gqa_batch_partial_step_sampled(lib, ratio, k):
    shape = SY.with_(SY.GQA7B_B8_N2048, n_layers=2, ratio=ratio)
    assert shape.k == k and shape.batch == 8
    _sampled_partial_step(lib, shape, [0, 5], seed=202)


def test_7b_gqa_two_sequences_dense_then_5_25(lib):
    shape = SY.with_(SY.GQA7B_B8_N2048, n_layers=2, batch=2, ratio=0.25)
    r = Run(lib, shape, prebuilt=_weights(shape))   # workspace sized for the 25 % step
    for t, k in enumerate([None, 103, 512]):
        if k is not None:
            _set_k(r, k)
        out = O.step(r.ocfg, r.ow, r.st, r.opol, dense=(t == 0))
        r.gpu_step(t == 0, None if t == 0 else out.idx, out.unmasked)
        r.compare_tokens(r.compare_state(TOL["bf16"], out.final_rows, out.idx))


def test_8b_single_sequence_approximate_attention_steps(lib):
    """DyLLM's FFN gate and approximate attention (French summary §2.A, §2.B) at
    full width on one 768-token sequence: the dense step, then two 10 % steps
    (the exact attention of 77 rows splits its keys among CTAs, so its softmax
    statistics come through the merge of the shares); the oracle decides, every
    cache of the mode is compared."""
    from test_gpu_next import _upd_forced
    shape = SY.with_(SY.DENSE8B_B1_N768, n_layers=2, ratio=0.10)
    _upd_forced(lib, shape, 1e-3, TOL["bf16"], 3, prebuilt=_weights(shape))
