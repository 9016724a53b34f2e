"""GPU parity of whole denoising steps (dllm_step) against the oracle.

Runs are compared step by step.  With forced decisions the GPU takes the
oracle's index lists and revealed positions, and its token state is
re-synchronised to the oracle's after each step; the caches evolve on their
own.  With its own decisions, every choice the GPU makes is checked against
the oracle's rule applied to the GPU's own inputs (bit-exact)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
import dllm_synth as SY
from _util import f64, max_abs_rel, TOL, oracle_cfg, oracle_policy
from _gpu import build, oracle_w_from, argmax_ok

pytestmark = pytest.mark.gpu
GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


class Run:
    def __init__(self, lib, shape, seed=0, prebuilt=None, **pol_kw):
        """prebuilt: (host weights, oracle weights, device weights) of this shape, to
        share one draw of the weights among several runs."""
        self.lib, self.s = lib, shape
        if prebuilt is None:
            self.model, self.ocfg, Wd, Wh = build(shape, seed=seed)
            self.ow = oracle_w_from(Wh)
        else:
            Wh, self.ow, Wd = prebuilt
            self.model = lib.Model(lib.cfg_from_shape(shape), Wd)
            self.ocfg = oracle_cfg(shape)
        B, N = shape.batch, shape.seq_len
        tok = SY.prompt_tokens(shape, seed=1)
        self.tokens = tok.cuda()
        self.cache = lib.Cache(self.model.cfg, B, N)
        self.opol = oracle_policy(shape, **pol_kw)
        self.pol = lib.make_policy(score_layer=self.opol.score_layer, alpha=self.opol.alpha,
                                   kind=self.opol.kind, mode=self.opol.mode, k=self.opol.k,
                                   tau=self.opol.tau, n_unmask=self.opol.n_unmask,
                                   gen_start=self.opol.gen_start, block_len=self.opol.block_len,
                                   select_from=self.opol.select_from,
                                   unmask_tau=self.opol.unmask_tau,
                                   refresh_every=self.opol.refresh_every,
                                   refresh_on_block=self.opol.refresh_on_block)
        self.k_cap = max(1, min(self.opol.k, N))
        self.ws = lib.Workspace(lib.dllm_step_workspace_size(self.model.cfg, B, N, self.pol))
        self.st = O.empty_state(self.ocfg, f64(tok).astype(np.int64))
        self.B, self.N = B, N

    def gpu_step(self, dense, forced_idx=None, forced_unmask=None):
        B, N, n = self.B, self.N, max(self.lib.dllm_unmask_capacity(self.pol), 1)
        idx = torch.full((B, self.k_cap), -1, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
        pos = torch.full((B, n), -5, dtype=torch.int32, device="cuda")
        sc = torch.zeros(B, N, dtype=torch.float32, device="cuda")
        fi = fc = fu = None
        if forced_idx is not None:
            a = np.full((B, self.k_cap), -1, dtype=np.int32)
            for b, r in enumerate(forced_idx):
                a[b, :len(r)] = r
            fi = torch.from_numpy(a).cuda()
            fc = torch.tensor([len(r) for r in forced_idx], dtype=torch.int32, device="cuda")
        if forced_unmask is not None:
            fu = torch.from_numpy(np.ascontiguousarray(forced_unmask, dtype=np.int32)).cuda()
        self.lib.dllm_step(self.model, self.cache, self.tokens, self.pol, dense, self.ws,
                           forced_idx=fi, forced_count=fc, forced_unmask_pos=fu, idx_out=idx,
                           count_out=cnt, pos_out=pos, scores_out=sc)
        torch.cuda.synchronize()
        assert self.ws.device_status() == 0
        return idx.cpu().numpy(), cnt.cpu().numpy(), pos.cpu().numpy(), sc.cpu().numpy()

    def _oracle_logits(self, final_rows, idx, b, p):
        j = np.nonzero(np.asarray(idx[b]) == p)[0]
        assert len(j), (b, p)   # only rows recomputed in this step have new logits
        n = O.store(O.rms_norm(final_rows[b][int(j[0])], self.ow.final_norm, self.ocfg.rms_eps),
                    self.ocfg.dtype)
        return n @ self.ow.lm_head.T

    def compare_state(self, tol, final_rows=None, idx=None):
        """Caches against the oracle's.  K/V and hidden references: max-abs-relative
        error < tol.  Confidence: within tol of the largest confidence, or, row by
        row, |ln conf_gpu - ln conf_oracle| <= 2 tol max|z| (ln conf = z_max -
        logsumexp(z) moves by at most twice a logit error; the logit tolerance is
        tol max|z|).  Predictions: equal, or a near tie of the oracle's logits.
        Accepted confidences and predictions are set to the oracle's, so that later
        steps start from the same state.  Returns the near-tie positions (b, p)."""
        c = self.cache
        for l in range(self.ocfg.n_layers):
            assert max_abs_rel(f64(c.k[l]), self.st.k[l]) < tol, ("k", l)
            assert max_abs_rel(f64(c.v[l]), self.st.v[l]) < tol, ("v", l)
        assert max_abs_rel(f64(c.h_ref), self.st.h_ref) < tol
        ctol = max(tol, TOL["f32"])
        cg, co = f64(c.conf), self.st.conf
        far = np.argwhere(np.abs(cg - co) >= ctol * max(np.abs(co).max(), 1e-30))
        for b, p in far:
            assert final_rows is not None, (b, p)
            z = self._oracle_logits(final_rows, idx, b, p)
            assert abs(np.log(cg[b, p]) - np.log(co[b, p])) <= 2.0 * tol * np.abs(z).max(), (b, p)
            self.cache.conf[b, p] = float(co[b, p])
        gp = f64(c.pred).astype(np.int64)
        ties = []
        for b, p in np.argwhere(gp != self.st.pred):
            # a different argmax must be a near tie of the oracle's logits
            assert final_rows is not None, (b, p)
            z = self._oracle_logits(final_rows, idx, b, p)
            assert argmax_ok(gp[b, p], z, TOL[self.ocfg.dtype]), (b, p)
            # accepted near tie: continue from the oracle's choice
            self.cache.pred[b, p] = int(self.st.pred[b, p])
            ties.append((int(b), int(p)))
        return ties

    def compare_tokens(self, ties):
        """Tokens equal the oracle's, except where a forced reveal took a near-tie
        prediction; then the oracle's tokens are taken over."""
        gt = f64(self.tokens).astype(np.int64)
        ok = np.ones_like(gt, dtype=bool)
        for b, p in ties:
            ok[b, p] = False
        np.testing.assert_array_equal(gt[ok], self.st.tokens[ok])
        self.tokens.copy_(torch.from_numpy(self.st.tokens.astype(np.int32)))


def test_step_tiny_f32_forced_decisions(lib):
    r = Run(lib, SY.TINY)
    for t in range(8):
        out = O.step(r.ocfg, r.ow, r.st, r.opol, dense=(t == 0))
        r.gpu_step(t == 0, None if t == 0 else out.idx, out.unmasked)
        r.compare_state(TOL["f32"], out.final_rows, out.idx)
        np.testing.assert_array_equal(f64(r.tokens).astype(np.int64), r.st.tokens)


def test_step_tiny_f32_own_decisions_follow_the_rules(lib):
    r = Run(lib, SY.TINY)
    gold = json.load(open(os.path.join(GOLD, "tiny_trajectory.json")))
    for t in range(8):
        tok_before = f64(r.tokens).astype(np.int64)
        conf_before = f64(r.cache.conf)
        href_before = f64(r.cache.h_ref)
        idx, cnt, pos, sc = r.gpu_step(dense=(t == 0))
        masked = tok_before == r.ocfg.mask_id
        if t > 0:
            h = r.ow.embed[tok_before]
            ora_scores = O.importance(O.variation(h, href_before, r.opol.kind), conf_before,
                                      masked, r.opol.alpha)
            assert max_abs_rel(sc, ora_scores) < TOL["f32"]
            for b in range(r.B):
                np.testing.assert_array_equal(idx[b, :cnt[b]], O.select_topk(sc[b], r.opol.k))
            assert [list(map(int, idx[b, :cnt[b]])) for b in range(r.B)] == gold["steps"][t]["idx"]
        conf_after = f64(r.cache.conf)
        pred_after = f64(r.cache.pred).astype(np.int64)
        t_ora = tok_before.copy()
        p_ora = O.unmask(conf_after, pred_after, t_ora, r.ocfg.mask_id, r.opol.gen_start,
                         r.opol.block_len, r.opol.n_unmask)
        np.testing.assert_array_equal(pos, p_ora)
        np.testing.assert_array_equal(f64(r.tokens).astype(np.int64), t_ora)
        assert pos.tolist() == gold["steps"][t]["unmasked"]
    assert f64(r.tokens).astype(np.int64).tolist() == gold["final_tokens"]


def _small_bf16(**kw):
    base = dict(dtype="bf16", n_layers=2, d=256, n_heads=2, n_kv_heads=2, head_dim=128, ffn=512,
                vocab=2048, batch=2, prompt_len=64, gen_len=128, block_len=32, n_unmask=4,
                ratio=0.25, alpha=0.5)
    base.update(kw)
    return SY.with_(SY.TINY, **base)


@pytest.mark.parametrize("score_layer", [0, 1])
def test_step_bf16_small_forced_decisions(lib, score_layer):
    shape = _small_bf16(score_layer=score_layer)
    r = Run(lib, shape)
    for t in range(6):
        out = O.step(r.ocfg, r.ow, r.st, r.opol, dense=(t == 0))
        r.gpu_step(t == 0, None if t == 0 else out.idx, out.unmasked)
        r.compare_state(TOL["bf16"], out.final_rows, out.idx)
        r.tokens.copy_(torch.from_numpy(r.st.tokens.astype(np.int32)))


def test_step_bf16_gqa_es_l1_forced(lib):
    shape = _small_bf16(n_heads=4, n_kv_heads=2, head_dim=64, batch=3)
    r = Run(lib, shape, kind=O.SCORE_ES_L1)
    for t in range(4):
        out = O.step(r.ocfg, r.ow, r.st, r.opol, dense=(t == 0))
        r.gpu_step(t == 0, None if t == 0 else out.idx, out.unmasked)
        r.compare_state(TOL["bf16"], out.final_rows, out.idx)
        r.tokens.copy_(torch.from_numpy(r.st.tokens.astype(np.int32)))


def test_step_zero_ratio_leaves_gpu_caches_untouched(lib):
    shape = _small_bf16()
    r = Run(lib, shape)
    r.gpu_step(True)
    snap = [t.clone() for t in r.cache.k + r.cache.v] + [r.cache.h_ref.clone(),
                                                          r.cache.conf.clone()]
    r.pol.k = 0
    r.ws = lib.Workspace(lib.dllm_step_workspace_size(r.model.cfg, r.B, r.N, r.pol))
    idx, cnt, pos, sc = r.gpu_step(False)
    assert np.all(cnt == 0)
    after = r.cache.k + r.cache.v + [r.cache.h_ref, r.cache.conf]
    for a, b in zip(snap, after):
        assert torch.equal(a, b)


def test_step_full_ratio_equals_dense_step_on_gpu(lib):
    shape = _small_bf16()
    r1, r2 = Run(lib, shape), Run(lib, shape)
    for r in (r1, r2):
        r.gpu_step(True)
    r1.pol.k = shape.seq_len
    r1.ws = lib.Workspace(lib.dllm_step_workspace_size(r1.model.cfg, r1.B, r1.N, r1.pol))
    r1.k_cap = shape.seq_len
    r1.gpu_step(False)
    r2.gpu_step(True)
    for a, b in zip(r1.cache.k + r1.cache.v + [r1.cache.h_ref, r1.cache.conf, r1.cache.pred],
                    r2.cache.k + r2.cache.v + [r2.cache.h_ref, r2.cache.conf, r2.cache.pred]):
        assert torch.equal(a, b)
    assert torch.equal(r1.tokens, r2.tokens)


def test_step_8b_width_two_layers_forced(lib):
    """The 8B step's launch configuration at full width (d 4096, 32 heads, FFN
    12288, vocab 126464, 1536 tokens with 512 prompt, 308 rows and 16 reveals per
    sequence per step) on 2 of its 32 sequences and 2 of its 32 layers: the
    dense first step and two partial steps with the oracle's decisions; every
    cache, the confidences and the predictions compared."""
    shape = SY.with_(SY.DENSE8B_B32_N1536, n_layers=2, batch=2)
    r = Run(lib, shape)
    for t in range(3):
        out = O.step(r.ocfg, r.ow, r.st, r.opol, dense=(t == 0))
        r.gpu_step(t == 0, None if t == 0 else out.idx, out.unmasked)
        r.compare_tokens(r.compare_state(TOL["bf16"], out.final_rows, out.idx))
