"""Pins of the oracle's step variants beyond the basic top-k step.

* Over-threshold unmasking (fast phase of "Accelerating Diffusion Large
  Language Models with SlowFast Sampling", German summary §2): brute force
  over small blocks with tied confidences, and its two limits.
* Response-only selection (DyLLM, French summary §2.C): brute force.
* Periodic refresh (ES-dLLM, Dutch summary "Methodologie" item 3): a refresh
  at every step is the vanilla generation written out independently; no
  refresh is the plain loop of steps; block refreshes fall where the block
  index floor(t * n / block_len) changes when every step reveals n tokens.
* Two skip points (ES-dLLM, German summary §2.B "Strategie"): keeping every
  row at the second point is the one-point step; keeping none leaves the
  layers from the second point on untouched; after a dense step a two-point
  step is a fixed point; the rows kept at the second point dominate the
  dropped ones by brute force.
* Incremental attention of stable rows (DyLLM, French summary §2.B): after
  some keys change, updating the cached statistics with the changed keys'
  old and new terms equals the attention over the updated keys computed
  directly; no change, every key changed and a key replaced by itself are
  the limits.
* Approximate attention inside a step (DyLLM, French summary §2.B): after
  any run of dense and partial steps, every row's cached context equals the
  attention of its cached query over the current K/V caches computed afresh,
  and its cached (m, l) are that attention's max and sum; with every row
  salient for the FFN the update changes nothing but the stable rows' caches.
* FFN gating on the attention context (DyLLM, French summary §2.A): every
  row salient is the plain layer; no row salient adds the cached FFN output
  to the post-attention residual (taken from the same model with its FFN
  output weight zeroed); after a dense step a gated step is a fixed point
  that runs no FFN.
"""
import itertools

import numpy as np
import pytest

import oracle as O
from dllm_synth import TINY, with_, model_weights, prompt_tokens
from _util import oracle_cfg, oracle_weights, oracle_policy, f64, max_abs_rel

RT = 1e-10


def _setup(shape=TINY, seed=0, **kw):
    s = with_(shape, **kw)
    cfg = oracle_cfg(s)
    W = oracle_weights(model_weights(s, seed=seed))
    tok = f64(prompt_tokens(s, seed=1)).astype(np.int64)
    return s, cfg, W, tok


# ----------------------------------------------------------------- unmask


def _brute_unmask(conf, tokens, mask_id, gen_start, block_len, n, tau):
    """Every masked position of the block above tau, or else the n best;
    "best" found by checking every subset against every outsider."""
    N = len(tokens)
    first = next((p for p in range(gen_start, N) if tokens[p] == mask_id), None)
    if first is None or n <= 0:
        return []
    start = gen_start + (first - gen_start) // block_len * block_len
    cand = [p for p in range(start, min(start + block_len, N)) if tokens[p] == mask_id]
    above = [p for p in cand if conf[p] > tau] if tau > 0 else []
    if tau > 0 and len(above) >= n:
        return sorted(above)

    def better(p, q):  # p ranks before q
        return conf[p] > conf[q] or (conf[p] == conf[q] and p < q)

    m = min(n, len(cand))
    for S in itertools.combinations(cand, m):
        rest = [q for q in cand if q not in S]
        if all(better(p, q) for p in S for q in rest):
            return sorted(S)
    raise AssertionError("no dominant subset")


def test_unmask_tau_brute_force():
    rng = np.random.default_rng(3)
    levels = np.array([0.05, 0.3, 0.3, 0.6, 0.9, 0.9, 0.97])
    mask_id = 99
    for _ in range(400):
        N = int(rng.integers(4, 13))
        gen_start = int(rng.integers(0, 3))
        block_len = int(rng.integers(1, 6))
        n = int(rng.integers(0, 4))
        tau = float(rng.choice([0.0, 0.3, 0.6, 0.95]))
        tokens = np.where(rng.random(N) < 0.6, mask_id, 1).astype(np.int64)
        conf = rng.choice(levels, N)
        got = O.unmask_positions(conf, tokens, mask_id, gen_start, block_len, n, tau)
        exp = _brute_unmask(conf, tokens, mask_id, gen_start, block_len, n, tau)
        assert list(got) == exp, (conf, tokens, gen_start, block_len, n, tau)


def test_unmask_tau_limits():
    rng = np.random.default_rng(4)
    mask_id = 7
    for _ in range(50):
        N, bl, n = 24, 8, 2
        tokens = np.where(rng.random(N) < 0.7, mask_id, 0).astype(np.int64)
        conf = rng.random(N)
        plain = O.unmask_positions(conf, tokens, mask_id, 0, bl, n)
        # a threshold no confidence reaches is the plain top-n rule
        assert list(O.unmask_positions(conf, tokens, mask_id, 0, bl, n, 2.0)) == list(plain)
        # a threshold every confidence passes reveals the whole current block
        blk = O.current_block(tokens, mask_id, 0, bl)
        if blk is None:
            continue
        whole = [p for p in range(*blk) if tokens[p] == mask_id]
        got = O.unmask_positions(conf, tokens, mask_id, 0, bl, n, 1e-30)
        assert list(got) == sorted(whole)
    assert O.unmask_capacity(4, 32, 0.0) == 4 and O.unmask_capacity(4, 32, 0.9) == 32


# ----------------------------------------------------------------- selection


def test_select_from_brute_force():
    rng = np.random.default_rng(5)
    for _ in range(300):
        N = int(rng.integers(1, 12))
        lo = int(rng.integers(0, N + 1))
        k = int(rng.integers(0, N + 2))
        sc = rng.choice(np.array([0.0, -0.0, 0.25, 0.25, 0.5, 1.0, np.nan]), (1, N))
        got = O.select(sc, O.SELECT_TOPK, k, 0.0, k, lo)[0]
        pos = list(range(lo, N))

        def key(p):
            v = sc[0, p]
            return (0, 0.0, -p) if np.isnan(v) else (1, float(v) + 0.0, -p)
        m = min(k, len(pos))
        exp = None
        for S in itertools.combinations(pos, m):
            rest = [q for q in pos if q not in S]
            if all(key(p) > key(q) for p in S for q in rest):
                exp = sorted(S)
                break
        assert list(got) == exp
        if lo == 0:
            assert list(got) == list(O.select(sc, O.SELECT_TOPK, k, 0.0, k)[0])


def test_response_only_step_keeps_prompt_caches():
    s, cfg, W, tok = _setup(n_layers=2)
    st = O.empty_state(cfg, tok)
    pol = oracle_policy(s, select_from=s.prompt_len, k=24)
    O.step(cfg, W, st, pol, dense=True)
    before = st.copy()
    out = O.step(cfg, W, st, pol, dense=False)
    assert all(len(a) == 24 and a.min() >= s.prompt_len for a in out.idx)
    P = s.prompt_len
    for l in range(cfg.n_layers):
        np.testing.assert_array_equal(st.k[l][:, :P], before.k[l][:, :P])
        np.testing.assert_array_equal(st.v[l][:, :P], before.v[l][:, :P])
    np.testing.assert_array_equal(st.h_ref[:, :P], before.h_ref[:, :P])


# ----------------------------------------------------------------- refresh


def _vanilla_generation(cfg, W, tok, pol, n_steps):
    """Every step a full forward of the current tokens; confidence and argmax of
    every masked position; the unmask rule."""
    tok = tok.copy()
    conf = np.zeros(tok.shape)
    pred = np.zeros(tok.shape, dtype=np.int64)
    for _ in range(n_steps):
        final = O.dense_forward(cfg, W, tok)
        for b in range(tok.shape[0]):
            m = np.nonzero(tok[b] == cfg.mask_id)[0]
            if len(m) == 0:
                continue
            n = O.store(O.rms_norm(final[b, m], W.final_norm, cfg.rms_eps), cfg.dtype)
            z = n @ np.asarray(W.lm_head).T
            zmax = z.max(axis=1, keepdims=True)
            conf[b, m] = 1.0 / np.exp(z - zmax).sum(axis=1)
            pred[b, m] = np.argmax(z, axis=1)
        O.unmask(conf, pred, tok, cfg.mask_id, pol.gen_start, pol.block_len, pol.n_unmask)
    return tok, conf


def test_refresh_every_step_is_the_vanilla_generation():
    s, cfg, W, tok = _setup(n_layers=2)
    pol = oracle_policy(s, refresh_every=1)
    st = O.empty_state(cfg, tok)
    dense_log, _ = O.generate(cfg, W, st, pol, 4)
    assert dense_log == [True] * 4
    tok_v, conf_v = _vanilla_generation(cfg, W, tok, pol, 4)
    np.testing.assert_array_equal(st.tokens, tok_v)
    m = conf_v > 0
    np.testing.assert_allclose(st.conf[m], conf_v[m], rtol=RT)


def test_no_refresh_is_the_plain_step_loop():
    s, cfg, W, tok = _setup()
    pol = oracle_policy(s)
    st = O.empty_state(cfg, tok)
    dense_log, pos_log = O.generate(cfg, W, st, pol, 5)
    assert dense_log == [True, False, False, False, False]
    st2 = O.empty_state(cfg, tok)
    for t in range(5):
        out = O.step(cfg, W, st2, pol, dense=(t == 0))
        np.testing.assert_array_equal(out.unmasked, pos_log[t])
    np.testing.assert_array_equal(st.tokens, st2.tokens)
    for a, b in zip(st.k + st.v, st2.k + st2.v):
        np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("block_len,n,R", [(16, 8, 0), (24, 8, 5), (64, 8, 3)])
def test_block_refresh_schedule(block_len, n, R):
    s, cfg, W, tok = _setup(block_len=block_len, n_unmask=n)
    pol = oracle_policy(s, refresh_on_block=True, refresh_every=R)
    st = O.empty_state(cfg, tok)
    T = 8
    dense_log, pos_log = O.generate(cfg, W, st, pol, T)
    exp = [t == 0 or (R > 0 and t % R == 0) or (t * n // block_len != (t - 1) * n // block_len)
           for t in range(T)]
    assert dense_log == exp
    assert all((p >= 0).sum() == n for p in pos_log)


# ----------------------------------------------------------------- two skip points


def _two_point_setup(k2, **kw):
    s, cfg, W, tok = _setup(n_layers=3, **kw)
    st = O.empty_state(cfg, tok)
    pol = oracle_policy(s, score_layer2=2, k2=k2)
    O.step(cfg, W, st, pol, dense=True)
    # change some generated tokens so the next step has real work
    rng = np.random.default_rng(9)
    P = s.prompt_len
    ch = rng.choice(np.arange(P, s.seq_len), 12, replace=False)
    st.tokens[0, ch] = rng.integers(0, cfg.vocab - 1, len(ch))
    return s, cfg, W, st, pol


def test_two_point_keeping_every_row_equals_one_point():
    s, cfg, W, st, pol = _two_point_setup(k2=10 ** 6)
    st1 = st.copy()
    out2 = O.step(cfg, W, st, pol, dense=False)
    pol1 = oracle_policy(s)
    out1 = O.step(cfg, W, st1, pol1, dense=False)
    for a, b in zip(out2.idx2, out1.idx):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(st.k + st.v, st1.k + st1.v):
        np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(st.tokens, st1.tokens)
    np.testing.assert_array_equal(st.conf, st1.conf)


def test_two_point_keeping_no_row_leaves_upper_layers():
    s, cfg, W, st, pol = _two_point_setup(k2=0)
    before = st.copy()
    out = O.step(cfg, W, st, pol, dense=False)
    assert all(len(a) == 0 for a in out.idx2)
    for l in range(2, cfg.n_layers):
        np.testing.assert_array_equal(st.k[l], before.k[l])
        np.testing.assert_array_equal(st.v[l], before.v[l])
    np.testing.assert_array_equal(st.conf, before.conf)
    np.testing.assert_array_equal(st.h_ref2, before.h_ref2)
    # the rows selected at the first point did run the layers below the second
    changed = [l for l in range(2) if not np.array_equal(st.k[l], before.k[l])]
    assert changed == [0, 1]


def test_two_point_fixed_point_after_dense():
    s, cfg, W, tok = _setup(n_layers=3)
    st = O.empty_state(cfg, tok)
    pol = oracle_policy(s, score_layer2=2, k2=9, n_unmask=0)
    O.step(cfg, W, st, pol, dense=True)
    ref = st.copy()
    O.step(cfg, W, st, pol, dense=False)
    for a, b in zip(st.k + st.v, ref.k + ref.v):
        np.testing.assert_allclose(a, b, rtol=RT, atol=RT)
    np.testing.assert_allclose(st.h_ref2, ref.h_ref2, rtol=RT, atol=RT)


def test_two_point_selection_brute_force():
    s, cfg, W, st, pol = _two_point_setup(k2=7)
    out = O.step(cfg, W, st.copy(), pol, dense=False)
    for b in range(len(out.idx)):
        pos, sc = out.idx[b], out.scores2[b]
        best = sorted(range(len(pos)), key=lambda j: _key(sc[j], pos[j]), reverse=True)[:7]
        # brute force: every kept row ranks above every dropped row
        kept = set(int(p) for p in out.idx2[b])
        for j in range(len(pos)):
            for i in range(len(pos)):
                if int(pos[i]) in kept and int(pos[j]) not in kept:
                    assert _key(sc[i], pos[i]) > _key(sc[j], pos[j])
        assert kept == set(int(pos[j]) for j in best)


def _key(v, p):
    v = float(v)
    return (0, 0.0, -int(p)) if np.isnan(v) else (1, v + 0.0, -int(p))


# ----------------------------------------------------------------- incremental attention


def _kv(rng, N, Hkv, hd, scale=1.0):
    return rng.normal(0, scale, (N, Hkv, hd)), rng.normal(0, 1.0, (N, Hkv, hd))


@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2)])
def test_attention_update_equals_attention_on_updated_keys(Hq, Hkv):
    rng = np.random.default_rng(21)
    N, hd, R = 40, 16, 7
    K, V = _kv(rng, N, Hkv, hd)
    q = rng.normal(0, 1.0, (R, Hq, hd))
    m, l, o = O.attention_stats(q, K, V)
    np.testing.assert_allclose(o, O.attention(q, K, V), rtol=1e-12, atol=1e-12)
    A = np.array([3, 9, 10, 27, 39])
    K2, V2 = K.copy(), V.copy()
    K2[A] = rng.normal(0, 2.0, (len(A), Hkv, hd))     # some new scores exceed the old max
    V2[A] = rng.normal(0, 1.0, (len(A), Hkv, hd))
    m2, l2, o2 = O.attention_update(q, m, l, o, K[A], V[A], K2[A], V2[A])
    me, le, oe = O.attention_stats(q, K2, V2)
    np.testing.assert_allclose(o2, oe, rtol=1e-10, atol=1e-10)
    # the same softmax: l e^m agrees (the reference max may stay above the new max)
    np.testing.assert_allclose(l2 * np.exp(m2 - me), le, rtol=1e-10)
    assert np.all(m2 >= me - 1e-12)


def test_attention_update_limits():
    rng = np.random.default_rng(22)
    N, Hkv, hd, R = 12, 2, 8, 5
    K, V = _kv(rng, N, Hkv, hd)
    q = rng.normal(0, 1.0, (R, 2, hd))
    m, l, o = O.attention_stats(q, K, V)
    # no key changed: nothing moves
    e = np.zeros((0, Hkv, hd))
    m2, l2, o2 = O.attention_update(q, m, l, o, e, e, e, e)
    np.testing.assert_allclose(o2, o, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(l2, l, rtol=1e-13)
    # every key changed: the attention over the new keys
    K2, V2 = _kv(rng, N, Hkv, hd)
    m2, l2, o2 = O.attention_update(q, m, l, o, K, V, K2, V2)
    np.testing.assert_allclose(o2, O.attention(q, K2, V2), rtol=1e-9, atol=1e-9)
    # a changed key replaced by itself: nothing moves
    A = np.array([0, 5])
    m2, l2, o2 = O.attention_update(q, m, l, o, K[A], V[A], K[A], V[A])
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------- FFN gating


def _gated_setup(**kw):
    s, cfg, W, tok = _setup(n_layers=2, **kw)
    st = O.empty_state(cfg, tok)
    return s, cfg, W, tok, st


def test_ffn_gate_every_row_salient_is_the_plain_layer():
    s, cfg, W, tok, st = _gated_setup()
    pol = oracle_policy(s, ffn_gate=True, ffn_tau=-1.0)
    plain = O.empty_state(cfg, tok)
    O.step(cfg, W, st, pol, dense=True)
    O.step(cfg, W, plain, oracle_policy(s), dense=True)
    for t in range(3):
        out = O.step(cfg, W, st, pol, dense=False)
        ref = O.step(cfg, W, plain, oracle_policy(s), dense=False)
        assert out.ffn_rows == [sum(len(a) for a in out.idx)] * cfg.n_layers
        for a, b in zip(out.final_rows, ref.final_rows):
            np.testing.assert_array_equal(a, b)   # f32 storage: the same sums, exactly
    np.testing.assert_array_equal(st.tokens, plain.tokens)


def test_ffn_gate_no_row_salient_reuses_the_cached_ffn():
    import dataclasses
    s, cfg, W, tok = _setup(n_layers=1)
    st = O.empty_state(cfg, tok)
    pol = oracle_policy(s, ffn_gate=True, ffn_tau=2.5)      # 1 - cos never exceeds 2
    O.step(cfg, W, st, pol, dense=True)
    st.tokens[0, s.prompt_len + 3] = 5                      # something to recompute
    ffn0 = st.ffn[0].copy()
    # the post-attention residual, from the plain layer of a model without FFN output
    W0 = dataclasses.replace(W, layers=[dataclasses.replace(W.layers[0],
                                                            w_down=np.zeros_like(W.layers[0].w_down))])
    st0 = st.copy()
    mid = O.step(cfg, W0, st0, oracle_policy(s), dense=False)
    out = O.step(cfg, W, st, pol, dense=False)
    assert out.ffn_rows == [0]
    np.testing.assert_array_equal(st.ffn[0], ffn0)
    np.testing.assert_array_equal(out.idx[0], mid.idx[0])
    np.testing.assert_allclose(out.final_rows[0], mid.final_rows[0] + ffn0[0, out.idx[0]],
                               rtol=1e-12, atol=1e-12)


def test_ffn_gate_fixed_point_after_dense():
    s, cfg, W, tok, st = _gated_setup(n_unmask=0)
    pol = oracle_policy(s, ffn_gate=True, ffn_tau=1e-9, n_unmask=0)
    O.step(cfg, W, st, pol, dense=True)
    ref = st.copy()
    out = O.step(cfg, W, st, pol, dense=False)
    # unchanged tokens: every context reproduces its cache, no FFN runs, and the rows
    # still come out as the dense pass computed them
    assert out.ffn_rows == [0] * cfg.n_layers
    for a, b in zip(st.k + st.v + st.ctx, ref.k + ref.v + ref.ctx):
        np.testing.assert_allclose(a, b, rtol=RT, atol=RT)
    full = O.dense_forward(cfg, W, tok)
    np.testing.assert_allclose(out.final_rows[0], full[0, out.idx[0]], rtol=RT, atol=RT)


def test_ffn_gate_threshold_splits_rows_by_context_change():
    s, cfg, W, tok, st = _gated_setup(n_unmask=0)
    pol = oracle_policy(s, ffn_gate=True, ffn_tau=0.0, n_unmask=0, alpha=0.0, k=32)
    O.step(cfg, W, st, pol, dense=True)
    st.tokens[0, s.prompt_len:s.prompt_len + 4] = [11, 12, 13, 14]
    out = O.step(cfg, W, st, pol, dense=False)
    # with tau 0 exactly the rows whose context moved at all run the FFN: in the first
    # recomputed layer every selected row sees the four changed keys
    assert 0 < out.ffn_rows[0] <= 32



# ----------------------------------------------------------------- approximate attention step


def _cached_attention_holds(cfg, st, tol):
    """Every row's cached context / statistics against a fresh attention of its
    cached query over the layer's K/V caches."""
    Hq, hd = cfg.n_heads, cfg.head_dim
    B, N = st.tokens.shape
    for l in range(cfg.n_layers):
        for b in range(B):
            q = st.q[l][b].reshape(N, Hq, hd)
            m, lsum, o = O.attention_stats(q, st.k[l][b], st.v[l][b])
            assert np.max(np.abs(st.ctx[l][b] - o.reshape(N, -1))) < tol * np.abs(o).max()
            lse = st.att_m[l][b] + np.log(st.att_l[l][b])
            assert np.max(np.abs(lse - (m + np.log(lsum)))) < tol * np.abs(m).max()


@pytest.mark.parametrize("tau", [-1.0, 1e-2])
def test_approximate_attention_tracks_the_caches(tau):
    """Stable rows keep their query, so their exactly updated statistics must be
    those of the attention over the updated keys: the invariant holds after the
    dense step and after every partial step (f32: no rounding anywhere)."""
    s, cfg, W, tok = _setup(n_layers=2)
    st = O.empty_state(cfg, tok)
    pol = oracle_policy(s, ffn_gate=True, ffn_tau=tau, attn_update=True)
    for t in range(5):
        out = O.step(cfg, W, st, pol, dense=(t == 0))
        _cached_attention_holds(cfg, st, 1e-9)
    assert sum(len(a) for a in out.idx) < tok.size    # stable rows existed


def test_approximate_attention_touches_only_the_stable_rows_caches():
    """With every row salient for the FFN, decisions never read the contexts, so
    a run with the update and one without agree on tokens, K/V, references,
    confidences, predictions and FFN outputs, and on the recomputed rows'
    contexts (up to the summation order of the two attention routines, 1e-10);
    only stable rows' contexts differ."""
    s, cfg, W, tok = _setup(n_layers=2)
    st1, st2 = O.empty_state(cfg, tok), O.empty_state(cfg, tok)
    p1 = oracle_policy(s, ffn_gate=True, ffn_tau=-1.0, attn_update=True)
    p2 = oracle_policy(s, ffn_gate=True, ffn_tau=-1.0)
    moved = 0
    for t in range(4):
        o1 = O.step(cfg, W, st1, p1, dense=(t == 0))
        o2 = O.step(cfg, W, st2, p2, dense=(t == 0))
        np.testing.assert_array_equal(st1.tokens, st2.tokens)
        np.testing.assert_array_equal(st1.pred, st2.pred)
        for a, b in zip(st1.k + st1.v + st1.ffn + [st1.h_ref, st1.conf],
                        st2.k + st2.v + st2.ffn + [st2.h_ref, st2.conf]):
            assert max_abs_rel(a, b) < RT
        for l in range(cfg.n_layers):
            for b, idx in enumerate(o1.idx):
                assert max_abs_rel(st1.ctx[l][b, idx], st2.ctx[l][b, idx]) < RT
                rest = np.setdiff1d(np.arange(tok.shape[1]), idx)
                moved += int(max_abs_rel(st1.ctx[l][b, rest], st2.ctx[l][b, rest]) > 1e-6)
    assert moved > 0
