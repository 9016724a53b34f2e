"""Step-level invariants of the oracle that the pages fix.

* Recomputing every row is the vanilla (full) pass [ES-dLLM / DyLLM problem
  statements]: a dense step reproduces a full forward pass.
* Skipped rows reuse cached values [ES-dLLM §2.B]: a step that selects no
  row leaves every cache bitwise untouched.
* Fixed point: after a dense pass, if no token changed, recomputing any
  subset of rows reproduces the dense values (up to the library matmul's
  summation order).
* Sequences are independent: permuting the batch permutes the results.
"""
import numpy as np

import oracle as O
from dllm_synth import TINY, with_, model_weights, prompt_tokens
from _util import oracle_cfg, oracle_weights, oracle_policy, f64


def _setup(shape=TINY, seed=0, **kw):
    s = with_(shape, **kw)
    cfg = oracle_cfg(s)
    W = oracle_weights(model_weights(s, seed=seed))
    tok = f64(prompt_tokens(s, seed=1)).astype(np.int64)
    return s, cfg, W, tok


# The library matmul may sum a row in a different order when the matrix has a
# different number of rows, so "reproduces" means equal to ~1e-12 relative in float64.
RT = 1e-10


def _states_equal(a: O.State, b: O.State):
    for x, y in zip(a.k + a.v, b.k + b.v):
        np.testing.assert_allclose(x, y, rtol=RT, atol=RT)
    np.testing.assert_array_equal(a.h_ref, b.h_ref)
    np.testing.assert_allclose(a.conf, b.conf, rtol=RT)
    np.testing.assert_array_equal(a.pred, b.pred)
    np.testing.assert_array_equal(a.tokens, b.tokens)


def test_dense_step_equals_full_forward():
    s, cfg, W, tok = _setup(n_layers=2)
    st = O.empty_state(cfg, tok)
    out = O.step(cfg, W, st, oracle_policy(s, n_unmask=0), dense=True)
    full = O.dense_forward(cfg, W, tok)
    np.testing.assert_allclose(out.final_rows[0], full[0], rtol=RT, atol=RT)


def test_zero_ratio_leaves_caches_untouched():
    s, cfg, W, tok = _setup()
    st = O.empty_state(cfg, tok)
    pol = oracle_policy(s)
    O.step(cfg, W, st, pol, dense=True)
    before = st.copy()
    out = O.step(cfg, W, st, oracle_policy(s, k=0), dense=False)
    assert all(len(a) == 0 for a in out.idx)
    for x, y in zip(before.k + before.v, st.k + st.v):
        np.testing.assert_array_equal(x, y)
    np.testing.assert_array_equal(before.h_ref, st.h_ref)
    np.testing.assert_array_equal(before.conf, st.conf)
    # the unmask still runs, from the cached confidence
    expect = before.tokens.copy()
    O.unmask(before.conf, before.pred, expect, cfg.mask_id, pol.gen_start, pol.block_len,
             pol.n_unmask)
    np.testing.assert_array_equal(st.tokens, expect)


def test_fixed_point_partial_reproduces_dense_rows():
    s, cfg, W, tok = _setup(n_layers=2, batch=2)
    st = O.empty_state(cfg, tok)
    dense_out = O.step(cfg, W, st, oracle_policy(s, n_unmask=0), dense=True)
    before = st.copy()
    rng = np.random.default_rng(3)
    forced = [np.sort(rng.choice(s.seq_len, 40, replace=False)) for _ in range(2)]
    out = O.step(cfg, W, st, oracle_policy(s, n_unmask=0), dense=False, forced_idx=forced)
    _states_equal(before, st)
    for b in range(2):
        np.testing.assert_allclose(out.final_rows[b], dense_out.final_rows[b][forced[b]],
                                   rtol=RT, atol=RT)


def test_full_ratio_partial_equals_dense_step():
    s, cfg, W, tok = _setup(n_layers=2)
    st = O.empty_state(cfg, tok)
    O.step(cfg, W, st, oracle_policy(s), dense=True)
    a, b = st.copy(), st.copy()
    O.step(cfg, W, a, oracle_policy(s, k=s.seq_len), dense=False)
    O.step(cfg, W, b, oracle_policy(s), dense=True)
    _states_equal(a, b)


def test_batch_permutation_equivariance():
    s, cfg, W, tok = _setup(batch=3)
    pol = oracle_policy(s)
    st = O.empty_state(cfg, tok)
    O.step(cfg, W, st, pol, dense=True)
    perm = np.array([2, 0, 1])
    sp = O.State(st.tokens[perm].copy(), [a[perm].copy() for a in st.k],
                 [a[perm].copy() for a in st.v], st.h_ref[perm].copy(), st.conf[perm].copy(),
                 st.pred[perm].copy())
    o1 = O.step(cfg, W, st, pol, dense=False)
    o2 = O.step(cfg, W, sp, pol, dense=False)
    for i, p in enumerate(perm):
        np.testing.assert_array_equal(o2.idx[i], o1.idx[p])
        np.testing.assert_array_equal(sp.k[0][i], st.k[0][p])
        np.testing.assert_array_equal(sp.tokens[i], st.tokens[p])


def test_selection_prefers_changed_rows_when_alpha_zero():
    # with the score taken on the embedding, only rows whose token changed move;
    # they must be the first chosen (score ~1 versus exactly 0 for the rest)
    s, cfg, W, tok = _setup()
    st = O.empty_state(cfg, tok)
    pol = oracle_policy(s)
    out0 = O.step(cfg, W, st, pol, dense=True)
    changed = out0.unmasked[0][out0.unmasked[0] >= 0]
    out1 = O.step(cfg, W, st, pol, dense=False)
    assert set(changed.tolist()) <= set(out1.idx[0].tolist())
    assert np.all(out1.scores[0][changed] > 0.5)
    others = np.setdiff1d(np.arange(s.seq_len), changed)
    assert np.all(out1.scores[0][others] == 0.0)


def test_tiny_generation_runs_to_completion():
    s, cfg, W, tok = _setup()
    st = O.empty_state(cfg, tok)
    pol = oracle_policy(s)
    O.step(cfg, W, st, pol, dense=True)
    for _ in range(7):
        O.step(cfg, W, st, pol, dense=False)
    assert not np.any(st.tokens == cfg.mask_id)
    assert np.all((st.tokens >= 0) & (st.tokens < cfg.vocab))
