"""GPU parity of the step variants: over-threshold unmasking ("Accelerating
Diffusion Large Language Models with SlowFast Sampling", German summary §2),
response-only selection (DyLLM, French summary §2.C) and the periodic
refresh of a generation (ES-dLLM, Dutch summary "Methodologie" item 3).
Index work is compared bit-exactly on identical inputs; whole steps and
generations against the oracle as in the step tests."""
import numpy as np
import pytest
import torch

import oracle as O
import dllm_synth as SY
from _util import f64, max_abs_rel, TOL
from test_gpu_step import Run, _small_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("tau", [0.0, 0.55, 0.97, 1e-30])
def test_unmask_tau_matches_oracle(lib, tau):
    g = torch.Generator().manual_seed(11)
    B, N, gen_start, bl, n, mask_id = 3, 200, 40, 32, 4, 999
    tokens = torch.randint(0, 900, (B, N), generator=g, dtype=torch.int32)
    tokens[:, gen_start:] = torch.where(torch.rand(B, N - gen_start, generator=g) < 0.8,
                                        torch.tensor(mask_id, dtype=torch.int32),
                                        tokens[:, gen_start:])
    tokens[1, gen_start:gen_start + 40] = 5          # sequence 1's first block is done
    conf = torch.round(torch.rand(B, N, generator=g) * 20) / 20   # ties
    pred = torch.randint(0, 900, (B, N), generator=g, dtype=torch.int32)
    pos = torch.full((B, bl), -7, dtype=torch.int32)
    t_gpu = tokens.cuda()
    p_gpu = pos.cuda()
    lib.dllm_unmask_tau(conf.cuda(), pred.cuda(), t_gpu, mask_id, gen_start, bl, n, tau, p_gpu)
    torch.cuda.synchronize()
    t_ora = f64(tokens).astype(np.int64)
    tau32 = float(np.float32(tau))   # the threshold the library compares in fp32
    p_ora = O.unmask(f64(conf), f64(pred).astype(np.int64), t_ora, mask_id, gen_start, bl, n,
                     tau32)
    cap = O.unmask_capacity(n, bl, tau)
    got = p_gpu.cpu().numpy()
    np.testing.assert_array_equal(got[:, :cap], p_ora)
    assert np.all(got[:, cap:] == -1)
    np.testing.assert_array_equal(t_gpu.cpu().numpy(), t_ora)


@pytest.mark.parametrize("lo,k", [(0, 50), (37, 50), (190, 50), (200, 5)])
def test_select_range_matches_oracle(lib, lo, k):
    g = torch.Generator().manual_seed(12)
    B, N = 4, 200
    sc = torch.round(torch.randn(B, N, generator=g) * 4) / 4
    sc[0, ::7] = float("nan")
    sc[1, ::5] = -0.0
    idx = torch.full((B, 64), -3, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    lib.dllm_select_range(sc.cuda(), idx, cnt, lo, lib.DLLM_SELECT_TOPK, k)
    torch.cuda.synchronize()
    ora = O.select(f64(sc), O.SELECT_TOPK, k, 0.0, 64, lo)
    for b in range(B):
        c = int(cnt[b])
        assert c == len(ora[b])
        np.testing.assert_array_equal(idx[b, :c].cpu().numpy(), ora[b])


def test_response_only_steps_tiny(lib):
    r = Run(lib, SY.TINY, select_from=SY.TINY.prompt_len)
    P = SY.TINY.prompt_len
    r.gpu_step(True)
    kv0 = [t[:, :P].clone() for t in r.cache.k + r.cache.v]
    for t in range(1, 5):
        tok_before = f64(r.tokens).astype(np.int64)
        href_before = f64(r.cache.h_ref)
        conf_before = f64(r.cache.conf)
        idx, cnt, pos, sc = r.gpu_step(False)
        masked = tok_before == r.ocfg.mask_id
        h = r.ow.embed[tok_before]
        ora = O.importance(O.variation(h, href_before, r.opol.kind), conf_before, masked,
                           r.opol.alpha)
        assert max_abs_rel(sc[:, P:], ora[:, P:]) < TOL["f32"]
        assert np.all(np.isneginf(sc[:, :P]))
        sel = O.select(sc, O.SELECT_TOPK, r.opol.k, 0.0, r.k_cap, P)
        for b in range(r.B):
            np.testing.assert_array_equal(idx[b, :cnt[b]], sel[b])
            assert idx[b, :cnt[b]].min() >= P
    for a, b in zip(kv0, [t[:, :P] for t in r.cache.k + r.cache.v]):
        assert torch.equal(a, b)


def test_threshold_unmask_inside_a_step(lib):
    shape = _small_bf16()
    r = Run(lib, shape)
    r.gpu_step(True)
    conf = f64(r.cache.conf)
    tok = f64(r.tokens).astype(np.int64)
    blk = O.current_block(tok[0], r.ocfg.mask_id, r.opol.gen_start, r.opol.block_len)
    m = [p for p in range(*blk) if tok[0, p] == r.ocfg.mask_id]
    tau = float(np.float32(np.quantile(conf[0, m], 0.3)))
    r.pol.unmask_tau = tau
    for t in range(2):
        tok_before = f64(r.tokens).astype(np.int64)
        idx, cnt, pos, sc = r.gpu_step(False)
        t_ora = tok_before.copy()
        p_ora = O.unmask(f64(r.cache.conf), f64(r.cache.pred).astype(np.int64), t_ora,
                         r.ocfg.mask_id, r.opol.gen_start, r.opol.block_len, r.opol.n_unmask,
                         tau)
        np.testing.assert_array_equal(pos, p_ora)
        np.testing.assert_array_equal(f64(r.tokens).astype(np.int64), t_ora)
        if t == 0:
            assert (p_ora[0] >= 0).sum() > r.opol.n_unmask   # the threshold did reveal more


def test_generate_tiny_matches_oracle(lib):
    shape = SY.with_(SY.TINY, block_len=16)
    r = Run(lib, shape, refresh_every=3, refresh_on_block=True)
    T = 8
    cap = lib.dllm_unmask_capacity(r.pol)
    pos_log = torch.full((T, r.B, cap), -9, dtype=torch.int32, device="cuda")
    ws = lib.Workspace(lib.dllm_generate_workspace_size(r.model.cfg, r.B, r.N, r.pol))
    dense = lib.dllm_generate(r.model, r.cache, r.tokens, r.pol, T, ws, pos_log=pos_log)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    d_ora, p_ora = O.generate(r.ocfg, r.ow, r.st, r.opol, T)
    assert dense == d_ora
    assert dense == [True, False, True, True, True, False, True, False]
    for t in range(T):
        np.testing.assert_array_equal(pos_log[t].cpu().numpy(), p_ora[t])
    np.testing.assert_array_equal(f64(r.tokens).astype(np.int64), r.st.tokens)
    r.compare_state(TOL["f32"])


def test_generate_equals_step_loop_bf16(lib):
    shape = _small_bf16()
    kw = dict(select_from=shape.prompt_len, refresh_every=2)
    r1, r2 = Run(lib, shape, **kw), Run(lib, shape, **kw)
    T = 5
    ws = lib.Workspace(lib.dllm_generate_workspace_size(r1.model.cfg, r1.B, r1.N, r1.pol))
    dense = lib.dllm_generate(r1.model, r1.cache, r1.tokens, r1.pol, T, ws)
    assert dense == [True, False, True, False, True]
    for t in range(T):
        r2.gpu_step(dense[t])
    torch.cuda.synchronize()
    assert torch.equal(r1.tokens, r2.tokens)
    for a, b in zip(r1.cache.k + r1.cache.v + [r1.cache.h_ref, r1.cache.conf, r1.cache.pred],
                    r2.cache.k + r2.cache.v + [r2.cache.h_ref, r2.cache.conf, r2.cache.pred]):
        assert torch.equal(a, b)


# ----------------------------------------------------------------- two skip points


def _pad(rows, width, fill=-1):
    a = np.full((len(rows), width), fill, dtype=np.int32)
    for b, r in enumerate(rows):
        a[b, :len(r)] = r
    return torch.from_numpy(a).cuda()


def _two_point_run(lib, shape, k2):
    r = Run(lib, shape, score_layer2=2, k2=k2)
    r.pol.score_layer2, r.pol.k2 = 2, k2
    r.cache = lib.Cache(r.model.cfg, r.B, r.N, second_ref=True)
    r.ws = lib.Workspace(lib.dllm_step_workspace_size(r.model.cfg, r.B, r.N, r.pol))
    r.k2_cap = max(1, min(k2, r.k_cap))
    return r


def _two_point_forced(lib, shape, k2, tol, steps):
    r = _two_point_run(lib, shape, k2)
    for t in range(steps):
        out = O.step(r.ocfg, r.ow, r.st, r.opol, dense=(t == 0))
        io = {"forced_unmask_pos": _pad(out.unmasked, out.unmasked.shape[1])}
        if t > 0:
            io.update(forced_idx=_pad(out.idx, r.k_cap),
                      forced_count=torch.tensor([len(a) for a in out.idx], dtype=torch.int32,
                                                device="cuda"),
                      forced_idx2=_pad(out.idx2, r.k2_cap),
                      forced_count2=torch.tensor([len(a) for a in out.idx2], dtype=torch.int32,
                                                 device="cuda"))
        lib.dllm_step_ex(r.model, r.cache, r.tokens, r.pol, t == 0, r.ws, **io)
        torch.cuda.synchronize()
        assert r.ws.device_status() == 0
        final_idx = out.idx2 if out.idx2 is not None else out.idx
        r.compare_state(tol, out.final_rows, final_idx)
        assert max_abs_rel(f64(r.cache.h_ref2), r.st.h_ref2) < tol
        r.tokens.copy_(torch.from_numpy(r.st.tokens.astype(np.int32)))
    return r


def test_two_point_tiny_f32_forced(lib):
    _two_point_forced(lib, SY.with_(SY.TINY, n_layers=3), 12, TOL["f32"], 5)


def test_two_point_bf16_forced(lib):
    _two_point_forced(lib, _small_bf16(n_layers=4), 10, TOL["bf16"], 4)


def test_two_point_own_decisions_follow_the_rule(lib):
    shape = SY.with_(SY.TINY, n_layers=3)
    r = _two_point_run(lib, shape, 12)
    lib.dllm_step_ex(r.model, r.cache, r.tokens, r.pol, True, r.ws)
    for t in range(1, 4):
        B = r.B
        idx = torch.full((B, r.k_cap), -1, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
        idx2 = torch.full((B, r.k2_cap), -1, dtype=torch.int32, device="cuda")
        cnt2 = torch.zeros(B, dtype=torch.int32, device="cuda")
        sc2 = torch.zeros(B, r.k_cap, dtype=torch.float32, device="cuda")
        lib.dllm_step_ex(r.model, r.cache, r.tokens, r.pol, False, r.ws, idx_out=idx,
                         count_out=cnt, idx2_out=idx2, count2_out=cnt2, scores2_out=sc2)
        torch.cuda.synchronize()
        assert r.ws.device_status() == 0
        for b in range(B):
            c = int(cnt[b])
            first = idx[b, :c].cpu().numpy()
            s2 = sc2[b, :c].cpu().numpy()
            keep = first[O.select_topk(s2, 12)]
            np.testing.assert_array_equal(idx2[b, :int(cnt2[b])].cpu().numpy(), keep)


# ----------------------------------------------------------------- incremental attention


def _lse(m, l):
    return np.asarray(m, dtype=np.float64) + np.log(np.asarray(l, dtype=np.float64))


def _update_case(lib, Hq, Hkv, hd, N, r_count, a_count, r_cap, a_cap):
    g = torch.Generator().manual_seed(31)
    B = len(r_count)
    kc = SY.normal((B, N, Hkv, hd), 1.0, 41, "cuda", "bf16")
    vc = SY.normal((B, N, Hkv, hd), 1.0, 42, "cuda", "bf16")
    q = SY.normal((B * r_cap, Hq * hd), 1.0, 43, "cuda", "bf16")
    o = torch.zeros_like(q)
    m = torch.zeros(B * r_cap, Hq, dtype=torch.float32, device="cuda")
    l = torch.zeros_like(m)
    rc = torch.tensor(r_count, dtype=torch.int32, device="cuda")
    lib.dllm_attention_stats_bf16(q, kc, vc, o, m, l, rc, r_cap)
    torch.cuda.synchronize()
    # statistics of the exact attention: the same log-sum-exp as the oracle's
    off = 0
    for b, c in enumerate(r_count):
        if c == 0:
            continue
        qb = f64(q[off:off + c]).reshape(c, Hq, hd)
        om, ol, oo = O.attention_stats(qb, f64(kc[b]), f64(vc[b]))
        assert np.max(np.abs(_lse(m[off:off + c].cpu(), l[off:off + c].cpu()) - _lse(om, ol))) < 2e-2
        assert max_abs_rel(f64(o[off:off + c]), O.store(oo, "bf16").reshape(c, -1)) < TOL["bf16"]
        off += c
    # change a_count[b] keys of each sequence (new keys larger: new scores pass the old max)
    k_new = torch.zeros(B * a_cap, Hkv, hd, dtype=torch.bfloat16, device="cuda")
    v_new, k_old, v_old = torch.zeros_like(k_new), torch.zeros_like(k_new), torch.zeros_like(k_new)
    kc2, vc2 = kc.clone(), vc.clone()
    aoff = 0
    for b, a in enumerate(a_count):
        pos = torch.randperm(N, generator=g)[:a].sort()[0].cuda()
        kn = (torch.randn(a, Hkv, hd, generator=g) * 1.8).to(torch.bfloat16).cuda()
        vn = torch.randn(a, Hkv, hd, generator=g).to(torch.bfloat16).cuda()
        k_old[aoff:aoff + a], v_old[aoff:aoff + a] = kc[b, pos], vc[b, pos]
        k_new[aoff:aoff + a], v_new[aoff:aoff + a] = kn, vn
        kc2[b, pos], vc2[b, pos] = kn, vn
        aoff += a
    ac = torch.tensor(a_count, dtype=torch.int32, device="cuda")
    o_before, m_before, l_before = o.clone(), m.clone(), l.clone()
    ws = lib.dllm_attention_update_bf16(q, o, m, l, rc, r_cap, k_new, v_new, k_old, v_old, ac,
                                        a_cap, Hkv)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    off = 0
    for b, c in enumerate(r_count):
        sl = slice(off, off + c)
        if c == 0:
            continue
        if a_count[b] == 0:
            assert torch.equal(o[sl], o_before[sl]) and torch.equal(m[sl], m_before[sl])
            assert torch.equal(l[sl], l_before[sl])
        else:
            qb = f64(q[sl]).reshape(c, Hq, hd)
            em, el, eo = O.attention_stats(qb, f64(kc2[b]), f64(vc2[b]))
            assert max_abs_rel(f64(o[sl]), O.store(eo, "bf16").reshape(c, -1)) < TOL["bf16"]
            assert np.max(np.abs(_lse(m[sl].cpu(), l[sl].cpu()) - _lse(em, el))) < 2e-2
        off += c


@pytest.mark.parametrize("Hq,Hkv,hd", [(4, 2, 128), (2, 2, 64)])
def test_attention_stats_and_update_match_oracle(lib, Hq, Hkv, hd):
    # the last sequence has no changed key
    _update_case(lib, Hq, Hkv, hd, 300, [150, 70, 33], [40, 7, 0], 150, 40)


def test_attention_update_several_pairs_per_cta(lib):
    """Enough sequences x heads that a CTA walks two pairs of query tiles, the
    last pair of a sequence holding one tile (or none)."""
    _update_case(lib, 32, 8, 64, 300, [600, 300, 257, 1, 0, 520, 88, 513],
                 [40, 7, 0, 13, 3, 128, 129, 1], 600, 129)


# ----------------------------------------------------------------- FFN gate


def _gated_run(lib, shape, tau):
    r = Run(lib, shape, ffn_gate=True, ffn_tau=tau)
    r.pol.ffn_gate, r.pol.ffn_tau = 1, tau
    r.cache = lib.Cache(r.model.cfg, r.B, r.N, ffn_gate=True)
    r.ws = lib.Workspace(lib.dllm_step_workspace_size(r.model.cfg, r.B, r.N, r.pol))
    return r


def _gated_forced(lib, shape, tau, tol, steps):
    r = _gated_run(lib, shape, tau)
    L = r.ocfg.n_layers
    for t in range(steps):
        out = O.step(r.ocfg, r.ow, r.st, r.opol, dense=(t == 0))
        rows = torch.full((L,), -1, dtype=torch.int32, device="cuda")
        io = {"forced_unmask_pos": _pad(out.unmasked, out.unmasked.shape[1]), "ffn_rows_out": rows}
        if t > 0:
            io.update(forced_idx=_pad(out.idx, r.k_cap),
                      forced_count=torch.tensor([len(a) for a in out.idx], dtype=torch.int32,
                                                device="cuda"))
        lib.dllm_step_ex(r.model, r.cache, r.tokens, r.pol, t == 0, r.ws, **io)
        torch.cuda.synchronize()
        assert r.ws.device_status() == 0
        assert rows.cpu().tolist() == out.ffn_rows
        r.compare_state(tol, out.final_rows, out.idx)
        for l in range(L):
            assert max_abs_rel(f64(r.cache.ctx[l]), r.st.ctx[l]) < tol, ("ctx", l)
            assert max_abs_rel(f64(r.cache.ffn[l]), r.st.ffn[l]) < tol, ("ffn", l)
        r.tokens.copy_(torch.from_numpy(r.st.tokens.astype(np.int32)))
    return r


@pytest.mark.parametrize("tau", [-1.0, 2.5])
def test_ffn_gate_tiny_f32_forced(lib, tau):
    _gated_forced(lib, SY.with_(SY.TINY, n_layers=2), tau, TOL["f32"], 5)


@pytest.mark.parametrize("tau", [-1.0, 2.5])
def test_ffn_gate_bf16_forced(lib, tau):
    _gated_forced(lib, _small_bf16(), tau, TOL["bf16"], 4)


def test_ffn_gate_fixed_point_bf16(lib):
    """After a dense step, a gated step over unchanged tokens finds every context
    where it was (up to rounding), runs no FFN and reproduces the dense rows."""
    shape = _small_bf16(n_unmask=0)
    r = _gated_run(lib, shape, 1e-3)
    lib.dllm_step_ex(r.model, r.cache, r.tokens, r.pol, True, r.ws)
    kv0 = [t.clone() for t in r.cache.k + r.cache.v]
    rows = torch.full((r.ocfg.n_layers,), -1, dtype=torch.int32, device="cuda")
    lib.dllm_step_ex(r.model, r.cache, r.tokens, r.pol, False, r.ws, ffn_rows_out=rows)
    torch.cuda.synchronize()
    assert r.ws.device_status() == 0
    assert rows.cpu().tolist() == [0] * r.ocfg.n_layers
    for a, b in zip(kv0, r.cache.k + r.cache.v):
        assert max_abs_rel(f64(b), f64(a)) < TOL["bf16"]


def _gated_mixed_forced(lib, shape, tau, tol, steps):
    """The gate at a threshold that splits the recomputed rows (DyLLM, French
    summary §2.A): the oracle decides every row of every layer, the GPU takes
    those decisions (forced_ffn, as forced_idx does for the selection), and the
    caches -- K/V, contexts, FFN outputs -- are compared after each step."""
    r = _gated_run(lib, shape, tau)
    L = r.ocfg.n_layers
    mixed = 0
    for t in range(steps):
        out = O.step(r.ocfg, r.ow, r.st, r.opol, dense=(t == 0))
        rows = torch.full((L,), -1, dtype=torch.int32, device="cuda")
        io = {"forced_unmask_pos": _pad(out.unmasked, out.unmasked.shape[1]), "ffn_rows_out": rows}
        if t > 0:
            io.update(forced_idx=_pad(out.idx, r.k_cap),
                      forced_count=torch.tensor([len(a) for a in out.idx], dtype=torch.int32,
                                                device="cuda"))
            fz = np.zeros((L, r.B * r.k_cap), dtype=np.uint8)
            first = L - len(out.ffn_salient)
            for j, sal in enumerate(out.ffn_salient):
                fz[first + j, :len(sal)] = sal
                mixed += int(0 < int(sal.sum()) < len(sal))
            io["forced_ffn"] = torch.from_numpy(fz).cuda()
        lib.dllm_step_ex(r.model, r.cache, r.tokens, r.pol, t == 0, r.ws, **io)
        torch.cuda.synchronize()
        assert r.ws.device_status() == 0
        assert rows.cpu().tolist() == out.ffn_rows
        r.compare_state(tol, out.final_rows, out.idx)
        for l in range(L):
            assert max_abs_rel(f64(r.cache.ctx[l]), r.st.ctx[l]) < tol, ("ctx", l)
            assert max_abs_rel(f64(r.cache.ffn[l]), r.st.ffn[l]) < tol, ("ffn", l)
        r.tokens.copy_(torch.from_numpy(r.st.tokens.astype(np.int32)))
    assert mixed > 0   # some layer-step ran the FFN on part of its rows only


def test_ffn_gate_mixed_threshold_bf16_forced(lib):
    _gated_mixed_forced(lib, _small_bf16(), 1e-3, TOL["bf16"], 4)


def test_ffn_gate_mixed_threshold_tiny_f32_forced(lib):
    _gated_mixed_forced(lib, SY.with_(SY.TINY, n_layers=2), 1e-2, TOL["f32"], 4)


def test_ffn_gate_own_decisions_follow_the_rule(lib):
    """The GPU's own gate at a mixed threshold: in every layer of every partial
    step, a recomputed row ran the FFN (its cached FFN output changed) exactly
    when 1 - cos(its new context, its previous context) > tau, evaluated here in
    float64 on the contexts the GPU stored; rows within 1e-5 of tau (where the
    kernel's fp32 cosine may fall on either side) are only counted."""
    tau, band = 1e-3, 1e-5
    shape = _small_bf16()
    r = _gated_run(lib, shape, tau)
    L, B = r.ocfg.n_layers, r.B
    lib.dllm_step_ex(r.model, r.cache, r.tokens, r.pol, True, r.ws)
    mixed = 0
    for t in range(1, 4):
        ctx0 = [f64(c) for c in r.cache.ctx]
        ffn0 = [c.clone() for c in r.cache.ffn]
        idx = torch.full((B, r.k_cap), -1, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
        rows = torch.full((L,), -1, dtype=torch.int32, device="cuda")
        lib.dllm_step_ex(r.model, r.cache, r.tokens, r.pol, False, r.ws, idx_out=idx,
                         count_out=cnt, ffn_rows_out=rows)
        torch.cuda.synchronize()
        assert r.ws.device_status() == 0
        sel = [(b, int(p)) for b in range(B) for p in idx[b, :int(cnt[b])].cpu().numpy()]
        bs = np.array([b for b, _ in sel])
        ps = np.array([p for _, p in sel])
        for l in range(L):
            ran = torch.any(r.cache.ffn[l] != ffn0[l], dim=-1).cpu().numpy()[bs, ps]
            assert int(ran.sum()) == int(rows[l])
            v = O.variation(f64(r.cache.ctx[l])[bs, ps], ctx0[l][bs, ps], O.SCORE_COS)
            clear = np.abs(v - tau) > band
            np.testing.assert_array_equal(ran[clear], (v > tau)[clear])
            mixed += int(0 < ran.sum() < len(ran))
    assert mixed > 0


def test_step_host_equals_device_step(lib):
    """dllm_step_host (token state in pinned host memory, copied in and out by the
    library on the stream) reproduces dllm_step on device tokens bit for bit."""
    shape = _small_bf16()
    r1, r2 = Run(lib, shape), Run(lib, shape)
    cap = max(lib.dllm_unmask_capacity(r1.pol), 1)
    ws_h = lib.Workspace(lib.dllm_step_host_workspace_size(r2.model.cfg, r2.B, r2.N, r2.pol))
    tok_h = r2.tokens.cpu().pin_memory()
    pos_h = torch.full((r2.B, cap), -9, dtype=torch.int32).pin_memory()
    for t in range(4):
        pos = torch.full((r1.B, cap), -9, dtype=torch.int32, device="cuda")
        lib.dllm_step(r1.model, r1.cache, r1.tokens, r1.pol, t == 0, r1.ws, pos_out=pos)
        lib.dllm_step_host(r2.model, r2.cache, tok_h, r2.pol, t == 0, ws_h, pos_h)
        torch.cuda.synchronize()
        assert torch.equal(r1.tokens.cpu(), tok_h)
        assert torch.equal(pos.cpu(), pos_h)
    assert ws_h.device_status() == 0
    for a, b in zip(r1.cache.k + r1.cache.v + [r1.cache.h_ref, r1.cache.conf, r1.cache.pred],
                    r2.cache.k + r2.cache.v + [r2.cache.h_ref, r2.cache.conf, r2.cache.pred]):
        assert torch.equal(a, b)


# ----------------------------------------------------------------- approximate attention step


def _upd_run(lib, shape, tau, prebuilt=None):
    r = Run(lib, shape, prebuilt=prebuilt, ffn_gate=True, ffn_tau=tau, attn_update=True)
    r.pol.ffn_gate, r.pol.ffn_tau, r.pol.attn_update = 1, tau, 1
    r.cache = lib.Cache(r.model.cfg, r.B, r.N, ffn_gate=True, attn_update=True)
    r.ws = lib.Workspace(lib.dllm_step_workspace_size(r.model.cfg, r.B, r.N, r.pol))
    return r


def _lse(m, l):
    return np.asarray(m, dtype=np.float64) + np.log(np.asarray(l, dtype=np.float64))


def _compare_upd_caches(r, tol):
    Hq = r.ocfg.n_heads
    for l in range(r.ocfg.n_layers):
        assert max_abs_rel(f64(r.cache.ctx[l]), r.st.ctx[l]) < tol, ("ctx", l)
        assert max_abs_rel(f64(r.cache.ffn[l]), r.st.ffn[l]) < tol, ("ffn", l)
        assert max_abs_rel(f64(r.cache.q[l]), r.st.q[l]) < tol, ("q", l)
        lse_g = _lse(f64(r.cache.att_m[l]), f64(r.cache.att_l[l]))
        lse_o = _lse(r.st.att_m[l], r.st.att_l[l])
        assert np.max(np.abs(lse_g - lse_o)) < tol * max(np.abs(lse_o).max(), 1.0), ("lse", l)


def _upd_forced(lib, shape, tau, tol, steps, prebuilt=None):
    """DyLLM's approximate attention inside partial steps (French summary §2.B):
    the GPU follows the oracle's selections, reveals and FFN-gate decisions; every
    cache -- K/V, contexts (the stable rows' ones updated incrementally), FFN
    outputs, queries and softmax statistics -- is compared after each step."""
    r = _upd_run(lib, shape, tau, prebuilt)
    L = r.ocfg.n_layers
    for t in range(steps):
        out = O.step(r.ocfg, r.ow, r.st, r.opol, dense=(t == 0))
        io = {"forced_unmask_pos": _pad(out.unmasked, out.unmasked.shape[1])}
        if t > 0:
            io.update(forced_idx=_pad(out.idx, r.k_cap),
                      forced_count=torch.tensor([len(a) for a in out.idx], dtype=torch.int32,
                                                device="cuda"))
            fz = np.zeros((L, r.B * r.k_cap), dtype=np.uint8)
            first = L - len(out.ffn_salient)
            for j, sal in enumerate(out.ffn_salient):
                fz[first + j, :len(sal)] = sal
            io["forced_ffn"] = torch.from_numpy(fz).cuda()
        lib.dllm_step_ex(r.model, r.cache, r.tokens, r.pol, t == 0, r.ws, **io)
        torch.cuda.synchronize()
        assert r.ws.device_status() == 0
        r.compare_tokens(r.compare_state(tol, out.final_rows, out.idx))
        _compare_upd_caches(r, tol)
    return r


def test_approximate_attention_step_bf16_forced(lib):
    _upd_forced(lib, _small_bf16(), 1e-3, TOL["bf16"], 4)


def test_approximate_attention_step_gqa_forced(lib):
    _upd_forced(lib, _small_bf16(n_heads=4, n_kv_heads=2, head_dim=64, batch=3), 1e-3,
                TOL["bf16"], 4)


def test_approximate_attention_step_own_run_tracks_its_caches(lib):
    """On its own decisions, after every step each row's cached context on the GPU
    equals the attention of its cached query over the GPU's current K/V caches
    (oracle attention in float64 on the GPU's caches; the invariant the oracle's
    step mode is pinned by), and its (m, l) give that attention's log-sum-exp."""
    shape = _small_bf16()
    r = _upd_run(lib, shape, 1e-3)
    Hq, hd = r.ocfg.n_heads, r.ocfg.head_dim
    for t in range(4):
        lib.dllm_step_ex(r.model, r.cache, r.tokens, r.pol, t == 0, r.ws)
        torch.cuda.synchronize()
        assert r.ws.device_status() == 0
        for l in range(r.ocfg.n_layers):
            for b in range(r.B):
                q = f64(r.cache.q[l][b]).reshape(r.N, Hq, hd)
                m, lsum, o = O.attention_stats(q, f64(r.cache.k[l][b]), f64(r.cache.v[l][b]))
                got = f64(r.cache.ctx[l][b])
                assert max_abs_rel(got, o.reshape(r.N, -1)) < TOL["bf16"], (t, l, b)
                lse = _lse(f64(r.cache.att_m[l][b]), f64(r.cache.att_l[l][b]))
                assert np.max(np.abs(lse - (m + np.log(lsum)))) < 2e-2 * max(np.abs(m).max(), 1), (t, l, b)
