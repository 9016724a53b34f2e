"""Pins of the CPU oracle against things other than itself.

Each test fixes a piece of the oracle with a closed form, a textbook or
library routine it must reduce to, brute force on tiny inputs, or an
invariant the pages state.  They run on the CPU (no GPU marker).
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special as sps
import torch
import torch.nn.functional as F

import oracle as O


# ---------------------------------------------------------------- bf16 storage

def test_bf16_round_hand_values():
    one = 1.0
    assert O.bf16_round(one) == 1.0
    assert O.bf16_round(1.0 + 2.0 ** -8) == 1.0                      # tie -> even (down)
    assert O.bf16_round(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6      # tie -> even (up)
    assert O.bf16_round(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7  # above tie -> up
    assert O.bf16_round(-3.0) == -3.0
    assert np.isinf(O.bf16_round(3.5e38))
    assert O.bf16_round(0.0) == 0.0


def test_bf16_round_matches_torch_on_float32_values():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-30).astype(np.float32),
        (rng.standard_normal(2000) * 1e30).astype(np.float32),
        # exact halfway points between neighbouring bf16 values
        (np.float32(1.0) + np.float32(2.0 ** -8) * np.arange(1, 200, 2, dtype=np.float32)),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


# ---------------------------------------------------------------- RMSNorm

def test_rms_norm_constant_row_closed_form():
    d, c, eps = 64, -3.0, 1e-5
    g = np.linspace(0.5, 1.5, d)
    out = O.rms_norm(np.full((2, d), c), g, eps)
    np.testing.assert_allclose(out, np.broadcast_to(c / math.sqrt(c * c + eps) * g, (2, d)),
                               rtol=1e-14)


def test_rms_norm_matches_torch_library():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 96)) * 3
    g = rng.standard_normal(96)
    ref = F.rms_norm(torch.from_numpy(x), (96,), torch.from_numpy(g), eps=1e-5).numpy()
    np.testing.assert_allclose(O.rms_norm(x, g, 1e-5), ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- RoPE

def test_rope_is_complex_rotation():
    rng = np.random.default_rng(2)
    R, H, hd = 7, 3, 16
    x = rng.standard_normal((R, H, hd))
    pos = rng.integers(0, 3000, R)
    theta = 5.0e5
    out = O.rope(x, pos, theta)
    half = hd // 2
    z = x[..., :half] + 1j * x[..., half:]
    rate = O.rope_inv_freq(hd, theta)
    zr = z * np.exp(1j * pos[:, None, None] * rate[None, None, :])
    np.testing.assert_allclose(out[..., :half], zr.real, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out[..., half:], zr.imag, rtol=1e-12, atol=1e-12)


def test_rope_frequencies_hand_values():
    # theta = 10000, hd = 4: pair 0 turns at rate 1, pair 1 at 10000^(-1/2) = 0.01
    np.testing.assert_allclose(O.rope_inv_freq(4, 10000.0), [1.0, 0.01], rtol=1e-15)
    x = np.zeros((1, 1, 4)); x[0, 0, 0] = 1.0; x[0, 0, 1] = 1.0
    out = O.rope(x, np.array([2]), 10000.0)
    np.testing.assert_allclose(out[0, 0], [math.cos(2), math.cos(0.02), math.sin(2),
                                           math.sin(0.02)], rtol=1e-14)


def test_rope_identity_at_zero_norm_preserving_relative():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 2, 64))
    np.testing.assert_array_equal(O.rope(x, np.zeros(4, int), 5e5), x)
    y = O.rope(x, np.array([1, 50, 700, 2047]), 5e5)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    q, k = x[:1], x[1:2]
    a = np.sum(O.rope(q, np.array([10]), 5e5) * O.rope(k, np.array([3]), 5e5))
    b = np.sum(O.rope(q, np.array([110]), 5e5) * O.rope(k, np.array([103]), 5e5))
    assert abs(a - b) < 1e-10
    np.testing.assert_array_equal(O.rope(x, np.array([1, 2, 3, 4]), 0.0), x)


# ---------------------------------------------------------------- attention

def test_attention_single_key_returns_value():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((3, 2, 8))
    K = rng.standard_normal((1, 2, 8))
    V = rng.standard_normal((1, 2, 8))
    out = O.attention(q, K, V)
    np.testing.assert_allclose(out, np.broadcast_to(V, (3, 2, 8)), rtol=1e-15)


def test_attention_equal_keys_give_mean():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((2, 1, 8))
    K = np.repeat(rng.standard_normal((1, 1, 8)), 6, axis=0)
    V = rng.standard_normal((6, 1, 8))
    np.testing.assert_allclose(O.attention(q, K, V)[:, 0], np.broadcast_to(V[:, 0].mean(0), (2, 8)),
                               rtol=1e-13)


def test_attention_two_keys_logistic_closed_form():
    # q.k1 - q.k2 = delta * sqrt(hd)  =>  weight of v1 = sigmoid(delta)
    hd, delta = 16, 0.7
    q = np.zeros((1, 1, hd)); q[0, 0, 0] = 1.0
    K = np.zeros((2, 1, hd)); K[0, 0, 0] = delta * math.sqrt(hd)
    V = np.zeros((2, 1, hd)); V[0, 0, 1] = 1.0; V[1, 0, 2] = 1.0
    out = O.attention(q, K, V)[0, 0]
    w = 1.0 / (1.0 + math.exp(-delta))
    np.testing.assert_allclose(out[1:3], [w, 1 - w], rtol=1e-14)


def test_attention_gqa_head_mapping():
    # 4 query heads over 2 KV heads: heads 0,1 read KV head 0; heads 2,3 read KV head 1
    q = np.ones((1, 4, 4))
    K = np.ones((1, 2, 4))
    V = np.zeros((1, 2, 4)); V[0, 0] = 1.0; V[0, 1] = 2.0
    out = O.attention(q, K, V)
    np.testing.assert_array_equal(out[0, :, 0], [1.0, 1.0, 2.0, 2.0])


def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(6)
    R, N, Hq, Hkv, hd = 5, 37, 6, 2, 16
    q = rng.standard_normal((R, Hq, hd))
    K = rng.standard_normal((N, Hkv, hd))
    V = rng.standard_normal((N, Hkv, hd))
    tq = torch.from_numpy(q).permute(1, 0, 2)                  # [Hq, R, hd]
    tk = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
    tv = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
    ref = F.scaled_dot_product_attention(tq, tk, tv, is_causal=False).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(O.attention(q, K, V), ref, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- whole layer

def _textbook_layer(x, w, pos, theta, eps, Hq, Hkv, hd):
    """A LLaMA-style pre-norm block written with torch library routines
    (rms_norm, complex RoPE via torch.polar, sdpa, silu), float64."""
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    x = t(x)
    n = F.rms_norm(x, (x.shape[-1],), t(w.attn_norm), eps=eps)
    R = x.shape[0]
    q = (n @ t(w.wq).T).view(R, Hq, hd)
    k = (n @ t(w.wk).T).view(R, Hkv, hd)
    v = (n @ t(w.wv).T).view(R, Hkv, hd)
    half = hd // 2
    j = torch.arange(half, dtype=torch.float64)
    freqs = torch.pow(torch.tensor(theta, dtype=torch.float64), -2.0 * j / hd)
    ang = t(pos)[:, None] * freqs[None, :]
    rot = torch.polar(torch.ones_like(ang), ang)[:, None, :]

    def rope(a):
        z = torch.complex(a[..., :half], a[..., half:]) * rot
        return torch.cat([z.real, z.imag], dim=-1)

    q, k = rope(q), rope(k)
    o = F.scaled_dot_product_attention(q.permute(1, 0, 2),
                                       k.permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0),
                                       v.permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0))
    x = x + o.permute(1, 0, 2).reshape(R, Hq * hd) @ t(w.wo).T
    n2 = F.rms_norm(x, (x.shape[-1],), t(w.ffn_norm), eps=eps)
    x = x + (F.silu(n2 @ t(w.w_gate).T) * (n2 @ t(w.w_up).T)) @ t(w.w_down).T
    return x.numpy(), k.numpy(), v.numpy()


def _rand_layer(rng, d, Hq, Hkv, hd, Fd, std=0.1):
    m = lambda r, c: rng.standard_normal((r, c)) * std
    return O.LayerW(1 + 0.1 * rng.standard_normal(d), m(Hq * hd, d), m(Hkv * hd, d),
                    m(Hkv * hd, d), m(d, Hq * hd), 1 + 0.1 * rng.standard_normal(d),
                    m(Fd, d), m(Fd, d), m(d, Fd))


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2)])
def test_layer_matches_textbook_block(Hq, Hkv):
    rng = np.random.default_rng(7)
    N, d, hd, Fd = 11, 32, 8, 40
    cfg = O.ModelCfg(1, d, Hq, Hkv, hd, Fd, 50, 1000.0, 1e-5, dtype=O.F32)
    w = _rand_layer(rng, d, Hq, Hkv, hd, Fd)
    x = rng.standard_normal((N, d))
    pos = np.arange(N)
    kc = np.zeros((1, N, Hkv, hd)); vc = np.zeros((1, N, Hkv, hd))
    out = O.layer_rows(cfg, w, x, np.zeros(N, int), pos, kc, vc)
    ref, rk, rv = _textbook_layer(x, w, pos, 1000.0, 1e-5, Hq, Hkv, hd)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(kc[0], rk, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(vc[0], rv, rtol=1e-11, atol=1e-11)


def test_silu_is_x_times_logistic():
    x = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(O.silu(x), x * sps.expit(x), rtol=1e-13, atol=1e-300)


# ---------------------------------------------------------------- confidence

def test_confidence_equal_logits():
    conf, pred = O.confidence(np.full((3, 1024), 0.37))
    np.testing.assert_array_equal(conf, np.full(3, 1.0 / 1024))
    np.testing.assert_array_equal(pred, [0, 0, 0])


def test_confidence_matches_softmax_library():
    rng = np.random.default_rng(8)
    z = rng.standard_normal((6, 777)) * 3
    conf, pred = O.confidence(z)
    p = sps.softmax(z, axis=-1)
    np.testing.assert_allclose(conf, p.max(-1), rtol=1e-13)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-13)
    np.testing.assert_array_equal(pred, p.argmax(-1))
    assert np.all(conf > 1.0 / 777) and np.all(conf <= 1.0)


def test_confidence_tie_goes_to_lowest_id_and_dominant_logit():
    z = np.zeros((2, 10)); z[0, 3] = z[0, 7] = 5.0; z[1, 9] = 200.0
    conf, pred = O.confidence(z)
    assert pred[0] == 3 and pred[1] == 9
    assert conf[1] == 1.0


# ---------------------------------------------------------------- variation / importance

def test_variation_special_cases():
    rng = np.random.default_rng(9)
    a = rng.standard_normal(64)
    b = rng.standard_normal(64); b -= a * (a @ b) / (a @ a)   # orthogonal to a
    h = np.stack([a, a, a, np.zeros(64), np.zeros(64)])
    r = np.stack([a, b, -a, a, np.zeros(64)])
    v = O.variation(h, r, O.SCORE_COS)
    assert v[0] == 0.0
    assert abs(v[1] - 1.0) < 1e-14
    assert abs(v[2] - 2.0) < 1e-14
    assert v[3] == 1.0 and v[4] == 0.0
    # ES L1 form: one coordinate moved by delta -> |delta| / (sqrt(d) * ||ref||)
    delta = -0.3
    h2 = a.copy(); h2[5] += delta
    ve = O.variation(h2[None], a[None], O.SCORE_ES_L1)[0]
    assert abs(ve - abs(delta) / (8.0 * np.linalg.norm(a))) < 1e-15
    assert O.variation(a[None], a[None], O.SCORE_ES_L1)[0] == 0.0
    assert np.isinf(O.variation(a[None], np.zeros((1, 64)), O.SCORE_ES_L1)[0])


@pytest.mark.parametrize("sigma,expect", [(0.5, 1 / math.sqrt(1.25)), (1e-3, 1 / math.sqrt(1 + 1e-6))])
def test_cosine_of_noisy_copy_closed_form(sigma, expect):
    # for h ~ N(0, I_d), h_ref = h + sigma * N(0, I_d): cos -> 1/sqrt(1 + sigma^2) as d grows
    rng = np.random.default_rng(10)
    h = rng.standard_normal((64, 4096))
    r = h + sigma * rng.standard_normal((64, 4096))
    cos = 1.0 - O.variation(h, r, O.SCORE_COS)
    assert abs(cos.mean() - expect) < 3e-3 * max(sigma, 1e-3) / 0.5 + 1e-9


def test_importance_worked_values():
    # alpha = 0.5: masked row c = 0.8, v = 0.2 -> 0.5; unmasked row ignores c
    v = np.array([0.2, 0.2, 0.0])
    conf = np.array([0.8, 0.8, 0.9])
    masked = np.array([1, 0, 1])
    np.testing.assert_allclose(O.importance(v, conf, masked, 0.5), [0.5, 0.1, 0.45], rtol=1e-15)
    np.testing.assert_allclose(O.importance(v, conf, masked, 0.0), v, rtol=0)


# ---------------------------------------------------------------- selection

def _brute_topk(s, k):
    """Pick the best remaining position k times with an explicit comparator."""
    def better(i, j):
        a, b = s[i], s[j]
        an, bn = math.isnan(a), math.isnan(b)
        if an != bn:
            return bn
        if not an and a != b:           # -0 == +0 here by IEEE comparison
            return a > b
        return i < j
    left = list(range(len(s)))
    chosen = []
    for _ in range(min(k, len(s))):
        best = left[0]
        for i in left[1:]:
            if better(i, best):
                best = i
        chosen.append(best)
        left.remove(best)
    return sorted(chosen)


def test_select_topk_brute_force_all_patterns():
    alphabet = [0.0, -0.0, 0.5, 1.0, float("nan"), -1.0]
    for n in range(1, 5):
        for pat in itertools.product(alphabet, repeat=n):
            s = np.array(pat)
            for k in range(0, n + 1):
                assert list(O.select_topk(s, k)) == _brute_topk(list(pat), k), (pat, k)


def test_select_topk_random_ties():
    rng = np.random.default_rng(11)
    for _ in range(200):
        n = int(rng.integers(1, 40))
        s = rng.integers(0, 4, n).astype(np.float64) / 4
        k = int(rng.integers(0, n + 1))
        assert list(O.select_topk(s, k)) == _brute_topk(list(s), k)


def test_select_thresh_brute_force():
    rng = np.random.default_rng(12)
    for _ in range(200):
        n = int(rng.integers(1, 30))
        s = rng.integers(0, 5, n).astype(np.float64) / 4
        tau = float(rng.integers(0, 5)) / 4
        cap = int(rng.integers(0, n + 1))
        over = [i for i in range(n) if s[i] > tau]
        expect = over if len(over) <= cap else _brute_topk([s[i] if i in over else float("nan")
                                                            for i in range(n)], cap)
        got, n_over = O.select_thresh(s, tau, cap)
        assert n_over == len(over)
        assert list(got) == expect


# ---------------------------------------------------------------- unmasking

def test_unmask_brute_force():
    rng = np.random.default_rng(13)
    M = 9
    for _ in range(300):
        N, gs, bl = 24, 8, int(rng.integers(1, 9))
        tok = rng.integers(0, 5, N)
        tok[gs:][rng.random(N - gs) < 0.6] = M
        conf = rng.integers(0, 4, N) / 4.0
        n = int(rng.integers(0, 5))
        got = O.unmask_positions(conf, tok, M, gs, bl, n)
        masked = [p for p in range(gs, N) if tok[p] == M]
        if not masked or n == 0:
            assert len(got) == 0
            continue
        blk = gs + ((masked[0] - gs) // bl) * bl
        cand = [p for p in masked if blk <= p < blk + bl]
        chosen = []
        for _ in range(min(n, len(cand))):
            best = None
            for p in cand:
                if p in chosen:
                    continue
                if best is None or conf[p] > conf[best] or (conf[p] == conf[best] and p < best):
                    best = p
            chosen.append(best)
        assert list(got) == sorted(chosen)


def test_cache_size_matches_page_figure():
    # ES-dLLM reports about 644 MB of cache per sample for LLaDA-8B at 1024 prompt + 256
    # generated tokens; the per-layer K/V of that shape alone is 640 MiB.
    b = O.kv_cache_bytes(32, 1024 + 256, 32, 128)
    assert b == 640 * 2 ** 20
    assert abs(b / 2 ** 20 - 644) / 644 < 0.01
