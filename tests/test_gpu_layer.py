"""GPU parity of one partial layer (dllm_partial_layer) against the oracle's
layer on the same rows, for fp32 and bf16 models, MHA and GQA, ragged
per-sequence counts, and the full 8B-shaped launch (32 x 1536, 308 rows per
sequence) checked on sampled sequences."""
import numpy as np
import pytest
import torch

import oracle as O
import dllm_synth as SY
from _util import f64, max_abs_rel, TOL, oracle_cfg
from _gpu import to_dev

pytestmark = pytest.mark.gpu


def _run_layer(lib, shape, B, N, counts, k_cap, seed=0, x_full=True, weights_on_gpu=False,
               check_seqs=None, kv_std=1.0):
    dt = shape.dtype
    tdt = SY.torch_dtype(dt)
    if weights_on_gpu:
        Wd = SY.model_weights(shape, seed=seed, device="cuda")
    else:
        Wd = to_dev(SY.model_weights(shape, seed=seed, device="cpu"))
    L = Wd["layers"][0]
    cfg = lib.cfg_from_shape(shape)
    lw = lib.layer_struct(L)
    rng = np.random.default_rng(seed + 1)
    idx = np.full((B, k_cap), -1, dtype=np.int32)
    for b, c in enumerate(counts):
        idx[b, :c] = np.sort(rng.choice(N, c, replace=False))
    kv_shape = (B, N, shape.n_kv_heads, shape.head_dim)
    kc = SY.normal(kv_shape, kv_std, seed + 2, "cuda", dt)
    vc = SY.normal(kv_shape, kv_std, seed + 3, "cuda", dt)
    h = SY.normal((B, N, shape.d), 1.0, seed + 4, "cuda", dt)
    kc0, vc0 = kc.clone(), vc.clone()
    x_out = torch.zeros(B * k_cap, shape.d, dtype=tdt, device="cuda")
    idx_t = torch.from_numpy(idx).cuda()
    cnt_t = torch.tensor(counts, dtype=torch.int32, device="cuda")
    ws = lib.Workspace(lib.dllm_partial_layer_workspace_size(cfg, B, N, k_cap))
    if x_full:
        lib.dllm_partial_layer(cfg, lw, h, x_out, idx_t, cnt_t, kc, vc, ws, x_in_is_full=True)
    else:
        xin = torch.zeros_like(x_out)
        off = 0
        for b, c in enumerate(counts):
            xin[off:off + c] = h[b, torch.from_numpy(idx[b, :c]).long().cuda()]
            off += c
        lib.dllm_partial_layer(cfg, lw, xin, x_out, idx_t, cnt_t, kc, vc, ws, x_in_is_full=False)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    # oracle, per checked sequence
    ocfg = oracle_cfg(shape)
    ow = O.LayerW(**{k: f64(v) for k, v in L.items()})
    seqs = range(B) if check_seqs is None else check_seqs
    offs = np.concatenate([[0], np.cumsum(counts)])
    tol = TOL[dt]
    for b in seqs:
        c = counts[b]
        kb, vb = f64(kc0[b:b + 1]), f64(vc0[b:b + 1])
        rows = idx[b, :c].astype(np.int64)
        x = f64(h[b])[rows]
        out = O.layer_rows(ocfg, ow, x, np.zeros(c, dtype=np.int64), rows, kb, vb)
        g = f64(x_out[offs[b]:offs[b] + c])
        if c:
            assert max_abs_rel(g, out) < tol, (b, max_abs_rel(g, out))
        gk, gv = f64(kc[b]), f64(vc[b])
        assert max_abs_rel(gk, kb[0]) < tol
        assert max_abs_rel(gv, vb[0]) < tol
        untouched = np.setdiff1d(np.arange(N), rows)
        np.testing.assert_array_equal(gk[untouched], f64(kc0[b])[untouched])
        np.testing.assert_array_equal(gv[untouched], f64(vc0[b])[untouched])


def test_layer_f32_tiny(lib):
    _run_layer(lib, SY.TINY, B=2, N=128, counts=[32, 17], k_cap=40)


def test_layer_f32_tiny_compact_input_no_rope(lib):
    _run_layer(lib, SY.with_(SY.TINY, rope_theta=0.0), B=1, N=128, counts=[32], k_cap=32,
               x_full=False)


@pytest.mark.parametrize("heads,kv,hd", [(2, 2, 128), (4, 2, 64), (8, 2, 64)])
def test_layer_bf16_small(lib, heads, kv, hd):
    shape = SY.with_(SY.TINY, dtype="bf16", d=256, n_heads=heads, n_kv_heads=kv, head_dim=hd,
                     ffn=512, vocab=2048)
    _run_layer(lib, shape, B=3, N=200, counts=[70, 33, 1], k_cap=70)


def test_layer_bf16_zero_rows_leave_cache(lib):
    shape = SY.with_(SY.TINY, dtype="bf16", d=256, n_heads=2, n_kv_heads=2, head_dim=128,
                     ffn=512, vocab=2048)
    _run_layer(lib, shape, B=2, N=64, counts=[0, 5], k_cap=8)


def test_layer_bf16_8b_shape_bench_launch(lib):
    """The launch the benchmark times: 32 sequences x 1536 tokens, 308 rows each,
    d 4096, 32 heads, FFN 12288; sequences 0 and 31 checked against the oracle."""
    shape = SY.with_(SY.DENSE8B_B32_N1536, n_layers=1)
    _run_layer(lib, shape, B=32, N=1536, counts=[308] * 32, k_cap=308, weights_on_gpu=True,
               check_seqs=[0, 31])


def test_layer_bf16_7b_gqa_shape(lib):
    shape = SY.with_(SY.GQA7B_B8_N2048, n_layers=1)
    _run_layer(lib, shape, B=2, N=2048, counts=[103, 250], k_cap=250, weights_on_gpu=True,
               check_seqs=[0, 1])


@pytest.mark.parametrize("B,N,counts", [(1, 1000, [77]), (1, 1100, [300]), (1, 4096, [5]),
                                        (2, 1536, [0, 40])])
def test_layer_bf16_few_rows_split_keys(lib, B, N, counts):
    """Few query rows over long sequences: the attention shares each sequence's
    keys among several CTAs and merges their partial outputs; ragged key tails
    (1000 and 1100 keys), an empty sequence and up to eight shares."""
    shape = SY.with_(SY.TINY, dtype="bf16", d=512, n_heads=4, n_kv_heads=2, head_dim=128,
                     ffn=1024, vocab=2048)
    _run_layer(lib, shape, B=B, N=N, counts=counts, k_cap=max(counts))


@pytest.mark.parametrize("B,N,counts", [(1, 1000, [77]), (2, 700, [300, 5])])
def test_layer_bf16_few_rows_split_keys_hd64(lib, B, N, counts):
    """The key split at head dim 64 (one query tile per CTA, two CTAs per SM)."""
    shape = SY.with_(SY.TINY, dtype="bf16", d=512, n_heads=8, n_kv_heads=4, head_dim=64,
                     ffn=1024, vocab=2048)
    _run_layer(lib, shape, B=B, N=N, counts=counts, k_cap=max(counts))


@pytest.mark.parametrize("heads,kv,hd", [(8, 8, 64), (8, 4, 128)])
def test_layer_bf16_many_sequences_mixed_counts(lib, heads, kv, hd):
    """A grid several waves deep (76 sequences): row counts cover a lone first
    query tile, a lone remainder after two full tiles, full pairs, one row and
    an empty sequence, for MHA and GQA."""
    shape = SY.with_(SY.TINY, dtype="bf16", d=512, n_heads=heads, n_kv_heads=kv, head_dim=hd,
                     ffn=1024, vocab=2048)
    pattern = [300, 100, 0, 200, 129, 1, 256, 257]
    counts = [pattern[i % len(pattern)] for i in range(76)]
    _run_layer(lib, shape, B=76, N=384, counts=counts, k_cap=300,
               check_seqs=[0, 1, 2, 3, 4, 5, 6, 7, 75])
