"""GPU parity of the partial attention alone (dllm_attention_bf16) against the
oracle's attention, and of a CUDA-graph-replayed step against the eager one."""
import numpy as np
import pytest
import torch

import oracle as O
import dllm_synth as SY
from _util import f64, max_abs_rel, TOL

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,N,Hq,Hkv,hd,counts", [
    (2, 200, 2, 2, 128, [70, 129]),        # ragged key tile, two query tiles
    (3, 1000, 4, 2, 64, [1, 256, 300]),    # GQA, hd 64, three query tiles
    (1, 2048, 28, 4, 128, [103]),          # 7B-class head layout
    (2, 64, 8, 8, 128, [0, 64]),           # a sequence with no rows, keys < one tile
    (2, 300, 2, 1, 128, [100, 257]),       # lone tiles split the keys 2 + 1 tiles (ragged)
])
def test_attention_matches_oracle(lib, B, N, Hq, Hkv, hd, counts):
    k_cap = max(max(counts), 1)
    M = B * k_cap
    q = SY.normal((M, Hq * hd), 1.0, 3, "cuda", "bf16")
    kc = SY.normal((B, N, Hkv, hd), 1.0, 4, "cuda", "bf16")
    vc = SY.normal((B, N, Hkv, hd), 1.0, 5, "cuda", "bf16")
    o = torch.zeros(M, Hq * hd, dtype=torch.bfloat16, device="cuda")
    cnt = torch.tensor(counts, dtype=torch.int32, device="cuda")
    ws = lib.dllm_attention_bf16(q, kc, vc, o, cnt, k_cap)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    off = 0
    for b, c in enumerate(counts):
        if c:
            ref = O.store(O.attention(f64(q[off:off + c]).reshape(c, Hq, hd), f64(kc[b]),
                                      f64(vc[b])), "bf16").reshape(c, Hq * hd)
            assert max_abs_rel(f64(o[off:off + c]), ref) < TOL["bf16"]
        off += c


def test_attention_large_score_range(lib):
    """Scores spread over a wide range force the reference-maximum raise and the
    in-TMEM rescale of the partial output."""
    B, N, Hq, hd = 1, 1024, 2, 128
    q = SY.normal((128, Hq * hd), 1.0, 6, "cuda", "bf16")
    k32 = SY.normal((B, N, Hq, hd), 1.0, 7, "cuda", "f32")
    ramp = torch.linspace(0.1, 6.0, N, device="cuda")[None, :, None, None]
    kc = (k32 * ramp).to(torch.bfloat16)           # later tiles carry larger logits
    vc = SY.normal((B, N, Hq, hd), 1.0, 8, "cuda", "bf16")
    o = torch.zeros_like(q)
    cnt = torch.tensor([128], dtype=torch.int32, device="cuda")
    lib.dllm_attention_bf16(q, kc, vc, o, cnt, 128)
    torch.cuda.synchronize()
    ref = O.store(O.attention(f64(q).reshape(128, Hq, hd), f64(kc[0]), f64(vc[0])),
                  "bf16").reshape(128, Hq * hd)
    assert max_abs_rel(f64(o), ref) < TOL["bf16"]


def test_graph_replay_equals_eager_step(lib):
    shape = SY.with_(SY.TINY, dtype="bf16", n_layers=2, d=256, n_heads=2, n_kv_heads=2,
                     head_dim=128, ffn=512, vocab=2048, batch=2, prompt_len=64, gen_len=128,
                     block_len=32, n_unmask=4, ratio=0.25, alpha=0.5)
    W = SY.model_weights(shape, seed=0, device="cuda")
    model = lib.Model(lib.cfg_from_shape(shape), W)
    pol = lib.make_policy(0, 0.5, 0, 0, shape.k, 0.0, 4, 64, 32)
    runs = []
    for use_graph in (False, True):
        tokens = SY.prompt_tokens(shape, seed=1).cuda()
        cache = lib.Cache(model.cfg, 2, shape.seq_len)
        ws = lib.Workspace(lib.dllm_step_workspace_size(model.cfg, 2, shape.seq_len, pol))
        lib.dllm_step(model, cache, tokens, pol, True, ws)
        lib.dllm_step(model, cache, tokens, pol, False, ws)
        if use_graph:
            g = lib.StepGraph(model, cache, tokens, pol, ws)
            for _ in range(3):
                g.replay()
        else:
            for _ in range(3):
                lib.dllm_step(model, cache, tokens, pol, False, ws)
        torch.cuda.synchronize()
        runs.append((tokens.clone(), [t.clone() for t in cache.k + cache.v], cache.conf.clone()))
    assert torch.equal(runs[0][0], runs[1][0])
    for a, b in zip(runs[0][1], runs[1][1]):
        assert torch.equal(a, b)
    assert torch.equal(runs[0][2], runs[1][2])
