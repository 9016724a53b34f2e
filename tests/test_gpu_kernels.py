"""GPU parity of the memory-bound kernels and of the tensor-core GEMM, through
the C ABI, against the CPU oracle (and, for the GEMM, a float64 library
matmul of the same bf16 inputs)."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import dllm_synth as SY
from _util import f64, max_abs_rel, TOL

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ GEMM

@pytest.mark.parametrize("M,N,K,splits,acc", [
    (1, 128, 64, 0, False),
    (77, 256, 4096, 0, False),
    (128, 512, 256, 1, False),
    (200, 384, 512, 0, True),
    (300, 4096, 1024, 0, False),
    (77, 4096, 4096, 4, True),
    (129, 200, 72, 1, False),
    (1000, 1024, 1024, 0, False),
    (2048, 2048, 2048, 1, False),
    (500, 1024, 4096, 0, False),     # four row tiles, few column tiles
    (400, 4096, 12288, 0, True),     # four row tiles, deep K, residual accumulate
    (257, 8192, 1024, 0, False),     # three row tiles, the last one holding one row
    (600, 1000, 512, 0, False),      # ragged last column tile
    (384, 640, 200, 0, True),        # ragged K (a partial last k-block), 1.5 row-tile pairs
    # one row tile, weight streaming (the planner's split-K clusters or wide tiles)
    (77, 4096, 4096, 0, True),       # O-shaped, residual accumulate
    (77, 12288, 4096, 0, False),     # QKV-shaped
    (1, 4096, 12288, 0, True),       # one row, down-shaped K
    (128, 2048, 4096, 0, False),     # a full row tile
    (100, 3000, 4096, 0, False),     # ragged last column tile
    (60, 2048, 4040, 0, True),       # ragged K (a partial last k-block)
])
def test_gemm_bf16(lib, M, N, K, splits, acc):
    A = SY.normal((M, K), 1.0, 11 + M, "cuda", "bf16")
    Bm = SY.normal((N, K), 0.05, 12 + N, "cuda", "bf16")
    C0 = SY.normal((M, N), 1.0, 13, "cuda", "bf16") if acc else torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    Cm = C0.clone()
    lib.dllm_gemm_bf16(A, Bm, Cm, accumulate=acc, splits=splits)
    torch.cuda.synchronize()
    ref = f64(A) @ f64(Bm).T + (f64(C0) if acc else 0.0)
    err = max_abs_rel(f64(Cm), ref)
    assert err < 1e-2, err


@pytest.mark.parametrize("M", [77, 300])
def test_gemm_split_k_is_deterministic(lib, M):
    A = SY.normal((M, 4096), 1.0, 3, "cuda", "bf16")
    Bm = SY.normal((4096, 4096), 0.02, 4, "cuda", "bf16")
    outs = []
    for _ in range(3):
        Cm = torch.zeros(M, 4096, dtype=torch.bfloat16, device="cuda")
        lib.dllm_gemm_bf16(A, Bm, Cm, splits=4)
        outs.append(Cm)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


# ------------------------------------------------------------------ score + confidence

def _score_case(lib, B, N, d, V, Mm, dtype, kind, alpha, seed=1):
    si = SY.score_inputs(B, N, d, V, Mm, seed=seed, device="cuda", dtype=dtype)
    conf = si.conf.clone()
    pred = si.pred.clone()
    scores = torch.empty(B, N, dtype=torch.float32, device="cuda")
    lib.dllm_score(si.h_cur, si.h_ref, conf, si.masked, scores, alpha, kind,
                   logits=si.logits, logit_pos=si.logit_pos, pred=pred)
    torch.cuda.synchronize()
    return si, conf, pred, scores


@pytest.mark.parametrize("dtype,kind", [("bf16", 0), ("bf16", 1), ("f32", 0), ("f32", 1)])
def test_score_small(lib, dtype, kind):
    B, N, d, V, Mm = 3, 300, 256, 1000, 50
    si, conf, pred, scores = _score_case(lib, B, N, d, V, Mm, dtype, kind, 0.5)
    ora_s, ora_c, ora_p = O.score_call(f64(si.h_cur), f64(si.h_ref), f64(si.conf),
                                       f64(si.pred), f64(si.masked), 0.5, kind,
                                       f64(si.logits), f64(si.logit_pos).astype(int))
    tol = TOL["f32"]
    assert max_abs_rel(f64(scores), ora_s) < tol
    assert max_abs_rel(f64(conf), ora_c) < tol
    g = f64(pred).astype(int)
    z = f64(si.logits)
    for b in range(B):
        for j, p in enumerate(f64(si.logit_pos).astype(int)[b]):
            if g[b, p] != ora_p[b, p]:
                assert z[b, j].max() - z[b, j, g[b, p]] <= 1e-6 * abs(z[b, j].max())


def test_score_and_select_full_size(lib):
    """Standalone score + select at 32 x 1024 x 4096 (bf16 hidden, 256 x 32768 logits)."""
    B, N, d, V, Mm, k = 32, 1024, 4096, 32768, 256, 256
    si, conf, pred, scores = _score_case(lib, B, N, d, V, Mm, "bf16", 0, 0.5)
    idx = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    count = torch.zeros(B, dtype=torch.int32, device="cuda")
    lib.dllm_select(scores, idx, count, lib.DLLM_SELECT_TOPK, k)
    torch.cuda.synchronize()
    g_scores = f64(scores)
    for b in (0, 13, 31):
        ora_s, ora_c, _ = O.score_call(f64(si.h_cur[b:b + 1]), f64(si.h_ref[b:b + 1]),
                                       f64(si.conf[b:b + 1]), f64(si.pred[b:b + 1]),
                                       f64(si.masked[b:b + 1]), 0.5, 0,
                                       f64(si.logits[b:b + 1]),
                                       f64(si.logit_pos[b:b + 1]).astype(int))
        assert max_abs_rel(g_scores[b:b + 1], ora_s) < TOL["bf16"]
        assert max_abs_rel(f64(conf[b:b + 1]), ora_c) < TOL["f32"]
    # selection: bit-exact against the oracle given the same scores
    s32 = scores.cpu().numpy()
    c = count.cpu().numpy()
    I = idx.cpu().numpy()
    for b in range(B):
        ref = O.select_topk(s32[b], k)
        assert c[b] == k
        np.testing.assert_array_equal(I[b, :c[b]], ref)


# ------------------------------------------------------------------ select edge cases

def _gpu_select(lib, scores_np, mode, k, tau, k_cap):
    B, N = scores_np.shape
    s = torch.from_numpy(np.ascontiguousarray(scores_np, dtype=np.float32)).cuda()
    idx = torch.full((B, k_cap), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    ws = lib.Workspace(lib.dllm_select_workspace_size(B, N))
    lib.dllm_select(s, idx, cnt, mode, k, tau, ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), cnt.cpu().numpy(), ws.device_status()


@pytest.mark.parametrize("N", [1, 7, 1000, 1025, 4096, 16384])
def test_select_topk_random(lib, N):
    rng = np.random.default_rng(N)
    B = 4
    s = rng.standard_normal((B, N)).astype(np.float32)
    s[1] = np.round(s[1] * 2) / 2          # many ties
    s[2] = 0.0                              # all equal
    s[3, ::3] = -0.0
    for k in sorted({0, 1, N // 3, N}):
        k_cap = max(k, 1)
        I, c, st = _gpu_select(lib, s, 0, k, 0.0, k_cap)
        assert st == 0
        for b in range(B):
            ref = O.select_topk(s[b], k)
            assert c[b] == len(ref)
            np.testing.assert_array_equal(I[b, :c[b]], ref)


def test_select_nan_inf_signed_zero(lib):
    s = np.array([[np.nan, 0.0, -0.0, np.inf, -np.inf, 1.0, np.nan, -0.0, 0.0, 2.0]],
                 dtype=np.float32)
    for k in range(0, 11):
        I, c, _ = _gpu_select(lib, s, 0, k, 0.0, max(k, 1))
        np.testing.assert_array_equal(I[0, :c[0]], O.select_topk(s[0], k))


def test_select_threshold_and_capacity(lib):
    rng = np.random.default_rng(5)
    s = rng.random((3, 777)).astype(np.float32)
    tau = 0.9
    n_over = (s > tau).sum(1)
    cap = int(n_over.min()) - 3              # clip at least one sequence
    I, c, st = _gpu_select(lib, s, 1, 0, tau, cap)
    assert st & lib.DLLM_DEV_CAPACITY
    for b in range(3):
        ref, nb = O.select_thresh(s[b], tau, cap)
        assert nb == n_over[b]
        np.testing.assert_array_equal(I[b, :c[b]], ref)
    I, c, st = _gpu_select(lib, s, 1, 0, 2.0, 8)   # nothing over the threshold
    assert st == 0 and np.all(c == 0)


# ------------------------------------------------------------------ unmask

def test_unmask_random(lib):
    rng = np.random.default_rng(9)
    for trial in range(40):
        B, N = 3, int(rng.integers(8, 300))
        gs = int(rng.integers(0, N))
        bl = int(rng.integers(1, 70))
        n = int(rng.integers(0, 12))
        M = 999
        tok = rng.integers(0, 50, (B, N)).astype(np.int32)
        tok[:, gs:][rng.random((B, N - gs)) < 0.5] = M
        if trial % 7 == 0:
            tok[0, gs:] = 3                 # nothing masked in sequence 0
        conf = (rng.integers(0, 6, (B, N)) / 8.0).astype(np.float32)
        pred = rng.integers(0, 50, (B, N)).astype(np.int32)
        t_gpu = torch.from_numpy(tok.copy()).cuda()
        pos = torch.full((B, max(n, 1)), -9, dtype=torch.int32, device="cuda")
        lib.dllm_unmask(torch.from_numpy(conf).cuda(), torch.from_numpy(pred).cuda(), t_gpu, M,
                        gs, bl, n, pos_out=pos if n else None)
        torch.cuda.synchronize()
        t_ora = tok.astype(np.int64).copy()
        p_ora = O.unmask(conf.astype(np.float64), pred.astype(np.int64), t_ora, M, gs, bl, n)
        np.testing.assert_array_equal(t_gpu.cpu().numpy(), t_ora)
        if n:
            np.testing.assert_array_equal(pos.cpu().numpy()[:, :n], p_ora)


def test_gemm_pair_stall_times_out_and_context_survives(lib):
    """Failure path of the CTA-pair GEMM: with one stage signal withheld the
    bounded wait runs out, every CTA drains and returns, the device status
    reports DLLM_DEV_TIMEOUT, and the same context then computes a correct GEMM."""
    M, N, K = 512, 1024, 512
    A = SY.normal((M, K), 1.0, 21, "cuda", "bf16")
    Bm = SY.normal((N, K), 0.05, 22, "cuda", "bf16")
    C = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    ws = lib.dllm_selftest_gemm_stall(A, Bm, C)
    torch.cuda.synchronize()
    assert ws.device_status() & lib.DLLM_DEV_TIMEOUT
    C2 = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    ws2 = lib.dllm_gemm_bf16(A, Bm, C2)
    torch.cuda.synchronize()
    assert ws2.device_status() == 0
    assert max_abs_rel(f64(C2), f64(A) @ f64(Bm).T) < 1e-2
