"""The C-ABI library loads, exports every entry point the header declares,
and rejects bad arguments on the host before touching the GPU (CPU tests)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dllm.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dllm_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_dllm_build", os.path.join(ROOT, "sparse_token_recompute_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    path = build.build()
    return C.CDLL(path)


def test_header_declares_the_step_entry_points():
    names = _declared()
    for n in ("dllm_score", "dllm_select", "dllm_partial_layer", "dllm_step", "dllm_unmask"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_host_only_calls(lib):
    lib.dllm_status_string.restype = C.c_char_p
    assert lib.dllm_status_string(0) == b"ok"
    assert b"workspace" in lib.dllm_status_string(3)
    assert lib.dllm_status_string(99) == b"unknown status"
    assert lib.dllm_version() >= 100


def test_bad_arguments_are_rejected_before_launch(lib):
    import sparse_token_recompute_b200 as S
    # negative sizes / bad enums / missing pointers: status codes, no CUDA work
    assert S._select(None, -1, 10, 0, 1, 0.0, None, None, 1, None, 0, None) == 1
    assert S._select(None, 1, 10, 7, 1, 0.0, None, None, 1, None, 0, None) == 1
    assert S._select(None, 1, 10, 0, 5, 0.0, None, None, 2, None, 0, None) == 5  # k > k_cap
    assert S._select(None, 1, 20000, 0, 5, 0.0, None, None, 8, None, 0, None) == 2
    assert S._unmask(None, None, None, 1, 10, 0, 0, 0, 1, None, None) == 1   # block_len 0
    assert S._unmask(None, None, None, 1, 10, 0, 0, 2048, 1, None, None) == 2
    assert S._score(None, None, 1, 4, 16, 5, None, None, 0, 0, None, None, None, 0.5, 0,
                    None, None) == 1  # bad dtype
    assert S._gemm(None, None, None, 4, 10, 64, 0, 0, None, 0, None) == 1
    cfg = S.make_cfg(1, 100, 4, 4, 64, 688, 1024, 5e5, 1e-5, 1023, "bf16")
    lw = S.LayerW()
    assert S._layer(C.byref(cfg), C.byref(lw), None, 1, None, None, None, 4, 1, 8, None, None,
                    None, 0, None) == 2  # d not a multiple of 128 on the bf16 path
    cfg = S.make_cfg(1, 256, 4, 3, 64, 688, 1024, 5e5, 1e-5, 1023, "f32")
    assert S._layer_ws(C.byref(cfg), 1, 8, 4) == 0  # heads not divisible by kv heads
    cfg = S.make_cfg(1, 256, 4, 4, 64, 688, 1024, 5e5, 1e-5, 1023, "f32")
    assert S._layer(C.byref(cfg), C.byref(lw), None, 1, None, None, None, 4, 1, 8, None, None,
                    None, 0, None) == 1  # null weights


def test_workspace_sizes_are_host_computable(lib):
    import sparse_token_recompute_b200 as S
    cfg = S.make_cfg(1, 256, 4, 4, 64, 688, 1024, 5e5, 1e-5, 1023, "f32")
    pol = S.make_policy(k=32, n_unmask=8, gen_start=64, block_len=64)
    a = S.dllm_step_workspace_size(cfg, 1, 128, pol)
    b = S.dllm_step_workspace_size(cfg, 2, 128, pol)
    assert 0 < a < b
    assert S.dllm_partial_layer_workspace_size(cfg, 1, 128, 32) > 0
    assert S.dllm_select_workspace_size(4, 100) >= 4


def test_gemm_plans_of_the_benchmarked_shapes(lib):
    """The host-side GEMM planner (no GPU: 148 SMs assumed) picks the plans the
    measurements behind it chose: CTA pairs for the QKV, O and down projections
    at 32 x 308 rows, single CTAs for gate/up and the LM head; at one sequence,
    weight-streaming plans that fill one wave (K splits for the narrow O and
    down projections) and a pair for QKV at 192 rows."""
    import sparse_token_recompute_b200 as S
    P = S.dllm_gemm_plan_info
    qkv, o, gu, down = (["qkv", 4096, [4096, 4096, 4096], 128], ["residual", 4096, [4096]],
                        ["swiglu", 4096, [12288, 12288]], ["residual", 12288, [4096]])

    def plan(spec, M):
        kind, K, segs, *hd = spec
        return P(kind, M, K, segs, *hd)

    M = 32 * 308
    for spec in (qkv, o, down):
        assert plan(spec, M) == {**plan(spec, M), "bn": 256, "splits": 1, "grid": 148, "pair": 1}
    assert plan(gu, M) == {"bn": 256, "splits": 1, "tiles_n": 96, "grid": 148, "pair": 0}
    assert P("lmhead", 8100, 4096, [126464])["pair"] == 0
    assert plan(qkv, 77) == {"bn": 128, "splits": 1, "tiles_n": 96, "grid": 96, "pair": 0}
    for spec in (o, down):
        assert plan(spec, 77) == {"bn": 128, "splits": 4, "tiles_n": 32, "grid": 128, "pair": 0}
    assert plan(qkv, 192) == {"bn": 256, "splits": 1, "tiles_n": 48, "grid": 96, "pair": 1}
    assert plan(o, 192)["pair"] == 0 and plan(o, 192)["splits"] == 4
    # no plan is wider than the SM count in one wave, except split K (one unit per CTA)
    for spec in (qkv, o, gu, down):
        for rows in (1, 77, 192, 384, 1000, 9856):
            p = plan(spec, rows)
            assert p["grid"] <= 148 or p["splits"] > 1
            assert p["pair"] in (0, 1) and (not p["pair"] or p["grid"] % 2 == 0)


def test_attention_plans_of_the_benchmarked_shapes(lib):
    """The host-side attention plan (no GPU: 148 SMs assumed): one query tile per
    CTA (two CTAs per SM) for an odd tile count of three or more and wherever the
    keys are split among CTAs; pairs of tiles sharing each K/V tile otherwise."""
    import sparse_token_recompute_b200 as S
    P = S.dllm_attention_plan_info
    plan = lambda *a, **kw: tuple(P(*a, **kw).values())
    assert plan(32, 308, 1536, 32, 128) == (1, 1, 3072)      # the 32-sequence step: 3 tiles
    assert plan(32, 308, 1536, 28, 128) == (1, 1, 2688)      # 7B GQA heads, 3 tiles
    assert plan(32, 256, 1536, 32, 128) == (2, 1, 1024)      # 2 tiles: pairs
    assert plan(32, 1536, 1536, 32, 128) == (2, 1, 6144)     # dense step: 12 tiles
    assert plan(32, 640, 1536, 32, 128)[0] == 1              # 5 tiles
    assert plan(1, 77, 768, 32, 128) == (1, 6, 192)          # one sequence: keys in 6 shares
    assert plan(1, 192, 768, 32, 128) == (1, 3, 192)
    assert plan(1, 77, 768, 32, 128, in_step=False) == (2, 1, 32)   # no scratch: no shares
    assert plan(8, 103, 2048, 28, 128) == (1, 1, 224)       # one wave singly, two in pairs
    assert plan(8, 205, 2048, 28, 128) == (2, 1, 224)
    # resident CTAs: one per SM with pairs, two per SM with one tile
    for args in [(1, 77, 768, 32, 128), (1, 384, 768, 32, 128), (2, 300, 4096, 8, 64)]:
        nt, shares, ctas = plan(*args)
        assert ctas <= (2 if nt == 1 else 1) * 148 or shares == 1
    with pytest.raises(RuntimeError):
        P(1, 77, 768, 32, 96)


def test_gemm_plan_rejects_bad_arguments(lib):
    import sparse_token_recompute_b200 as S
    segs = (C.c_int32 * 3)(4096, 4096, 4096)
    out = (C.c_int32 * 5)()
    assert S._gemm_plan(9, 100, 64, C.cast(segs, C.c_void_p), 1, 0, C.cast(out, C.c_void_p)) == 1
    assert S._gemm_plan(3, 100, 64, C.cast(segs, C.c_void_p), 1, 128, C.cast(out, C.c_void_p)) == 1
    assert S._gemm_plan(0, 0, 64, C.cast(segs, C.c_void_p), 1, 0, C.cast(out, C.c_void_p)) == 1
    assert S._gemm_plan(0, 100, 64, None, 1, 0, C.cast(out, C.c_void_p)) == 1


def test_host_buffer_step_validates_before_any_copy(lib):
    """dllm_step_host rejects a missing token buffer, a bad shape and a small
    workspace before it enqueues a copy; its workspace adds the token and
    revealed-position buffers to the step's."""
    import sparse_token_recompute_b200 as S
    cfg = S.make_cfg(1, 256, 4, 4, 64, 688, 1024, 5e5, 1e-5, 1023, "f32")
    pol = S.make_policy(k=32, n_unmask=8, gen_start=64, block_len=64)
    step = S.dllm_step_workspace_size(cfg, 2, 128, pol)
    host = S.dllm_step_host_workspace_size(cfg, 2, 128, pol)
    assert host >= step + 2 * 128 * 4 + 2 * 8 * 4
    m = S.ModelW()
    c = S.CacheS()
    tok = (C.c_int32 * 256)()
    assert S._step_host(C.byref(cfg), C.byref(m), C.byref(c), None, 2, 128, C.byref(pol), 0,
                        None, None, 0, None) == 1
    assert S._step_host(C.byref(cfg), C.byref(m), C.byref(c), C.cast(tok, C.c_void_p), -1, 128,
                        C.byref(pol), 0, None, None, 0, None) == 1
    assert S._step_host(C.byref(cfg), C.byref(m), C.byref(c), C.cast(tok, C.c_void_p), 2, 128,
                        C.byref(pol), 0, None, None, 0, None) == 3
    bad = S.make_cfg(1, 256, 4, 3, 64, 688, 1024, 5e5, 1e-5, 1023, "f32")
    assert S._step_host(C.byref(bad), C.byref(m), C.byref(c), C.cast(tok, C.c_void_p), 2, 128,
                        C.byref(pol), 0, None, None, 0, None) == 2
