"""Host-side logic of bench.py on CPU: the command line it must accept, that
every option the code reads is one the parser defines, and the roofline
arithmetic of its JSON line (hand-computed values)."""
import ast
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import dllm_synth as SY  # noqa: E402


def _parse(argv):
    old = sys.argv
    sys.argv = ["bench.py"] + argv
    try:
        return bench.parse()
    finally:
        sys.argv = old


def test_contract_command_lines_parse():
    a = _parse([])
    assert (a.gpus, a.steps, a.warmup, a.impl) == (1, 10, 3, "ours")
    a = _parse(["--gpus", "8", "--steps", "5", "--warmup", "3", "--impl", "reference"])
    assert (a.gpus, a.steps, a.warmup, a.impl) == (8, 5, 3, "reference")
    assert _parse(["--no-bs1", "--no-gqa", "--no-cpu-baseline"]).no_bs1


def test_every_option_read_is_defined():
    """Each `args.<name>` in bench.py exists on the parsed namespace."""
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    used = {n.attr for n in ast.walk(tree)
            if isinstance(n, ast.Attribute) and isinstance(n.value, ast.Name)
            and n.value.id == "args"}
    defined = set(vars(_parse([])))
    assert used and used <= defined, sorted(used - defined)


def test_job_throughput_is_weak_scaling():
    # 32 sequences x 16 reveals per rank, 4 ranks, slowest rank 128 ms
    assert bench.job_tokens_per_s(4, 512, 128.0) == pytest.approx(4 * 512 / 0.128)
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_gemm_bytes_per_launch_by_hand():
    s = SY.with_(SY.DENSE8B_B32_N1536)
    M, d, q, kv, f = 32 * 308, 4096, 4096, 4096, 12288
    qkv = M * d + (q + 2 * kv) * d + M * (q + 2 * kv)
    o = M * q + d * q + 2 * M * d
    gu = M * d + 2 * f * d + M * f
    down = M * f + d * f + 2 * M * d
    assert bench.gemm_bytes_per_launch(s) == 2 * (qkv + o + gu + down) / 4
    assert round(bench.gemm_bytes_per_launch(s)) == 432013312


def test_single_sequence_roofline_by_hand():
    s = SY.with_(bench.BS1, ratio=0.10)          # 77 of 768 rows, 8B
    r = bench.step_roofline(s, 5.0, 6550.0, 1640.0)
    p_layer = 4096 * 3 * 4096 + 4096 * 4096 + 3 * 4096 * 12288
    nbytes = (32 * p_layer + s.vocab * 4096) * 2 + 32 * 768 * 2 * 4096 * 2 + 32 * 77 * 2 * 4096 * 2
    flops = 32 * (2.0 * 77 * p_layer + 4.0 * 77 * 768 * 4096)
    assert r["bytes"] == nbytes and r["flops"] == pytest.approx(flops)
    assert r["bound"] == "hbm"                    # intensity ~72 flop/B, ridge ~250
    assert r["hbm_frac"] == pytest.approx(nbytes / 5e-3 / 1e9 / 6550.0, abs=1e-4)
    full = bench.step_roofline(SY.with_(bench.BS1, ratio=1.0), 12.0, 6550.0, 1640.0)
    assert full["bound"] == "tensor"              # 768 rows: ~700 flop/B


def test_hbm_kernels_by_hand():
    s = bench.SHAPE                              # 32 x 1536, d 4096, 308 rows/seq
    prof = {"score": [10, 1.5], "gather": [10, 0.4], "select": [10, 0.2], "attention": [320, 180.0]}
    r = bench.hbm_kernels(s, prof, 6550.0)
    score = 2 * 32 * 1536 * 4096 * 2 + 32 * 1536 * 12
    assert r["score"]["bytes_per_launch"] == score
    assert r["score"]["frac"] == pytest.approx(score / 0.15e-3 / 1e9 / 6550.0, abs=1e-4)
    assert r["gather"]["bytes_per_launch"] == 3 * 32 * 308 * 4096 * 2
    assert r["select"]["bound"] == "latency"
    assert "attention" not in r
    assert bench.hbm_kernels(s, {}, 6550.0) == {"peak_gbs": 6550.0}


def test_generation_from_sample_by_hand():
    """Whole generation = dense step + 63 partial steps, each 32 sequences x 32 layers
    of the one-sequence one-layer sample plus the sequence's LM head."""
    s = bench.SHAPE
    gen, dense, partial = bench.generation_from_sample(s, 0.5, 0.25, 2.0, 1.5)
    assert dense == 32 * (32 * 2.0 + 1.5)
    assert partial == 32 * (32 * 0.5 + 0.25)
    assert gen == dense + 63 * partial


def test_clock_summaries_merge(tmp_path):
    """Samples of several windows summarise as one: median SM clock of the loaded
    samples, every throttle reason seen."""
    rows = [
        ["0, u, 1400, 1965, 900, 0x4, Not Active, Not Active, Not Active, Active",
         "0, u, 1500, 1965, 950, 0x0, Not Active, Not Active, Not Active, Not Active"],
        ["0, u, 1300, 1965, 990, 0x4, Not Active, Not Active, Not Active, Active",
         "0, u, 210, 1965, 90, 0x0, Not Active, Not Active, Not Active, Not Active"]]
    cl = []
    for i, rr in enumerate(rows):
        c = bench.Clocks("u")
        c.path = str(tmp_path / f"c{i}.csv")
        open(c.path, "w").write("\n".join(rr) + "\n")
        cl.append(c)
    m = bench.Clocks.merge(cl)
    assert m["samples"] == 4 and m["sm_mhz"] == 1400.0 and m["reasons"] == ["sw_power_cap"]
    assert cl[1].summary()["sm_mhz"] == 1300.0    # the idle 210 MHz sample is not under load
