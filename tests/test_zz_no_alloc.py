"""The workspace-free partial attention (dllm_attention_bf16_noalloc).

It serves callers that cannot allocate device memory -- code running during
CUDA-graph capture, servers with pre-carved memory pools, plugins that only
receive their tensors -- by keeping its scratch in a fixed array inside the
library.  These tests call it through the C ABI and check that two calls in a
row give the same result as dllm_attention_bf16 with a caller workspace, and
that a batch larger than the fixed scratch is refused.  The file is collected
last so that a failure here never hides the result of another test.
"""
import ctypes as C

import pytest
import torch

import dllm_synth as SY
from _util import f64, max_abs_rel, TOL

pytestmark = pytest.mark.gpu


def _inputs(B, N, Hq, Hkv, hd, counts, seed):
    k_cap = max(max(counts), 1)
    q = SY.normal((B * k_cap, Hq * hd), 1.0, seed, "cuda", "bf16")
    kc = SY.normal((B, N, Hkv, hd), 1.0, seed + 1, "cuda", "bf16")
    vc = SY.normal((B, N, Hkv, hd), 1.0, seed + 2, "cuda", "bf16")
    cnt = torch.tensor(counts, dtype=torch.int32, device="cuda")
    return q, kc, vc, cnt, k_cap


def test_noalloc_matches_workspace_entry_on_two_calls(lib):
    cases = [(3, 700, 4, 2, 128, [200, 5, 77], 11),   # first call: sets the scratch up
             (2, 1536, 8, 8, 64, [0, 300], 21)]       # second call: other sizes, same scratch
    for B, N, Hq, Hkv, hd, counts, seed in cases:
        q, kc, vc, cnt, k_cap = _inputs(B, N, Hq, Hkv, hd, counts, seed)
        ref = torch.zeros_like(q)
        out = torch.full_like(q, 7.0)
        lib.dllm_attention_bf16(q, kc, vc, ref, cnt, k_cap)
        lib.dllm_attention_bf16_noalloc(q, kc, vc, out, cnt, k_cap)
        torch.cuda.synchronize()
        off = 0
        for c in counts:
            if c:
                assert max_abs_rel(f64(out[off:off + c]), f64(ref[off:off + c])) < TOL["bf16"]
            off += c


def test_noalloc_refuses_more_sequences_than_its_scratch(lib):
    B = lib.DLLM_NOALLOC_MAX_SEQS + 1
    dummy = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    p = dummy.data_ptr()
    st = lib._attn_noalloc(p, p, p, p, cnt.data_ptr(), B, 1, 16, 1, 1, 64,
                           torch.cuda.current_stream().cuda_stream)
    assert st == 5  # DLLM_ERR_CAPACITY, nothing launched
