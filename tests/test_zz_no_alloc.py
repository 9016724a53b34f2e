"""The workspace-free partial attention (dllm_attention_bf16_noalloc).

It serves callers that cannot allocate device memory -- servers that carve
all device memory into fixed pools before they serve, plugins and operators
that only receive the tensors they compute on -- by keeping its scratch in a
fixed array inside the library.  These tests call it through the C ABI and
check, on two calls in a row (the second reusing the scratch the first left
behind), that its output equals dllm_attention_bf16's with a caller workspace
and the oracle's attention (DyLLM, French summary §1 and §2.B: every selected
query attends to all keys of its sequence, no mask), and that a batch larger
than the fixed scratch is refused.  The file is collected last so that a
failure here never hides the result of another test.
"""
import numpy as np
import pytest
import torch

import oracle as O
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


def test_noalloc_matches_workspace_entry_and_oracle_on_two_calls(lib):
    cases = [(3, 700, 4, 2, 128, [200, 5, 77], 11),   # first call: sets the scratch up
             (2, 1536, 8, 8, 64, [0, 300], 21)]       # second call: other sizes, same scratch
    for B, N, Hq, Hkv, hd, counts, seed in cases:
        q, kc, vc, cnt, k_cap = _inputs(B, N, Hq, Hkv, hd, counts, seed)
        ref = torch.zeros_like(q)
        out = torch.full_like(q, 7.0)
        lib.dllm_attention_bf16(q, kc, vc, ref, cnt, k_cap)
        lib.dllm_attention_bf16_noalloc(q, kc, vc, out, cnt, k_cap)
        torch.cuda.synchronize()
        # the compact rows are packed by sequence: count[b] rows at sum(count[:b])
        off = 0
        for b, c in enumerate(counts):
            if c:
                got = f64(out[off:off + c])
                assert max_abs_rel(got, f64(ref[off:off + c])) < TOL["bf16"]
                qb = f64(q[off:off + c]).reshape(c, Hq, hd)
                ora = O.store(O.attention(qb, f64(kc[b]), f64(vc[b])), "bf16").reshape(c, -1)
                assert max_abs_rel(got, ora) < TOL["bf16"], (B, N, b)
            off += c
        # rows past the packed total are not written
        assert torch.all(out[off:] == 7.0)


def test_noalloc_refuses_more_sequences_than_its_scratch(lib):
    B = lib.DLLM_NOALLOC_MAX_SEQS + 1
    dummy = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    p = dummy.data_ptr()
    st = lib._attn_noalloc(p, p, p, p, cnt.data_ptr(), B, 1, 16, 1, 1, 64,
                           torch.cuda.current_stream().cuda_stream)
    assert st == 5  # DLLM_ERR_CAPACITY, nothing launched
