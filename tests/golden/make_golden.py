"""Writes tests/golden/tiny_trajectory.json from the CPU oracle alone.

The file records the decisions (selected positions, revealed positions,
final tokens) of the 8-step generation on the tiny 1-layer fp32 model with
seeded synthetic weights and prompt.  It is a regression record of the
oracle, not an independent pin; the pins live in tests/test_oracle_*.py.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path[:0] = [ROOT, os.path.dirname(HERE)]

import numpy as np  # noqa: E402

import oracle as O  # noqa: E402
from dllm_synth import TINY, model_weights, prompt_tokens  # noqa: E402
from _util import oracle_cfg, oracle_weights, oracle_policy, f64  # noqa: E402


def trajectory():
    s = TINY
    cfg = oracle_cfg(s)
    W = oracle_weights(model_weights(s, seed=0))
    st = O.empty_state(cfg, f64(prompt_tokens(s, seed=1)).astype(np.int64))
    pol = oracle_policy(s)
    steps = []
    for t in range(8):
        out = O.step(cfg, W, st, pol, dense=(t == 0))
        steps.append({"idx": [a.tolist() for a in out.idx],
                      "unmasked": out.unmasked.tolist()})
    return {"shape": s.name, "steps": steps, "final_tokens": st.tokens.tolist()}


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_trajectory.json"), "w") as f:
        json.dump(trajectory(), f)
    print("wrote", os.path.join(HERE, "tiny_trajectory.json"))
