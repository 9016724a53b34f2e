"""The oracle against the constants the pages print and its own recorded
tiny trajectory (tests/golden/)."""
import json
import os

import oracle as O
from golden.make_golden import trajectory

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_page_constants_used_by_oracle():
    c = _load("pages_constants.json")
    assert O.Policy().alpha == c["importance_alpha"]["value"]
    mb = c["cache_mb_per_sample_llada8b_1024p_256g"]["value"]
    kv = O.kv_cache_bytes(32, 1024 + 256, 32, 128) / 2 ** 20
    assert abs(kv - mb) / mb < 0.01
    # the early-skip depths of an 8B model (32 layers) fall on whole layers
    assert [32 * f for f in c["early_skip_depth_fractions"]["value"]] == [4.0, 8.0]


def test_tiny_trajectory_matches_record():
    rec = _load("tiny_trajectory.json")
    now = trajectory()
    assert now["steps"] == rec["steps"]
    assert now["final_tokens"] == rec["final_tokens"]
