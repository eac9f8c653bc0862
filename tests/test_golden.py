"""The oracle still computes what tests/golden/make_golden.py froze (no GPU)."""
import json
import os

import numpy as np

from joint_audio_video_flash_b200 import synth, workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle_rows.json")


def test_oracle_matches_frozen_rows(oracle):
    from tests.golden.make_golden import input_digest
    with open(GOLDEN) as f:
        data = json.load(f)
    _, calls = workloads.configs()["tiny"]
    assert [c.name for c in calls] == [g["name"] for g in data["calls"]]
    for c, g in zip(calls, data["calls"]):
        q, k, v = synth.make_qkv(c.batch, c.q_len, c.kv_len, c.heads, c.head_dim, c.seed)
        assert input_digest(q, k, v) == g["input_sha256"], "seeded input generator drifted"
        o, lse = oracle.attention(q, k, v, c.scale, kv_valid_len=c.kv_valid_len, rows=g["rows"],
                                  return_lse=True)
        want = np.array([[float.fromhex(x) for x in r] for r in g["out"]])
        np.testing.assert_allclose(o, want, rtol=1e-14, atol=1e-16)
        np.testing.assert_allclose(lse, [float.fromhex(x) for x in g["lse"]], rtol=1e-14)
