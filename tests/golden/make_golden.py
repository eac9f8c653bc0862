"""Writes tiny_oracle_rows.json: fp64 oracle outputs on the tiny workload.

Calls only the oracle (and the seeded input generator).  The file freezes the
oracle's arithmetic: a later change to it shows up as a mismatch in
tests/test_golden.py and has to be justified by the passage it follows.
Run from the repository root:  python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from joint_audio_video_flash_b200 import synth, workloads  # noqa: E402
from oracle import oracle  # noqa: E402


def input_digest(q, k, v):
    h = hashlib.sha256()
    for t in (q, k, v):
        h.update(oracle._bits(t).tobytes())
    return h.hexdigest()


def main():
    _, calls = workloads.configs()["tiny"]
    out = {"source": "oracle/attention_oracle.c via tests/golden/make_golden.py", "calls": []}
    for c in calls:
        q, k, v = synth.make_qkv(c.batch, c.q_len, c.kv_len, c.heads, c.head_dim, c.seed)
        rows = synth.sample_rows(c.batch, c.q_len, c.heads, per_head=2, seed=c.seed,
                                 full_heads=()).tolist()
        o, lse = oracle.attention(q, k, v, c.scale, kv_valid_len=c.kv_valid_len, rows=rows,
                                  return_lse=True)
        out["calls"].append({
            "name": c.name, "seed": c.seed, "shape": [c.batch, c.q_len, c.kv_len, c.heads,
                                                      c.head_dim], "kv_valid_len": c.kv_valid_len,
            "scale": c.scale, "input_sha256": input_digest(q, k, v), "rows": rows,
            "out": [[float(x).hex() for x in r] for r in o], "lse": [float(x).hex() for x in lse],
        })
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_rows.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(path)


if __name__ == "__main__":
    main()
