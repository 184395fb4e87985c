"""Writes oracle_tiny.json: the oracle's outputs on tiny seeded cases.

A regression lock on the oracle itself -- a later change to its arithmetic
must change this file, and the commit that does so must say why.  Calls only
``oracle/`` and the seeded generators.  Run from the repository root:
``python tests/golden/make_oracle_tiny.py``.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from synth import normal_bf16, paged_kv, rng, uniform_bf16  # noqa: E402


def cases():
    g = rng(1234)
    x = normal_bf16(g, (2, 8))
    w = uniform_bf16(g, (8,), 0.5, 1.5)
    W = normal_bf16(g, (3, 8), std=0.02)
    kv = paged_kv(g, [5, 19], num_kv_heads=1, head_dim=4)
    q = normal_bf16(g, (2, 2, 4))
    rows = oracle.decode_rows(q, kv.seq_lens)
    o, lse = oracle.attention(*rows, 2, kv.k_cache, kv.v_cache, kv.block_table, want_lse=True)
    return {
        "seed": 1234,
        "rmsnorm": {"x": x.tolist(), "w": w.tolist(), "eps": 1e-6,
                    "y": oracle.rmsnorm(x, w, 1e-6).tolist()},
        "matmul": {"a": x.tolist(), "w": W.tolist(), "c": oracle.matmul(x, W).tolist()},
        "attention": {"k_cache": kv.k_cache.tolist(), "v_cache": kv.v_cache.tolist(),
                      "block_table": kv.block_table.tolist(), "seq_lens": kv.seq_lens.tolist(),
                      "q": q.tolist(), "Hq": 2, "o": o.tolist(), "lse": lse.tolist()},
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "oracle_tiny.json"), "w") as f:
        json.dump(cases(), f, indent=None, separators=(",", ":"))
        f.write("\n")
