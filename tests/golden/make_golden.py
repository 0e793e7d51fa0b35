"""Writes tests/golden/tiny_oracle.json from the FP64 oracle only.

The pages print no attention values, so this fixture is a regression pin of the
oracle itself on the tiny workload (1 x 64 frames, d_model 128, 2 heads, seed 0):
any later change to the oracle's arithmetic shows up as a mismatch here.
Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from speech_encoder_attention_b200 import inputs  # noqa: E402


def main():
    spec = inputs.ENCODER_WORKLOADS["tiny"]
    inp = inputs.make_encoder_inputs(spec)
    out, qkv = oracle.encoder_attention(inp.x, inp.w_qkv, inp.b_q, inp.b_v, spec.batch, spec.t,
                                        spec.n_heads, return_qkv=True)
    rng = np.random.default_rng(1234)
    o_idx = [(int(r), int(c)) for r, c in zip(rng.integers(0, 64, 32), rng.integers(0, 128, 32))]
    q_idx = [(int(r), int(c)) for r, c in zip(rng.integers(0, 64, 32), rng.integers(0, 384, 32))]
    doc = {
        "what": "FP64 oracle values on the tiny workload (seed 0); regression pin of the oracle",
        "source": "written by tests/golden/make_golden.py from oracle/ only",
        "out": [[r, c, float(out[r, c])] for r, c in o_idx],
        "qkv": [[r, c, float(qkv[r, c])] for r, c in q_idx],
        "out_l2": float(np.linalg.norm(out)),
        "qkv_l2": float(np.linalg.norm(qkv)),
    }
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
