"""Writes tests/golden/tiny_oracle.json and tiny_options.json from the FP64
oracle only.

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
    options()


def options_case():
    """The seeded inputs of the options fixture: 3 sequences of 40 keys with
    16-row query blocks, 2 heads; the q8_tiny projection."""
    rng = np.random.default_rng(4321)
    q = inputs.random_f16(rng, (3 * 16, 128))
    k = inputs.random_f16(rng, (3 * 40, 128))
    v = inputs.random_f16(rng, (3 * 40, 128))
    sinks = np.array([0.7, -1.3], np.float32)
    return q, k, v, sinks, inputs.make_q8_inputs(inputs.Q8_WORKLOADS["q8_tiny"])


def options():
    """Writes tiny_options.json: the range family (lengths, causal, band) with
    sinks, and the Q8_0 projection, from the oracle alone."""
    q, k, v, sinks, q8 = options_case()
    att = oracle.range_attention(q, k, v, 3, 16, 40, 2, q_lens=[16, 9, 0], kv_lens=[40, 25, 7], window=12,
                                 causal=True, sinks=sinks)
    proj = oracle.qkv_projection_q8_0(q8.x, q8.w_blocks, q8.b_q, q8.b_v)
    rng = np.random.default_rng(99)
    a_idx = [(int(r), int(c)) for r, c in zip(rng.integers(0, 48, 40), rng.integers(0, 128, 40))]
    p_idx = [(int(r), int(c)) for r, c in zip(rng.integers(0, 5, 40), rng.integers(0, 768, 40))]
    doc = {
        "what": "FP64 oracle values: causal band attention with lengths and sinks; the Q8_0 projection "
                "(q8_tiny); regression pin of the oracle",
        "source": "written by tests/golden/make_golden.py from oracle/ only",
        "attention": [[r, c, float(att[r, c])] for r, c in a_idx],
        "attention_l2": float(np.linalg.norm(att)),
        "q8_projection": [[r, c, float(proj[r, c])] for r, c in p_idx],
        "q8_projection_l2": float(np.linalg.norm(proj)),
    }
    with open(os.path.join(HERE, "tiny_options.json"), "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
