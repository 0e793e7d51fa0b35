"""The oracle against its stored regression fixture (written by
tests/golden/make_golden.py from the oracle alone)."""
import json
import os

import numpy as np

import oracle
from speech_encoder_attention_b200 import inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_oracle_matches_fixture():
    with open(os.path.join(HERE, "golden", "tiny_oracle.json")) as f:
        doc = json.load(f)
    spec = inputs.ENCODER_WORKLOADS["tiny"]
    inp = inputs.make_encoder_inputs(spec)
    out, qkv = oracle.encoder_attention(inp.x, inp.w_qkv, inp.b_q, inp.b_v, 1, 64, 2, return_qkv=True)
    for r, c, val in doc["out"]:
        assert abs(out[r, c] - val) <= 1e-12 * max(1.0, abs(val))
    for r, c, val in doc["qkv"]:
        assert abs(qkv[r, c] - val) <= 1e-12 * max(1.0, abs(val))
    assert abs(np.linalg.norm(out) - doc["out_l2"]) <= 1e-10
    assert abs(np.linalg.norm(qkv) - doc["qkv_l2"]) <= 1e-10


def test_options_oracle_matches_fixture():
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "golden", "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    with open(os.path.join(HERE, "golden", "tiny_options.json")) as f:
        doc = json.load(f)
    q, k, v, sinks, q8 = mg.options_case()
    att = oracle.range_attention(q, k, v, 3, 16, 40, 2, q_lens=[16, 9, 0], kv_lens=[40, 25, 7], window=12,
                                 causal=True, sinks=sinks)
    proj = oracle.qkv_projection_q8_0(q8.x, q8.w_blocks, q8.b_q, q8.b_v)
    for r, c, val in doc["attention"]:
        assert abs(att[r, c] - val) <= 1e-12 * max(1.0, abs(val))
    for r, c, val in doc["q8_projection"]:
        assert abs(proj[r, c] - val) <= 1e-12 * max(1.0, abs(val))
    assert abs(np.linalg.norm(att) - doc["attention_l2"]) <= 1e-10
    assert abs(np.linalg.norm(proj) - doc["q8_projection_l2"]) <= 1e-10
