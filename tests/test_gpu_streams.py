"""The library under CUDA graph capture and under back-to-back launches.

Every kernel is launched programmatically (its prologue may overlap the
previous kernel in the stream), so these check that results stay exact when
calls follow each other closely, when they are replayed from a captured
graph, and that no bounded wait expires on the way."""
import numpy as np
import pytest

import oracle
from speech_encoder_attention_b200 import attn, inputs
from tests.gpu_util import assert_parity, to_dev, to_np64

pytestmark = pytest.mark.gpu


def torch_mod():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def check_error_word():
    st, word = attn.debug_error_word()
    assert st == attn.ATTN_OK and word == 0, f"device error word {word:#x}"


def test_encoder_step_replayed_from_a_cuda_graph():
    torch = torch_mod()
    spec = inputs.ENCODER_WORKLOADS["window"]
    inp = inputs.make_encoder_inputs(spec)
    d = spec.d_model
    x, w, bq, bv = (to_dev(a) for a in (inp.x, inp.w_qkv, inp.b_q, inp.b_v))
    qkv = torch.empty(spec.t, 3 * d, dtype=torch.float16, device="cuda")
    out = torch.empty(spec.t, d, dtype=torch.float16, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):  # warm up (one-time device setup) outside the capture
        attn.attn_qkv_pack(x, w, bq, bv, out=qkv)
        attn.attn_forward(qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:], 1, spec.t, spec.t, spec.n_heads, out=out)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        attn.attn_qkv_pack(x, w, bq, bv, out=qkv)
        attn.attn_forward(qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:], 1, spec.t, spec.t, spec.n_heads, out=out)
    ref = oracle.encoder_attention(inp.x, inp.w_qkv, inp.b_q, inp.b_v, 1, spec.t, spec.n_heads)
    for _ in range(3):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert_parity(to_np64(out), ref, what="graph replay")
    check_error_word()


def test_split_paths_replayed_from_a_cuda_graph():
    """The verify calls (split key ranges plus their combine launches),
    captured once and replayed with new query values."""
    torch = torch_mod()
    spec = inputs.VERIFY_WORKLOADS["verify"]
    inp = inputs.make_verify_inputs(spec)
    q, kc, vc, ke, ve = (to_dev(a) for a in (inp.q, inp.k_cache, inp.v_cache, inp.k_enc, inp.v_enc))
    bits = to_dev(inp.bits.view(np.int32))
    ws_bytes = max(attn.workspace_size(1, spec.t_q, spec.slots, spec.n_heads, attn.MASK_SLOTMASK),
                   attn.workspace_size(1, spec.t_q, spec.t_enc, spec.n_heads))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    o_self = torch.empty_like(q)
    o_cross = torch.empty_like(q)

    def step():
        attn.attn_forward(q, kc, vc, 1, spec.t_q, spec.slots, spec.n_heads, mask_kind=attn.MASK_SLOTMASK,
                          bits=bits, out=o_self, workspace=ws)
        attn.attn_cross(q, ke, ve, 1, spec.t_q, spec.t_enc, spec.n_heads, out=o_cross, workspace=ws)

    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    rng = np.random.default_rng(90)
    for _ in range(2):
        q_host = inputs.random_f16(rng, inp.q.shape)
        q.copy_(to_dev(q_host))
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        assert_parity(to_np64(o_self), oracle.slotmask_attention(q_host, inp.k_cache, inp.v_cache, inp.bits,
                                                                  spec.n_heads), what="graph slotmask")
        assert_parity(to_np64(o_cross), oracle.cross_attention(q_host, inp.k_enc, inp.v_enc, spec.n_heads),
                      what="graph cross")
    check_error_word()


def test_back_to_back_calls_of_every_kind():
    """Alternating projections, range, bitmask, cross and Q8_0 calls on one
    stream, many times, with each call's output read by the next call."""
    torch = torch_mod()
    rng = np.random.default_rng(91)
    t, heads, d = 300, 4, 256
    x = inputs.random_f16(rng, (2 * t, d))
    w = inputs.random_f16(rng, (3 * d, d), 0.02)
    bq, bv = inputs.random_f16(rng, (d,), 0.01), inputs.random_f16(rng, (d,), 0.01)
    q8 = inputs.make_q8_inputs(inputs.Q8Spec("s", 2 * t, d, 92))
    allowed = rng.random((t, t)) < 0.1
    allowed[:, 0] = True
    bits = inputs.pack_bits(allowed)
    dx, dw, dbq, dbv = to_dev(x), to_dev(w), to_dev(bq), to_dev(bv)
    dq8, dbits = to_dev(q8.w_blocks), to_dev(bits.view(np.int32))
    lens = to_dev(np.array([t, 171], np.int32))
    for _ in range(30):
        qkv = attn.attn_qkv_pack(dx, dw, dbq, dbv)
        a = attn.attn_forward(qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:], 2, t, t, heads,
                              mask_kind=attn.MASK_BAND, window=50, causal=True, q_lens=lens, kv_lens=lens)
        b = attn.attn_forward(a, qkv[:, d:2 * d], qkv[:, 2 * d:], 2, t, t, heads, mask_kind=attn.MASK_SLOTMASK,
                              bits=dbits)
        c = attn.attn_cross(b[:16], qkv[:, d:2 * d], qkv[:, 2 * d:], 1, 16, 2 * t, heads)
        qkv8 = attn.attn_qkv_pack_q8_0(dx, dq8, dbq, dbv)
    torch.cuda.synchronize()
    check_error_word()
    r_qkv = oracle.qkv_projection(x, w, bq, bv)
    r_a = oracle.range_attention(r_qkv[:, :d], r_qkv[:, d:2 * d], r_qkv[:, 2 * d:], 2, t, t, heads,
                                 q_lens=[t, 171], kv_lens=[t, 171], window=50, causal=True)
    # the oracle runs the whole chain from the original inputs
    r_b = np.concatenate([oracle.attention(r_a[s * t:(s + 1) * t], r_qkv[s * t:(s + 1) * t, d:2 * d],
                                           r_qkv[s * t:(s + 1) * t, 2 * d:], heads, allowed) for s in range(2)])
    r_c = oracle.cross_attention(r_b[:16], r_qkv[:, d:2 * d], r_qkv[:, 2 * d:], heads)
    assert_parity(to_np64(qkv), r_qkv, what="back-to-back qkv")
    assert_parity(to_np64(a), r_a, what="back-to-back band")
    assert_parity(to_np64(b), r_b, what="back-to-back slotmask")
    assert_parity(to_np64(c), r_c, what="back-to-back cross")
    assert_parity(to_np64(qkv8), oracle.qkv_projection_q8_0(x, q8.w_blocks, bq, bv), what="back-to-back q8")
