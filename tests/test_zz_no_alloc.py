"""attn_cross_static_scratch: cross-attention for callers that may not allocate
device memory (a host that owns every device allocation through its own pool,
or a real-time decode loop that must not allocate between frames).

It runs the split-KV cross-attention with its partials in the library's fixed
device array instead of a caller workspace (splits of more than 8 parts; up to
8 parts merge inside a thread-block cluster and need no scratch). Two calls
with different queries on such a shape, enqueued back to back on one stream
with no synchronisation between them (the second reuses the array the first
one wrote), must each match the FP64 oracle and the workspace entry point
attn_cross within the parity tolerance;
a call after a warm-up must allocate no device memory; and a shape whose
split needs more than the fixed 4 MiB must be refused. This file is named to
be collected last."""
import ctypes
import types

import numpy as np
import pytest

import oracle
from speech_encoder_attention_b200 import attn, inputs
from tests.gpu_util import assert_parity, to_dev, to_np64

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 4 << 20


def _mat(t):
    return attn.AttnMat(ctypes.c_void_p(t.data_ptr()), t.stride(0))


class _Shape:
    """The verify block's 80 queries over 12000 encoder frames with 2 heads:
    long enough a key range that the split takes more than 8 parts, so it
    keeps its partials in scratch memory (shorter splits merge inside a
    thread-block cluster and need none)."""
    t_q, t_enc, n_heads, d_model = 80, 12000, 2, 128


def _verify_cross_inputs():
    spec = _Shape()
    rng = np.random.default_rng(5)
    inp = types.SimpleNamespace(q=inputs.random_f16(rng, (spec.t_q, spec.d_model)),
                                k_enc=inputs.random_f16(rng, (spec.t_enc, spec.d_model)),
                                v_enc=inputs.random_f16(rng, (spec.t_enc, spec.d_model)))
    # a second block of queries, so the two calls' partials differ
    q2 = inputs.random_f16(np.random.default_rng([5, 99]), inp.q.shape)
    return spec, inp, q2


def test_static_scratch_matches_oracle_and_workspace_entry_point_back_to_back():
    import torch
    assert torch.cuda.is_available()
    lib = attn.load_library()
    spec, inp, q2_host = _verify_cross_inputs()
    ke, ve = to_dev(inp.k_enc), to_dev(inp.v_enc)
    qs = [to_dev(inp.q), to_dev(q2_host)]
    d = spec.d_model
    # the shape splits its key range into more parts than a cluster merges,
    # so the scratch is really used
    need = attn.workspace_size(1, spec.t_q, spec.t_enc, spec.n_heads, attn.MASK_FULL)
    assert 0 < need <= STATIC_SCRATCH_BYTES
    assert attn.debug_plan(1, spec.t_q, spec.t_enc, spec.n_heads, attn.MASK_FULL,
                           num_sms=torch.cuda.get_device_properties(0).multi_processor_count)["kv_splits"] > 8

    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    outs = [torch.full((spec.t_q, d), float("nan"), dtype=torch.float16, device="cuda") for _ in qs]
    for q, out in zip(qs, outs):  # no synchronisation between the two calls
        st = lib.attn_cross_static_scratch(_mat(q), _mat(ke), _mat(ve), 1, spec.t_q, spec.t_enc, spec.n_heads,
                                           64, 0.125, _mat(out), stream)
        assert st == attn.ATTN_OK, attn.status_string(st)
    torch.cuda.synchronize()
    wants = [attn.attn_cross(q, ke, ve, 1, spec.t_q, spec.t_enc, spec.n_heads) for q in qs]
    torch.cuda.synchronize()
    for call, (q_host, out, want) in enumerate(zip((inp.q, q2_host), outs, wants)):
        ref = oracle.cross_attention(q_host, inp.k_enc, inp.v_enc, spec.n_heads)
        assert_parity(to_np64(out), ref, what=f"static scratch call {call} vs oracle")
        assert_parity(to_np64(out), to_np64(want), what=f"static scratch call {call} vs attn_cross")
    assert attn.debug_error_word() == (attn.ATTN_OK, 0)


def test_static_scratch_allocates_nothing():
    import torch
    lib = attn.load_library()
    spec, inp, _ = _verify_cross_inputs()
    q, ke, ve = (to_dev(a) for a in (inp.q, inp.k_enc, inp.v_enc))
    out = torch.empty(spec.t_q, spec.d_model, dtype=torch.float16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        st = lib.attn_cross_static_scratch(_mat(q), _mat(ke), _mat(ve), 1, spec.t_q, spec.t_enc, spec.n_heads,
                                           64, 0.125, _mat(out), stream)
        assert st == attn.ATTN_OK, attn.status_string(st)
        torch.cuda.synchronize()

    call()  # warm-up: the device set-up and lazy module loading happen here
    free0, allocated0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(3):
        call()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == allocated0


def test_static_scratch_refuses_splits_larger_than_the_array():
    import torch
    lib = attn.load_library()
    # 16 query tiles of one head over 18 key tiles: 9 splits (more than a
    # cluster merges), whose partials need 9 x 2048 x 264 bytes > 4 MiB
    t_q, t_enc, heads = 128 * 16, 2304, 1
    rng = np.random.default_rng(0)
    q = to_dev(inputs.random_f16(rng, (t_q, 64)))
    k = to_dev(inputs.random_f16(rng, (t_enc, 64)))
    v = to_dev(inputs.random_f16(rng, (t_enc, 64)))
    assert attn.workspace_size(1, t_q, t_enc, heads, attn.MASK_FULL) > STATIC_SCRATCH_BYTES
    out = torch.zeros(t_q, 64, dtype=torch.float16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.attn_cross_static_scratch(_mat(q), _mat(k), _mat(v), 1, t_q, t_enc, heads, 64, 0.125, _mat(out),
                                       stream)
    torch.cuda.synchronize()
    assert st == attn.ATTN_ERR_INVALID
    assert torch.count_nonzero(out) == 0, "a refused call must launch nothing"
