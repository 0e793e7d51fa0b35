"""GPU parity of the Q8_0-weight projection (attn_qkv_pack_q8_0) against the
FP64 oracle, which dequantizes the 34-byte blocks exactly: the seeded decoder
workloads, ragged row counts across the 128-row tile, no bias, strided
operands, identity rows that select dequantized weight columns, and the
boundary cases of the int8 range and of the block scales."""
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


def run(x, blocks, bq, bv, out=None):
    torch = torch_mod()
    got = attn.attn_qkv_pack_q8_0(to_dev(x), to_dev(blocks), None if bq is None else to_dev(bq),
                                  None if bv is None else to_dev(bv), out=out)
    torch.cuda.synchronize()
    st, word = attn.debug_error_word()
    assert st == attn.ATTN_OK and word == 0, f"device error word {word:#x}"
    return got


@pytest.mark.parametrize("name", ["q8_tiny", "q8_verify"])
def test_q8_workloads(name):
    inp = inputs.make_q8_inputs(inputs.Q8_WORKLOADS[name])
    got = run(inp.x, inp.w_blocks, inp.b_q, inp.b_v)
    assert_parity(to_np64(got), oracle.qkv_projection_q8_0(inp.x, inp.w_blocks, inp.b_q, inp.b_v), what=name)


@pytest.mark.parametrize("rows,d", [(1, 256), (127, 512), (128, 256), (129, 1280), (300, 768), (1000, 256)])
def test_q8_ragged_rows(rows, d):
    inp = inputs.make_q8_inputs(inputs.Q8Spec("r", rows, d, rows + d))
    got = run(inp.x, inp.w_blocks, inp.b_q, inp.b_v)
    assert_parity(to_np64(got), oracle.qkv_projection_q8_0(inp.x, inp.w_blocks, inp.b_q, inp.b_v),
                  what=f"q8 rows={rows} d={d}")


def test_q8_without_bias_and_strided_operands():
    torch = torch_mod()
    inp = inputs.make_q8_inputs(inputs.Q8Spec("s", 70, 512, 3))
    d = 512
    xs = torch.zeros(70, d + 64, dtype=torch.float16, device="cuda")
    xs[:, :d] = to_dev(inp.x)
    out = torch.full((70, 3 * d + 32), 7.0, dtype=torch.float16, device="cuda")
    got = attn.attn_qkv_pack_q8_0(xs[:, :d], to_dev(inp.w_blocks), out=out[:, :3 * d])
    torch.cuda.synchronize()
    zero = np.zeros(d, np.float16)
    assert_parity(to_np64(got), oracle.qkv_projection_q8_0(inp.x, inp.w_blocks, zero, zero), what="q8 no bias")
    assert (out[:, 3 * d:] == 7.0).all(), "padding columns of the output view were written"


def test_q8_identity_rows_select_dequantized_columns():
    inp = inputs.make_q8_inputs(inputs.Q8Spec("i", 1, 256, 4))
    d = 256
    x = np.eye(d, dtype=np.float16)[:130]          # 130 rows: two row tiles
    got = to_np64(run(x, inp.w_blocks, inp.b_q, inp.b_v))
    w = oracle.dequantize_q8_0(inp.w_blocks, d)
    bias = np.concatenate([inp.b_q, np.zeros(d), inp.b_v]).astype(np.float64)
    # |d*q| <= 127 * 6e-4 < 0.08 and |bias| < 0.05: the GPU rounds d*q to fp16
    # (half an ulp at 2^-4 scale: 2^-15) and then the sum with the bias (again
    # at most 2^-15), so the absolute error is below 2^-14 = 6.1e-5.
    for c in (0, 31, 32, 129):
        np.testing.assert_allclose(got[c], w[:, c] + bias, rtol=0, atol=6.2e-5)


def test_q8_extreme_codes_and_scales():
    rng = np.random.default_rng(5)
    d, rows = 256, 40
    n = 3 * d
    qs = rng.choice(np.array([-128, -127, 0, 1, 127], dtype=np.int8), size=(n, d))
    scales = rng.choice(np.array([0.0, 6.1e-5, 1e-3, 0.5, -0.25], dtype=np.float16), size=(n, d // 32))
    blocks = inputs.pack_q8_0(scales, qs)
    # x small enough that the outputs stay O(1) (|W| reaches 64): the absolute
    # tolerance is sized for O(1) outputs, where an fp16 half-ulp is <= 2^-11
    x = inputs.random_f16(rng, (rows, d), 0.002)
    zero = np.zeros(d, np.float16)
    got = run(x, blocks, zero, zero)
    assert_parity(to_np64(got), oracle.qkv_projection_q8_0(x, blocks, zero, zero), what="q8 extreme codes")
