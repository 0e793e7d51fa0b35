"""GPU parity: the CUDA path (through the C ABI) against the FP64 oracle on the
same seeded inputs, element by element, within rel-L2 1e-3 and max-abs 5e-3.

Covers the five workloads at their full sizes (the 8-window one in the launch
configuration the benchmark times), ragged and edge sizes that span several
tiles and a tail, every mask mode, the split-KV path and its opt-out, and
invariants that hold at any size."""
import numpy as np
import pytest

import oracle
from speech_encoder_attention_b200 import attn, inputs
from tests.gpu_util import assert_parity, to_dev, to_np64

pytestmark = pytest.mark.gpu

SCALE = 0.125


def torch_mod():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def run_encoder(inp, mask_kind=attn.MASK_FULL, chunk_len=0):
    torch = torch_mod()
    s = inp.spec
    x, w, bq, bv = (to_dev(a) for a in (inp.x, inp.w_qkv, inp.b_q, inp.b_v))
    qkv = attn.attn_qkv_pack(x, w, bq, bv)
    d = s.d_model
    out = attn.attn_forward(qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:], s.batch, s.t, s.t, s.n_heads,
                            mask_kind=mask_kind, chunk_len=chunk_len)
    torch.cuda.synchronize()
    return to_np64(qkv), to_np64(out)


def check_error_word():
    st, word = attn.debug_error_word()
    assert st == attn.ATTN_OK and word == 0, f"device error word {word:#x}"


# ---------------------------------------------------------------------------
# the five workloads
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "window"])
def test_encoder_full_window(name):
    spec = inputs.ENCODER_WORKLOADS[name]
    inp = inputs.make_encoder_inputs(spec)
    qkv, out = run_encoder(inp)
    ref_out, ref_qkv = oracle.encoder_attention(inp.x, inp.w_qkv, inp.b_q, inp.b_v, spec.batch, spec.t,
                                                spec.n_heads, return_qkv=True)
    assert_parity(qkv, ref_qkv, what=f"{name} qkv")
    assert_parity(out, ref_out, what=f"{name} attention")
    check_error_word()


def test_encoder_eight_windows_full_size():
    """The benchmarked workload, in the benchmark's launch configuration."""
    spec = inputs.ENCODER_WORKLOADS["windows8"]
    inp = inputs.make_encoder_inputs(spec)
    qkv, out = run_encoder(inp)
    ref_out, ref_qkv = oracle.encoder_attention(inp.x, inp.w_qkv, inp.b_q, inp.b_v, spec.batch, spec.t,
                                                spec.n_heads, return_qkv=True)
    assert_parity(qkv, ref_qkv, what="windows8 qkv")
    assert_parity(out, ref_out, what="windows8 attention")
    for b in range(spec.batch):
        rows = slice(b * spec.t, (b + 1) * spec.t)
        assert_parity(out[rows], ref_out[rows], what=f"windows8 window {b}")
    check_error_word()


def test_encoder_chunked():
    spec = inputs.ENCODER_WORKLOADS["chunks"]
    inp = inputs.make_encoder_inputs(spec)
    qkv, out = run_encoder(inp, attn.MASK_CHUNK, spec.chunk_len)
    ref_out, ref_qkv = oracle.encoder_attention(inp.x, inp.w_qkv, inp.b_q, inp.b_v, 1, spec.t, spec.n_heads,
                                                mask="chunk", chunk_len=spec.chunk_len, return_qkv=True)
    assert_parity(qkv, ref_qkv, what="chunks qkv")
    assert_parity(out, ref_out, what="chunks attention")
    # the short last chunk on its own
    assert_parity(out[2200:], ref_out[2200:], what="chunks last (125-frame) chunk")
    check_error_word()


@pytest.mark.parametrize("split", [True, False])
def test_verify_tree_and_cross(split):
    torch = torch_mod()
    spec = inputs.VERIFY_WORKLOADS["verify"]
    inp = inputs.make_verify_inputs(spec)
    q, kc, vc, bits, ke, ve = (to_dev(a) for a in (inp.q, inp.k_cache, inp.v_cache,
                                                    inp.bits.view(np.int32), inp.k_enc, inp.v_enc))
    o_self = attn.attn_forward(q, kc, vc, 1, spec.t_q, spec.slots, spec.n_heads,
                               mask_kind=attn.MASK_SLOTMASK, bits=bits, split=split)
    o_cross = attn.attn_cross(q, ke, ve, 1, spec.t_q, spec.t_enc, spec.n_heads, split=split)
    torch.cuda.synchronize()
    assert_parity(to_np64(o_self), oracle.slotmask_attention(inp.q, inp.k_cache, inp.v_cache, inp.bits,
                                                              spec.n_heads), what="verify self")
    assert_parity(to_np64(o_cross), oracle.cross_attention(inp.q, inp.k_enc, inp.v_enc, spec.n_heads),
                  what="verify cross")
    check_error_word()


# ---------------------------------------------------------------------------
# QKV projection: ragged shapes
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("rows,d", [(1, 64), (65, 128), (129, 64), (300, 192), (1000, 1280), (127, 384)])
def test_qkv_projection_shapes(rows, d):
    torch = torch_mod()
    rng = np.random.default_rng(rows * 7 + d)
    x = inputs.random_f16(rng, (rows, d))
    w = inputs.random_f16(rng, (3 * d, d), 0.02)
    bq = inputs.random_f16(rng, (d,), 0.01)
    bv = inputs.random_f16(rng, (d,), 0.01)
    got = attn.attn_qkv_pack(to_dev(x), to_dev(w), to_dev(bq), to_dev(bv))
    torch.cuda.synchronize()
    assert_parity(to_np64(got), oracle.qkv_projection(x, w, bq, bv), what=f"qkv {rows}x{d}")


@pytest.mark.parametrize("rows,d", [(4096, 256), (4097, 512), (5000, 1280), (8191, 1024), (4500, 320)])
def test_qkv_projection_on_cta_pairs(rows, d):
    """Row counts that take the CTA-pair projection (256 x 256 tiles over two
    SMs): whole and ragged pair tiles, a last tile whose second CTA has no
    row, and a width (3 x 320) that is not a multiple of 256, which falls
    back to single-CTA tiles."""
    torch = torch_mod()
    rng = np.random.default_rng(rows + d)
    x = inputs.random_f16(rng, (rows, d))
    w = inputs.random_f16(rng, (3 * d, d), 0.02)
    bq = inputs.random_f16(rng, (d,), 0.01)
    bv = inputs.random_f16(rng, (d,), 0.01)
    if rows == 4097:
        bq = bv = None
    big = torch.full((rows, 3 * d + 32), 7.0, dtype=torch.float16, device="cuda")
    out = big[:, :3 * d]
    attn.attn_qkv_pack(to_dev(x), to_dev(w), None if bq is None else to_dev(bq), None if bv is None else to_dev(bv),
                       out=out)
    torch.cuda.synchronize()
    zero = np.zeros(d, dtype=np.float16)
    want = oracle.qkv_projection(x, w, zero if bq is None else bq, zero if bv is None else bv)
    assert_parity(to_np64(out), want, what=f"qkv pairs {rows}x{d}")
    assert torch.all(big[:, 3 * d:] == 7.0), "wrote outside the output view"
    check_error_word()


def test_qkv_projection_without_bias_and_padded_output():
    torch = torch_mod()
    rng = np.random.default_rng(5)
    rows, d = 200, 128
    x = inputs.random_f16(rng, (rows, d))
    w = inputs.random_f16(rng, (3 * d, d), 0.02)
    big = torch.full((rows, 3 * d + 64), 7.0, dtype=torch.float16, device="cuda")
    out = big[:, :3 * d]
    attn.attn_qkv_pack(to_dev(x), to_dev(w), None, None, out=out)
    torch.cuda.synchronize()
    assert_parity(to_np64(out), oracle.qkv_projection(x, w, np.zeros(d), np.zeros(d)), what="qkv no bias")
    assert torch.all(big[:, 3 * d:] == 7.0), "wrote outside the output view"


def test_qkv_identity_rows_select_weight_columns():
    torch = torch_mod()
    d = 128
    rng = np.random.default_rng(6)
    w = inputs.random_f16(rng, (3 * d, d))
    bq = inputs.random_f16(rng, (d,))
    bv = inputs.random_f16(rng, (d,))
    got = to_np64(attn.attn_qkv_pack(to_dev(np.eye(d, dtype=np.float16)), to_dev(w), to_dev(bq), to_dev(bv)))
    torch.cuda.synchronize()
    bias = np.concatenate([bq, np.zeros(d), bv]).astype(np.float64)
    want = w.astype(np.float64).T + bias
    # one product and one bias add, rounded once to fp16
    np.testing.assert_allclose(got, want, rtol=2e-3, atol=2e-3)


# ---------------------------------------------------------------------------
# attention: edge sizes and masks (random q, k, v)
# ---------------------------------------------------------------------------

def rand_qkv(rng, batch, t_q, t_kv, heads, std=1.0):
    c = heads * 64
    return (inputs.random_f16(rng, (batch * t_q, c), std), inputs.random_f16(rng, (batch * t_kv, c), std),
            inputs.random_f16(rng, (batch * t_kv, c), std))


def oracle_batched(q, k, v, batch, t_q, t_kv, heads, allowed):
    out = np.zeros((batch * t_q, heads * 64))
    for b in range(batch):
        out[b * t_q:(b + 1) * t_q] = oracle.attention(q[b * t_q:(b + 1) * t_q], k[b * t_kv:(b + 1) * t_kv],
                                                      v[b * t_kv:(b + 1) * t_kv], heads, allowed)
    return out


@pytest.mark.parametrize("t", [1, 2, 63, 64, 65, 127, 128, 129, 255, 257, 700])
def test_full_self_attention_lengths(t):
    torch = torch_mod()
    rng = np.random.default_rng(t)
    batch, heads = 2, 2
    q, k, v = rand_qkv(rng, batch, t, t, heads)
    got = attn.attn_forward(to_dev(q), to_dev(k), to_dev(v), batch, t, t, heads)
    torch.cuda.synchronize()
    assert_parity(to_np64(got), oracle_batched(q, k, v, batch, t, t, heads, oracle.allowed_full(t, t)),
                  what=f"full t={t}")


@pytest.mark.parametrize("clen", [1, 7, 64, 100, 128, 150, 200, 256, 517, 2000])
def test_chunk_lengths(clen):
    torch = torch_mod()
    t = 517
    rng = np.random.default_rng(clen)
    q, k, v = rand_qkv(rng, 2, t, t, 2)
    got = attn.attn_forward(to_dev(q), to_dev(k), to_dev(v), 2, t, t, 2, mask_kind=attn.MASK_CHUNK,
                            chunk_len=clen)
    torch.cuda.synchronize()
    assert_parity(to_np64(got), oracle_batched(q, k, v, 2, t, t, 2, oracle.allowed_chunk(t, clen)),
                  what=f"chunk len={clen}")


@pytest.mark.parametrize("t_q,t_kv,density", [(16, 45, 0.5), (80, 448, 0.2), (200, 300, 0.05),
                                              (130, 1000, 0.01), (33, 129, 1.0)])
def test_slotmask_random(t_q, t_kv, density):
    torch = torch_mod()
    rng = np.random.default_rng(t_q + t_kv)
    batch, heads = 2, 2
    q, k, v = rand_qkv(rng, batch, t_q, t_kv, heads)
    allowed = rng.random((t_q, t_kv)) < density
    allowed[0] = False                      # a row with nothing allowed -> zeros
    allowed[min(1, t_q - 1), :] = False
    allowed[min(1, t_q - 1), t_kv - 1] = True   # a single slot, in the last word
    bits = inputs.pack_bits(allowed)
    got = attn.attn_forward(to_dev(q), to_dev(k), to_dev(v), batch, t_q, t_kv, heads,
                            mask_kind=attn.MASK_SLOTMASK, bits=to_dev(bits.view(np.int32)))
    torch.cuda.synchronize()
    got = to_np64(got)
    assert_parity(got, oracle_batched(q, k, v, batch, t_q, t_kv, heads, allowed),
                  what=f"slotmask {t_q}x{t_kv}")
    assert np.all(got[0] == 0.0) and np.all(got[t_q] == 0.0)


def test_slotmask_skips_empty_tiles_and_ignores_bits_past_the_end():
    torch = torch_mod()
    rng = np.random.default_rng(3)
    t_q, t_kv = 64, 600
    q, k, v = rand_qkv(rng, 1, t_q, t_kv, 2)
    allowed = np.zeros((t_q, t_kv), bool)
    allowed[:, 0:5] = True          # tile 0
    allowed[:, 590:600] = True      # tile 4 (partial); tiles 1..3 are empty
    bits = inputs.pack_bits(allowed)
    bits[:, -1] |= np.uint32(0xFFFF0000)   # bits past slot 599 must be ignored
    got = attn.attn_forward(to_dev(q), to_dev(k), to_dev(v), 1, t_q, t_kv, 2, mask_kind=attn.MASK_SLOTMASK,
                            bits=to_dev(bits.view(np.int32)))
    torch.cuda.synchronize()
    assert_parity(to_np64(got), oracle.attention(q, k, v, 2, allowed), what="slotmask sparse tiles")


@pytest.mark.parametrize("t_q,t_enc", [(1, 1), (16, 100), (80, 1500), (200, 1500), (5, 3000)])
def test_cross_shapes(t_q, t_enc):
    torch = torch_mod()
    rng = np.random.default_rng(t_q * 3 + t_enc)
    q, k, v = rand_qkv(rng, 2, t_q, t_enc, 4)
    got = attn.attn_cross(to_dev(q), to_dev(k), to_dev(v), 2, t_q, t_enc, 4)
    torch.cuda.synchronize()
    assert_parity(to_np64(got), oracle_batched(q, k, v, 2, t_q, t_enc, 4, oracle.allowed_full(t_q, t_enc)),
                  what=f"cross {t_q}x{t_enc}")


def test_large_logits_do_not_overflow():
    torch = torch_mod()
    rng = np.random.default_rng(9)
    q, k, v = rand_qkv(rng, 1, 300, 300, 2, std=4.0)  # logits with std ~16
    got = attn.attn_forward(to_dev(q), to_dev(k), to_dev(v), 1, 300, 300, 2)
    torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, 2, oracle.allowed_full(300, 300))
    # v has std 4 here, so scale the absolute bound with it
    assert_parity(to_np64(got), ref, abs_tol=4 * 5e-3, what="large logits")


@pytest.mark.parametrize("order", ["growing", "shrinking", "mixed"])
def test_row_max_jumps_between_key_tiles(order):
    """Key tiles whose logits jump by far more than the softmax's exponent
    headroom from one tile to the next (the range kernel computes a tile's
    exponentials against the reference of earlier tiles and must redo the tile
    and rescale O and the row sums when a row's max outgrows it): keys
    [512, 1024) are scaled up 6x, so their logits reach ~20 natural units
    above those of the first tiles. "mixed" shrinks every other query row
    twenty-fold, so those rows never outgrow their reference while their
    neighbours in the same warp do."""
    torch = torch_mod()
    rng = np.random.default_rng({"growing": 31, "shrinking": 32, "mixed": 33}[order])
    t, heads = 1300, 2
    q = rng.standard_normal((t, heads * 64))
    k = rng.standard_normal((t, heads * 64))
    v = rng.standard_normal((t, heads * 64))
    big = slice(512, 1024) if order != "shrinking" else slice(0, 512)
    k[big] *= 6.0
    if order == "mixed":
        q[1::2] *= 0.05
    q, k, v = (a.astype(np.float16) for a in (q, k, v))
    got = attn.attn_forward(to_dev(q), to_dev(k), to_dev(v), 1, t, t, heads)
    torch.cuda.synchronize()
    check_error_word()
    ref = oracle.attention(q, k, v, heads, oracle.allowed_full(t, t))
    assert_parity(to_np64(got), ref, what=f"row max jumps ({order})")


def test_output_view_padding_untouched_and_strided_inputs():
    torch = torch_mod()
    rng = np.random.default_rng(10)
    t, heads = 300, 2
    q, k, v = rand_qkv(rng, 1, t, t, heads)
    big_q = torch.zeros(t, 256 + 64, dtype=torch.float16, device="cuda")
    big_q[:, 64:192] = to_dev(q)
    big = torch.full((t, 128 + 72), 3.0, dtype=torch.float16, device="cuda")
    out = big[:, 8:136]
    attn.attn_forward(big_q[:, 64:192], to_dev(k), to_dev(v), 1, t, t, heads, out=out)
    torch.cuda.synchronize()
    assert_parity(to_np64(out), oracle.attention(q, k, v, heads, oracle.allowed_full(t, t)), what="strided")
    assert torch.all(big[:, :8] == 3.0) and torch.all(big[:, 136:] == 3.0)


# ---------------------------------------------------------------------------
# invariants on the GPU
# ---------------------------------------------------------------------------

def test_constant_values_come_back():
    """W_v = 0 and b_v = c: every output row equals c (closed form)."""
    torch = torch_mod()
    spec = inputs.ENCODER_WORKLOADS["window"]
    inp = inputs.make_encoder_inputs(spec)
    d = spec.d_model
    w = inp.w_qkv.copy()
    w[2 * d:] = 0
    c = np.random.default_rng(1).uniform(-1, 1, d).astype(np.float16)
    inp2 = inputs.EncoderInputs(spec, inp.x, w, inp.b_q, c)
    _, out = run_encoder(inp2)
    want = np.tile(c.astype(np.float64), (spec.t, 1))
    assert_parity(out, want, what="constant V")


def test_full_mode_is_permutation_equivariant():
    torch = torch_mod()
    spec = inputs.ENCODER_WORKLOADS["window"]
    inp = inputs.make_encoder_inputs(spec)
    perm = np.random.default_rng(2).permutation(spec.t)
    _, a = run_encoder(inp)
    _, b = run_encoder(inputs.EncoderInputs(spec, inp.x[perm], inp.w_qkv, inp.b_q, inp.b_v))
    assert_parity(b, a[perm], what="permutation")


def test_chunk_equals_independent_sequences_on_gpu():
    """CHUNK(200) over 2325 frames == each chunk run as its own FULL sequence."""
    torch = torch_mod()
    spec = inputs.ENCODER_WORKLOADS["chunks"]
    inp = inputs.make_encoder_inputs(spec)
    x, w, bq, bv = (to_dev(a) for a in (inp.x, inp.w_qkv, inp.b_q, inp.b_v))
    qkv = attn.attn_qkv_pack(x, w, bq, bv)
    d = spec.d_model
    chunked = attn.attn_forward(qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:], 1, spec.t, spec.t, spec.n_heads,
                                mask_kind=attn.MASK_CHUNK, chunk_len=200)
    pieces = []
    for c0 in range(0, spec.t, 200):
        n = min(200, spec.t - c0)
        sl = qkv[c0:c0 + n]
        pieces.append(attn.attn_forward(sl[:, :d], sl[:, d:2 * d], sl[:, 2 * d:], 1, n, n, spec.n_heads,
                                        split=False))
    torch.cuda.synchronize()
    indep = torch.cat(pieces)
    assert torch.equal(chunked, indep), "CHUNK differs from independent chunks"


def test_slotmask_all_ones_equals_full_and_single_bit_returns_value():
    torch = torch_mod()
    rng = np.random.default_rng(11)
    t_q, t_kv = 80, 448
    q, k, v = rand_qkv(rng, 1, t_q, t_kv, 2)
    ones = inputs.pack_bits(np.ones((t_q, t_kv), bool))
    a = attn.attn_forward(to_dev(q), to_dev(k), to_dev(v), 1, t_q, t_kv, 2, mask_kind=attn.MASK_SLOTMASK,
                          bits=to_dev(ones.view(np.int32)))
    b = attn.attn_forward(to_dev(q), to_dev(k), to_dev(v), 1, t_q, t_kv, 2)
    sel = rng.integers(0, t_kv, t_q)
    one = inputs.pack_bits(np.eye(t_kv, dtype=bool)[sel])
    c = attn.attn_forward(to_dev(q), to_dev(k), to_dev(v), 1, t_q, t_kv, 2, mask_kind=attn.MASK_SLOTMASK,
                          bits=to_dev(one.view(np.int32)))
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    np.testing.assert_allclose(to_np64(c), v[sel].astype(np.float64), rtol=1e-3, atol=1e-4)


# ---------------------------------------------------------------------------
# bounded waits
# ---------------------------------------------------------------------------

def test_timeout_probe_reports_and_clears():
    torch_mod()
    assert attn.debug_error_word()[0] == attn.ATTN_OK
    assert attn.debug_timeout_probe(2_000_000) == attn.ATTN_OK   # 2 ms
    st, word = attn.debug_error_word()
    assert st == attn.ATTN_ERR_TIMEOUT and word != 0
    assert attn.debug_error_word() == (attn.ATTN_OK, 0)
    # the context is still usable
    test_full_self_attention_lengths(65)


# ---------------------------------------------------------------------------
# maximum sizes and many units
# ---------------------------------------------------------------------------

def test_slotmask_at_the_slot_limit():
    """65,536 slots (16 tile-flag words of 32 key tiles): bits spread over the
    whole range, including the very last slot."""
    torch = torch_mod()
    t_q, t_kv, heads = 8, 65536, 1
    rng = np.random.default_rng(70)
    q, k, v = rand_qkv(rng, 1, t_q, t_kv, heads)
    allowed = rng.random((t_q, t_kv)) < 0.002
    allowed[:, -1] = True
    allowed[0, :] = False
    allowed[0, 40000] = True
    bits = inputs.pack_bits(allowed)
    got = attn.attn_forward(to_dev(q), to_dev(k), to_dev(v), 1, t_q, t_kv, heads, mask_kind=attn.MASK_SLOTMASK,
                            bits=to_dev(bits.view(np.int32)))
    torch.cuda.synchronize()
    assert_parity(to_np64(got), oracle.attention(q, k, v, heads, allowed), what="slotmask 65536 slots")
    check_error_word()


def test_many_units_per_persistent_cta():
    """1,024 short sequences: each persistent CTA walks several units."""
    torch = torch_mod()
    batch, t, heads = 512, 100, 2
    rng = np.random.default_rng(71)
    q, k, v = rand_qkv(rng, batch, t, t, heads)
    got = attn.attn_forward(to_dev(q), to_dev(k), to_dev(v), batch, t, t, heads)
    torch.cuda.synchronize()
    want = oracle_batched(q, k, v, batch, t, t, heads, oracle.allowed_full(t, t))
    assert_parity(to_np64(got), want, what="512 sequences")
    check_error_word()
