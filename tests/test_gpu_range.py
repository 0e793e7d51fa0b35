"""GPU parity of the range family's options and of attention sinks: the CUDA
path (through the C ABI) against the FP64 oracle on seeded inputs, element by
element, within rel-L2 1e-3 and max-abs 5e-3.

Per-sequence lengths (padding never attends nor is seen; padding rows are 0),
the causal flag with the query block at the end of its keys, the band (sliding
window), CHUNK with lengths, sinks on every mask kind and on the split-KV
path, and the degenerate cases: window 1, empty rows, zero-length sequences,
more queries than keys, a sink that takes all the weight."""
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


def rand_qkv(rng, batch, t_q, t_kv, heads):
    c = heads * 64
    return (inputs.random_f16(rng, (batch * t_q, c)), inputs.random_f16(rng, (batch * t_kv, c)),
            inputs.random_f16(rng, (batch * t_kv, c)))


def i32(a):
    return to_dev(np.asarray(a, dtype=np.int32))


def f32(a):
    return to_dev(np.asarray(a, dtype=np.float32))


def run(q, k, v, batch, t_q, t_kv, heads, split=True, **kw):
    torch = torch_mod()
    dev = {}
    for key in ("q_lens", "kv_lens"):
        if kw.get(key) is not None:
            dev[key] = i32(kw[key])
    if kw.get("sinks") is not None:
        dev["sinks"] = f32(kw["sinks"])
    opts = {key: kw[key] for key in ("mask_kind", "chunk_len", "window", "causal") if key in kw}
    got = attn.attn_forward(to_dev(q), to_dev(k), to_dev(v), batch, t_q, t_kv, heads, split=split, **opts, **dev)
    torch.cuda.synchronize()
    st, word = attn.debug_error_word()
    assert st == attn.ATTN_OK and word == 0, f"device error word {word:#x}"
    return to_np64(got)


def want(q, k, v, batch, t_q, t_kv, heads, **kw):
    kw = dict(kw)
    kind = kw.pop("mask_kind", attn.MASK_FULL)
    if kind != attn.MASK_CHUNK:
        kw.pop("chunk_len", None)
    return oracle.range_attention(q, k, v, batch, t_q, t_kv, heads, **kw)


def check(q, k, v, batch, t_q, t_kv, heads, what, split=True, **kw):
    got = run(q, k, v, batch, t_q, t_kv, heads, split=split, **kw)
    ref = want(q, k, v, batch, t_q, t_kv, heads, **kw)
    assert_parity(got, ref, what=what)
    return got, ref


# ---------------------------------------------------------------------------
# causal
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("t", [1, 2, 65, 128, 129, 300, 700])
def test_causal_square(t):
    rng = np.random.default_rng(100 + t)
    q, k, v = rand_qkv(rng, 2, t, t, 2)
    check(q, k, v, 2, t, t, 2, f"causal t={t}", causal=True)


@pytest.mark.parametrize("t_q,t_kv,batch", [(16, 448, 5), (80, 1500, 1), (130, 257, 2), (200, 100, 2),
                                            (1, 700, 3)])
def test_causal_query_block_at_the_end_of_its_keys(t_q, t_kv, batch):
    rng = np.random.default_rng(t_q * 7 + t_kv)
    q, k, v = rand_qkv(rng, batch, t_q, t_kv, 2)
    got, _ = check(q, k, v, batch, t_q, t_kv, 2, f"causal {t_q}x{t_kv}", causal=True)
    if t_q > t_kv:  # rows at negative positions see no key
        np.testing.assert_array_equal(got[: t_q - t_kv - 1], 0.0)


@pytest.mark.parametrize("split", [True, False])
def test_causal_split_and_unsplit_agree_with_oracle(split):
    rng = np.random.default_rng(5)
    q, k, v = rand_qkv(rng, 1, 80, 1500, 4)
    check(q, k, v, 1, 80, 1500, 4, f"causal split={split}", split=split, causal=True)


# ---------------------------------------------------------------------------
# narrow query tiles (at most 32 rows: the rows in every lane quadrant, each
# softmax warp a quarter of the key columns, four partials merged per row)
# ---------------------------------------------------------------------------

NARROW_CASES = [  # (t_q, t_kv, batch, heads, options)
    (1, 1, 3, 2, {}), (1, 700, 3, 2, {}), (7, 129, 5, 3, {}), (16, 448, 5, 4, {}), (31, 1000, 2, 2, {}),
    (32, 256, 4, 2, {}), (16, 448, 5, 4, {"causal": True}), (20, 10, 3, 2, {"causal": True}),
    (32, 100, 2, 2, {"causal": True}), (16, 300, 4, 2, {"mask_kind": attn.MASK_BAND, "window": 50}),
    (16, 448, 5, 2, {"sinks": [0.5, -1.0]}), (16, 448, 5, 2, {"sinks": [2.0, 0.0], "causal": True}),
    (24, 500, 4, 2, {"q_lens": [24, 9, 0, 17], "kv_lens": [500, 33, 200, 0]}),
]


@pytest.mark.parametrize("case", range(len(NARROW_CASES)))
def test_narrow_query_tiles(case):
    t_q, t_kv, batch, heads, opts = NARROW_CASES[case]
    # unsplit (the narrow layout needs one unit per CTA and no key split)
    assert batch * heads <= 148 and t_q <= 32
    rng = np.random.default_rng(900 + case)
    q, k, v = rand_qkv(rng, batch, t_q, t_kv, heads)
    got, _ = check(q, k, v, batch, t_q, t_kv, heads, f"narrow {t_q}x{t_kv} {opts}", split=False, **opts)
    if opts.get("q_lens") is not None:
        for b, n in enumerate(opts["q_lens"]):
            np.testing.assert_array_equal(got[b * t_q + n:(b + 1) * t_q], 0.0)


def test_narrow_and_wide_layouts_agree():
    """33 rows take the 128-row layout, 32 the narrow one: the first 32 rows
    of a 33-row block (FULL, no split) match the 32-row block within rounding."""
    rng = np.random.default_rng(77)
    q, k, v = rand_qkv(rng, 1, 33, 600, 2)
    wide = run(q, k, v, 1, 33, 600, 2, split=False)
    narrow = run(q[:32], k, v, 1, 32, 600, 2, split=False)
    assert_parity(narrow, wide[:32], rel_tol=1e-3, abs_tol=2e-3, what="narrow vs wide")


# ---------------------------------------------------------------------------
# band (sliding window)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("window", [1, 2, 64, 127, 128, 129, 300, 2000])
def test_band_windows(window):
    t = 517
    rng = np.random.default_rng(200 + window)
    q, k, v = rand_qkv(rng, 2, t, t, 2)
    got, ref = check(q, k, v, 2, t, t, 2, f"band w={window}", mask_kind=attn.MASK_BAND, window=window)
    if window == 1:  # each row sees only itself
        np.testing.assert_allclose(got, v.astype(np.float64), rtol=0, atol=2e-3)


@pytest.mark.parametrize("window", [1, 100, 256])
def test_band_causal(window):
    t = 400
    rng = np.random.default_rng(300 + window)
    q, k, v = rand_qkv(rng, 2, t, t, 2)
    check(q, k, v, 2, t, t, 2, f"band+causal w={window}", mask_kind=attn.MASK_BAND, window=window, causal=True)


def test_band_rectangular_and_split():
    rng = np.random.default_rng(7)
    q, k, v = rand_qkv(rng, 1, 80, 1500, 4)
    check(q, k, v, 1, 80, 1500, 4, "band 80x1500", mask_kind=attn.MASK_BAND, window=300)


# ---------------------------------------------------------------------------
# per-sequence lengths
# ---------------------------------------------------------------------------

def test_lengths_self_attention_padding_rows_are_zero():
    t = 517
    lens = [517, 300, 1, 0, 129, 128]
    rng = np.random.default_rng(11)
    q, k, v = rand_qkv(rng, len(lens), t, t, 2)
    got, _ = check(q, k, v, len(lens), t, t, 2, "lengths", q_lens=lens, kv_lens=lens)
    for b, n in enumerate(lens):
        np.testing.assert_array_equal(got[b * t + n:(b + 1) * t], 0.0)


def test_lengths_equal_truncated_sequences_run_alone():
    torch = torch_mod()
    t, lens = 300, [300, 173, 64]
    rng = np.random.default_rng(12)
    q, k, v = rand_qkv(rng, len(lens), t, t, 2)
    got = run(q, k, v, len(lens), t, t, 2, q_lens=lens, kv_lens=lens)
    for b, n in enumerate(lens):
        r = slice(b * t, b * t + n)
        alone = attn.attn_forward(to_dev(q[r]), to_dev(k[r]), to_dev(v[r]), 1, n, n, 2)
        torch.cuda.synchronize()
        assert_parity(got[r], to_np64(alone), rel_tol=2e-3, abs_tol=2e-3, what=f"length {n} vs alone")


@pytest.mark.parametrize("split", [True, False])
def test_key_lengths_only_cross_style(split):
    rng = np.random.default_rng(13)
    kv_lens = [1500, 700, 1]
    q, k, v = rand_qkv(rng, 3, 80, 1500, 2)
    check(q, k, v, 3, 80, 1500, 2, f"kv_lens split={split}", split=split, kv_lens=kv_lens)


def test_lengths_with_causal_per_sequence_offsets():
    rng = np.random.default_rng(14)
    t_q, t_kv = 32, 300
    q_lens, kv_lens = [16, 32, 5, 0], [100, 300, 5, 50]
    q, k, v = rand_qkv(rng, 4, t_q, t_kv, 2)
    check(q, k, v, 4, t_q, t_kv, 2, "lens+causal", q_lens=q_lens, kv_lens=kv_lens, causal=True)


@pytest.mark.parametrize("clen", [7, 128, 200])
def test_chunk_with_lengths(clen):
    t = 517
    lens = [517, 350, 199]
    rng = np.random.default_rng(400 + clen)
    q, k, v = rand_qkv(rng, 3, t, t, 2)
    check(q, k, v, 3, t, t, 2, f"chunk {clen} + lens", mask_kind=attn.MASK_CHUNK, chunk_len=clen,
          q_lens=lens, kv_lens=lens)


def test_lengths_out_of_range_are_clamped():
    t = 200
    rng = np.random.default_rng(15)
    q, k, v = rand_qkv(rng, 2, t, t, 2)
    got = run(q, k, v, 2, t, t, 2, q_lens=[-5, 10 ** 6], kv_lens=[10 ** 6, -1])
    ref = want(q, k, v, 2, t, t, 2, q_lens=[0, t], kv_lens=[t, 0])
    assert_parity(got, ref, what="clamped lengths")


# ---------------------------------------------------------------------------
# sinks
# ---------------------------------------------------------------------------

SINKS4 = [0.5, -1.0, 8.0, -np.inf]


@pytest.mark.parametrize("t", [1, 129, 517])
def test_sinks_full(t):
    rng = np.random.default_rng(500 + t)
    q, k, v = rand_qkv(rng, 2, t, t, 4)
    check(q, k, v, 2, t, t, 4, f"sinks t={t}", sinks=SINKS4)


@pytest.mark.parametrize("split", [True, False])
def test_sinks_split_path(split):
    rng = np.random.default_rng(16)
    q, k, v = rand_qkv(rng, 1, 80, 1500, 4)
    check(q, k, v, 1, 80, 1500, 4, f"sinks split={split}", split=split, sinks=SINKS4)


def test_sinks_with_causal_band_and_lengths():
    rng = np.random.default_rng(17)
    t_q, t_kv = 48, 400
    q, k, v = rand_qkv(rng, 3, t_q, t_kv, 4)
    check(q, k, v, 3, t_q, t_kv, 4, "sinks+band+causal+lens", mask_kind=attn.MASK_BAND, window=64, causal=True,
          q_lens=[48, 16, 0], kv_lens=[400, 100, 3], sinks=SINKS4)


def test_sink_that_takes_all_the_weight_gives_zero():
    rng = np.random.default_rng(18)
    q, k, v = rand_qkv(rng, 1, 100, 100, 2)
    got = run(q, k, v, 1, 100, 100, 2, sinks=[80.0, 0.0])
    assert np.abs(got[:, :64]).max() == 0.0
    assert_parity(got, want(q, k, v, 1, 100, 100, 2, sinks=[80.0, 0.0]), what="dominant sink")


def test_sinks_with_slotmask_verify_workload():
    torch = torch_mod()
    spec = inputs.VERIFY_WORKLOADS["verify"]
    inp = inputs.make_verify_inputs(spec)
    sinks = np.linspace(-2.0, 3.0, spec.n_heads).astype(np.float32)
    got = attn.attn_forward(to_dev(inp.q), to_dev(inp.k_cache), to_dev(inp.v_cache), 1, spec.t_q, spec.slots,
                            spec.n_heads, mask_kind=attn.MASK_SLOTMASK, bits=to_dev(inp.bits.view(np.int32)),
                            sinks=f32(sinks))
    torch.cuda.synchronize()
    allowed = oracle.allowed_from_bits(inp.bits, spec.slots)
    ref = oracle.attention(inp.q, inp.k_cache, inp.v_cache, spec.n_heads, allowed, sinks=sinks)
    assert_parity(to_np64(got), ref, what="slotmask + sinks")


# ---------------------------------------------------------------------------
# the benchmarked workloads of these options, at full size, in the bench's
# launch configuration
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["varlen8", "band8"])
def test_encoder_workload_full_size(name):
    torch = torch_mod()
    spec = inputs.ENCODER_WORKLOADS[name]
    inp = inputs.make_encoder_inputs(spec)
    lens = inputs.encoder_lengths(spec)
    d = spec.d_model
    x, w, bq, bv = (to_dev(a) for a in (inp.x, inp.w_qkv, inp.b_q, inp.b_v))
    qkv = attn.attn_qkv_pack(x, w, bq, bv)
    dl = None if lens is None else i32(lens)
    kind = attn.MASK_BAND if spec.mask == "band" else attn.MASK_FULL
    out = attn.attn_forward(qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:], spec.batch, spec.t, spec.t, spec.n_heads,
                            mask_kind=kind, window=spec.band, q_lens=dl, kv_lens=dl, split=False)
    torch.cuda.synchronize()
    ref_qkv = oracle.qkv_projection(inp.x, inp.w_qkv, inp.b_q, inp.b_v)
    ref = oracle.range_attention(ref_qkv[:, :d], ref_qkv[:, d:2 * d], ref_qkv[:, 2 * d:], spec.batch, spec.t, spec.t,
                                 spec.n_heads, q_lens=lens, kv_lens=lens, window=spec.band)
    got = to_np64(out)
    assert_parity(to_np64(qkv), ref_qkv, what=f"{name} qkv")
    assert_parity(got, ref, what=f"{name} attention")
    for b in range(spec.batch):
        n = spec.t if lens is None else int(lens[b])
        assert_parity(got[b * spec.t:b * spec.t + n], ref[b * spec.t:b * spec.t + n], what=f"{name} window {b}")
        np.testing.assert_array_equal(got[b * spec.t + n:(b + 1) * spec.t], 0.0)
    st, word = attn.debug_error_word()
    assert st == attn.ATTN_OK and word == 0


@pytest.mark.parametrize("name", ["drafter", "drafter_causal"])
def test_drafter_workload(name):
    torch = torch_mod()
    spec = inputs.DRAFTER_WORKLOADS[name]
    inp = inputs.make_drafter_inputs(spec)
    ws = attn.workspace_size(spec.beams, spec.t_q, spec.t_kv, spec.n_heads, attn.MASK_FULL)
    workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device="cuda")
    out = attn.attn_forward(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), spec.beams, spec.t_q, spec.t_kv,
                            spec.n_heads, causal=spec.causal, sinks=f32(inp.sinks), workspace=workspace)
    torch.cuda.synchronize()
    ref = oracle.range_attention(inp.q, inp.k, inp.v, spec.beams, spec.t_q, spec.t_kv, spec.n_heads,
                                 causal=spec.causal, sinks=inp.sinks)
    assert_parity(to_np64(out), ref, what=name)
    st, word = attn.debug_error_word()
    assert st == attn.ATTN_OK and word == 0


def test_many_units_without_keys_back_to_back():
    """Units whose rows see no key (all padding) are skipped by every role; a
    CTA that meets several in a row must not get a barrier phase ahead. Many
    calls over a batch full of empty and one-row sequences, then the device
    error word must still be clear."""
    torch = torch_mod()
    t, heads = 1500, 20
    lens = [0, 1, 0, 130, 0, 0, 1500, 574, 0, 1, 129, 0, 0, 0, 256, 0]
    rng = np.random.default_rng(19)
    q, k, v = rand_qkv(rng, len(lens), t, t, heads)
    dq, dk, dv, dl = to_dev(q), to_dev(k), to_dev(v), i32(lens)
    for _ in range(300):
        out = attn.attn_forward(dq, dk, dv, len(lens), t, t, heads, q_lens=dl, kv_lens=dl, split=False)
    torch.cuda.synchronize()
    st, word = attn.debug_error_word()
    assert st == attn.ATTN_OK and word == 0, f"device error word {word:#x}"
    got = to_np64(out)
    sel = [0, 1, 3, 6, 10]
    qs = np.concatenate([q[b * t:(b + 1) * t] for b in sel])
    ks = np.concatenate([k[b * t:(b + 1) * t] for b in sel])
    vs = np.concatenate([v[b * t:(b + 1) * t] for b in sel])
    ref = oracle.range_attention(qs, ks, vs, len(sel), t, t, heads, q_lens=[lens[b] for b in sel],
                                 kv_lens=[lens[b] for b in sel])
    assert_parity(np.concatenate([got[b * t:(b + 1) * t] for b in sel]), ref, what="empty-unit stress")
    for b, n in enumerate(lens):
        np.testing.assert_array_equal(got[b * t + n:(b + 1) * t], 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_drafter_projection_reuses_cached_context_rows(causal):
    """The drafter's packed projection with K/V row reuse, through the public
    entry points: each beam's packed [context + block, 3d] buffer holds the
    context rows' q/k/v from an earlier projection (computed once, reused);
    a step projects only the block's rows into their rows of the buffer and
    attends from the block's queries over every key of the buffer, with the
    causal flag and sinks. Must equal the oracle's projection of all rows
    followed by the same attention."""
    torch = torch_mod()
    rng = np.random.default_rng(41 + causal)
    beams, ctx, block, heads = 3, 150, 16, 4
    d = heads * 64
    t_kv = ctx + block
    w = inputs.random_f16(rng, (3 * d, d), 0.02)
    bq, bv = inputs.random_f16(rng, (d,), 0.01), inputs.random_f16(rng, (d,), 0.01)
    x = inputs.random_f16(rng, (beams * t_kv, d))
    sinks = rng.standard_normal(heads).astype(np.float32)
    dw, dbq, dbv, ds = to_dev(w), to_dev(bq), to_dev(bv), f32(sinks)
    cache = torch.zeros(beams * t_kv, 3 * d, dtype=torch.float16, device="cuda")
    dx = to_dev(x)
    for b in range(beams):  # context rows: projected once
        r0 = b * t_kv
        attn.attn_qkv_pack(dx[r0:r0 + ctx], dw, dbq, dbv, out=cache[r0:r0 + ctx])
    outs = []
    for b in range(beams):  # the step: the block's rows only, then attention over the whole buffer
        r0 = b * t_kv
        attn.attn_qkv_pack(dx[r0 + ctx:r0 + t_kv], dw, dbq, dbv, out=cache[r0 + ctx:r0 + t_kv])
        seq = cache[r0:r0 + t_kv]
        outs.append(attn.attn_forward(seq[ctx:, :d], seq[:, d:2 * d], seq[:, 2 * d:], 1, block, t_kv, heads,
                                      causal=causal, sinks=ds))
    torch.cuda.synchronize()
    got = np.concatenate([to_np64(o) for o in outs])
    qkv = oracle.qkv_projection(x, w, bq, bv)
    ref = []
    for b in range(beams):
        rows = qkv[b * t_kv:(b + 1) * t_kv]
        ref.append(oracle.range_attention(rows[ctx:, :d], rows[:, d:2 * d], rows[:, 2 * d:], 1, block, t_kv, heads,
                                          causal=causal, sinks=sinks))
    assert_parity(got, np.concatenate(ref), what=f"drafter step causal={causal}")
