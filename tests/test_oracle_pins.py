"""Pins for the FP64 oracle against facts fixed by the pages and by mathematics.

None of these re-types the oracle's own formula: each compares it with a closed
form, an invariant the pages state, or a brute-force pure-Python loop on tiny
inputs, chosen so that a dropped term, a wrong sign or index, a transposed
operand, a wrong scale or a wrong mask bit order fails at least one test.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
from speech_encoder_attention_b200 import inputs

SCALE = 0.125  # 1/sqrt(64)


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# packed QKV projection
# ---------------------------------------------------------------------------

def test_qkv_bruteforce_loops():
    rng = _rng(1)
    d, rows = 4, 3
    x = rng.standard_normal((rows, d))
    w = rng.standard_normal((3 * d, d))
    bq = rng.standard_normal(d)
    bv = rng.standard_normal(d)
    got = oracle.qkv_projection(x, w, bq, bv)
    for r in range(rows):
        for j in range(3 * d):
            acc = 0.0
            for c in range(d):
                acc += x[r][c] * w[j][c]
            if j < d:
                acc += bq[j]
            elif j >= 2 * d:
                acc += bv[j - 2 * d]
            assert got[r, j] == pytest.approx(acc, abs=1e-12)


def test_qkv_identity_rows_pick_weight_columns():
    rng = _rng(2)
    d = 8
    w = rng.standard_normal((3 * d, d))
    bq, bv = rng.standard_normal(d), rng.standard_normal(d)
    got = oracle.qkv_projection(np.eye(d), w, bq, bv)
    bias = np.concatenate([bq, np.zeros(d), bv])
    for c in range(d):
        np.testing.assert_allclose(got[c], w[:, c] + bias, rtol=0, atol=1e-14)


def test_qkv_bias_split_k_has_no_bias():
    d = 6
    bq = np.arange(1, d + 1, dtype=np.float64)
    bv = -np.arange(1, d + 1, dtype=np.float64)
    got = oracle.qkv_projection(np.zeros((2, d)), np.ones((3 * d, d)), bq, bv)
    np.testing.assert_array_equal(got[:, :d], np.tile(bq, (2, 1)))
    np.testing.assert_array_equal(got[:, d:2 * d], 0.0)
    np.testing.assert_array_equal(got[:, 2 * d:], np.tile(bv, (2, 1)))


# ---------------------------------------------------------------------------
# softmax attention: closed forms
# ---------------------------------------------------------------------------

def test_softmax_rows_sum_to_one():
    rng = _rng(3)
    t_q, t_kv = 9, 37
    q, k, v = (rng.standard_normal((t, 64)) for t in (t_q, t_kv, t_kv))
    allowed = rng.random((t_q, t_kv)) < 0.4
    allowed[0] = False
    _, st = oracle.attention(q, k, v, 1, allowed, return_stats=True)
    p = st[0]["p"]
    sums = p.sum(axis=1)
    nonempty = allowed.any(axis=1)
    np.testing.assert_allclose(sums[nonempty] / st[0]["l"][nonempty], 1.0, atol=1e-15)
    assert np.all(p[~allowed] == 0.0)
    # the max-shifted weights peak at exactly 1 on every nonempty row
    np.testing.assert_array_equal(p[nonempty].max(axis=1), 1.0)


def test_two_keys_tanh_closed_form():
    """With two keys, softmax-weighted averaging is a logistic blend:
    o = (v0 + v1)/2 + (v0 - v1)/2 * tanh((s0 - s1)/2), s = <q,k>/8."""
    rng = _rng(4)
    for _ in range(20):
        q = rng.standard_normal((1, 64)) * 2
        k = rng.standard_normal((2, 64))
        v = rng.standard_normal((2, 64))
        s0, s1 = (q[0] @ k[0]) / 8.0, (q[0] @ k[1]) / 8.0
        want = (v[0] + v[1]) / 2 + (v[0] - v[1]) / 2 * math.tanh((s0 - s1) / 2)
        got = oracle.attention(q, k, v, 1, np.ones((1, 2), bool))
        np.testing.assert_allclose(got[0], want, rtol=1e-12, atol=1e-13)


def test_constant_values_return_the_constant():
    rng = _rng(5)
    t = 23
    q, k = rng.standard_normal((t, 128)), rng.standard_normal((t, 128))
    c = rng.standard_normal(128)
    v = np.tile(c, (t, 1))
    for allowed in (oracle.allowed_full(t, t), oracle.allowed_chunk(t, 5)):
        got = oracle.attention(q, k, v, 2, allowed)
        np.testing.assert_allclose(got, np.tile(c, (t, 1)), rtol=1e-13, atol=1e-14)


def test_encoder_constant_v_through_projection():
    """W_v = 0 and b_v = c make every value row equal c, so every output row is c."""
    spec = inputs.EncoderSpec("t", 2, 33, 128, 2, "full", 0, 11)
    inp = inputs.make_encoder_inputs(spec)
    w = inp.w_qkv.copy()
    w[256:] = 0
    c = np.linspace(-1, 1, 128).astype(np.float16)
    out = oracle.encoder_attention(inp.x, w, inp.b_q, c, 2, 33, 2)
    np.testing.assert_allclose(out, np.tile(c.astype(np.float64), (66, 1)), rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("mode", ["full", "chunk", "slotmask"])
def test_zero_queries_give_uniform_mean(mode):
    """q = 0 makes every allowed score equal, so each row is the plain mean of
    the allowed value rows."""
    rng = _rng(6)
    t = 19
    k, v = rng.standard_normal((t, 64)), rng.standard_normal((t, 64))
    q = np.zeros((t, 64))
    if mode == "full":
        allowed = oracle.allowed_full(t, t)
    elif mode == "chunk":
        allowed = oracle.allowed_chunk(t, 4)
    else:
        allowed = rng.random((t, t)) < 0.5
        allowed[np.arange(t), np.arange(t)] = True
    got = oracle.attention(q, k, v, 1, allowed)
    for i in range(t):
        np.testing.assert_allclose(got[i], v[allowed[i]].mean(axis=0), rtol=1e-12, atol=1e-13)


def test_scale_and_sign_pinned_by_one_hot_keys():
    """q = a*e0, k_j = b_j*e0: weights are softmax(a*b_j/8); compare against a
    hand-evaluated two-point softmax."""
    a = 4.0
    b = np.array([1.0, -2.0])
    q = np.zeros((1, 64)); q[0, 0] = a
    k = np.zeros((2, 64)); k[:, 0] = b
    v = np.zeros((2, 64)); v[0, 1] = 1.0; v[1, 1] = 0.0
    got = oracle.attention(q, k, v, 1, np.ones((1, 2), bool))
    # weight of key 0 = 1 / (1 + exp(a*(b1-b0)/8)) = 1 / (1 + exp(-1.5))
    assert got[0, 1] == pytest.approx(1.0 / (1.0 + math.exp(-1.5)), rel=1e-14)


def test_large_logits_stay_finite():
    rng = _rng(7)
    q = rng.standard_normal((4, 64)) * 300
    k = rng.standard_normal((6, 64)) * 300
    v = rng.standard_normal((6, 64))
    got = oracle.attention(q, k, v, 1, np.ones((4, 6), bool))
    assert np.isfinite(got).all()
    # with logits this far apart each row collapses onto its best key
    s = q @ k.T
    np.testing.assert_allclose(got, v[s.argmax(axis=1)], atol=1e-9)


# ---------------------------------------------------------------------------
# FULL: bidirectional, permutation equivariant
# ---------------------------------------------------------------------------

def test_full_is_permutation_equivariant():
    spec = inputs.EncoderSpec("t", 1, 41, 128, 2, "full", 0, 12)
    inp = inputs.make_encoder_inputs(spec)
    perm = _rng(8).permutation(41)
    a = oracle.encoder_attention(inp.x, inp.w_qkv, inp.b_q, inp.b_v, 1, 41, 2)
    b = oracle.encoder_attention(inp.x[perm], inp.w_qkv, inp.b_q, inp.b_v, 1, 41, 2)
    np.testing.assert_allclose(b, a[perm], rtol=1e-12, atol=1e-14)


def test_single_frame_returns_its_value():
    rng = _rng(9)
    q, k, v = (rng.standard_normal((1, 128)) for _ in range(3))
    np.testing.assert_allclose(oracle.attention(q, k, v, 2, np.ones((1, 1), bool)), v, rtol=1e-15)


def test_full_is_bidirectional_future_frames_matter():
    """Changing the last frame's key/value changes the first frame's output."""
    rng = _rng(10)
    t = 8
    q, k, v = (rng.standard_normal((t, 64)) for _ in range(3))
    a = oracle.attention(q, k, v, 1, oracle.allowed_full(t, t))
    v2 = v.copy(); v2[-1] += 1.0
    b = oracle.attention(q, k, v2, 1, oracle.allowed_full(t, t))
    assert np.abs(a[0] - b[0]).max() > 1e-3


# ---------------------------------------------------------------------------
# CHUNK: each chunk an independent sequence
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("t,clen", [(2325 // 25, 8), (50, 7), (64, 64), (65, 64), (31, 1)])
def test_chunk_equals_independent_sequences(t, clen):
    rng = _rng(11)
    q, k, v = (rng.standard_normal((t, 128)) for _ in range(3))
    got = oracle.attention(q, k, v, 2, oracle.allowed_chunk(t, clen))
    for c0 in range(0, t, clen):
        sl = slice(c0, min(c0 + clen, t))
        n = sl.stop - sl.start
        want = oracle.attention(q[sl], k[sl], v[sl], 2, oracle.allowed_full(n, n))
        np.testing.assert_allclose(got[sl], want, rtol=1e-12, atol=1e-14)


def test_chunk_len_one_returns_values_and_long_chunk_is_full():
    rng = _rng(12)
    t = 17
    q, k, v = (rng.standard_normal((t, 64)) for _ in range(3))
    np.testing.assert_allclose(oracle.attention(q, k, v, 1, oracle.allowed_chunk(t, 1)), v, rtol=1e-15)
    full = oracle.attention(q, k, v, 1, oracle.allowed_full(t, t))
    for clen in (t, t + 1, 1000):
        np.testing.assert_array_equal(oracle.attention(q, k, v, 1, oracle.allowed_chunk(t, clen)), full)


def _window_rows_bruteforce(qkv, rows, n_heads, d):
    """Pure-Python attention of the frames `rows` (global row indices) among
    themselves only, from a packed qkv matrix: the definition of one window (or
    one chunk) encoded on its own."""
    q = [qkv[r, :d].tolist() for r in rows]
    k = [qkv[r, d:2 * d].tolist() for r in rows]
    v = [qkv[r, 2 * d:].tolist() for r in rows]
    return _brute_force(q, k, v, [list(range(len(rows)))] * len(rows), n_heads)


def test_encoder_windows_attend_only_within_themselves():
    """Each window of a batch is its own bidirectional sequence: the batched
    encoder path equals, window by window, brute-force attention over that
    window's frames alone (windows carry different offsets, so a window that
    saw another window's keys would differ)."""
    batch, t, d, heads = 3, 13, 128, 2
    spec = inputs.EncoderSpec("t", batch, t, d, heads, "full", 0, 21, True)
    inp = inputs.make_encoder_inputs(spec)
    got = oracle.encoder_attention(inp.x, inp.w_qkv, inp.b_q, inp.b_v, batch, t, heads)
    qkv = oracle.qkv_projection(inp.x, inp.w_qkv, inp.b_q, inp.b_v)
    for b in range(batch):
        rows = list(range(b * t, (b + 1) * t))
        want = _window_rows_bruteforce(qkv, rows, heads, d)
        np.testing.assert_allclose(got[b * t:(b + 1) * t], want, rtol=1e-12, atol=1e-13)
    # the same frames run as one long sequence give a different answer
    whole = _window_rows_bruteforce(qkv, list(range(t)) + list(range(t, 2 * t)), heads, d)
    assert np.abs(whole[:t] - got[:t]).max() > 1e-4


def test_encoder_chunk_mode_equals_independent_chunks():
    """CHUNK(len) through the batched encoder path: every chunk of every window
    (chunks restart at each window's frame 0, the last one short) equals
    brute-force attention over that chunk's frames alone."""
    batch, t, clen, d, heads = 2, 12, 5, 128, 2
    spec = inputs.EncoderSpec("t", batch, t, d, heads, "chunk", clen, 22, True)
    inp = inputs.make_encoder_inputs(spec)
    got = oracle.encoder_attention(inp.x, inp.w_qkv, inp.b_q, inp.b_v, batch, t, heads,
                                   mask="chunk", chunk_len=clen)
    qkv = oracle.qkv_projection(inp.x, inp.w_qkv, inp.b_q, inp.b_v)
    spans = []
    for b in range(batch):
        for c0 in range(0, t, clen):
            spans.append(list(range(b * t + c0, b * t + min(c0 + clen, t))))
    assert [len(s) for s in spans] == [5, 5, 2, 5, 5, 2]
    for rows in spans:
        want = _window_rows_bruteforce(qkv, rows, heads, d)
        np.testing.assert_allclose(got[rows], want, rtol=1e-12, atol=1e-13)
    full = oracle.encoder_attention(inp.x, inp.w_qkv, inp.b_q, inp.b_v, batch, t, heads)
    assert np.abs(full - got).max() > 1e-4


def test_chunk_boundaries_by_hand():
    a = oracle.allowed_chunk(7, 3)
    want = np.array([[1, 1, 1, 0, 0, 0, 0],
                     [1, 1, 1, 0, 0, 0, 0],
                     [1, 1, 1, 0, 0, 0, 0],
                     [0, 0, 0, 1, 1, 1, 0],
                     [0, 0, 0, 1, 1, 1, 0],
                     [0, 0, 0, 1, 1, 1, 0],
                     [0, 0, 0, 0, 0, 0, 1]], dtype=bool)
    np.testing.assert_array_equal(a, want)


# ---------------------------------------------------------------------------
# SLOTMASK: brute force over exactly the allowed slots
# ---------------------------------------------------------------------------

def _brute_force(q, k, v, allowed_lists, n_heads, dh=64):
    """Pure-Python loops: for each row and head, softmax over the listed slots."""
    out = [[0.0] * (n_heads * dh) for _ in range(len(q))]
    for i in range(len(q)):
        slots = allowed_lists[i]
        if not slots:
            continue
        for h in range(n_heads):
            base = h * dh
            scores = []
            for j in slots:
                dot = 0.0
                for e in range(dh):
                    dot += q[i][base + e] * k[j][base + e]
                scores.append(dot / math.sqrt(dh))
            top = max(scores)
            w = [math.exp(s - top) for s in scores]
            tot = sum(w)
            for e in range(dh):
                acc = 0.0
                for wj, j in zip(w, slots):
                    acc += wj * v[j][base + e]
                out[i][base + e] = acc / tot
    return np.array(out)


def test_slotmask_every_pattern_one_row_eight_slots():
    rng = _rng(13)
    q = rng.standard_normal((1, 64))
    k = rng.standard_normal((8, 64))
    v = rng.standard_normal((8, 64))
    for pattern in range(256):
        bits = np.array([[pattern]], dtype=np.uint32)
        got = oracle.slotmask_attention(q, k, v, bits, 1)
        slots = [j for j in range(8) if (pattern >> j) & 1]
        want = _brute_force(q.tolist(), k.tolist(), v.tolist(), [slots], 1)
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


def test_slotmask_random_multiword_bruteforce():
    rng = _rng(14)
    rows, slots, heads = 6, 45, 2
    q = rng.standard_normal((rows, 64 * heads))
    k = rng.standard_normal((slots, 64 * heads))
    v = rng.standard_normal((slots, 64 * heads))
    allowed = rng.random((rows, slots)) < 0.3
    allowed[2] = False
    allowed[3, 33] = True  # a bit in the second word
    bits = inputs.pack_bits(allowed)
    assert bits.shape == (rows, 2)
    got = oracle.slotmask_attention(q, k, v, bits, heads)
    lists = [[j for j in range(slots) if allowed[i, j]] for i in range(rows)]
    want = _brute_force(q.tolist(), k.tolist(), v.tolist(), lists, heads)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(got[2], 0.0)


def test_slotmask_special_cases():
    rng = _rng(15)
    slots = 40
    q = rng.standard_normal((3, 64))
    k, v = rng.standard_normal((slots, 64)), rng.standard_normal((slots, 64))
    for j in (0, 5, 31, 32, 39):
        bits = inputs.pack_bits(np.eye(slots, dtype=bool)[[j] * 3])
        np.testing.assert_allclose(oracle.slotmask_attention(q, k, v, bits, 1), np.tile(v[j], (3, 1)), rtol=1e-15)
    ones = inputs.pack_bits(np.ones((3, slots), bool))
    np.testing.assert_array_equal(oracle.slotmask_attention(q, k, v, ones, 1),
                                  oracle.attention(q, k, v, 1, oracle.allowed_full(3, slots)))


def test_bit_order_is_lsb_first():
    bits = np.array([[0b101, 1 << 1]], dtype=np.uint32)
    got = oracle.allowed_from_bits(bits, 40)
    want = np.zeros(40, bool); want[[0, 2, 33]] = True
    np.testing.assert_array_equal(got[0], want)


# ---------------------------------------------------------------------------
# cross-attention: t_q != t_kv, heads independent
# ---------------------------------------------------------------------------

def test_cross_attention_bruteforce_rectangular():
    rng = _rng(16)
    t_q, t_kv, heads = 3, 5, 2
    q = rng.standard_normal((t_q, 64 * heads))
    k = rng.standard_normal((t_kv, 64 * heads))
    v = rng.standard_normal((t_kv, 64 * heads))
    got = oracle.cross_attention(q, k, v, heads)
    want = _brute_force(q.tolist(), k.tolist(), v.tolist(), [list(range(t_kv))] * t_q, heads)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


def test_heads_do_not_mix():
    rng = _rng(17)
    t = 10
    q, k, v = (rng.standard_normal((t, 128)) for _ in range(3))
    a = oracle.attention(q, k, v, 2, oracle.allowed_full(t, t))
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[:, 64:] = rng.standard_normal((t, 64))
    k2[:, 64:] = rng.standard_normal((t, 64))
    v2[:, 64:] = rng.standard_normal((t, 64))
    b = oracle.attention(q2, k2, v2, 2, oracle.allowed_full(t, t))
    np.testing.assert_array_equal(a[:, :64], b[:, :64])
    assert np.abs(a[:, 64:] - b[:, 64:]).max() > 1e-3


# ---------------------------------------------------------------------------
# range family: per-sequence lengths, causal, band (hand-written patterns)
# ---------------------------------------------------------------------------

def _m(rows):
    return np.array(rows, dtype=bool)


def test_range_masks_by_hand():
    # causal, square: keys up to and including the row itself
    np.testing.assert_array_equal(oracle.allowed_range(4, 4, causal=True),
                                  _m([[1, 0, 0, 0], [1, 1, 0, 0], [1, 1, 1, 0], [1, 1, 1, 1]]))
    # causal, 2 queries at the end of 5 keys: positions 3 and 4
    np.testing.assert_array_equal(oracle.allowed_range(2, 5, causal=True),
                                  _m([[1, 1, 1, 1, 0], [1, 1, 1, 1, 1]]))
    # band of window 2: |i - j| < 2
    np.testing.assert_array_equal(oracle.allowed_range(5, 5, window=2),
                                  _m([[1, 1, 0, 0, 0], [1, 1, 1, 0, 0], [0, 1, 1, 1, 0],
                                      [0, 0, 1, 1, 1], [0, 0, 0, 1, 1]]))
    # band + causal: the row itself and the one before it
    np.testing.assert_array_equal(oracle.allowed_range(5, 5, window=2, causal=True),
                                  _m([[1, 0, 0, 0, 0], [1, 1, 0, 0, 0], [0, 1, 1, 0, 0],
                                      [0, 0, 1, 1, 0], [0, 0, 0, 1, 1]]))
    # lengths: 2 valid query rows, 3 valid keys of a 4-frame buffer
    np.testing.assert_array_equal(oracle.allowed_range(4, 4, q_len=2, kv_len=3),
                                  _m([[1, 1, 1, 0], [1, 1, 1, 0], [0, 0, 0, 0], [0, 0, 0, 0]]))
    # causal with lengths: the 2 queries are positions 1 and 2 of 3 keys
    np.testing.assert_array_equal(oracle.allowed_range(4, 4, q_len=2, kv_len=3, causal=True),
                                  _m([[1, 1, 0, 0], [1, 1, 1, 0], [0, 0, 0, 0], [0, 0, 0, 0]]))
    # chunks of 3 with the 2 queries at positions 4 and 5 of 6 keys: chunk 1
    np.testing.assert_array_equal(oracle.allowed_range(2, 6, chunk_len=3),
                                  _m([[0, 0, 0, 1, 1, 1], [0, 0, 0, 1, 1, 1]]))
    # more queries than keys: positions -1 and 0; causal leaves row 0 empty
    np.testing.assert_array_equal(oracle.allowed_range(2, 1, causal=True), _m([[0], [1]]))


def test_range_special_cases_reduce_to_known_masks():
    t = 7
    np.testing.assert_array_equal(oracle.allowed_range(t, t), oracle.allowed_full(t, t))
    np.testing.assert_array_equal(oracle.allowed_range(t, t, window=t), oracle.allowed_full(t, t))
    np.testing.assert_array_equal(oracle.allowed_range(t, t, window=1), np.eye(t, dtype=bool))
    np.testing.assert_array_equal(oracle.allowed_range(t, t, chunk_len=3), oracle.allowed_chunk(t, 3))
    np.testing.assert_array_equal(oracle.allowed_range(t, t, causal=True, window=t),
                                  np.tril(np.ones((t, t), bool)))


def test_zero_queries_give_prefix_window_and_length_means():
    rng = _rng(21)
    t = 9
    v = rng.standard_normal((t, 64))
    q = np.zeros((t, 64))
    k = rng.standard_normal((t, 64))
    causal = oracle.range_attention(q, k, v, 1, t, t, 1, causal=True)
    for i in range(t):
        np.testing.assert_allclose(causal[i], v[: i + 1].mean(axis=0), rtol=1e-13, atol=1e-15)
    band = oracle.range_attention(q, k, v, 1, t, t, 1, window=3)
    for i in range(t):
        np.testing.assert_allclose(band[i], v[max(0, i - 2): i + 3].mean(axis=0), rtol=1e-13, atol=1e-15)
    lens = oracle.range_attention(q, k, v, 1, t, t, 1, q_lens=[5], kv_lens=[4])
    for i in range(5):
        np.testing.assert_allclose(lens[i], v[:4].mean(axis=0), rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(lens[5:], 0.0)


def test_lengths_equal_the_truncated_sequences():
    """Masking the padding must give what the shortened sequence gives alone
    (a valid frame never attends to the padding)."""
    rng = _rng(22)
    t, heads, lens = 12, 2, [12, 7, 1, 0]
    q, k, v = (rng.standard_normal((len(lens) * t, 64 * heads)) for _ in range(3))
    got = oracle.range_attention(q, k, v, len(lens), t, t, heads, q_lens=lens, kv_lens=lens)
    for b, n in enumerate(lens):
        r = slice(b * t, b * t + n)
        if n:
            want = oracle.attention(q[r], k[r], v[r], heads, oracle.allowed_full(n, n))
            np.testing.assert_allclose(got[r], want, rtol=1e-13, atol=1e-15)
        np.testing.assert_array_equal(got[b * t + n:(b + 1) * t], 0.0)


def test_range_bruteforce_causal_band_lengths():
    rng = _rng(23)
    t_q, t_kv, heads = 5, 8, 2
    q = rng.standard_normal((t_q, 64 * heads))
    k = rng.standard_normal((t_kv, 64 * heads))
    v = rng.standard_normal((t_kv, 64 * heads))
    # q_len 4, kv_len 7: positions 3, 4, 5, 6; causal band of 3 -> keys p-2 .. p
    lists = [[1, 2, 3], [2, 3, 4], [3, 4, 5], [4, 5, 6], []]
    got = oracle.range_attention(q, k, v, 1, t_q, t_kv, heads, q_lens=[4], kv_lens=[7], window=3, causal=True)
    want = _brute_force(q.tolist(), k.tolist(), v.tolist(), lists, heads)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# attention sinks
# ---------------------------------------------------------------------------

def test_sink_two_keys_closed_form():
    s0, s1, sigma = 0.75, -1.25, 0.5
    q = np.zeros((1, 64)); q[0, 0] = 8.0  # scale 1/8: scores equal k[:, 0]
    k = np.zeros((2, 64)); k[0, 0], k[1, 0] = s0, s1
    v = np.zeros((2, 64)); v[0, 1], v[1, 1] = 3.0, -2.0
    got = oracle.attention(q, k, v, 1, oracle.allowed_full(1, 2), sinks=np.array([sigma]))
    den = math.exp(sigma) + math.exp(s0) + math.exp(s1)
    assert got[0, 1] == pytest.approx((3.0 * math.exp(s0) - 2.0 * math.exp(s1)) / den, rel=1e-14)
    np.testing.assert_array_equal(np.delete(got[0], 1), 0.0)


def test_sink_minus_inf_is_no_sink_and_zero_queries_close_form():
    rng = _rng(24)
    t, heads = 6, 2
    q, k, v = (rng.standard_normal((t, 64 * heads)) for _ in range(3))
    a = oracle.allowed_range(t, t, causal=True)
    np.testing.assert_allclose(oracle.attention(q, k, v, heads, a, sinks=np.array([-np.inf, -np.inf])),
                               oracle.attention(q, k, v, heads, a), rtol=1e-14, atol=1e-16)
    sig = np.array([0.3, -2.0])
    got = oracle.attention(np.zeros_like(q), k, v, heads, a, sinks=sig)
    for i in range(t):
        for h in range(heads):
            cols = slice(64 * h, 64 * h + 64)
            want = v[: i + 1, cols].sum(axis=0) / (math.exp(sig[h]) + i + 1)
            np.testing.assert_allclose(got[i, cols], want, rtol=1e-13, atol=1e-15)


def test_sink_edge_cases():
    rng = _rng(25)
    t = 5
    q, k, v = (rng.standard_normal((t, 128)) for _ in range(3))
    a = oracle.allowed_full(t, t)
    a[2] = False
    big = oracle.attention(q, k, v, 2, a, sinks=np.array([60.0, 0.0]))
    assert np.abs(big[:, :64]).max() < 1e-15   # the sink takes almost all the weight
    np.testing.assert_array_equal(big[2], 0.0)  # empty row stays zero
    # changing head 1's sink leaves head 0 exactly as it was
    other = oracle.attention(q, k, v, 2, a, sinks=np.array([60.0, -5.0]))
    np.testing.assert_array_equal(big[:, :64], other[:, :64])
    assert np.abs(big[:, 64:] - other[:, 64:]).max() > 1e-3


# ---------------------------------------------------------------------------
# Q8_0 weights: 34-byte blocks, little-endian fp16 scale then 32 signed bytes
# ---------------------------------------------------------------------------

def test_q8_0_one_block_by_hand():
    # scale 0.5 is fp16 0x3800 -> bytes 00 38; q = 1, -2, 3, 127, -128, 0, ...
    block = bytes([0x00, 0x38, 0x01, 0xFE, 0x03, 0x7F, 0x80] + [0] * 27)
    assert len(block) == 34
    w = oracle.dequantize_q8_0(np.frombuffer(block, dtype=np.uint8)[None, :], 32)
    want = [0.5, -1.0, 1.5, 63.5, -64.0] + [0.0] * 27
    np.testing.assert_array_equal(w[0], want)


def test_q8_0_block_boundaries_and_rows_by_hand():
    # row 0: block 0 scale 1.0 (0x3C00), all q = 2; block 1 scale -0.25 (0xB400), all q = -4
    # row 1: block 0 scale 2.0 (0x4000), q[t] = t; block 1 scale 0 -> zeros
    r0 = bytes([0x00, 0x3C] + [2] * 32 + [0x00, 0xB4] + [0xFC] * 32)
    r1 = bytes([0x00, 0x40] + list(range(32)) + [0x00, 0x00] + [0x55] * 32)
    w = oracle.dequantize_q8_0(np.frombuffer(r0 + r1, dtype=np.uint8).reshape(2, 68), 64)
    np.testing.assert_array_equal(w[0, :32], 2.0)
    np.testing.assert_array_equal(w[0, 32:], 1.0)      # -0.25 * -4
    np.testing.assert_array_equal(w[1, :32], 2.0 * np.arange(32))
    np.testing.assert_array_equal(w[1, 32:], 0.0)


def test_q8_0_projection_bruteforce_over_bytes():
    import struct
    spec = inputs.Q8Spec("pin", 3, 64, 31)
    inp = inputs.make_q8_inputs(spec)
    d = 64
    got = oracle.qkv_projection_q8_0(inp.x, inp.w_blocks, inp.b_q, inp.b_v)
    raw = inp.w_blocks
    for r in range(3):
        for j in range(3 * d):
            acc = 0.0
            for c in range(d):
                blk = raw[j, (c // 32) * 34:(c // 32) * 34 + 34].tobytes()
                scale = struct.unpack("<e", blk[:2])[0]
                q = blk[2 + c % 32]
                q = q - 256 if q > 127 else q
                acc += float(inp.x[r, c]) * scale * q
            if j < d:
                acc += float(inp.b_q[j])
            elif j >= 2 * d:
                acc += float(inp.b_v[j - 2 * d])
            assert got[r, j] == pytest.approx(acc, rel=1e-12, abs=1e-12)
