"""FP64 CPU oracle for the Whisper-style attention pass.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The CUDA library never calls it and shares no code with it.

What it computes is the plain definition, step by step, in float64 with no
blocking, fusion or reordering beyond what the definition states. NumPy's
matmul serves as the library primitive for the dot products.

* Packed QKV projection -- the edda PR ("Add Edda ASR with DFlash2 speculative
  decoding", PR description and the commit note on the encoder) replaces three
  projections by one packed one. With the packed weight W (q rows, then k rows,
  then v rows): qkv[r, j] = sum_c x[r, c] * W[j, c] + bias[j], where bias is b_q
  on the q third, 0 on the k third (Whisper's key projection has no bias) and
  b_v on the v third.
* Scaled-dot-product attention with a per-row allowed set A_i. The PR's flash
  path gives the same transcripts as the path that materialises the scores, so
  the oracle materialises them: s_ij = scale * <q_i, k_j>, m_i = max over A_i,
  p_ij = exp(s_ij - m_i) on A_i and 0 elsewhere, l_i = sum_j p_ij,
  o_i = sum_j p_ij v_j / l_i. A row whose allowed set is empty yields 0 (the
  pages are silent on that case; zero is the reading taken).
* Allowed sets: FULL = every key (the Whisper encoder is fully bidirectional:
  BuzzASR "danish" discussion #1, the reply on the padded region); CHUNK(len) =
  keys in the same len-frame chunk of the same sequence (higgs-audio-v3-stt model
  card, "Architecture note (chunked encoder)": each chunk is encoded on its own
  with within-chunk attention); SLOTMASK = the explicit per-row bitmask of a
  token tree over a position-indexed cache (edda PR description: each beam's
  mask row admits only its ancestors; block verification over KV slots indexed
  by position).

* Range family with per-sequence lengths, a causal flag and a band (the
  drafter page, "Add causal attention and attention sinks to DFlash" PR text
  and diff: the draft block's internal attention is non-causal unless the model
  says causal; an optional sliding window; the higgs model card: valid frames
  must not attend to silence padding; BuzzASR discussion: a shortened
  500-position encoder input). Readings where the pages are silent: query row i
  of a sequence with q_len valid rows and kv_len valid keys sits at key position
  p_i = i + (kv_len - q_len) (the query block is the last q_len positions);
  rows i >= q_len are padding and yield 0; keys j >= kv_len are never allowed;
  causal keeps j <= p_i; a band of window w keeps |p_i - j| < w; CHUNK keeps
  floor(p_i / len) == floor(j / len).
* Attention sinks (same PR: optional per-head "attn_sinks" passed to the
  attention). Reading: a sink is one extra logit sigma_h per head, in the units
  of the scaled scores, that joins the softmax normalisation and carries no
  value vector: o_i = sum_j e^{s_ij} v_j / (e^{sigma_h} + sum_j e^{s_ij}).
  sigma = -inf is no sink. A row with no allowed key yields 0.

* Q8_0 weights for the projection (edda PR, results table: "Q8_0 decoder").
  The pages name the GGUF Q8_0 type without defining it; the reading taken is
  its published layout: each weight row is a run of 34-byte blocks, a
  little-endian fp16 scale d followed by 32 signed bytes q, and block b of
  row j holds W[j, 32b + t] = d * q[t]. The projection is then the packed one
  above with that W, dequantized exactly (a float64 product).

Inputs arrive as fp16 arrays and are widened to float64 exactly. Nothing is
rounded in between; the output stays float64.
"""
from __future__ import annotations

import numpy as np

HEAD_DIM = 64


def _f64(a: np.ndarray) -> np.ndarray:
    return np.asarray(a).astype(np.float64)


def packed_bias(b_q: np.ndarray, b_v: np.ndarray) -> np.ndarray:
    """The 3d-long bias of the packed projection: [b_q | 0 | b_v]."""
    b_q = _f64(b_q)
    return np.concatenate([b_q, np.zeros_like(b_q), _f64(b_v)])


def qkv_projection(x: np.ndarray, w_qkv: np.ndarray, b_q: np.ndarray, b_v: np.ndarray) -> np.ndarray:
    """qkv = x . W^T + [b_q | 0 | b_v] in float64.  x [rows, d], W [3d, d] -> [rows, 3d]."""
    return _f64(x) @ _f64(w_qkv).T + packed_bias(b_q, b_v)


Q8_0_BLOCK = 32          # weights per block
Q8_0_BLOCK_BYTES = 34    # fp16 scale + 32 int8


def dequantize_q8_0(blocks: np.ndarray, cols: int) -> np.ndarray:
    """Q8_0 rows (uint8 [rows, cols / 32 * 34]) -> float64 weights [rows, cols]:
    per block, the fp16 scale times each signed byte."""
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    rows = blocks.shape[0]
    nb = cols // Q8_0_BLOCK
    if cols % Q8_0_BLOCK or blocks.shape[1] != nb * Q8_0_BLOCK_BYTES:
        raise ValueError("expected [rows, cols/32 * 34] bytes with cols a multiple of 32")
    b = blocks.reshape(rows, nb, Q8_0_BLOCK_BYTES)
    d = b[:, :, :2].copy().view("<f2").astype(np.float64)          # [rows, nb, 1]
    q = b[:, :, 2:].copy().view(np.int8).astype(np.float64)        # [rows, nb, 32]
    return (d * q).reshape(rows, cols)


def qkv_projection_q8_0(x: np.ndarray, w_blocks: np.ndarray, b_q: np.ndarray, b_v: np.ndarray) -> np.ndarray:
    """The packed projection with Q8_0 weights: x . W^T + [b_q | 0 | b_v], W
    dequantized exactly from its blocks. x [rows, d], blocks [3d, d/32 * 34]."""
    d = np.asarray(x).shape[1]
    return qkv_projection(x, dequantize_q8_0(w_blocks, d), b_q, b_v)


# ----------------------------------------------------------------------------
# allowed sets
# ----------------------------------------------------------------------------

def allowed_full(t_q: int, t_kv: int) -> np.ndarray:
    return np.ones((t_q, t_kv), dtype=bool)


def allowed_chunk(t: int, chunk_len: int) -> np.ndarray:
    """allowed(i, j) <=> floor(i / len) == floor(j / len), frames counted from the
    start of the sequence; the last chunk may be short."""
    if chunk_len <= 0:
        raise ValueError("chunk_len must be positive")
    c = np.arange(t) // chunk_len
    return c[:, None] == c[None, :]


def allowed_from_bits(bits: np.ndarray, t_kv: int) -> np.ndarray:
    """allowed(i, j) <=> bit (j % 32) of word (j // 32) of row i is set."""
    bits = np.asarray(bits, dtype=np.uint32)
    j = np.arange(t_kv)
    return ((bits[:, j // 32] >> (j % 32).astype(np.uint32)) & 1).astype(bool)


def allowed_range(t_q: int, t_kv: int, *, q_len: int | None = None, kv_len: int | None = None,
                  chunk_len: int = 0, window: int = 0, causal: bool = False) -> np.ndarray:
    """Allowed set of the range family for one sequence, element by element
    from the definitions in the module docstring: valid query row (i < q_len),
    valid key (j < kv_len), and each requested condition on the query position
    p_i = i + (kv_len - q_len)."""
    q_len = t_q if q_len is None else q_len
    kv_len = t_kv if kv_len is None else kv_len
    i = np.arange(t_q)[:, None]
    j = np.arange(t_kv)[None, :]
    pos = i + (kv_len - q_len)
    a = (i < q_len) & (j < kv_len)
    if chunk_len:
        if chunk_len < 0:
            raise ValueError("chunk_len must be positive")
        a &= np.floor_divide(pos, chunk_len) == j // chunk_len
    if causal:
        a &= j <= pos
    if window:
        if window < 0:
            raise ValueError("window must be positive")
        a &= np.abs(pos - j) < window
    return a


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------

def attention_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, allowed: np.ndarray,
                   scale: float, return_stats: bool = False, sink: float | None = None):
    """One head: q [t_q, dh], k/v [t_kv, dh] (float64), allowed [t_q, t_kv].
    sink: optional extra logit of the normalisation (no value vector)."""
    if sink is not None:
        return _attention_head_sink(q, k, v, allowed, scale, float(sink))
    s = scale * (q @ k.T)
    s_masked = np.where(allowed, s, -np.inf)
    nonempty = allowed.any(axis=1)
    m = np.where(nonempty, s_masked.max(axis=1), 0.0)
    p = np.where(allowed, np.exp(s_masked - m[:, None]), 0.0)
    l = p.sum(axis=1)
    o = np.zeros((q.shape[0], v.shape[1]), dtype=np.float64)
    o[nonempty] = (p[nonempty] @ v) / l[nonempty, None]
    if return_stats:
        return o, {"s": s, "m": m, "l": l, "p": p}
    return o


def _attention_head_sink(q, k, v, allowed, scale, sink):
    """The softmax over the allowed keys plus the sink logit, shifted by the
    largest of them; the sink's share of the weight multiplies nothing."""
    s = scale * (q @ k.T)
    s_masked = np.where(allowed, s, -np.inf)
    nonempty = allowed.any(axis=1)
    o = np.zeros((q.shape[0], v.shape[1]), dtype=np.float64)
    if not nonempty.any():
        return o
    m = np.maximum(s_masked[nonempty].max(axis=1), sink)
    p = np.where(allowed[nonempty], np.exp(s_masked[nonempty] - m[:, None]), 0.0)
    l = p.sum(axis=1) + np.exp(sink - m)
    o[nonempty] = (p @ v) / l[:, None]
    return o


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, n_heads: int, allowed: np.ndarray,
              scale: float = 1.0 / np.sqrt(HEAD_DIM), head_dim: int = HEAD_DIM,
              return_stats: bool = False, sinks: np.ndarray | None = None):
    """Multi-head attention for one sequence. q [t_q, H*dh], k/v [t_kv, H*dh];
    head h uses columns [h*dh, (h+1)*dh) of each. Returns o [t_q, H*dh] float64.
    sinks: optional [H] per-head sink logits."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    o = np.zeros((q.shape[0], n_heads * head_dim), dtype=np.float64)
    stats = []
    if sinks is not None and return_stats:
        raise ValueError("stats are not exported with sinks")
    for h in range(n_heads):
        cols = slice(h * head_dim, (h + 1) * head_dim)
        sink = None if sinks is None else float(np.asarray(sinks, dtype=np.float64)[h])
        res = attention_head(q[:, cols], k[:, cols], v[:, cols], allowed, scale, return_stats, sink)
        if return_stats:
            o[:, cols], st = res
            stats.append(st)
        else:
            o[:, cols] = res
    if return_stats:
        return o, stats
    return o


def encoder_attention(x: np.ndarray, w_qkv: np.ndarray, b_q: np.ndarray, b_v: np.ndarray,
                      batch: int, t: int, n_heads: int, mask: str = "full", chunk_len: int = 0,
                      scale: float = 1.0 / np.sqrt(HEAD_DIM), return_qkv: bool = False):
    """Packed projection followed by self-attention of each of ``batch``
    sequences of ``t`` frames. mask is "full" or "chunk"."""
    d = x.shape[1]
    qkv = qkv_projection(x, w_qkv, b_q, b_v)
    allowed = allowed_full(t, t) if mask == "full" else allowed_chunk(t, chunk_len)
    out = np.zeros((batch * t, d), dtype=np.float64)
    for b in range(batch):
        rows = slice(b * t, (b + 1) * t)
        out[rows] = attention(qkv[rows, :d], qkv[rows, d:2 * d], qkv[rows, 2 * d:], n_heads, allowed, scale)
    if return_qkv:
        return out, qkv
    return out


def slotmask_attention(q, k_cache, v_cache, bits, n_heads, scale=1.0 / np.sqrt(HEAD_DIM)):
    """Block verification over a position-indexed cache with an explicit
    allowed-slot bitmask (one row of words per query row, shared by all heads)."""
    return attention(q, k_cache, v_cache, n_heads, allowed_from_bits(bits, k_cache.shape[0]), scale)


def cross_attention(q, k_enc, v_enc, n_heads, scale=1.0 / np.sqrt(HEAD_DIM)):
    """Decoder queries attending to every encoder frame (t_q != t_kv allowed)."""
    return attention(q, k_enc, v_enc, n_heads, allowed_full(q.shape[0], k_enc.shape[0]), scale)



def range_attention(q, k, v, batch, t_q, t_kv, n_heads, *, q_lens=None, kv_lens=None, chunk_len=0,
                    window=0, causal=False, sinks=None, scale=1.0 / np.sqrt(HEAD_DIM)):
    """Self- or cross-attention of ``batch`` sequences (rows [b*t_q, (b+1)*t_q)
    of q, [b*t_kv, (b+1)*t_kv) of k and v) under the range family: per-sequence
    valid lengths, CHUNK, band, causal, and optional per-head sinks."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    out = np.zeros((batch * t_q, n_heads * HEAD_DIM), dtype=np.float64)
    for b in range(batch):
        allowed = allowed_range(t_q, t_kv, q_len=None if q_lens is None else int(q_lens[b]),
                                kv_len=None if kv_lens is None else int(kv_lens[b]),
                                chunk_len=chunk_len, window=window, causal=causal)
        qr, kr = slice(b * t_q, (b + 1) * t_q), slice(b * t_kv, (b + 1) * t_kv)
        out[qr] = attention(q[qr], k[kr], v[kr], n_heads, allowed, scale, sinks=sinks)
    return out
