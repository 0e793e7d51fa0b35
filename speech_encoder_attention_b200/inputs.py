"""Seeded synthetic inputs for the Whisper-style attention pass.

This module only draws random numbers and builds input structure (shapes,
distributions, the token tree and its allowed-slot bitmask). It contains none
of the arithmetic of the attention pass itself, so that the FP64 oracle and the
CUDA path can both be fed from it without sharing any computation.

Workloads (sizes follow the pages' encoder and decoder):

* ``tiny``      -- 1 sequence of 64 frames, d_model 128, 2 heads of 64 (seed 0).
* ``window``    -- one 30 s Whisper-large-v3 window: 1500 frames, d_model 1280,
                   20 heads of 64, full bidirectional mask (seed 2). The 1500-frame
                   window is the one the edda PR ("Add Edda ASR with DFlash2
                   speculative decoding", PR description) describes for its encoder.
* ``windows8``  -- 8 such windows with one shared weight set; each window's x
                   carries its own scalar offset drawn from U(-0.5, 0.5) (seed 3).
* ``chunks``    -- a higgs-style chunked encode: 12 chunks of up to 200 frames
                   (11 x 200 + 125 = 2325 frames), chunk-local mask (seed 4). The
                   4 s chunk rule is the higgs-audio-v3-stt model card's
                   "Architecture note (chunked encoder)"; 4 s at 50 frames/s = 200.
* ``varlen8``   -- 8 windows of up to 1500 frames with per-window valid lengths
                   drawn uniformly from [500, 1500] (seed 6; lengths from the
                   generator stream [6, 1]): the shortened 500-position input
                   (1000 mel frames; BuzzASR discussion) up to a full window. The
                   frames past a window's length are padding that no valid frame
                   may attend to (higgs model card: attending to the silence
                   padding corrupts the conditioning).
* ``band8``     -- 8 full windows under a sliding-window band of 256 frames
                   (seed 7). The drafter PR adds a sliding window without a size;
                   256 frames (~5 s) is this recipe's choice.
* ``drafter`` / ``drafter_causal`` -- the drafter's block attention: 5 beams,
                   each a block of 16 queries (anchor + 15 drafts) at the end of
                   448 keys (432 context positions + the block), 20 heads of 64,
                   per-head sink logits ~ N(0, 1) (seeds 8, 9). Non-causal inside
                   the block by default, causal when the model says so (drafter PR).
* ``q8_tiny`` / ``q8_verify`` -- the packed projection with Q8_0 weights for
                   the decoder's verify block (edda PR results table: Q8_0
                   decoder): 5 x 256 and 80 x 1280 (the 5 beams x 16 rows of
                   the verify block) rows, q uniform int8, block scales uniform
                   in [2e-4, 6e-4] (seeds 10, 11).
* ``verify``    -- decoder block verification over a token tree: 5 beams x
                   (anchor + 15 drafts) = 80 query rows over a 448-slot KV cache,
                   each row limited to its ancestors, plus cross-attention of the
                   same rows to 1500 encoder frames (seed 5). Block size and the
                   ancestor rule come from the edda PR description (block
                   verification of up to 15 drafted tokens; token-tree KV cache
                   whose mask rows admit only ancestors).

Distributions: x ~ N(0, 1); packed W_qkv ~ N(0, 0.02^2); b_q, b_v ~ N(0, 0.01^2);
verify Q, K, V ~ N(0, 1). Everything is rounded once to IEEE fp16.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

HEAD_DIM = 64


@dataclasses.dataclass(frozen=True)
class EncoderSpec:
    name: str
    batch: int
    t: int
    d_model: int
    n_heads: int
    mask: str  # "full" or "chunk"
    chunk_len: int
    seed: int
    window_offset: bool = False
    band: int = 0          # BAND window in frames (mask == "band")
    varlen: bool = False   # per-window valid lengths, see encoder_lengths


ENCODER_WORKLOADS: Dict[str, EncoderSpec] = {
    "tiny": EncoderSpec("tiny", 1, 64, 128, 2, "full", 0, 0),
    "window": EncoderSpec("window", 1, 1500, 1280, 20, "full", 0, 2),
    "windows8": EncoderSpec("windows8", 8, 1500, 1280, 20, "full", 0, 3, True),
    "chunks": EncoderSpec("chunks", 1, 2325, 1280, 20, "chunk", 200, 4),
    "varlen8": EncoderSpec("varlen8", 8, 1500, 1280, 20, "full", 0, 6, True, varlen=True),
    "band8": EncoderSpec("band8", 8, 1500, 1280, 20, "band", 0, 7, True, band=256),
}


def encoder_lengths(spec: EncoderSpec) -> Optional[np.ndarray]:
    """Valid frames of each window (int32 [batch]) of a varlen workload, else None:
    uniform integers in [500, t] from the generator stream [seed, 1]."""
    if not spec.varlen:
        return None
    rng = np.random.default_rng([spec.seed, 1])
    return rng.integers(500, spec.t + 1, size=spec.batch).astype(np.int32)


@dataclasses.dataclass(frozen=True)
class DrafterSpec:
    name: str
    n_heads: int
    d_model: int
    block: int     # queries per beam: anchor + drafts, at the end of the keys
    beams: int     # independent sequences
    context: int   # key positions before the block
    causal: bool   # block-internal attention causal (else bidirectional)
    seed: int

    @property
    def t_q(self) -> int:
        return self.block

    @property
    def t_kv(self) -> int:
        return self.context + self.block


DRAFTER_WORKLOADS: Dict[str, DrafterSpec] = {
    "drafter": DrafterSpec("drafter", 20, 1280, 16, 5, 432, False, 8),
    "drafter_causal": DrafterSpec("drafter_causal", 20, 1280, 16, 5, 432, True, 9),
}


@dataclasses.dataclass
class DrafterInputs:
    spec: DrafterSpec
    q: np.ndarray      # [beams * block, d_model] float16
    k: np.ndarray      # [beams * (context + block), d_model] float16
    v: np.ndarray      # [beams * (context + block), d_model] float16
    sinks: np.ndarray  # [n_heads] float32 sink logits


@dataclasses.dataclass(frozen=True)
class Q8Spec:
    name: str
    rows: int      # decoder rows projected at once
    d_model: int
    seed: int


Q8_WORKLOADS: Dict[str, Q8Spec] = {
    "q8_tiny": Q8Spec("q8_tiny", 5, 256, 10),
    "q8_verify": Q8Spec("q8_verify", 80, 1280, 11),
}


@dataclasses.dataclass
class Q8Inputs:
    spec: Q8Spec
    x: np.ndarray         # [rows, d_model] float16
    w_blocks: np.ndarray  # [3 * d_model, d_model / 32 * 34] uint8 Q8_0 rows
    scales: np.ndarray    # [3 * d_model, d_model / 32] float16 (the blocks' scales, for inspection)
    qs: np.ndarray        # [3 * d_model, d_model] int8 (the blocks' bytes, for inspection)
    b_q: np.ndarray       # [d_model] float16
    b_v: np.ndarray       # [d_model] float16


def pack_q8_0(scales: np.ndarray, qs: np.ndarray) -> np.ndarray:
    """Lay out per-block fp16 scales [rows, nb] and int8 values [rows, nb * 32]
    as Q8_0 rows: per block, the scale's two little-endian bytes, then the
    32 signed bytes. Byte layout only; no arithmetic on the values."""
    rows, nb = scales.shape
    out = np.empty((rows, nb, 34), dtype=np.uint8)
    out[:, :, :2] = np.ascontiguousarray(scales.astype("<f2")).view(np.uint8).reshape(rows, nb, 2)
    out[:, :, 2:] = np.ascontiguousarray(qs.astype(np.int8)).view(np.uint8).reshape(rows, nb, 32)
    return out.reshape(rows, nb * 34)


def make_q8_inputs(spec: Q8Spec) -> Q8Inputs:
    """Random Q8_0 weights drawn directly in their stored form: q uniform in
    [-127, 127], scales uniform in [2e-4, 6e-4] (the block scale of N(0, 0.02^2)
    weights, max|w| / 127), rounded to fp16; x ~ N(0, 1); biases ~ N(0, 0.01^2)."""
    rng = np.random.default_rng(spec.seed)
    d = spec.d_model
    if d % 32:
        raise ValueError("d_model must be a multiple of 32")
    n = 3 * d
    qs = rng.integers(-127, 128, size=(n, d)).astype(np.int8)
    scales = rng.uniform(2e-4, 6e-4, size=(n, d // 32)).astype(np.float16)
    x = _normal_f16(rng, (spec.rows, d))
    b_q = _normal_f16(rng, (d,), 0.01)
    b_v = _normal_f16(rng, (d,), 0.01)
    return Q8Inputs(spec, x, pack_q8_0(scales, qs), scales, qs, b_q, b_v)


def make_drafter_inputs(spec: DrafterSpec) -> DrafterInputs:
    rng = np.random.default_rng(spec.seed)
    d = spec.d_model
    q = _normal_f16(rng, (spec.beams * spec.t_q, d))
    k = _normal_f16(rng, (spec.beams * spec.t_kv, d))
    v = _normal_f16(rng, (spec.beams * spec.t_kv, d))
    sinks = rng.standard_normal(spec.n_heads).astype(np.float32)
    return DrafterInputs(spec, q, k, v, sinks)


@dataclasses.dataclass(frozen=True)
class VerifySpec:
    name: str
    n_heads: int
    d_model: int
    block: int          # anchor + drafts per beam
    beams: int
    prompt_slots: int   # shared committed prefix at the start of the cache
    beam_steps: int     # beam-search steps already in the cache before the block
    t_enc: int          # encoder frames for cross-attention
    seed: int

    @property
    def t_q(self) -> int:
        return self.block * self.beams

    @property
    def slots(self) -> int:
        return self.prompt_slots + self.beam_steps * self.beams + self.t_q


VERIFY_WORKLOADS: Dict[str, VerifySpec] = {
    "verify": VerifySpec("verify", 20, 1280, 16, 5, 8, 72, 1500, 5),
}


@dataclasses.dataclass
class EncoderInputs:
    spec: EncoderSpec
    x: np.ndarray      # [batch * t, d_model] float16
    w_qkv: np.ndarray  # [3 * d_model, d_model] float16 (q rows, k rows, v rows)
    b_q: np.ndarray    # [d_model] float16
    b_v: np.ndarray    # [d_model] float16


@dataclasses.dataclass
class VerifyInputs:
    spec: VerifySpec
    q: np.ndarray        # [t_q, d_model] float16
    k_cache: np.ndarray  # [slots, d_model] float16
    v_cache: np.ndarray  # [slots, d_model] float16
    parent: np.ndarray   # [slots] int64, -1 for the root
    bits: np.ndarray     # [t_q, words_per_row] uint32 allowed-slot bitmask
    query_slot: np.ndarray  # [t_q] int64: the cache slot each query row occupies
    k_enc: np.ndarray    # [t_enc, d_model] float16
    v_enc: np.ndarray    # [t_enc, d_model] float16


def _normal_f16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    return (rng.standard_normal(shape) * std).astype(np.float16)


def make_encoder_inputs(spec: EncoderSpec, batch: Optional[int] = None) -> EncoderInputs:
    """Draw x, W_qkv, b_q, b_v for an encoder workload.

    ``batch`` may override the spec's window count (used to build a bounded
    sample); the draws for windows [0, batch) do not depend on the override.
    """
    b = spec.batch if batch is None else batch
    rng = np.random.default_rng(spec.seed)
    d = spec.d_model
    w = _normal_f16(rng, (3 * d, d), 0.02)
    b_q = _normal_f16(rng, (d,), 0.01)
    b_v = _normal_f16(rng, (d,), 0.01)
    xs = []
    for _ in range(b):
        xw = rng.standard_normal((spec.t, d))
        if spec.window_offset:
            xw = xw + rng.uniform(-0.5, 0.5)
        xs.append(xw.astype(np.float16))
    x = np.concatenate(xs, axis=0)
    return EncoderInputs(spec, x, w, b_q, b_v)


def words_per_row(slots: int) -> int:
    return (slots + 31) // 32


def pack_bits(allowed: np.ndarray) -> np.ndarray:
    """Pack a boolean [rows, slots] matrix LSB-first into uint32 words:
    slot j is bit (j % 32) of word (j // 32)."""
    rows, slots = allowed.shape
    wpr = words_per_row(slots)
    padded = np.zeros((rows, wpr * 32), dtype=np.uint64)
    padded[:, :slots] = allowed.astype(np.uint64)
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    words = (padded.reshape(rows, wpr, 32) * weights).sum(axis=2)
    return words.astype(np.uint32)


def unpack_bits(bits: np.ndarray, slots: int) -> np.ndarray:
    rows, wpr = bits.shape
    j = np.arange(slots)
    return ((bits[:, j // 32] >> (j % 32).astype(np.uint32)) & 1).astype(bool)


def make_token_tree(spec: VerifySpec, rng: np.random.Generator):
    """Seeded token tree over the position-indexed cache.

    Slots [0, prompt) form the committed prompt chain. Then ``beam_steps``
    beam-search steps each give every beam a fresh slot whose parent is drawn
    uniformly among the previous step's slots (the first step hangs off the
    last prompt slot). The verify block follows: beam b's anchor sits at slot
    ``base + block*b`` with beam b's last-step slot as parent, and its drafts
    chain one after another. Returns (parent, query_slot)."""
    slots = spec.slots
    parent = np.full(slots, -1, dtype=np.int64)
    for s in range(1, spec.prompt_slots):
        parent[s] = s - 1
    prev = [spec.prompt_slots - 1] * spec.beams
    nxt = spec.prompt_slots
    for _ in range(spec.beam_steps):
        cur = []
        for _b in range(spec.beams):
            parent[nxt] = prev[int(rng.integers(0, spec.beams))]
            cur.append(nxt)
            nxt += 1
        prev = cur
    query_slot = np.zeros(spec.t_q, dtype=np.int64)
    for b in range(spec.beams):
        for i in range(spec.block):
            slot = nxt + spec.block * b + i
            parent[slot] = prev[b] if i == 0 else slot - 1
            query_slot[spec.block * b + i] = slot
    return parent, query_slot


def ancestors_mask(parent: np.ndarray, query_slot: np.ndarray) -> np.ndarray:
    """Boolean [rows, slots]: row r admits its own slot and every ancestor."""
    allowed = np.zeros((len(query_slot), len(parent)), dtype=bool)
    for r, s in enumerate(query_slot):
        while s >= 0:
            allowed[r, s] = True
            s = parent[s]
    return allowed


def make_verify_inputs(spec: VerifySpec) -> VerifyInputs:
    rng = np.random.default_rng(spec.seed)
    parent, query_slot = make_token_tree(spec, rng)
    d = spec.d_model
    q = _normal_f16(rng, (spec.t_q, d))
    k_cache = _normal_f16(rng, (spec.slots, d))
    v_cache = _normal_f16(rng, (spec.slots, d))
    k_enc = _normal_f16(rng, (spec.t_enc, d))
    v_enc = _normal_f16(rng, (spec.t_enc, d))
    bits = pack_bits(ancestors_mask(parent, query_slot))
    return VerifyInputs(spec, q, k_cache, v_cache, parent, bits, query_slot, k_enc, v_enc)


def random_bits(rng: np.random.Generator, rows: int, slots: int, density: float) -> np.ndarray:
    """Random allowed-slot bitmask (for edge-case tests)."""
    return pack_bits(rng.random((rows, slots)) < density)


def random_f16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    return _normal_f16(rng, shape, std)
