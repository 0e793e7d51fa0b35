"""The C ABI: the library loads, exports every entry point include/attn.h
declares, and rejects invalid arguments on the host before any CUDA call (so
these run without a GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

from speech_encoder_attention_b200 import attn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")

# Fake, 16-byte aligned device addresses: validation must fail before any of
# them is used.
P = 0x7F0000000000
P2 = 0x7F0010000000
P3 = 0x7F0020000000
P4 = 0x7F0030000000


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:attn_status|size_t|const char \*)\s*(attn_\w+)\(", text, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("attn_qkv_pack", "attn_forward", "attn_cross", "attn_workspace_size",
                     "attn_status_string", "attn_debug_error_word", "attn_debug_timeout_probe"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(attn.SIGNATURES)


def test_status_strings(lib):
    for code in range(5):
        s = attn.status_string(code)
        assert s.startswith("ATTN_")
    assert "UNKNOWN" in attn.status_string(99)


def m(ptr, stride):
    return attn.AttnMat(ctypes.c_void_p(ptr), stride)


def full():
    return attn.make_mask(attn.MASK_FULL)


def call_forward(lib, q=None, k=None, v=None, out=None, batch=1, t_q=64, t_kv=64, heads=2, hd=64,
                 mask=None, scale=0.125, ws=0, ws_bytes=0):
    q = q or m(P, 128)
    k = k or m(P2, 128)
    v = v or m(P3, 128)
    out = out or m(P4, 128)
    return lib.attn_forward(q, k, v, batch, t_q, t_kv, heads, hd, mask or full(), scale, out,
                            ctypes.c_void_p(ws), ws_bytes, None)


@pytest.mark.parametrize("kw", [
    dict(batch=0), dict(t_q=0), dict(t_kv=-1), dict(heads=0), dict(hd=128), dict(hd=32),
    dict(scale=0.0), dict(scale=-1.0), dict(scale=float("nan")), dict(scale=float("inf")),
    dict(q=m(0, 128)), dict(k=m(P2 + 8, 128)), dict(v=m(P3, 100)), dict(out=m(P4, 64)),
    dict(out=m(P + 64, 128)),                      # output overlaps q
    dict(ws=P4 + 0x10000008, ws_bytes=1 << 20),    # misaligned workspace
    dict(ws=0, ws_bytes=16),                       # bytes without a buffer
    dict(batch=70000),
])
def test_forward_rejects_invalid_arguments(lib, kw):
    assert call_forward(lib, **kw) == attn.ATTN_ERR_INVALID


def test_forward_rejects_bad_masks(lib):
    mk = attn.AttnMask()
    mk.kind = 7
    assert call_forward(lib, mask=mk) == attn.ATTN_ERR_INVALID
    mk = attn.AttnMask(); mk.kind = attn.MASK_CHUNK; mk.chunk_len = 0
    assert call_forward(lib, mask=mk) == attn.ATTN_ERR_INVALID
    mk = attn.AttnMask(); mk.kind = attn.MASK_CHUNK; mk.chunk_len = 16
    assert call_forward(lib, mask=mk, t_q=64, t_kv=32) == attn.ATTN_ERR_INVALID  # CHUNK needs t_q == t_kv
    mk = attn.AttnMask(); mk.kind = attn.MASK_SLOTMASK; mk.bits = 0; mk.words_per_row = 2
    assert call_forward(lib, mask=mk) == attn.ATTN_ERR_INVALID                  # no bits
    mk = attn.AttnMask(); mk.kind = attn.MASK_SLOTMASK; mk.bits = P4 + 0x1000000; mk.words_per_row = 1
    assert call_forward(lib, mask=mk, t_kv=64) == attn.ATTN_ERR_INVALID         # 1 word < 64 slots
    mk = attn.AttnMask(); mk.kind = attn.MASK_SLOTMASK; mk.bits = P4 + 0x1000002; mk.words_per_row = 2
    assert call_forward(lib, mask=mk, t_kv=64) == attn.ATTN_ERR_INVALID         # misaligned bits
    mk = attn.AttnMask(); mk.kind = attn.MASK_FULL; mk.flags = 2
    assert call_forward(lib, mask=mk) == attn.ATTN_ERR_INVALID


def test_forward_rejects_bad_range_options(lib):
    def mk(kind=attn.MASK_FULL, **kw):
        x = attn.AttnMask(); x.kind = kind
        for key, val in kw.items():
            setattr(x, key, val)
        return x
    assert call_forward(lib, mask=mk(window=4)) == attn.ATTN_ERR_INVALID                # window on FULL
    assert call_forward(lib, mask=mk(attn.MASK_BAND)) == attn.ATTN_ERR_INVALID           # BAND needs window
    assert call_forward(lib, mask=mk(attn.MASK_BAND, window=-3)) == attn.ATTN_ERR_INVALID
    assert call_forward(lib, mask=mk(causal=2)) == attn.ATTN_ERR_INVALID
    assert call_forward(lib, mask=mk(q_lens=P4 + 0x1000002)) == attn.ATTN_ERR_INVALID    # misaligned
    assert call_forward(lib, mask=mk(kv_lens=P4 + 0x1000001)) == attn.ATTN_ERR_INVALID
    slot = dict(bits=P4 + 0x1000000, words_per_row=2)
    assert call_forward(lib, mask=mk(attn.MASK_SLOTMASK, causal=1, **slot)) == attn.ATTN_ERR_INVALID
    assert call_forward(lib, mask=mk(attn.MASK_SLOTMASK, kv_lens=P4 + 0x2000000, **slot)) == attn.ATTN_ERR_INVALID
    assert call_forward(lib, mask=mk(attn.MASK_CHUNK, chunk_len=16, window=8)) == attn.ATTN_ERR_INVALID


def test_forward_sinks_validates_like_forward(lib):
    args = [m(P, 128), m(P2, 128), m(P3, 128), 1, 64, 64, 2, 64, full(), ctypes.c_void_p(P4 + 0x1000000),
            0.125, m(P4, 128), ctypes.c_void_p(0), 0, None]
    bad = list(args); bad[9] = ctypes.c_void_p(P4 + 0x1000002)   # misaligned sinks
    assert lib.attn_forward_sinks(*bad) == attn.ATTN_ERR_INVALID
    bad = list(args); bad[3] = 0
    assert lib.attn_forward_sinks(*bad) == attn.ATTN_ERR_INVALID
    bad = list(args); bad[11] = m(P + 64, 128)                     # output overlaps q
    assert lib.attn_forward_sinks(*bad) == attn.ATTN_ERR_INVALID


def test_cross_rejects_invalid_arguments(lib):
    args = [m(P, 128), m(P2, 128), m(P3, 128), 1, 80, 1500, 2, 64, 0.125, m(P4, 128),
            ctypes.c_void_p(0), 0, None]
    bad = list(args); bad[5] = 0
    assert lib.attn_cross(*bad) == attn.ATTN_ERR_INVALID
    bad = list(args); bad[7] = 80
    assert lib.attn_cross(*bad) == attn.ATTN_ERR_INVALID
    bad = list(args); bad[0] = m(P + 4, 128)
    assert lib.attn_cross(*bad) == attn.ATTN_ERR_INVALID


@pytest.mark.parametrize("case", [
    dict(rows=0), dict(d=0), dict(d=96), dict(d=-64),
    dict(x=m(0, 128)), dict(x=m(P, 120)), dict(x=m(P + 2, 128)),
    dict(w=0), dict(w=P2 + 4), dict(bq=P3 + 2), dict(out=m(P4, 256)), dict(out=m(P4 + 8, 384)),
    dict(out=m(P + 128, 384)),   # output overlaps x
])
def test_qkv_pack_rejects_invalid_arguments(lib, case):
    x = case.get("x", m(P, 128))
    w = case.get("w", P2)
    bq = case.get("bq", P3)
    out = case.get("out", m(P4, 384))
    st = lib.attn_qkv_pack(x, ctypes.c_void_p(w), ctypes.c_void_p(bq), ctypes.c_void_p(0),
                           case.get("rows", 64), case.get("d", 128), out, None)
    assert st == attn.ATTN_ERR_INVALID


def test_timeout_probe_rejects_out_of_range_limits(lib):
    assert lib.attn_debug_timeout_probe(10, None) == attn.ATTN_ERR_INVALID
    assert lib.attn_debug_timeout_probe(10 ** 10, None) == attn.ATTN_ERR_INVALID


def test_workspace_size_of_invalid_sizes_is_zero(lib):
    assert lib.attn_workspace_size(0, 80, 1500, 20, 64, 0) == 0
    assert lib.attn_workspace_size(1, 80, 1500, 20, 32, 0) == 0
    assert lib.attn_workspace_size(1, 80, 1500, 20, 64, attn.MASK_CHUNK) == 0


@pytest.mark.parametrize("case", [
    dict(rows=0), dict(d=128), dict(d=384), dict(d=0),          # d_model must be a multiple of 256
    dict(x=m(0, 256)), dict(x=m(P, 200)), dict(w=0), dict(w=P2 + 2), dict(bq=P3 + 4),
    dict(out=m(P4, 512)),                                        # row stride < 3*d_model
    dict(out=m(P2 + 64, 768)),                                   # output overlaps the weights
])
def test_qkv_pack_q8_0_rejects_invalid_arguments(lib, case):
    x = case.get("x", m(P, 256))
    st = lib.attn_qkv_pack_q8_0(x, ctypes.c_void_p(case.get("w", P2)), ctypes.c_void_p(case.get("bq", P3)),
                                ctypes.c_void_p(0), case.get("rows", 16), case.get("d", 256),
                                case.get("out", m(P4, 768)), None)
    assert st == attn.ATTN_ERR_INVALID


def test_slotmask_slot_limit_is_enforced(lib):
    mk = attn.AttnMask(); mk.kind = attn.MASK_SLOTMASK; mk.bits = P4 + 0x1000000; mk.words_per_row = 2049
    assert call_forward(lib, mask=mk, t_kv=65537) == attn.ATTN_ERR_INVALID


# ---------------------------------------------------------------------------
# host launch plan (no device needed)
# ---------------------------------------------------------------------------

def test_plan_of_the_benchmarked_and_one_window_steps(lib):
    p = attn.debug_plan(8, 1500, 1500, 20, proj_rows=12000, d_model=1280)
    assert (p["q_tiles"], p["kv_splits"], p["units"], p["workspace_bytes"]) == (12, 1, 8 * 20 * 12, 0)
    # 12000 rows take the CTA-pair projection (256 x 256 tiles on two SMs)
    assert p["proj_tile_n"] == 512
    # below 4096 rows: 32 x 15 wide tiles = 3.2 waves against 32 x 20 narrow = 4.3: wide
    assert attn.debug_plan(1, 4000, 4000, 20, proj_rows=4000, d_model=1280)["proj_tile_n"] == 256
    # a width that is not a multiple of 256 never takes the pair tiles
    assert attn.debug_plan(1, 4500, 4500, 5, proj_rows=4500, d_model=320)["proj_tile_n"] in (192, 256)
    # 12 x 15 = 180 wide tiles = 2 waves, 12 x 20 = 240 narrow = 2 waves of smaller tiles: narrow
    assert attn.debug_plan(1, 1500, 1500, 20, proj_rows=1500, d_model=1280)["proj_tile_n"] == 192


@pytest.mark.parametrize("t,clen", [(2325, 200), (517, 7), (517, 128), (517, 150), (300, 1)])
def test_plan_chunk_segments_are_whole_chunks(lib, t, clen):
    p = attn.debug_plan(1, t, t, 2, attn.MASK_CHUNK, clen)
    seg = clen if clen >= 128 else (128 // clen) * clen  # one chunk, or as many whole chunks as fit 128 rows
    assert p["seg_len"] == seg and p["seg_len"] % clen == 0
    assert p["tiles_per_seg"] == -(-seg // 128)
    assert p["q_tiles"] == -(-t // seg) * p["tiles_per_seg"]
    assert p["kv_splits"] == 1 and p["workspace_bytes"] == 0  # CHUNK tiles already fill the GPU


def test_plan_chunk_at_least_the_sequence_is_full(lib):
    a = attn.debug_plan(2, 300, 300, 2, attn.MASK_CHUNK, 300)
    b = attn.debug_plan(2, 300, 300, 2, attn.MASK_FULL)
    assert a == b


@pytest.mark.parametrize("kind,t_q,t_kv,heads,sms", [
    (attn.MASK_SLOTMASK, 80, 448, 20, 148),   # the verify block: 4 key tiles
    (attn.MASK_FULL, 80, 1500, 20, 148),      # cross-attention: 12 key tiles
    (attn.MASK_BAND, 16, 448, 5, 148),
    (attn.MASK_FULL, 80, 1500, 20, 64),
])
def test_plan_splits_short_query_blocks(lib, kind, t_q, t_kv, heads, sms):
    p = attn.debug_plan(1, t_q, t_kv, heads, kind, num_sms=sms)
    base = heads * -(-t_q // 128)
    n_kv = -(-t_kv // 128)
    assert base * 2 <= sms  # these cases qualify for a split
    want = min(n_kv, max(1, sms // base))
    per = -(-n_kv // want)
    splits = -(-n_kv // per)
    assert (p["kv_splits"], p["kv_tiles_per_split"]) == (splits, per)
    assert p["kv_splits"] * p["kv_tiles_per_split"] >= n_kv > (p["kv_splits"] - 1) * p["kv_tiles_per_split"]
    assert p["units"] == base * splits
    rows = splits * heads * t_q
    if splits <= 8:  # merged inside a cluster of `splits` CTAs: no workspace
        assert p["cluster_merge"] == 1 and p["workspace_bytes"] == 0
    else:
        assert p["cluster_merge"] == 0
        assert p["workspace_bytes"] == rows * 64 * 4 + rows * 2 * 4  # partial O, then (m, l)


def test_plan_long_splits_use_the_workspace(lib):
    # one head of 80 queries over 12000 keys: 94 key tiles over up to 148 CTAs
    p = attn.debug_plan(1, 80, 12000, 1, attn.MASK_FULL, num_sms=148)
    assert p["kv_splits"] > 8 and p["cluster_merge"] == 0
    assert p["workspace_bytes"] == p["kv_splits"] * 80 * (64 * 4 + 2 * 4)
    # the verify block's cross-attention: 6 splits, merged in clusters
    p = attn.debug_plan(1, 80, 1500, 20, attn.MASK_FULL, num_sms=148)
    assert (p["kv_splits"], p["cluster_merge"], p["workspace_bytes"]) == (6, 1, 0)


def test_plan_narrow_tiles_for_decode_sized_blocks(lib):
    # the drafter: 5 beams x 16 queries, 20 heads -> 100 one-tile units, no split
    p = attn.debug_plan(5, 16, 448, 20, num_sms=148)
    assert (p["kv_splits"], p["units"], p["narrow"]) == (1, 100, 1)
    assert attn.debug_plan(5, 32, 448, 20, num_sms=148)["narrow"] == 1      # up to 32 rows
    assert attn.debug_plan(5, 33, 448, 20, num_sms=148)["narrow"] == 0      # more rows: the 128-row layout
    assert attn.debug_plan(5, 16, 448, 20, attn.MASK_BAND, num_sms=148)["narrow"] == 1
    assert attn.debug_plan(8, 16, 448, 20, num_sms=148)["narrow"] == 0      # 160 units: more than one per SM
    p = attn.debug_plan(1, 16, 448, 20, num_sms=148)                         # 20 units: the key split instead
    assert p["kv_splits"] > 1 and p["narrow"] == 0
    assert attn.debug_plan(5, 16, 448, 20, attn.MASK_SLOTMASK, num_sms=148)["narrow"] == 0


def test_plan_does_not_split_when_units_fill_the_gpu(lib):
    p = attn.debug_plan(1, 80, 1500, 80, num_sms=148)  # 80 units: more than half of 148
    assert p["kv_splits"] == 1 and p["workspace_bytes"] == 0
    p = attn.debug_plan(1, 80, 100, 20, num_sms=148)    # a single key tile: nothing to split
    assert p["kv_splits"] == 1


def test_plan_rejects_invalid_requests(lib):
    info = attn.AttnPlanInfo()
    assert lib.attn_debug_plan(0, 1, 1, 1, 0, 0, 148, 0, 0, ctypes.byref(info)) == attn.ATTN_ERR_INVALID
    assert lib.attn_debug_plan(1, 1, 1, 1, 0, 0, 0, 0, 0, ctypes.byref(info)) == attn.ATTN_ERR_INVALID
    assert lib.attn_debug_plan(1, 1, 1, 1, 9, 0, 148, 0, 0, ctypes.byref(info)) == attn.ATTN_ERR_INVALID
    assert lib.attn_debug_plan(1, 8, 8, 1, attn.MASK_CHUNK, 0, 148, 0, 0, ctypes.byref(info)) == attn.ATTN_ERR_INVALID
    assert lib.attn_debug_plan(1, 1, 1, 1, 0, 0, 148, 0, 0, None) == attn.ATTN_ERR_INVALID


def call_static_scratch(lib, q=None, k=None, v=None, out=None, batch=1, t_q=80, t_enc=1500, heads=2, hd=64,
                        scale=0.125):
    return lib.attn_cross_static_scratch(q or m(P, 128), k or m(P2, 128), v or m(P3, 128), batch, t_q, t_enc,
                                         heads, hd, scale, out or m(P4, 128), None)


@pytest.mark.parametrize("kw", [
    dict(batch=0), dict(t_q=0), dict(t_enc=-1), dict(heads=0), dict(hd=128), dict(scale=0.0),
    dict(q=m(0, 128)), dict(k=m(P2 + 8, 128)), dict(v=m(P3, 100)), dict(out=m(P + 64, 128)),
])
def test_static_scratch_rejects_invalid_arguments_before_any_cuda_call(lib, kw):
    """The fixed-scratch cross-attention checks its arguments before it looks
    at the device: here, with no usable device, an invalid call must still say
    ATTN_ERR_INVALID (a device query would have failed with another status)."""
    assert call_static_scratch(lib, **kw) == attn.ATTN_ERR_INVALID


def test_division_by_launch_constants():
    """The attention kernels divide by launch constants (key splits, query
    tiles, heads, chunk length) as umulhi(n, m) >> s with l = ceil(log2 d),
    m = ceil(2^(31 + l) / d), s = l - 1 (the host computes m and s): exact for
    every 0 <= n < 2^31, checked here densely at both ends of that range."""
    def magic(d):
        if d <= 1:
            return 0, 0
        l = (d - 1).bit_length()
        return ((1 << (31 + l)) + d - 1) // d, l - 1

    rng = np.random.default_rng(3)
    divisors = list(range(1, 2049)) + [2 ** k + e for k in range(11, 31) for e in (-1, 0, 1)] + [2 ** 31 - 1]
    for d in divisors:
        m, s = magic(d)
        assert m < 2 ** 32
        n = np.concatenate([np.arange(0, 600), np.arange(2 ** 31 - 600, 2 ** 31),
                            rng.integers(0, 2 ** 31, 200)]).astype(object)
        q = n if m == 0 else ((n * m) >> 32) >> s
        assert all(q == n // d), d
