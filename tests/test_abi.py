"""The C ABI: the library loads, exports every entry point include/attn.h
declares, and rejects invalid arguments on the host before any CUDA call (so
these run without a GPU)."""
import ctypes
import os
import re

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
    mk = attn.AttnMask(); mk.kind = attn.MASK_FULL; mk.reserved = 1
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
