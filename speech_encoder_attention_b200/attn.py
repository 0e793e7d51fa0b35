"""Python binding of libattn.so (the C ABI in include/attn.h).

Argument marshalling only: every step of the attention pass runs in the CUDA
library. Tensors must be CUDA fp16 tensors (uint32 for the SLOTMASK bits);
the library is loaded on first use and a missing library raises. There is no
CPU fallback.

The function names match the C entry points:
    attn_qkv_pack(x, w_qkv, b_q, b_v, out=None)        -> qkv
    attn_qkv_pack_q8_0(x, w_q8_0, b_q, b_v, out=None)  -> qkv
    attn_forward(q, k, v, batch, t_q, t_kv, n_heads, mask=..., out=None) -> out
      (split=False sets ATTN_FLAG_NO_SPLIT)
    attn_forward with sinks=...                          -> attn_forward_sinks
    attn_cross(q, k_enc, v_enc, batch, t_q, t_enc, n_heads, out=None)   -> out
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libattn.so")

ATTN_OK = 0
ATTN_ERR_INVALID = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_CUDA = 3
ATTN_ERR_TIMEOUT = 4

ATTN_FLAG_NO_SPLIT = 1

MASK_FULL = 0
MASK_CHUNK = 1
MASK_SLOTMASK = 2
MASK_BAND = 3

HEAD_DIM = 64
DEFAULT_SCALE = 0.125  # 1/sqrt(64)


class AttnMat(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("row_stride", ctypes.c_int64)]


class AttnMask(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32),
        ("chunk_len", ctypes.c_int32),
        ("bits", ctypes.c_void_p),
        ("words_per_row", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("causal", ctypes.c_int32),
        ("flags", ctypes.c_int32),
        ("q_lens", ctypes.c_void_p),
        ("kv_lens", ctypes.c_void_p),
    ]


class AttnPlanInfo(ctypes.Structure):
    _fields_ = [
        ("seg_len", ctypes.c_int32),
        ("tiles_per_seg", ctypes.c_int32),
        ("q_tiles", ctypes.c_int32),
        ("kv_splits", ctypes.c_int32),
        ("kv_tiles_per_split", ctypes.c_int32),
        ("proj_tile_n", ctypes.c_int32),
        ("units", ctypes.c_int64),
        ("workspace_bytes", ctypes.c_size_t),
        ("cluster_merge", ctypes.c_int32),
        ("narrow", ctypes.c_int32),
    ]


# (name, restype, argtypes) of every exported entry point.
SIGNATURES = {
    "attn_qkv_pack": (ctypes.c_int, [AttnMat, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_int64, ctypes.c_int32, AttnMat, ctypes.c_void_p]),
    "attn_qkv_pack_q8_0": (ctypes.c_int, [AttnMat, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_int64, ctypes.c_int32, AttnMat, ctypes.c_void_p]),
    "attn_forward": (ctypes.c_int, [AttnMat, AttnMat, AttnMat, ctypes.c_int32, ctypes.c_int32,
                                    ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, AttnMask,
                                    ctypes.c_float, AttnMat, ctypes.c_void_p, ctypes.c_size_t,
                                    ctypes.c_void_p]),
    "attn_forward_sinks": (ctypes.c_int, [AttnMat, AttnMat, AttnMat, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, AttnMask,
                                          ctypes.c_void_p, ctypes.c_float, AttnMat, ctypes.c_void_p,
                                          ctypes.c_size_t, ctypes.c_void_p]),
    "attn_cross": (ctypes.c_int, [AttnMat, AttnMat, AttnMat, ctypes.c_int32, ctypes.c_int32,
                                  ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                                  AttnMat, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "attn_cross_static_scratch": (ctypes.c_int, [AttnMat, AttnMat, AttnMat, ctypes.c_int32, ctypes.c_int32,
                                                 ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                 ctypes.c_float, AttnMat, ctypes.c_void_p]),
    "attn_workspace_size": (ctypes.c_size_t, [ctypes.c_int32] * 6),
    "attn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "attn_debug_error_word": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint32)]),
    "attn_debug_timeout_probe": (ctypes.c_int, [ctypes.c_int64, ctypes.c_void_p]),
    "attn_debug_plan": (ctypes.c_int, [ctypes.c_int32] * 7 + [ctypes.c_int64, ctypes.c_int32,
                                                              ctypes.POINTER(AttnPlanInfo)]),
}

_lib = None
_lock = threading.Lock()


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def load_library(path: str = LIB_PATH):
    """Loads libattn.so (built in-tree by ``python -m speech_encoder_attention_b200.build``)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"libattn.so not found at {path}; build it with "
                               "`python -m speech_encoder_attention_b200.build` (needs nvcc)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load_library().attn_status_string(status).decode()


def _check(status: int, where: str):
    if status != ATTN_OK:
        raise AttnError(status, where)


def _stream_ptr(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _mat(t, cols: Optional[int] = None) -> AttnMat:
    """A 2-D CUDA fp16 tensor (or a column view of one) as {ptr, row_stride}."""
    import torch
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor (there is no CPU path)")
    if t.dtype != torch.float16:
        raise ValueError(f"expected float16, got {t.dtype}")
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit column stride")
    return AttnMat(ctypes.c_void_p(t.data_ptr()), t.stride(0))


def _ptr(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor (there is no CPU path)")
    return ctypes.c_void_p(t.data_ptr())


def attn_qkv_pack(x, w_qkv, b_q=None, b_v=None, out=None, stream=None):
    """qkv = x . W^T + [b_q | 0 | b_v].  x [rows, d], W [3d, d] -> [rows, 3d] fp16."""
    import torch
    lib = load_library()
    rows, d = x.shape
    if w_qkv.shape != (3 * d, d) or not w_qkv.is_contiguous() or w_qkv.dtype != torch.float16:
        raise ValueError("w_qkv must be a contiguous [3*d_model, d_model] fp16 tensor")
    for b in (b_q, b_v):
        if b is not None and (b.shape != (d,) or b.dtype != torch.float16 or not b.is_contiguous()):
            raise ValueError("biases must be contiguous [d_model] fp16 tensors")
    if out is None:
        out = torch.empty(rows, 3 * d, dtype=torch.float16, device=x.device)
    st = lib.attn_qkv_pack(_mat(x), _ptr(w_qkv), _ptr(b_q), _ptr(b_v), rows, d, _mat(out),
                           _stream_ptr(stream))
    _check(st, "attn_qkv_pack")
    return out


def attn_qkv_pack_q8_0(x, w_q8_0, b_q=None, b_v=None, out=None, stream=None):
    """qkv = x . W^T + [b_q | 0 | b_v] with Q8_0 weights: w_q8_0 is a contiguous
    uint8 CUDA tensor [3*d, d/32*34] (per block: fp16 scale, 32 int8)."""
    import torch
    lib = load_library()
    rows, d = x.shape
    if w_q8_0.dtype != torch.uint8 or w_q8_0.shape != (3 * d, d // 32 * 34) or not w_q8_0.is_contiguous():
        raise ValueError("w_q8_0 must be a contiguous [3*d_model, d_model/32*34] uint8 tensor")
    for b in (b_q, b_v):
        if b is not None and (b.shape != (d,) or b.dtype != torch.float16 or not b.is_contiguous()):
            raise ValueError("biases must be contiguous [d_model] fp16 tensors")
    if out is None:
        out = torch.empty(rows, 3 * d, dtype=torch.float16, device=x.device)
    st = lib.attn_qkv_pack_q8_0(_mat(x), _ptr(w_q8_0), _ptr(b_q), _ptr(b_v), rows, d, _mat(out),
                                _stream_ptr(stream))
    _check(st, "attn_qkv_pack_q8_0")
    return out


def _lens_ptr(t):
    import torch
    if t is None:
        return 0
    if t.dtype != torch.int32 or t.dim() != 1 or not t.is_contiguous():
        raise ValueError("sequence lengths must be a contiguous [batch] int32 CUDA tensor")
    return _ptr(t).value or 0


def make_mask(kind: int = MASK_FULL, chunk_len: int = 0, bits=None, window: int = 0, causal: bool = False,
              q_lens=None, kv_lens=None) -> AttnMask:
    import torch
    m = AttnMask()
    m.kind = kind
    m.chunk_len = chunk_len
    m.window = window
    m.causal = 1 if causal else 0
    m.flags = 0
    m.q_lens = _lens_ptr(q_lens)
    m.kv_lens = _lens_ptr(kv_lens)
    if kind == MASK_SLOTMASK:
        if bits is None or bits.dtype not in (torch.int32, torch.uint32) or bits.dim() != 2:
            raise ValueError("SLOTMASK needs a [t_q, words_per_row] int32/uint32 CUDA tensor")
        if not bits.is_contiguous():
            raise ValueError("mask bits must be contiguous")
        m.bits = _ptr(bits).value or 0
        m.words_per_row = bits.shape[1]
    else:
        m.bits = 0
        m.words_per_row = 0
    return m


def workspace_size(batch, t_q, t_kv, n_heads, mask_kind=MASK_FULL, head_dim=HEAD_DIM) -> int:
    return int(load_library().attn_workspace_size(batch, t_q, t_kv, n_heads, head_dim, mask_kind))


def _workspace(nbytes: int, device, workspace=None):
    import torch
    if nbytes == 0:
        return None, 0
    if workspace is not None:
        return workspace, workspace.numel() * workspace.element_size()
    return torch.empty(nbytes, dtype=torch.uint8, device=device), nbytes


def attn_forward(q, k, v, batch, t_q, t_kv, n_heads, mask_kind=MASK_FULL, chunk_len=0, bits=None,
                 scale=DEFAULT_SCALE, out=None, workspace=None, split=True, stream=None, window=0,
                 causal=False, q_lens=None, kv_lens=None, sinks=None):
    """Masked multi-head flash attention. q [batch*t_q, >=H*64] (or a column
    view of the packed qkv buffer), k/v [batch*t_kv, >=H*64]; returns out
    [batch*t_q, H*64] fp16. window / causal / q_lens / kv_lens select the
    range family's band, causal flag and per-sequence lengths ([batch] int32
    CUDA tensors); sinks ([n_heads] fp32 CUDA tensor) calls attn_forward_sinks."""
    import torch
    lib = load_library()
    mask = make_mask(mask_kind, chunk_len, bits, window, causal, q_lens, kv_lens)
    if not split:
        mask.flags = ATTN_FLAG_NO_SPLIT
    if out is None:
        out = torch.empty(batch * t_q, n_heads * HEAD_DIM, dtype=torch.float16, device=q.device)
    need = workspace_size(batch, t_q, t_kv, n_heads, mask_kind) if split else 0
    ws, ws_bytes = _workspace(need, q.device, workspace) if split else (None, 0)
    if sinks is None:
        st = lib.attn_forward(_mat(q), _mat(k), _mat(v), batch, t_q, t_kv, n_heads, HEAD_DIM, mask,
                              float(scale), _mat(out), _ptr(ws), ws_bytes, _stream_ptr(stream))
        _check(st, "attn_forward")
        return out
    if sinks.dtype != torch.float32 or sinks.dim() != 1 or not sinks.is_contiguous():
        raise ValueError("sinks must be a contiguous [n_heads] float32 CUDA tensor")
    st = lib.attn_forward_sinks(_mat(q), _mat(k), _mat(v), batch, t_q, t_kv, n_heads, HEAD_DIM, mask,
                                _ptr(sinks), float(scale), _mat(out), _ptr(ws), ws_bytes, _stream_ptr(stream))
    _check(st, "attn_forward_sinks")
    return out


def attn_cross(q, k_enc, v_enc, batch, t_q, t_enc, n_heads, scale=DEFAULT_SCALE, out=None,
               workspace=None, split=True, stream=None):
    """Decoder queries against every encoder frame (FULL, t_q != t_enc allowed).
    split=False passes no workspace: a split that needs one does not happen, a
    split merged inside a cluster still does (attn_cross takes no flags; use
    attn_forward with split=False for a fixed summation order)."""
    import torch
    lib = load_library()
    if out is None:
        out = torch.empty(batch * t_q, n_heads * HEAD_DIM, dtype=torch.float16, device=q.device)
    need = workspace_size(batch, t_q, t_enc, n_heads, MASK_FULL) if split else 0
    ws, ws_bytes = _workspace(need, q.device, workspace) if split else (None, 0)
    st = lib.attn_cross(_mat(q), _mat(k_enc), _mat(v_enc), batch, t_q, t_enc, n_heads, HEAD_DIM,
                        float(scale), _mat(out), _ptr(ws), ws_bytes, _stream_ptr(stream))
    _check(st, "attn_cross")
    return out


def encoder_layer_attention(x, w_qkv, b_q, b_v, batch, t, n_heads, mask_kind=MASK_FULL,
                            chunk_len=0, qkv=None, out=None, stream=None):
    """The encoder attention pass: packed projection, then attention read in
    place from the packed buffer (q, k, v are column views of it)."""
    d = x.shape[1]
    qkv = attn_qkv_pack(x, w_qkv, b_q, b_v, out=qkv, stream=stream)
    return attn_forward(qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:], batch, t, t, n_heads,
                        mask_kind=mask_kind, chunk_len=chunk_len, out=out, stream=stream)


def debug_error_word(stream=None):
    """Synchronises the stream; returns (status, raw word) and clears the word."""
    w = ctypes.c_uint32(0)
    st = load_library().attn_debug_error_word(_stream_ptr(stream), ctypes.byref(w))
    return st, w.value


def debug_timeout_probe(limit_ns: int, stream=None) -> int:
    return load_library().attn_debug_timeout_probe(int(limit_ns), _stream_ptr(stream))


def debug_plan(batch, t_q, t_kv, n_heads, mask_kind=MASK_FULL, chunk_len=0, num_sms=148, proj_rows=0,
               d_model=0) -> dict:
    """The launch plan the library would choose on a GPU with num_sms SMs (host arithmetic only)."""
    info = AttnPlanInfo()
    st = load_library().attn_debug_plan(batch, t_q, t_kv, n_heads, mask_kind, chunk_len, num_sms, proj_rows,
                                        d_model, ctypes.byref(info))
    _check(st, "attn_debug_plan")
    return {name: getattr(info, name) for name, _ in AttnPlanInfo._fields_}
