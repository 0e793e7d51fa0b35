"""B200 (sm_100a) Whisper-style attention pass: packed QKV projection and
flash attention with FULL / CHUNK / SLOTMASK masks, behind a C ABI.

The CUDA library is loaded lazily by ``speech_encoder_attention_b200.attn``;
there is no CPU fallback.
"""
__all__ = ["attn", "inputs"]
