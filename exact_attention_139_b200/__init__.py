"""Exact scaled-dot-product attention for NVIDIA B200 (sm_100a).

The compute lives in ``libattn_b200.so`` (CUDA, C ABI declared in ``include/attn.h``);
``exact_attention_139_b200.attn`` is the thin ctypes binding over it and raises at import
when the library is missing. ``exact_attention_139_b200.inputs`` holds the seeded synthetic
input generators (no attention arithmetic); ``exact_attention_139_b200.shard`` splits a
layer's heads over ranks.
"""
__all__ = ["attn", "inputs", "shard"]
