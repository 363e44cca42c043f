"""Closed-form KV-cache size — test oracle.

Test infrastructure (see ``oracle/__init__``).

[COMPRESS] "1. The KV cache memory problem" states the estimate
    KV bytes = 2 * L * n_kv_heads * head_dim * seq_len * batch * bytes_per_element
(2 for K and V, L layers), with bytes_per_element 2 for FP16, 1 for FP8,
0.5 for INT4 and 0.25 for INT2, and works it for LLaMA-2-70B (80 layers,
8 KV heads, head_dim 128) at 4096 tokens (about 1.34 GB) and 128K tokens
(about 42.9 GB). [LIMITS] (opening paragraph and "TL;DR") works the same
product for a 70B Llama-3 at 32k in BF16 (about 10.7 GB per request), and
[76X] "2. How much memory the KV cache takes" gives the per-token form
(2 * layers * kv_heads * head_dim * bytes; about 40 KB for 10 attention layers,
8 KV heads, head_dim 128, FP16).

The formula counts element bytes only; the per-token scales a quantised cache
also stores are counted separately (``scale_bytes``).
"""

from __future__ import annotations

from fractions import Fraction

BYTES_PER_ELEMENT = {"fp16": Fraction(2), "bf16": Fraction(2), "fp8": Fraction(1),
                     "e5m2": Fraction(1), "int8": Fraction(1), "int8c": Fraction(1),
                     "int8t": Fraction(1), "int4": Fraction(1, 2),
                     "int2": Fraction(1, 4)}


def kv_bytes(layers, n_kv_heads, head_dim, seq_len, batch, bytes_per_element):
    """Exact KV bytes by the closed form (a Fraction, so 0.5 / 0.25 stay exact)."""
    return 2 * layers * n_kv_heads * head_dim * seq_len * batch * Fraction(bytes_per_element)


def per_token_kv_bytes(layers, n_kv_heads, head_dim, bytes_per_element):
    """K and V bytes one token adds across all layers."""
    return kv_bytes(layers, n_kv_heads, head_dim, 1, 1, bytes_per_element)


def scale_bytes(layers, n_kv_heads, seq_len, batch, fmt):
    """Bytes of the per-token, per-KV-head BF16 metadata of K and V:
    one scale (FP8) or a scale and a zero point (INT8) per row; none for BF16."""
    per_row = {"bf16": 0, "fp16": 0, "fp8": 2, "e5m2": 2, "int8": 4, "int8c": 0, "int8t": 0}[fmt]
    return 2 * layers * n_kv_heads * seq_len * batch * per_row


def static_scale_bytes(layers, n_kv_heads, head_dim, fmt):
    """Bytes of the static BF16 scales of K and V: one per (KV head, channel)
    for per-channel INT8, one per cache for per-tensor INT8; independent of the
    number of tokens."""
    per_cache = {"int8c": n_kv_heads * head_dim * 2, "int8t": 2}.get(fmt, 0)
    return 2 * layers * per_cache
