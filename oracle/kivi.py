"""KIVI-style low-bit KV cache: K quantized per channel, V per token, the most
recent tokens kept in full precision — test oracle.

Test infrastructure (see ``oracle/__init__``).

What the pages fix
------------------
* [COMPRESS] "2.1" (the asymmetry): K has a few outlier channels and V a
  per-token distribution, so K is quantized per channel and V per token (the
  KIVI finding).
* [COMPRESS] "3.1", "KIVI": an asymmetric 2-bit method, K per channel and V
  per token; the most recent tokens stay in full precision as a residual
  (sliding window); no tuning.
* [LIMITS] "Formats you will actually meet": the mixed-precision 4-bit
  variants (KIVI, KVQuant, ZipCache) quantize K per channel and V per token;
  4-bit storage is 25% of BF16 ([LIMITS] opening paragraph).

Readings taken where the pages are silent
-----------------------------------------
* Asymmetric uniform quantizer with b bits (b = 2 or 4) over a group of
  values: ``z = bf16_rne(min x)``, ``s = bf16_rne(f32(max x - min x) /
  (2^b - 1))`` (f32 arithmetic), ``c = clamp(rint(f32(x - z) / s), 0,
  2^b - 1)``, dequantized ``c * s + z``; a group with ``s == 0`` stores code 0
  and dequantizes to z.
* K groups: one (KV head, channel) over 128 consecutive positions of a
  sequence (one 128-token tile of the paged cache); V groups: one (position,
  KV head) over its D channels.
* Residual: the positions after the last complete 128-position group (at
  most 127) stay in BF16, K and V alike; a group is quantized when it
  completes.
* Metadata (s, z) is BF16: K 4 bytes per (group, KV head, channel), V 4 bytes
  per (position, KV head). A zero minimum or range is stored as +0 (the pages
  give no sign of zero; numpy's min / max leave it to the order of the values).
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_round

GROUP = 128


def asym_params(x, axis, bits):
    """(s, z) as float32 BF16 values of the groups of x reduced along `axis`."""
    a = np.asarray(x, dtype=np.float32)
    lo = np.min(a, axis=axis).astype(np.float32)
    hi = np.max(a, axis=axis).astype(np.float32)
    # a zero minimum or range is +0: numpy's reductions leave the sign of a
    # zero result to the order they visit the values in (adding +0 maps -0 to +0)
    z = bf16_round(lo) + np.float32(0.0)
    s = bf16_round((hi - lo).astype(np.float32) / np.float32(2 ** bits - 1)) + np.float32(0.0)
    return s, z


def asym_quantize(x, axis, bits):
    """(codes uint8, s, z): c = clamp(rint(f32(x - z) / s), 0, 2^b - 1) per
    group along `axis`; a zero scale gives code 0."""
    a = np.asarray(x, dtype=np.float32)
    s, z = asym_params(a, axis, bits)
    se = np.expand_dims(s, axis)
    ze = np.expand_dims(z, axis)
    safe = np.where(se == 0, np.float32(1.0), se).astype(np.float32)
    q = np.rint((a - ze).astype(np.float32) / safe)
    q = np.clip(q, 0, 2 ** bits - 1)
    q = np.where(se == 0, 0, q)
    return q.astype(np.uint8), s, z


def asym_dequantize(codes, s, z, axis) -> np.ndarray:
    """float64 values c * s + z, (s, z) broadcast along `axis`."""
    c = np.asarray(codes).astype(np.float64)
    return c * np.expand_dims(np.asarray(s, np.float64), axis) + np.expand_dims(np.asarray(z, np.float64), axis)


def quantize_sequence(K, V, bits=2, group=GROUP):
    """One sequence's cache as the format stores it.

    K, V: [n][Hk][D] BF16 values (as float32), positions in order.
    Returns dict: 'n_groups', 'k_codes' [g][group][Hk][D], 'k_s', 'k_z'
    [g][Hk][D], 'v_codes' [g*group][Hk][D], 'v_s', 'v_z' [g*group][Hk], and the
    residual 'k_res', 'v_res' [n - g*group][Hk][D] (BF16 values)."""
    K = np.asarray(K, dtype=np.float32)
    V = np.asarray(V, dtype=np.float32)
    n = K.shape[0]
    g = n // group
    m = g * group
    kg = K[:m].reshape(g, group, *K.shape[1:])
    kc, ks, kz = asym_quantize(kg, axis=1, bits=bits)          # per (group, head, channel)
    vc, vs, vz = asym_quantize(V[:m], axis=-1, bits=bits)      # per (position, head)
    return {"n_groups": g, "k_codes": kc, "k_s": ks, "k_z": kz, "v_codes": vc, "v_s": vs,
            "v_z": vz, "k_res": bf16_round(K[m:]), "v_res": bf16_round(V[m:])}


def dequantize_sequence(st, group=GROUP):
    """float64 K, V [n][Hk][D] of a quantize_sequence result: the quantized
    groups followed by the full-precision residual."""
    g = st["n_groups"]
    kq = asym_dequantize(st["k_codes"], st["k_s"], st["k_z"], axis=1)
    kq = kq.reshape(g * group, *kq.shape[2:]) if g else kq.reshape(0, *st["k_res"].shape[1:])
    vq = asym_dequantize(st["v_codes"], st["v_s"], st["v_z"], axis=-1)
    K = np.concatenate([kq, st["k_res"].astype(np.float64)])
    V = np.concatenate([vq.reshape(-1, *st["v_res"].shape[1:]), st["v_res"].astype(np.float64)])
    return K, V


def bytes_per_token(n_kv_heads, head_dim, bits=2, group=GROUP):
    """Stored bytes per quantized token (K and V, all KV heads): the codes, V's
    per-token (s, z), and K's per-group (s, z) spread over the group."""
    codes = 2 * n_kv_heads * head_dim * bits / 8
    v_meta = n_kv_heads * 4
    k_meta = n_kv_heads * head_dim * 4 / group
    return codes + v_meta + k_meta
