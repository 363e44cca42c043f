"""Codecs of the quantized KV cache: OCP FP8 E4M3 and E5M2, INT8 asymmetric,
BF16 scales.

Test infrastructure (see ``oracle/__init__``): plain numpy, element by element
in meaning, vectorised only for speed.

What the pages fix
------------------
* [LIMITS] "Formats you will actually meet": E4M3 carries more precision and
  less range than E5M2 and is the format used for K/V; INT8 per-token
  asymmetric gives each token's K and each token's V its own
  (scale, zero_point) pair.
* [COMPRESS] "3.1 Quantization techniques": E4M3 has 4 exponent and 3 mantissa
  bits. (That section quotes a +-240 range, which is the FNUZ variant; the OCP
  variant used here saturates at 448.)
* [LIMITS] "What KV cache quantization actually is": quantisation happens only
  when a token is stored, the scale is computed from the full BF16 values, and
  the per-token / per-head scales are themselves kept in BF16.

Readings taken where the pages are silent (each is a stated choice)
-------------------------------------------------------------------
* FP8 scale: ``s = bf16_rne(f32(amax) / 448)`` with an IEEE f32 division; the
  code is ``e4m3_rne_satfinite(f32(x) / f32(s))``, again an IEEE f32 division
  by the *stored* BF16 scale (no reciprocal multiply).
* E5M2 (the pages name it as the wider-range, lower-precision FP8 variant)
  follows the same rule with its own maximum: ``s = bf16_rne(amax / 57344)``,
  ``code = e5m2_rne_satfinite(x / s)``.
* INT8: codes are signed [-128, 127]; the range is widened to contain 0,
  ``s = bf16_rne((xmax - xmin) / 255)`` in f32,
  ``zp = clamp(-128 - rint(xmin / s), -128, 127)`` (an integer, exact in BF16),
  ``c = clamp(rint(x / s) + zp, -128, 127)``, ``deq = (c - zp) * s``;
  ``rint`` rounds half to even.
* A zero scale (all-zero row, or a BF16 underflow) stores ``s = 0, zp = 0`` and
  all-zero codes, so every value dequantises to 0.
* Per-channel and per-tensor INT8 ([LIMITS] "Formats you will actually meet":
  one scale per head_dim slice is faster on hardware and slightly less
  accurate; one scale for the whole cache is cheapest and loses most). The
  pages give one scale and no zero point, and say nothing of where the scale
  comes from; read as symmetric codes with a static BF16 scale fixed before
  the tokens arrive (given by the caller): ``c = clamp(rint(f32(x) / f32(s)),
  -127, 127)``, ``deq = c * s``; ``s <= 0`` stores code 0. Per channel means
  one scale per (KV head, channel), for K and for V separately; per tensor one
  for all of K and one for all of V. ``int8_static_calibrate`` is one way to
  fix such scales from sample data (max |x| / 127, rounded to BF16); the path
  takes them as inputs.
"""

from __future__ import annotations

import numpy as np
import torch

E4M3_MAX = 448.0
E4M3_NAN_CODE = 0x7F


# --------------------------------------------------------------------------- BF16
def bf16_round(x) -> np.ndarray:
    """Round f32 values to BF16 (round to nearest, ties to even); returned as f32.

    Uses the library conversion of PyTorch on the CPU (a library primitive)."""
    a = np.asarray(x, dtype=np.float32)
    t = torch.from_numpy(np.ascontiguousarray(a.reshape(-1)))
    return t.to(torch.bfloat16).to(torch.float32).numpy().reshape(a.shape)


def bf16_bits(x) -> np.ndarray:
    """The 16-bit pattern of BF16 values given as f32 (which must be exact BF16)."""
    a = np.asarray(x, dtype=np.float32)
    flat = np.ascontiguousarray(a.reshape(-1))
    return ((flat.view(np.uint32) >> 16).astype(np.uint16)).reshape(a.shape)


def bf16_from_bits(bits) -> np.ndarray:
    """f32 values of 16-bit BF16 patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


# --------------------------------------------------------------------------- E4M3
def e4m3_decode(codes) -> np.ndarray:
    """Value (float64) of each OCP E4M3 byte.

    Bit 7 is the sign, bits 6..3 the exponent field e (bias 7), bits 2..0 the
    mantissa m. e == 0 encodes subnormals m/8 * 2^-6; otherwise the value is
    (1 + m/8) * 2^(e - 7). The pattern e == 15, m == 7 is NaN; the format has
    no infinities, so the largest finite magnitude is (1 + 6/8) * 2^8 = 448.
    """
    c = np.asarray(codes).astype(np.int64) & 0xFF
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    subnormal = (m / 8.0) * 2.0 ** -6
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    val = sign * np.where(e == 0, subnormal, normal)
    return np.where((e == 15) & ((c & 0x7) == 7), np.nan, val)


# The 127 non-negative finite magnitudes, indexed by their code 0x00..0x7E.
# The code order is the value order, so this table is sorted.
_E4M3_MAGNITUDES = e4m3_decode(np.arange(0x7F))


def e4m3_encode(x) -> np.ndarray:
    """Encode f32 values to OCP E4M3 codes (uint8): round to nearest, ties to even,
    saturating to +-448.

    Definition used: the nearest finite E4M3 value to x (exact comparison in
    float64, where every f32 and every E4M3 value is exact). On a tie the code
    with an even mantissa (even code) wins. Magnitudes above 448 give 448
    ("satfinite"). The sign is kept, so negative values that round to zero
    give 0x80. NaN gives 0x7F.
    """
    xf = np.asarray(x, dtype=np.float32)
    mag = np.abs(xf.astype(np.float64))
    tab = _E4M3_MAGNITUDES
    hi = np.searchsorted(tab, mag, side="left")         # first magnitude >= |x|
    hi = np.clip(hi, 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    d_lo = mag - tab[lo]
    d_hi = tab[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(mag >= tab[hi], hi, code)            # exact hit (includes 0)
    code = np.where(mag >= E4M3_MAX, 0x7E, code)         # satfinite
    code = code.astype(np.int64)
    code = np.where(np.signbit(xf), code | 0x80, code)
    code = np.where(np.isnan(xf), E4M3_NAN_CODE, code)
    return code.astype(np.uint8)


# --------------------------------------------------------------------------- E5M2
E5M2_MAX = 57344.0
E5M2_NAN_CODE = 0x7F


def e5m2_decode(codes) -> np.ndarray:
    """Value (float64) of each OCP E5M2 byte.

    Bit 7 is the sign, bits 6..2 the exponent field e (bias 15), bits 1..0 the
    mantissa m. e == 0 encodes subnormals m/4 * 2^-14; e == 31 encodes +-inf
    (m == 0) and NaN (m != 0); otherwise the value is (1 + m/4) * 2^(e - 15),
    so the largest finite magnitude is (1 + 3/4) * 2^15 = 57344.
    """
    c = np.asarray(codes).astype(np.int64) & 0xFF
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    e = (c >> 2) & 0x1F
    m = (c & 0x3).astype(np.float64)
    subnormal = (m / 4.0) * 2.0 ** -14
    normal = (1.0 + m / 4.0) * np.exp2(e.astype(np.float64) - 15.0)
    val = sign * np.where(e == 0, subnormal, normal)
    val = np.where((e == 31) & ((c & 0x3) == 0), sign * np.inf, val)
    return np.where((e == 31) & ((c & 0x3) != 0), np.nan, val)


# The 124 non-negative finite magnitudes, codes 0x00..0x7B, in value order.
_E5M2_MAGNITUDES = e5m2_decode(np.arange(0x7C))


def e5m2_encode(x) -> np.ndarray:
    """Encode f32 values to OCP E5M2 codes (uint8): round to nearest, ties to even,
    saturating to +-57344 (infinities too). Same definition as e4m3_encode over
    the E5M2 value set: nearest finite value, the even code on a tie, the sign
    kept (-0 -> 0x80), NaN -> 0x7F.
    """
    xf = np.asarray(x, dtype=np.float32)
    mag = np.abs(xf.astype(np.float64))
    tab = _E5M2_MAGNITUDES
    top = len(tab) - 1                                    # 0x7B
    hi = np.clip(np.searchsorted(tab, mag, side="left"), 0, top)
    lo = np.clip(hi - 1, 0, top)
    d_lo = mag - tab[lo]
    d_hi = tab[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(mag >= tab[hi], hi, code)            # exact hit (includes 0)
    code = np.where(mag >= E5M2_MAX, top, code)          # satfinite
    code = code.astype(np.int64)
    code = np.where(np.signbit(xf), code | 0x80, code)
    code = np.where(np.isnan(xf), E5M2_NAN_CODE, code)
    return code.astype(np.uint8)


def e5m2_scale(rows) -> np.ndarray:
    """BF16 scale per row, as f32: ``s = bf16_rne(amax / 57344)`` (IEEE f32 division)."""
    r = np.asarray(rows, dtype=np.float32)
    amax = np.max(np.abs(r), axis=-1).astype(np.float32)
    return bf16_round(amax / np.float32(E5M2_MAX))


def e5m2_quantize(rows):
    """(codes uint8[..., D], scales f32[...]): code = e5m2_encode(f32(x) / f32(s))
    with the stored BF16 scale; a zero scale gives all-zero codes."""
    r = np.asarray(rows, dtype=np.float32)
    s = e5m2_scale(r)
    safe = np.where(s == 0.0, np.float32(1.0), s).astype(np.float32)
    codes = e5m2_encode(r / safe[..., None])
    codes = np.where((s == 0.0)[..., None], np.uint8(0), codes).astype(np.uint8)
    return codes, s


def e5m2_dequantize(codes, scales) -> np.ndarray:
    """float64 values of E5M2 codes: e5m2(c) * s, exact."""
    return e5m2_decode(codes) * np.asarray(scales, dtype=np.float64)[..., None]


# --------------------------------------------------------------------------- FP8 per-token scale
# All row functions take an array [..., D]: each row along the last axis is one
# token's K (or V) for one KV head, and gets its own scale.

def fp8_scale(rows) -> np.ndarray:
    """BF16 scale per row, as f32: ``s = bf16_rne(amax / 448)``.

    amax = max |x| over the head_dim values of the row (exact in f32); the
    division is an IEEE f32 division."""
    r = np.asarray(rows, dtype=np.float32)
    amax = np.max(np.abs(r), axis=-1).astype(np.float32)
    return bf16_round(amax / np.float32(E4M3_MAX))


def fp8_quantize(rows):
    """(codes uint8[..., D], scales f32[...]) for rows of K or V.

    code = e4m3_encode(f32(x) / f32(s)) with the stored BF16 scale s; a row
    whose scale is zero gets all-zero codes."""
    r = np.asarray(rows, dtype=np.float32)
    s = fp8_scale(r)
    safe = np.where(s == 0.0, np.float32(1.0), s).astype(np.float32)
    codes = e4m3_encode(r / safe[..., None])
    codes = np.where((s == 0.0)[..., None], np.uint8(0), codes).astype(np.uint8)
    return codes, s


def fp8_dequantize(codes, scales) -> np.ndarray:
    """float64 values of FP8 codes: e4m3(c) * s, exact (4 x 8 significant bits)."""
    return e4m3_decode(codes) * np.asarray(scales, dtype=np.float64)[..., None]


# --------------------------------------------------------------------------- INT8 asymmetric
def int8_params(rows):
    """(scales f32[...] holding BF16 values, zero_points int64[...]) per row.

    The range of a row is [xmin, xmax] widened to contain 0:
    xmin = min(0, min x), xmax = max(0, max x). In f32 with IEEE rounding,
    s = bf16_rne((xmax - xmin) / 255) and zp = clamp(-128 - rint(xmin / s),
    -128, 127), so that xmin lands on the lowest code -128. A zero scale gives
    (0, 0)."""
    r = np.asarray(rows, dtype=np.float32)
    xmin = np.minimum(np.float32(0.0), np.min(r, axis=-1)).astype(np.float32)
    xmax = np.maximum(np.float32(0.0), np.max(r, axis=-1)).astype(np.float32)
    span = (xmax - xmin).astype(np.float32)
    s = bf16_round(span / np.float32(255.0))
    safe = np.where(s == 0.0, np.float32(1.0), s).astype(np.float32)
    zp = -128 - np.rint(xmin / safe).astype(np.int64)
    zp = np.clip(zp, -128, 127)
    zp = np.where(s == 0.0, 0, zp).astype(np.int64)
    return s, zp


def int8_quantize(rows):
    """(codes int8[..., D], scales f32[...], zero_points int64[...]) for rows:
    c = clamp(rint(f32(x) / f32(s)) + zp, -128, 127); zero scale -> zero codes."""
    r = np.asarray(rows, dtype=np.float32)
    s, zp = int8_params(r)
    safe = np.where(s == 0.0, np.float32(1.0), s).astype(np.float32)
    q = np.rint(r / safe[..., None]).astype(np.int64) + zp[..., None]
    q = np.clip(q, -128, 127)
    q = np.where((s == 0.0)[..., None], 0, q)
    return q.astype(np.int8), s, zp


def int8_dequantize(codes, scales, zero_points) -> np.ndarray:
    """float64 values of INT8 codes: (c - zp) * s."""
    c = np.asarray(codes).astype(np.int64)
    zp = np.asarray(zero_points, dtype=np.int64)[..., None]
    return (c - zp).astype(np.float64) * np.asarray(scales, dtype=np.float64)[..., None]


def int8_clip_range(scales, zero_points):
    """Per row, the interval representable without clipping:
    [(-128 - zp) s, (127 - zp) s]."""
    s = np.asarray(scales, dtype=np.float64)
    zp = np.asarray(zero_points, dtype=np.int64)
    return (-128 - zp) * s, (127 - zp) * s


# --------------------------------------------------------------------------- INT8 symmetric, static scales
def int8_static_quantize(x, scales) -> np.ndarray:
    """int8 codes of values x[..., D] under given scales that broadcast against
    x (per channel: [Hk][D] against [..., Hk, D]; per tensor: a scalar):
    c = clamp(rint(f32(x) / f32(s)), -127, 127); 0 where s <= 0 or s is NaN."""
    r = np.asarray(x, dtype=np.float32)
    s = np.broadcast_to(np.asarray(scales, dtype=np.float32), r.shape)
    ok = s > 0
    safe = np.where(ok, s, np.float32(1.0)).astype(np.float32)
    with np.errstate(over="ignore"):
        q = np.rint(r / safe)
    q = np.clip(q, -127, 127)
    return np.where(ok, q, 0).astype(np.int8)


def int8_static_dequantize(codes, scales) -> np.ndarray:
    """float64 values of static-scale INT8 codes: c * s (s broadcast as in
    int8_static_quantize)."""
    c = np.asarray(codes).astype(np.float64)
    return c * np.broadcast_to(np.asarray(scales, dtype=np.float64), c.shape)


def int8_static_calibrate(x, per_channel=True) -> np.ndarray:
    """Static scales from sample values x[..., Hk, D]: bf16_rne(f32(max |x|) /
    127) over every axis but (Hk, D) (per channel, shape [Hk][D]) or over all
    of x (per tensor, shape [1])."""
    a = np.abs(np.asarray(x, dtype=np.float32))
    if per_channel:
        amax = a.reshape(-1, a.shape[-2], a.shape[-1]).max(axis=0)
    else:
        amax = np.array([a.max()], dtype=np.float32)
    return bf16_round(amax.astype(np.float32) / np.float32(127.0))

