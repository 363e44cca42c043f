"""The decode kernel multiplies the stored codes on the tensor cores, so the
other operand (the query of S = K·q, the softmax weights of O = V·P) has to be
given in the codes' own operand type. It is split into parts whose weighted sum
restores it. This file checks, on the host, the precision each split claims
(the kernel's arithmetic restated in numpy float32; the E4M3 rounding is the
oracle's codec, which is pinned against PyTorch's float8_e4m3fn elsewhere):

* query, FP8 cache: x = q * 2^e with max |x| in [128, 256); hi = E4M3(x),
  lo = E4M3(16 (x - hi)); hi + lo / 16 equals x exactly for every BF16 x with
  2^-6 <= |x| < 256 (both parts inside E4M3's range and precision);
* query, INT8 cache: x in [-64, 64); three integer parts (weights 1, 2^-7,
  2^-14), each inside the s8 range; error at most 2^-15;
* weights, FP8 cache: y in [0, 256) (the largest weight of a tile lands in
  [128, 256)); four E4M3 parts, each the rounded residual of the part before
  times 16; relative error at most 2^-18 for y >= 1/4, and at most 2^-11
  absolute (2^-18 of the tile's largest weight) below, where the last parts
  fall into E4M3's subnormal range;
* weights, INT8 cache: Y = rint(y 2^16) < 2^24 split into three bytes that
  restore Y exactly;
* weights, BF16 cache: hi + mid + lo of three BF16 roundings, relative error
  at most 2^-24.

"What KV cache quantization actually is" ("KV cache quantization: what
FP8/INT8 K and V really give") puts the dequantized product right before the
matmuls; these splits are how the kernel forms that product from the codes
without converting them.
"""

import numpy as np

from oracle import formats as F


def _e4m3(x):
    return F.e4m3_decode(F.e4m3_encode(np.asarray(x, np.float32))).astype(np.float32)


def _all_bf16(lo, hi):
    """Every positive BF16 value in [lo, hi), as float32."""
    bits = (np.arange(0x0000, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    return bits[(bits >= lo) & (bits < hi)]


def test_fp8_query_parts_are_exact_for_every_bf16():
    x = _all_bf16(2.0 ** -6, 256.0)
    x = np.concatenate([x, -x])
    hi = _e4m3(x)
    lo = _e4m3(np.float32(16.0) * (x - hi))
    assert np.array_equal(hi + lo / np.float32(16.0), x)


def test_int8_query_parts():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.uniform(-64, 64, 200_000), [-64.0, -63.5, 0.5, 63.49]]).astype(np.float32)
    x0 = np.rint(x)
    r0 = (x - x0) * np.float32(128)
    x1 = np.rint(r0)
    x2 = np.rint((r0 - x1) * np.float32(128))
    for p in (x0, x1, x2):
        assert np.all(np.abs(p) <= 64)
    back = x0.astype(np.float64) + x1 / 128.0 + x2 / 16384.0
    assert np.max(np.abs(back - x)) <= 2.0 ** -15


def test_fp8_weight_parts():
    rng = np.random.default_rng(2)
    y = np.concatenate([rng.uniform(0, 256, 100_000), 2.0 ** rng.uniform(-12, 8, 100_000)]).astype(np.float32)
    parts, r = [], y.copy()
    for j in range(4):
        p = _e4m3(r)
        parts.append(p)
        r = (r - p) * np.float32(16.0)
    back = sum(p.astype(np.float64) / 16.0 ** j for j, p in enumerate(parts))
    err = np.abs(back - y)
    big = y >= 0.25
    assert np.all(err[big] <= 2.0 ** -18 * y[big])
    assert np.all(err <= 2.0 ** -11)


def test_int8_weight_bytes():
    rng = np.random.default_rng(3)
    y = rng.uniform(0, 255.99, 100_000).astype(np.float32)
    Y = np.rint(y.astype(np.float64) * 65536).astype(np.int64)
    assert np.all(Y < 2 ** 24)
    b2, b1, b0 = (Y >> 16) & 0xFF, (Y >> 8) & 0xFF, Y & 0xFF
    assert np.array_equal(b2 * 65536 + b1 * 256 + b0, Y)
    assert np.all(np.abs(Y / 65536.0 - y) <= 2.0 ** -17)


def test_bf16_weight_parts():
    rng = np.random.default_rng(4)
    p = rng.uniform(0, 1, 200_000).astype(np.float32)
    hi = F.bf16_round(p)
    r1 = p - hi
    mid = F.bf16_round(r1)
    lo = F.bf16_round(r1 - mid)
    back = hi.astype(np.float64) + mid + lo
    assert np.all(np.abs(back - p) <= 2.0 ** -24 * p + 1e-45)


def test_a_single_fp8_query_part_is_not_enough():
    """Planted simplification: hi alone loses the low mantissa bits of BF16."""
    x = _all_bf16(1.0, 256.0)
    assert not np.array_equal(_e4m3(x), x)
