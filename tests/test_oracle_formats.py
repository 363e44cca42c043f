"""Pins of the oracle's codecs against facts fixed outside the oracle.

Sources: "KV cache quantization: what FP8/INT8 K and V really give, and their
limits" (notes under the formats table: E4M3 for K/V, INT8 per-token
asymmetric with a (scale, zero_point) pair); "KV Cache compression", section
3.1 (E4M3 = 4 exponent + 3 mantissa bits). OCP FP8 E4M3 is the variant (max
448, no infinities, one NaN pattern per sign).

Each pin comes from somewhere the oracle does not: PyTorch's float8_e4m3fn
library conversion, a brute-force nearest search, an integer bit-level
rounding written here, hand-worked rows under tests/golden/, and the INT8
error bound of the affine quantiser.
"""

from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import formats as F
from tests.conftest import read_golden

# ----------------------------------------------------------------------------- helpers (independent)


def f32_bits(x):
    return np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.int64)


def e4m3_by_bits(x):
    """f32 -> E4M3 code by integer rounding of the f32 bit pattern (RNE, satfinite).

    Written from IEEE binary32 and OCP E4M3, independently of the oracle: the
    24-bit significand is shifted down to the target precision and rounded
    with the usual guard/sticky rule."""
    out = []
    for b in f32_bits(np.ravel(x)).tolist():
        sign = (b >> 31) & 1
        e = (b >> 23) & 0xFF
        m = b & 0x7FFFFF
        if e == 0xFF:
            out.append(0x7F if m else (0x7E | (sign << 7)))
            continue
        if e == 0:                      # f32 subnormal: far below 2^-10 -> zero
            out.append(sign << 7)
            continue
        sig = m | 0x800000              # value = sig * 2^(e - 150)
        E = e - 127                     # value in [2^E, 2^(E+1))
        if E >= -6:                     # E4M3 normal range: keep 4 significant bits
            shift = 20
        else:                           # E4M3 subnormal: multiples of 2^-9
            shift = 20 + (-6 - E)
        if shift >= 32:
            out.append(sign << 7)
            continue
        q = sig >> shift
        rem = sig & ((1 << shift) - 1)
        half = 1 << (shift - 1)
        if rem > half or (rem == half and (q & 1)):
            q += 1
        if E >= -6:
            if q == 16:                 # carried into the next binade
                q = 8
                E += 1
            code_e = E + 7
            mant = q - 8
            if code_e > 15 or (code_e == 15 and mant == 7):
                code = 0x7E             # satfinite
            else:
                code = (code_e << 3) | mant
        else:
            code = q                    # q in 0..8; q == 8 is the smallest normal 2^-6 (code 0x08)
        out.append(code | (sign << 7))
    return np.asarray(out, dtype=np.uint8).reshape(np.shape(x))


def e4m3_brute_force(x):
    """Nearest finite E4M3 value with the sign of x, ties to the even code: a
    plain search over the 127 codes of that sign, with exact rational distances."""
    vals = [Fraction(v) if np.isfinite(v) else None for v in F.e4m3_decode(np.arange(256)).tolist()]
    out = []
    for xv in np.ravel(np.asarray(x, dtype=np.float32)).astype(np.float64).tolist():
        if np.isnan(xv):
            out.append(0x7F)
            continue
        codes = range(0x80, 0xFF) if np.signbit(xv) else range(0x00, 0x7F)
        if np.isinf(xv):
            out.append(0xFE if xv < 0 else 0x7E)    # nearest finite to an infinity
            continue
        xq = Fraction(xv)
        best, pick = None, None
        for c in codes:
            d = abs(vals[c] - xq)
            if best is None or d < best or (d == best and c % 2 == 0):
                best, pick = d, c
        out.append(pick)
    return np.asarray(out, dtype=np.uint8).reshape(np.shape(x))


def bf16_by_bits(x):
    """f32 -> BF16 (as f32) by integer round-to-nearest-even on the bit pattern."""
    b = f32_bits(x)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return (r & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


# ----------------------------------------------------------------------------- E4M3 decode


def test_e4m3_decode_matches_torch_float8_for_all_256_codes():
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = F.e4m3_decode(codes)
    assert np.array_equal(np.isnan(lib), np.isnan(ours))
    fin = ~np.isnan(lib)
    assert np.array_equal(lib[fin], ours[fin])
    assert np.array_equal(np.signbit(lib[fin]), np.signbit(ours[fin]))


def test_e4m3_decode_value_set_and_landmarks():
    # the positive finite values: 8 subnormals m * 2^-9, then (8 + m) * 2^(e - 10)
    expect = sorted({m * 2.0 ** -9 for m in range(8)} |
                    {(8 + m) * 2.0 ** (e - 10) for e in range(1, 16) for m in range(8)
                     if not (e == 15 and m == 7)})
    got = F.e4m3_decode(np.arange(0x7F))
    assert list(got) == expect
    assert np.all(np.diff(got) > 0)                      # code order == value order
    assert np.array_equal(F.e4m3_decode(np.arange(0x80, 0xFF)), -got)
    lm = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
          0x38: 1.0, 0x76: 224.0, 0x6E: 112.0, 0x7E: 448.0, 0xFE: -448.0}
    for c, v in lm.items():
        assert F.e4m3_decode(np.array([c]))[0] == v
    assert np.isnan(F.e4m3_decode(np.array([0x7F, 0xFF]))).all()
    assert np.signbit(F.e4m3_decode(np.array([0x80]))[0])


# ----------------------------------------------------------------------------- E4M3 encode


def test_e4m3_round_trip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = F.e4m3_decode(codes).astype(np.float32)
    vals[codes == 0x80] = np.float32(-0.0)
    assert np.array_equal(F.e4m3_encode(vals), codes)


def test_e4m3_encode_special_cases():
    cases = [
        (0.0, 0x00), (-0.0, 0x80), (-1e-30, 0x80), (1e-30, 0x00),
        (2.0 ** -10, 0x00),            # tie between 0 and 2^-9 -> even code 0
        (3 * 2.0 ** -10, 0x02),        # tie between 2^-9 (0x01) and 2^-8 (0x02) -> even
        (2.0 ** -10 * 1.0000001, 0x01),
        (448.0, 0x7E), (449.0, 0x7E), (464.0, 0x7E), (480.0, 0x7E), (1e6, 0x7E),
        (float("inf"), 0x7E), (-float("inf"), 0xFE), (-500.0, 0xFE),
        (1.0, 0x38), (1.0625, 0x38),   # 1 + 1/16 is the tie between 1 and 1.125 -> even (1.0)
        (1.1875, 0x3A),                # tie between 1.125 (0x39) and 1.25 (0x3A) -> even
        (240.0, 0x77), (232.0, 0x76),  # 232 is the tie between 224 (0x76) and 240 (0x77)
    ]
    xs = np.array([c[0] for c in cases], dtype=np.float32)
    want = np.array([c[1] for c in cases], dtype=np.uint8)
    assert np.array_equal(F.e4m3_encode(xs), want), (F.e4m3_encode(xs), want)
    assert F.e4m3_encode(np.array([np.nan], dtype=np.float32))[0] == 0x7F


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32) * np.float32(40),
        (rng.random(200_000).astype(np.float32) - np.float32(0.5)) * np.float32(920),
        rng.standard_normal(50_000).astype(np.float32) * np.float32(0.01),
    ])
    x = x[np.abs(x) < 464]                  # torch turns >= 480 into NaN instead of saturating
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_encode(x), lib)


def test_e4m3_encode_exhaustive_bf16_vs_brute_force_and_bits():
    bits = np.arange(1 << 16, dtype=np.uint32)
    x = (bits << 16).view(np.float32)
    x = x[~np.isnan(x)]
    ours = F.e4m3_encode(x)
    assert np.array_equal(ours, e4m3_by_bits(x))
    # the brute-force search is slow in Python: check a stride of the set plus all
    # values within the E4M3 range
    sel = np.concatenate([np.arange(0, x.size, 37), np.nonzero(np.abs(x) <= 480)[0][::3]])
    assert np.array_equal(ours[sel], e4m3_brute_force(x[sel]))


def test_e4m3_encode_tie_neighbourhoods_vs_bits():
    vals = F.e4m3_decode(np.arange(0x7F))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)    # exact in f32
    near = []
    for m in mids:
        b = int(np.array([m], dtype=np.float32).view(np.uint32)[0])
        for d in (-2, -1, 0, 1, 2):
            if b + d >= 0:
                near.append(np.array([b + d], dtype=np.uint32).view(np.float32)[0])
    near = np.array(near, dtype=np.float32)
    near = np.concatenate([near, -near])
    ours = F.e4m3_encode(near)
    assert np.array_equal(ours, e4m3_by_bits(near))
    assert np.array_equal(ours, e4m3_brute_force(near))


def test_e4m3_encode_random_f32_vs_bits():
    rng = np.random.default_rng(7)
    b = rng.integers(0, 1 << 32, size=300_000, dtype=np.uint64).astype(np.uint32)
    x = b.view(np.float32)
    x = x[~np.isnan(x)]
    assert np.array_equal(F.e4m3_encode(x), e4m3_by_bits(x))


# ----------------------------------------------------------------------------- BF16


def test_bf16_round_matches_bit_rounding():
    rng = np.random.default_rng(3)
    b = rng.integers(0, 1 << 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    x = b.view(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) < 3e38)]
    ties = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)], dtype=np.float32)
    x = np.concatenate([x, ties])
    assert np.array_equal(F.bf16_round(x).view(np.uint32), bf16_by_bits(x).view(np.uint32))
    assert F.bf16_round(np.float32(1 + 2.0 ** -8)) == 1.0               # tie -> even
    assert F.bf16_round(np.float32(1 + 3 * 2.0 ** -8)) == 1 + 2.0 ** -6  # tie -> even (up)


# ----------------------------------------------------------------------------- FP8 rows


def test_fp8_worked_row():
    rows = read_golden("fp8_worked_row.txt")
    scale_bits = int(rows[0][1], 16)
    xs = np.array([float(r[0]) for r in rows[1:]], dtype=np.float32)
    want = np.array([int(r[1], 16) for r in rows[1:]], dtype=np.uint8)
    codes, s = F.fp8_quantize(xs)
    assert int(F.bf16_bits(s)) == scale_bits
    assert np.array_equal(codes, want)


def test_fp8_scale_special_rows():
    codes, s = F.fp8_quantize(np.zeros((3, 64), dtype=np.float32))
    assert np.all(s == 0) and np.all(codes == 0)
    row = np.linspace(-448, 448, 64, dtype=np.float32)
    row = F.bf16_round(row)
    codes, s = F.fp8_quantize(row)
    assert s == 1.0                                  # amax 448 -> scale exactly 1
    assert np.array_equal(codes, F.e4m3_encode(row))
    # a scale that underflows BF16 (amax tiny) stores zero and zero codes
    tiny = np.full(8, 1e-45, dtype=np.float32)
    codes, s = F.fp8_quantize(tiny)
    assert s == 0 and np.all(codes == 0)


def test_fp8_error_bound_random_rows():
    """Inside the E4M3 range the stored value is within half a step of x:
    |x - deq| <= |x| / 16 for E4M3 normals and <= 2^-10 s for subnormals."""
    rng = np.random.default_rng(11)
    rows = F.bf16_round(rng.standard_normal((2000, 128)).astype(np.float32) *
                        np.exp(rng.normal(0, 3, size=(2000, 1))).astype(np.float32))
    codes, s = F.fp8_quantize(rows)
    deq = F.fp8_dequantize(codes, s)
    x = rows.astype(np.float64)
    in_range = np.abs(x / s[:, None]) <= 448
    bound = np.maximum(np.abs(x) / 16, 2.0 ** -10 * s[:, None]) * (1 + 2.0 ** -20)
    assert np.all(np.abs(x - deq)[in_range] <= bound[in_range])
    # the largest element may saturate only because s was rounded down to BF16
    amax_deq = np.max(np.abs(deq), axis=1)
    assert np.all(amax_deq <= 448 * s + 0)


# ----------------------------------------------------------------------------- INT8 rows


def test_int8_worked_rows():
    for name, vals, sbits, zp, codes in read_golden("int8_worked_rows.txt"):
        x = np.array([float(t) for t in vals.split()], dtype=np.float32)
        c, s, z = F.int8_quantize(x)
        assert int(F.bf16_bits(s)) == int(sbits, 16), name
        assert int(z) == int(zp), name
        assert c.tolist() == [int(t) for t in codes.split()], name


def _int8_rows():
    rng = np.random.default_rng(5)
    rows = [rng.normal(0.3, 1.0, size=(500, 128)),
            rng.normal(0.0, 1.0, size=(500, 128)) * 50,
            np.abs(rng.normal(0, 1, size=(200, 128))),            # all positive
            -np.abs(rng.normal(0, 1, size=(200, 128))),           # all negative
            np.full((5, 128), 3.25), np.full((5, 128), -0.7),     # all equal
            np.zeros((5, 128))]
    spike = rng.normal(0, 1, size=(50, 128))
    spike[:, 17] = 400.0                                          # one outlier per row
    rows.append(spike)
    return F.bf16_round(np.concatenate(rows).astype(np.float32))


def test_int8_half_scale_bound_inside_clip_range():
    x = _int8_rows()
    c, s, zp = F.int8_quantize(x)
    deq = F.int8_dequantize(c, s, zp)
    lo, hi = F.int8_clip_range(s, zp)
    xd = x.astype(np.float64)
    inside = (xd >= lo[:, None]) & (xd <= hi[:, None])
    # s/2 exactly, plus the f32 rounding of x/s (one ulp of a value below 2^8)
    slack = np.abs(xd / np.where(s == 0, 1, s)[:, None]) * 2.0 ** -23 * s[:, None]
    err = np.abs(xd - deq)
    assert np.all(err[inside] <= (s[:, None] / 2 + slack)[inside])
    assert np.all((c >= -128) & (c <= 127))
    zero_rows = s == 0
    assert np.all(c[zero_rows] == 0) and np.all(deq[zero_rows] == 0)
    # the clip range covers nearly all of [xmin, xmax]: only the BF16 rounding of s
    # may leave the very ends outside
    frac_outside = 1 - inside[~zero_rows].mean()
    assert frac_outside < 0.01


def test_int8_brute_force_small_rows():
    rng = np.random.default_rng(9)
    for _ in range(200):
        x = F.bf16_round(rng.normal(rng.normal(0, 2), abs(rng.normal(0, 3)) + 1e-3,
                                    size=6).astype(np.float32))
        c, s, zp = F.int8_quantize(x)
        if s == 0:
            continue
        for xi, ci in zip(x.tolist(), c.tolist()):
            t = np.float32(xi) / np.float32(s)               # the f32 quotient
            cands = np.arange(-128, 128)
            d = np.abs((cands - zp).astype(np.float64) - np.float64(t))
            best = d.min()
            ok = cands[d == best]
            ok = ok[(ok - zp) % 2 == 0] if ok.size > 1 else ok  # half-way -> even integer
            assert ci == ok[0]


def test_int8_zero_point_landmarks():
    # all positive rows: xmin widened to 0 -> zp = -128; all negative: xmax = 0
    c, s, zp = F.int8_quantize(np.array([[1.0, 2.0, 4.0]], dtype=np.float32))
    assert zp[0] == -128 and c[0, 0] >= -128
    c, s, zp = F.int8_quantize(np.array([[-1.0, -2.0, -4.0]], dtype=np.float32))
    assert c[0].min() == -128
    # symmetric range: zp near 0
    c, s, zp = F.int8_quantize(np.array([[-3.0, 3.0]], dtype=np.float32))
    assert abs(int(zp[0])) <= 1


# ----------------------------------------------------------------------------- scale rounding


def _scale_rows():
    rows = read_golden("fp8_scale_rounding.txt")
    return [(fmt, np.float32(amax), int(bits, 16)) for fmt, amax, bits, _ in rows]


def test_scale_rounding_rows_are_exact_f32_inputs():
    """The fixture's amax values are f32 numbers as written (no rounding on read)."""
    for fmt, amax, _ in _scale_rows():
        assert float(amax) == float(np.float64(amax))


def test_fp8_and_e5m2_scale_rounding_rows():
    """Hand-worked scales: RNE of the f32 quotient, ties to even, IEEE division.
    Each row puts amax at the front of a row of smaller values, so the scale is
    taken through the full quantize path too."""
    for fmt, amax, bits in _scale_rows():
        row = np.array([amax, amax / np.float32(4), -amax / np.float32(8)], dtype=np.float32)
        if fmt == "fp8":
            s = F.fp8_scale(row)
            _, s2 = F.fp8_quantize(row)
        else:
            s = F.e5m2_scale(row)
            _, s2 = F.e5m2_quantize(row)
        assert int(F.bf16_bits(s)) == bits, (fmt, float(amax), hex(int(F.bf16_bits(s))), hex(bits))
        assert int(F.bf16_bits(s2)) == bits
        # the sign of amax does not matter
        s3 = F.fp8_scale(-row) if fmt == "fp8" else F.e5m2_scale(-row)
        assert int(F.bf16_bits(s3)) == bits


def test_e5m2_worked_row():
    rows = read_golden("e5m2_worked_row.txt")
    scale_bits = int(rows[0][1], 16)
    xs = np.array([float(r[0]) for r in rows[1:]], dtype=np.float32)
    want = np.array([int(r[1], 16) for r in rows[1:]], dtype=np.uint8)
    codes, s = F.e5m2_quantize(xs)
    assert int(F.bf16_bits(s)) == scale_bits
    assert np.array_equal(codes, want)
