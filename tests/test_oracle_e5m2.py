"""Pins of the oracle's E5M2 codec ("KV cache quantization: what FP8/INT8 K and V
really give" "Formats you will actually meet": E5M2 is the FP8 variant with
more range and less precision than E4M3; OCP definition: 5 exponent bits, bias
15, 2 mantissa bits, infinities and NaNs at exponent 31, largest finite 57344).

Pinned against PyTorch's float8_e5m2 (a library implementation of the same
definition), the value set written out from the definition, an exact-rational
brute-force nearest search, and the error bound of round-to-nearest.
"""

from fractions import Fraction

import numpy as np
import torch

from oracle import formats as F
from oracle import paged as P
from oracle import sizes as S


def _brute(x):
    """Nearest finite E5M2 value by exact rational comparison; ties to the even
    code; saturating; the sign kept."""
    vals = [Fraction(float(v)) for v in F.e5m2_decode(np.arange(0x7C))]
    out = []
    for xi in np.asarray(x, dtype=np.float32):
        mag = abs(Fraction(float(xi)))
        best, bd = 0, None
        for c, v in enumerate(vals):
            d = abs(v - mag)
            if bd is None or d < bd or (d == bd and c % 2 == 0):
                best, bd = c, d
        if mag >= Fraction(57344):
            best = 0x7B
        if np.signbit(xi):
            best |= 0x80
        out.append(best)
    return np.array(out, dtype=np.uint8)


def test_e5m2_decode_matches_torch_for_all_256_codes():
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes.copy()).view(torch.float8_e5m2).to(torch.float64).numpy()
    ours = F.e5m2_decode(codes)
    assert np.array_equal(np.isnan(lib), np.isnan(ours))
    fin = ~np.isnan(lib)
    assert np.array_equal(lib[fin], ours[fin])
    assert np.array_equal(np.signbit(lib[fin]), np.signbit(ours[fin]))


def test_e5m2_value_set_and_landmarks():
    # positive finite values: 4 subnormals m * 2^-16, then (4 + m) * 2^(e - 17), e = 1..30
    expect = sorted({m * 2.0 ** -16 for m in range(4)} |
                    {(4 + m) * 2.0 ** (e - 17) for e in range(1, 31) for m in range(4)})
    got = F.e5m2_decode(np.arange(0x7C))
    assert list(got) == expect
    assert np.all(np.diff(got) > 0)
    lm = {0x00: 0.0, 0x01: 2.0 ** -16, 0x04: 2.0 ** -14, 0x3C: 1.0, 0x3D: 1.25,
          0x7B: 57344.0, 0xFB: -57344.0}
    for c, v in lm.items():
        assert F.e5m2_decode(np.array([c]))[0] == v
    assert F.e5m2_decode(np.array([0x7C]))[0] == np.inf
    assert F.e5m2_decode(np.array([0xFC]))[0] == -np.inf
    assert np.isnan(F.e5m2_decode(np.array([0x7D, 0x7E, 0x7F, 0xFF]))).all()


def test_e5m2_round_trip_all_finite_codes():
    codes = np.array([c for c in range(256) if (c & 0x7F) < 0x7C], dtype=np.uint8)
    vals = F.e5m2_decode(codes).astype(np.float32)
    vals[codes == 0x80] = np.float32(-0.0)
    assert np.array_equal(F.e5m2_encode(vals), codes)


def test_e5m2_encode_special_cases():
    cases = [
        (0.0, 0x00), (-0.0, 0x80), (2.0 ** -17, 0x00),    # tie between 0 and 2^-16 -> even 0
        (3 * 2.0 ** -17, 0x02),                            # tie 2^-16 / 2^-15 -> even code 0x02
        (1.0, 0x3C), (1.125, 0x3C),                        # tie between 1 and 1.25 -> even (1.0)
        (1.375, 0x3E),                                     # tie between 1.25 and 1.5 -> even 0x3E
        (57344.0, 0x7B), (60000.0, 0x7B), (1e9, 0x7B),     # saturating
        (float("inf"), 0x7B), (-float("inf"), 0xFB),
    ]
    xs = np.array([c[0] for c in cases], dtype=np.float32)
    want = np.array([c[1] for c in cases], dtype=np.uint8)
    assert np.array_equal(F.e5m2_encode(xs), want), (F.e5m2_encode(xs), want)
    assert F.e5m2_encode(np.array([np.nan], dtype=np.float32))[0] == 0x7F


def test_e5m2_encode_matches_torch_in_range():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32) * np.float32(3000),
        rng.standard_normal(100_000).astype(np.float32) * np.float32(1e-3),
        (rng.random(100_000).astype(np.float32) - np.float32(0.5)) * np.float32(120000),
    ])
    x = x[np.abs(x) < 61440]                # torch overflows to inf from the 57344/inf midpoint
    lib = torch.from_numpy(x).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(F.e5m2_encode(x), lib)


def test_e5m2_encode_ties_vs_exact_brute_force():
    vals = F.e5m2_decode(np.arange(0x7C))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)      # exact in f32
    near = []
    for m in mids[::3]:
        b = int(np.array([m], dtype=np.float32).view(np.uint32)[0])
        for d in (-1, 0, 1):
            near.append(np.array([b + d], dtype=np.uint32).view(np.float32)[0])
    near = np.array(near, dtype=np.float32)
    near = np.concatenate([near, -near, np.array([57344, 70000, -1e6], dtype=np.float32)])
    assert np.array_equal(F.e5m2_encode(near), _brute(near))


def test_e5m2_quantize_error_bound_and_zero_rows():
    rng = np.random.default_rng(5)
    rows = (rng.standard_normal((400, 128)) * rng.uniform(0.01, 50, size=(400, 1))).astype(np.float32)
    rows[:3] = 0.0
    c, s = F.e5m2_quantize(rows)
    assert np.all(s[:3] == 0) and np.all(c[:3] == 0)
    deq = F.e5m2_dequantize(c, s)
    # RNE to 3 significant bits: |err| <= 2^-3 |x / s| * s, plus half the subnormal
    # spacing 2^-17 * s, plus the f32 rounding of x / s
    x = rows.astype(np.float64)
    bound = (2.0 ** -3 * np.abs(x) + 2.0 ** -17 * s[:, None] +
             np.abs(x) * 2.0 ** -23)
    assert np.all(np.abs(x - deq) <= bound)
    # the scale maps the row maximum onto the top of the E5M2 range
    amax = np.max(np.abs(x[3:]), axis=1)
    top = np.abs(F.e5m2_decode(c[3:])).max(axis=1) * s[3:]
    assert np.all(np.abs(top - amax) <= 2.0 ** -3 * amax)


def test_e5m2_pool_and_sizes():
    pool = P.LogicalPool("e5m2", 4, 2, 16, 64)
    rng = np.random.default_rng(2)
    k = rng.standard_normal((5, 2, 64)).astype(np.float32)
    v = rng.standard_normal((5, 2, 64)).astype(np.float32)
    pool.append(k, v, np.array([0, 1, 17, 33, 50]))
    K, V = pool.gather(np.array([0, 1, 2, 3]), 2)
    c, s = F.e5m2_quantize(k[:2])
    assert np.array_equal(K, F.e5m2_dequantize(c, s))
    assert S.kv_bytes(1, 8, 128, 4096, 1, S.BYTES_PER_ELEMENT["e5m2"]) == \
        S.kv_bytes(1, 8, 128, 4096, 1, S.BYTES_PER_ELEMENT["fp8"])
    assert S.scale_bytes(1, 8, 100, 2, "e5m2") == S.scale_bytes(1, 8, 100, 2, "fp8")


def test_a_wrong_exponent_bias_is_caught():
    """Planted mistake: decode with bias 16 instead of 15 fails the library check."""
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes.copy()).view(torch.float8_e5m2).to(torch.float64).numpy()
    wrong = F.e5m2_decode(codes) / 2.0
    fin = np.isfinite(lib) & (lib != 0)
    assert not np.array_equal(lib[fin], wrong[fin])
