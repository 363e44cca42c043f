"""Pins of the oracle's static-scale INT8 codec ("KV cache quantization: what
FP8/INT8 K and V really give", "Formats you will actually meet": a per-channel
scale per head_dim slice, or one per-tensor scale, beside per-token INT8).

The reading: symmetric codes c = clamp(rint(x / s), -127, 127) with a given
BF16 scale s, dequantised as c * s. Pinned by hand-worked values, the
round-to-nearest error bound, an exact-rational brute-force nearest code on
small inputs, broadcasting identities, the calibration rule's landmarks and
planted mistakes.
"""

from fractions import Fraction

import numpy as np

from oracle import formats as F
from oracle import paged as P
from oracle import sizes as S


def test_hand_worked_codes():
    s = np.float32(0.5)
    #            x:  0   -0   0.5  -0.5  0.25  0.75  1.25  -1.25  63.5  63.75  64   -70
    x = np.array([0, -0.0, 0.5, -0.5, 0.25, 0.75, 1.25, -1.25, 63.5, 63.75, 64, -70], np.float32)
    # x / s:        0    0    1    -1   0.5   1.5   2.5   -2.5   127  127.5  128  -140
    want = [0, 0, 1, -1, 0, 2, 2, -2, 127, 127, 127, -127]   # ties to even, saturation at +-127
    assert F.int8_static_quantize(x, s).tolist() == want


def test_zero_and_nan_scales_give_zero_codes():
    x = np.array([[1.0, -3.0], [5.0, 7.0]], np.float32)
    sc = np.array([[0.0, np.nan], [-1.0, 0.5]], np.float32)
    assert F.int8_static_quantize(x, sc).tolist() == [[0, 0], [0, 14]]


def test_error_bound_inside_the_range():
    rng = np.random.default_rng(3)
    s = F.bf16_round(rng.uniform(1e-3, 10, size=(4, 64)).astype(np.float32))
    x = (rng.uniform(-127, 127, size=(500, 4, 64)) * s).astype(np.float32)
    c = F.int8_static_quantize(x, s)
    deq = F.int8_static_dequantize(c, s)
    # half a step, plus one f32 rounding of x / s
    bound = s.astype(np.float64) / 2 + np.abs(x.astype(np.float64)) * 2.0 ** -23
    assert np.all(np.abs(deq - x) <= bound)


def test_brute_force_nearest_code():
    rng = np.random.default_rng(4)
    s = np.float32(0.375)
    x = np.concatenate([(rng.standard_normal(300) * 30).astype(np.float32),
                        (np.arange(-130, 131) * np.float32(0.1875)).astype(np.float32)])   # ties
    got = F.int8_static_quantize(x, s)
    for xi, ci in zip(x, got):
        q = Fraction(float(xi)) / Fraction(float(s))        # exact quotient; its f32 rounding
        # crosses no half-integer for these inputs (the ties are exact in f32)
        best = min(range(-127, 128), key=lambda c: (abs(q - c), c % 2))   # nearest, ties to even
        assert ci == best, (xi, ci, best)


def test_per_tensor_is_per_channel_with_equal_entries():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((50, 3, 16)).astype(np.float32) * 4
    s = np.float32(0.0625)
    a = F.int8_static_quantize(x, np.array([s], np.float32))
    b = F.int8_static_quantize(x, np.full((3, 16), s, np.float32))
    assert np.array_equal(a, b)


def test_calibration_maps_the_maximum_to_the_top_code():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((200, 2, 8)).astype(np.float32) * np.arange(1, 9, dtype=np.float32)
    x = F.bf16_round(x)
    sc = F.int8_static_calibrate(x, per_channel=True)
    assert sc.shape == (2, 8)
    assert np.array_equal(sc, F.bf16_round(np.abs(x).max(axis=0) / np.float32(127)))
    c = F.int8_static_quantize(x, sc)
    assert np.all(np.abs(c).reshape(-1, 16).max(axis=0) == 127)
    st = F.int8_static_calibrate(x, per_channel=False)
    assert st.shape == (1,) and st[0] == F.bf16_round(np.float32(np.abs(x).max()) / np.float32(127))


def test_pool_stores_static_codes():
    rng = np.random.default_rng(7)
    ks = F.bf16_round(rng.uniform(0.01, 0.05, size=(2, 32)).astype(np.float32))
    vs = F.bf16_round(np.array([0.02], np.float32))
    pool = P.LogicalPool("int8c", 4, 2, 16, 32, k_static=ks, v_static=ks)
    k = rng.standard_normal((5, 2, 32)).astype(np.float32)
    v = rng.standard_normal((5, 2, 32)).astype(np.float32)
    pool.append(k, v, np.array([0, 1, 17, 33, 50]))
    K, V = pool.gather(np.array([0, 1, 2, 3]), 2)
    assert np.array_equal(K, F.int8_static_dequantize(F.int8_static_quantize(k[:2], ks), ks))
    pt = P.LogicalPool("int8t", 4, 2, 16, 32, k_static=vs, v_static=vs)
    pt.append(k, v, np.array([0, 1, 17, 33, 50]))
    K, _ = pt.gather(np.array([0, 1]), 2)
    assert np.array_equal(K, F.int8_static_quantize(k[:2], vs[0]).astype(np.float64) * float(vs[0]))


def test_sizes():
    assert S.static_scale_bytes(80, 8, 128, "int8c") == 2 * 80 * 8 * 128 * 2
    assert S.static_scale_bytes(80, 8, 128, "int8t") == 2 * 80 * 2
    assert S.scale_bytes(1, 8, 4096, 1, "int8c") == 0
    assert S.kv_bytes(1, 8, 128, 4096, 1, S.BYTES_PER_ELEMENT["int8c"]) == \
        S.kv_bytes(1, 8, 128, 4096, 1, S.BYTES_PER_ELEMENT["int8"])


def test_planted_mistakes_are_caught(monkeypatch):
    """Round half away from zero, or an asymmetric clamp at -128, each fail a pin."""
    x = np.array([0.25, 0.75, 1.25, -70], np.float32)
    s = np.float32(0.5)
    away = np.clip(np.sign(x / s) * np.floor(np.abs(x / s) + 0.5), -127, 127).astype(np.int8)
    assert away.tolist() != F.int8_static_quantize(x, s).tolist()
    asym = np.clip(np.rint(x / s), -128, 127).astype(np.int8)
    assert asym.tolist() != F.int8_static_quantize(x, s).tolist()
