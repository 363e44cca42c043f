"""Pins of the KIVI-style oracle (K per channel, V per token, low-bit
asymmetric codes, full-precision residual): "KV Cache compression" 2.1 and
3.1 "KIVI", and "KV cache quantization: what FP8/INT8 K and V really give"
("Formats you will actually meet", the mixed-precision 4-bit row; 4-bit
storage is 25% of BF16).

Pinned by hand-worked codes (exact grids, ties to even), the rounding bound,
an exact-rational brute-force nearest level, the per-channel / per-token axis
identity, exact residual and constant groups, the pages' claim that per-channel
K beats per-token K when K has outlier channels, the 25% figure, and planted
mistakes.
"""

from fractions import Fraction

import numpy as np

from oracle import attention as A
from oracle import formats as F
from oracle import kivi as Q


def test_hand_worked_groups():
    x = np.array([[0, 1, 2, 3], [-1, 0.5, 2, 2], [5, 5, 5, 5]], np.float32)
    c, s, z = Q.asym_quantize(x, axis=-1, bits=2)
    assert c.tolist() == [[0, 1, 2, 3], [0, 2, 3, 3], [0, 0, 0, 0]]   # 1.5 -> 2 (even)
    assert s.tolist() == [1.0, 1.0, 0.0] and z.tolist() == [0.0, -1.0, 5.0]
    assert np.array_equal(Q.asym_dequantize(c, s, z, -1)[0], x[0])
    assert np.array_equal(Q.asym_dequantize(c, s, z, -1)[2], x[2])  # zero range: exact
    c4, s4, z4 = Q.asym_quantize(np.arange(16, dtype=np.float32)[None] * 0.5, axis=-1, bits=4)
    assert c4.tolist() == [list(range(16))] and s4[0] == 0.5


def test_rounding_bound():
    rng = np.random.default_rng(1)
    for bits in (2, 4):
        x = F.bf16_round((rng.standard_normal((300, 64)) * rng.uniform(0.1, 20, (300, 1))).astype(np.float32))
        c, s, z = Q.asym_quantize(x, axis=-1, bits=bits)
        deq = Q.asym_dequantize(c, s, z, -1)
        xd = x.astype(np.float64)
        lo, hi = xd.min(axis=-1), xd.max(axis=-1)
        top = z.astype(np.float64) + (2 ** bits - 1) * s.astype(np.float64)
        bound = (s / 2.0 + np.abs(z - lo) + np.maximum(0.0, hi - top) + np.abs(xd).max(axis=-1) * 2.0 ** -22)
        assert np.all(np.abs(deq - xd) <= bound[:, None])


def test_brute_force_nearest_level():
    rng = np.random.default_rng(2)
    x = F.bf16_round(rng.uniform(-3, 5, (40, 8)).astype(np.float32))
    c, s, z = Q.asym_quantize(x, axis=-1, bits=2)
    for i in range(x.shape[0]):
        for j in range(x.shape[1]):
            t = (Fraction(float(x[i, j])) - Fraction(float(z[i]))) / Fraction(float(s[i]))
            best = min(range(4), key=lambda k: (abs(t - k), k % 2))
            assert c[i, j] == best


def test_per_channel_is_per_token_of_the_transpose():
    rng = np.random.default_rng(3)
    K = F.bf16_round(rng.standard_normal((128, 2, 16)).astype(np.float32))
    c1, s1, z1 = Q.asym_quantize(K, axis=0, bits=2)                       # per (head, channel)
    c2, s2, z2 = Q.asym_quantize(np.transpose(K, (1, 2, 0)), axis=-1, bits=2)
    assert np.array_equal(c1, np.transpose(c2, (2, 0, 1)))
    assert np.array_equal(s1, s2) and np.array_equal(z1, z2)


def test_residual_and_groups():
    rng = np.random.default_rng(4)
    n = 128 * 2 + 37
    K = F.bf16_round(rng.standard_normal((n, 2, 32)).astype(np.float32))
    V = F.bf16_round(rng.standard_normal((n, 2, 32)).astype(np.float32))
    st = Q.quantize_sequence(K, V, bits=2)
    assert st["n_groups"] == 2 and st["k_res"].shape[0] == 37
    Kd, Vd = Q.dequantize_sequence(st)
    assert Kd.shape == K.shape and Vd.shape == V.shape
    assert np.array_equal(Kd[256:], K[256:].astype(np.float64))      # residual exact
    assert np.array_equal(Vd[256:], V[256:].astype(np.float64))
    assert not np.array_equal(Kd[:256], K[:256].astype(np.float64))  # groups quantized
    # a short sequence is all residual: attention equals the BF16 attention
    st = Q.quantize_sequence(K[:100], V[:100])
    Kd, Vd = Q.dequantize_sequence(st)
    q = rng.standard_normal((1, 4, 32))
    assert np.array_equal(A.decode_attention(q, [(Kd, Vd)], 0.2, 2),
                          A.decode_attention(q, [(K[:100].astype(np.float64), V[:100].astype(np.float64))], 0.2, 2))


def test_per_channel_keys_win_with_outlier_channels():
    """The pages' reason for the asymmetry: a few K channels carry outliers."""
    rng = np.random.default_rng(5)
    K = rng.standard_normal((128, 1, 64)).astype(np.float32)
    K[:, :, [3, 17, 40, 55]] *= 20
    K = F.bf16_round(K)
    pc = Q.asym_dequantize(*Q.asym_quantize(K, axis=0, bits=4), axis=0)
    pt = Q.asym_dequantize(*Q.asym_quantize(K, axis=-1, bits=4), axis=-1)
    err_c = np.linalg.norm(pc - K) / np.linalg.norm(K)
    err_t = np.linalg.norm(pt - K) / np.linalg.norm(K)
    assert err_c < err_t
    # per token, the outliers take the range of every row and the ordinary
    # channels lose most of their precision; per channel they keep it
    keep = np.ones(64, bool)
    keep[[3, 17, 40, 55]] = False
    norm_c = np.linalg.norm((pc - K)[..., keep]) / np.linalg.norm(K[..., keep])
    norm_t = np.linalg.norm((pt - K)[..., keep]) / np.linalg.norm(K[..., keep])
    assert norm_c < 0.2 * norm_t


def test_four_bit_codes_are_a_quarter_of_bf16():
    codes_only = 2 * 8 * 128 * 4 / 8
    assert codes_only / (2 * 8 * 128 * 2) == 0.25
    assert Q.bytes_per_token(8, 128, bits=4) == codes_only + 8 * 4 + 8 * 128 * 4 / 128
    assert Q.bytes_per_token(8, 128, bits=2) < Q.bytes_per_token(8, 128, bits=4)


def test_planted_mistakes_are_caught():
    x = np.array([[-1, 0.5, 2, 2]], np.float32)
    c, s, z = Q.asym_quantize(x, axis=-1, bits=2)
    floor_codes = np.clip(np.floor((x - z[:, None]) / s[:, None]), 0, 3)
    assert floor_codes.tolist() != c.tolist()                  # truncation instead of rint
    g = np.arange(4, dtype=np.float32)[None]
    c2, s2, z2 = Q.asym_quantize(g, axis=-1, bits=2)
    wrong_s = (g.max() - g.min()) / 4                          # 2^b instead of 2^b - 1 levels
    assert np.rint(g / wrong_s).tolist() != c2.tolist()


def test_zero_minimum_and_range_are_plus_zero():
    """Groups whose minimum or range is zero store +0 whatever the order of
    +0 and -0 among the values (a canonical sign, reading in the oracle)."""
    for row in ([0.0, -0.0, 0.0, -0.0], [-0.0, 0.0, -0.0, 0.0], [-0.0, -0.0, 1.0, 2.0]):
        x = np.array([row], np.float32)
        c, s, z = Q.asym_quantize(x, axis=-1, bits=2)
        assert not np.signbit(z[0]) and z[0] == 0
    c, s, z = Q.asym_quantize(np.array([[-0.0, 0.0, -0.0, 0.0]], np.float32), axis=-1, bits=4)
    assert not np.signbit(s[0]) and s[0] == 0 and c.tolist() == [[0, 0, 0, 0]]
