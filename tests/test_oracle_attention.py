"""Pins of the oracle's attention, paging and size formula.

Sources: "From FP8 KV cache to INT4 weight-only" (Core concepts 1: decode
attends one query against the whole cached K/V; 2: PagedAttention maps each
request to fixed-size blocks of a pool); "KV Cache compression", section 1
(closed-form KV bytes with worked examples) and 5.1 (quantise at store,
dequantise before attention); "Fitting 76x concurrent requests with an FP8 KV
cache", section 2 (per-token K/V bytes); "KV cache quantization: what FP8/INT8
K and V really give" (opening paragraph / TL;DR: 70B at 32k in BF16).

Pins: the softmax row sums to one; a single cached token returns its value;
identical keys give the mean of V; a brute-force scalar loop with math.exp;
PyTorch's scaled_dot_product_attention in float64 with its GQA mapping; the
storage permutation invariance of paging; the pages' printed sizes.
"""

import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import formats as F
from oracle import paged as P
from oracle import sizes as S
from tests.conftest import read_golden


def _rand(rng, *shape):
    return F.bf16_round(rng.standard_normal(shape).astype(np.float32))


# ----------------------------------------------------------------------------- attention invariants


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(0)
    for n in (1, 2, 17, 300):
        w = A.softmax_weights(rng.standard_normal(64), rng.standard_normal((n, 64)) * 5, 0.125)
        assert abs(w.sum() - 1.0) < 1e-12 and np.all(w >= 0)


def test_single_token_returns_value():
    rng = np.random.default_rng(1)
    v = rng.standard_normal((1, 128))
    out = A.attend_one(rng.standard_normal(128), rng.standard_normal((1, 128)), v, 0.1)
    assert np.array_equal(out, v[0])


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(2)
    k = np.tile(rng.standard_normal(64), (50, 1))
    v = rng.standard_normal((50, 64))
    out = A.attend_one(rng.standard_normal(64), k, v, 0.125)
    assert np.allclose(out, v.mean(axis=0), atol=1e-13, rtol=0)


def test_empty_context_gives_zero():
    out = A.attend_one(np.ones(8), np.zeros((0, 8)), np.zeros((0, 8)), 1.0)
    assert np.array_equal(out, np.zeros(8))


def test_brute_force_scalar_loop():
    rng = np.random.default_rng(3)
    q, k, v = rng.standard_normal(6), rng.standard_normal((5, 6)), rng.standard_normal((5, 6))
    s = [sum(q[d] * k[t][d] for d in range(6)) * 0.3 for t in range(5)]
    e = [math.exp(x) for x in s]
    z = sum(e)
    want = [sum(e[t] / z * v[t][d] for t in range(5)) for d in range(6)]
    assert np.allclose(A.attend_one(q, k, v, 0.3), want, atol=1e-14, rtol=0)


def test_decode_attention_matches_torch_sdpa_gqa():
    rng = np.random.default_rng(4)
    B, Hq, Hk, D = 3, 8, 2, 32
    ctx = [5, 1, 40]
    q = rng.standard_normal((B, Hq, D))
    kv = [(rng.standard_normal((n, Hk, D)), rng.standard_normal((n, Hk, D))) for n in ctx]
    ours = A.decode_attention(q, kv, 0.17, Hk)
    for b in range(B):
        K, V = kv[b]
        qt = torch.from_numpy(q[b][:, None, :])                 # [Hq][1][D]
        kt = torch.from_numpy(np.ascontiguousarray(K.transpose(1, 0, 2)))  # [Hk][n][D]
        vt = torch.from_numpy(np.ascontiguousarray(V.transpose(1, 0, 2)))
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, scale=0.17, enable_gqa=True)[:, 0, :].numpy()
        assert np.allclose(ours[b], ref, atol=1e-12, rtol=0)


# ----------------------------------------------------------------------------- paging


def test_slot_of_positions():
    row = np.array([7, 2, 5])
    assert P.slot_of(row, 0, 16) == 7 * 16
    assert P.slot_of(row, 15, 16) == 7 * 16 + 15
    assert P.slot_of(row, 16, 16) == 2 * 16
    assert P.slot_of(row, 40, 16) == 5 * 16 + 8


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "int8"])
def test_paged_storage_is_permutation_invariant(fmt):
    """The same tokens appended through two different block tables gather back
    to identical K/V, equal to quantising the rows directly."""
    rng = np.random.default_rng(5)
    Hk, D, bs, n = 2, 64, 16, 45
    k, v = _rand(rng, n, Hk, D), _rand(rng, n, Hk, D)
    nb = 8
    outs = []
    for row in (np.array([0, 1, 2]), np.array([6, 0, 3])):
        pool = P.LogicalPool(fmt, nb, Hk, bs, D)
        pool.append(k, v, P.slot_of(row, np.arange(n), bs))
        outs.append(pool.gather(row, n))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    if fmt == "fp8":
        c, s = F.fp8_quantize(k)
        assert np.array_equal(outs[0][0], F.fp8_dequantize(c, s))
    elif fmt == "int8":
        c, s, z = F.int8_quantize(v)
        assert np.array_equal(outs[0][1], F.int8_dequantize(c, s, z))
    else:
        assert np.array_equal(outs[0][0], k.astype(np.float64))


def test_append_skips_negative_slots_and_rejects_overflow():
    pool = P.LogicalPool("fp8", 2, 1, 16, 8)
    k = np.ones((2, 1, 8), dtype=np.float32)
    pool.append(k, k, np.array([-1, 3]))
    assert np.all(pool.k[0, 0, 3] != 0) and np.all(pool.k[0, 0, 0] == 0)
    with pytest.raises(IndexError):
        pool.append(k, k, np.array([0, 32]))


def test_gqa_mapping_uses_contiguous_groups():
    """Query head h reads KV head h // G: give each KV head a constant V and check."""
    Hq, Hk, D = 8, 2, 4
    K = np.zeros((3, Hk, D))
    V = np.zeros((3, Hk, D))
    V[:, 0, :], V[:, 1, :] = 1.0, 2.0
    out = A.decode_attention(np.zeros((1, Hq, D)), [(K, V)], 1.0, Hk)
    assert np.array_equal(out[0, :, 0], [1, 1, 1, 1, 2, 2, 2, 2])


# ----------------------------------------------------------------------------- sizes


def test_closed_form_reproduces_printed_sizes():
    unit = {"GB": 10 ** 9, "KB": 10 ** 3}
    for name, L, hk, hd, n, b, bpe, printed, u, _src in read_golden("kv_size_examples.txt"):
        got = S.kv_bytes(int(L), int(hk), int(hd), int(n), int(b), Fraction(bpe))
        # printed figures are rounded (or truncated) to their last shown digit
        digits = len(printed.split(".")[1]) if "." in printed else 0
        step = Fraction(1, 10 ** digits)
        val = got / unit[u]
        assert abs(val - Fraction(printed)) < step, (name, float(val), printed)


def test_closed_form_exact_bytes():
    assert S.kv_bytes(80, 8, 128, 4096, 1, 2) == 1_342_177_280
    assert S.kv_bytes(80, 8, 128, 131072, 1, 2) == 42_949_672_960
    assert S.kv_bytes(80, 8, 128, 32768, 1, 2) == 10_737_418_240
    assert S.per_token_kv_bytes(10, 8, 128, 2) == 40_960
    # 8-bit formats halve the element bytes, 4-bit quarter them
    assert S.kv_bytes(80, 8, 128, 4096, 1, 1) * 2 == S.kv_bytes(80, 8, 128, 4096, 1, 2)
    assert S.kv_bytes(80, 8, 128, 4096, 1, "1/2") * 4 == S.kv_bytes(80, 8, 128, 4096, 1, 2)
    # INT8 carries more metadata than FP8 (scale + zero point vs scale)
    assert S.scale_bytes(80, 8, 4096, 1, "int8") > S.scale_bytes(80, 8, 4096, 1, "fp8") > 0
