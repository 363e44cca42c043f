"""Plant plausible mistakes in the oracle (CPU only) and check that a pin fails.

This shows that the pins are not vacuous: a wrong exponent bias, a tie rule
that rounds away from zero, a flipped zero-point sign, a GQA mapping that
interleaves instead of grouping, a dropped softmax scale, or an FP8 / E5M2 scale
that truncates, rounds ties up or multiplies by a reciprocal each break at least
one pin test.
"""

import numpy as np
import pytest

import oracle.attention as A
import oracle.formats as F
from tests import test_oracle_attention as TA
from tests import test_oracle_formats as TF


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_wrong_exponent_bias_is_caught(monkeypatch):
    good = F.e4m3_decode

    def bias8(codes):
        return good(codes) / 2.0
    monkeypatch.setattr(F, "e4m3_decode", bias8)
    assert _fails(TF.test_e4m3_decode_matches_torch_float8_for_all_256_codes)


def test_ties_away_from_zero_is_caught(monkeypatch):
    tab = F._E4M3_MAGNITUDES

    def away(x):
        xf = np.asarray(x, dtype=np.float32)
        mag = np.abs(xf.astype(np.float64))
        hi = np.clip(np.searchsorted(tab, mag), 0, 0x7E)
        lo = np.clip(hi - 1, 0, 0x7E)
        code = np.where(tab[hi] - mag <= mag - tab[lo], hi, lo)     # ties go up
        code = np.where(mag >= 448, 0x7E, code).astype(np.int64)
        code = np.where(np.signbit(xf), code | 0x80, code)
        return code.astype(np.uint8)
    monkeypatch.setattr(F, "e4m3_encode", away)
    assert _fails(TF.test_e4m3_encode_special_cases)


def test_flipped_zero_point_is_caught(monkeypatch):
    good = F.int8_params

    def flipped(rows):
        s, zp = good(rows)
        return s, np.clip(-zp, -128, 127)
    monkeypatch.setattr(F, "int8_params", flipped)
    assert _fails(TF.test_int8_worked_rows)


def test_interleaved_gqa_mapping_is_caught(monkeypatch):
    def interleaved(q, kv_per_seq, sm_scale, n_kv_heads):
        q = np.asarray(q, dtype=np.float64)
        B, Hq, D = q.shape
        out = np.zeros((B, Hq, D))
        for b in range(B):
            K, V = kv_per_seq[b]
            for h in range(Hq):
                out[b, h] = A.attend_one(q[b, h], K[:, h % n_kv_heads], V[:, h % n_kv_heads], sm_scale)
        return out
    monkeypatch.setattr(A, "decode_attention", interleaved)
    assert _fails(TA.test_gqa_mapping_uses_contiguous_groups)
    assert _fails(TA.test_decode_attention_matches_torch_sdpa_gqa)


def test_dropped_softmax_scale_is_caught(monkeypatch):
    good = A.attend_one
    monkeypatch.setattr(A, "attend_one", lambda q, k, v, s: good(q, k, v, 1.0))
    assert _fails(TA.test_decode_attention_matches_torch_sdpa_gqa)


# --------------------------------------------------------------------------- FP8 / E5M2 scale rounding
def _bf16_truncate(x):
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    return (a.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)


def _bf16_half_up(x):
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    return ((a.view(np.uint32) + np.uint32(0x8000)) & np.uint32(0xFFFF0000)).view(np.float32)


@pytest.mark.parametrize("fmt", ["fp8", "e5m2"])
@pytest.mark.parametrize("rounding", ["truncate", "half_up", "reciprocal"])
def test_wrong_scale_rounding_is_caught(monkeypatch, fmt, rounding):
    M = np.float32(F.E4M3_MAX if fmt == "fp8" else F.E5M2_MAX)

    def scale(rows):
        r = np.asarray(rows, dtype=np.float32)
        amax = np.max(np.abs(r), axis=-1).astype(np.float32)
        if rounding == "reciprocal":
            return F.bf16_round(amax * (np.float32(1.0) / M))
        q = amax / M
        return _bf16_truncate(q) if rounding == "truncate" else _bf16_half_up(q)
    monkeypatch.setattr(F, "fp8_scale" if fmt == "fp8" else "e5m2_scale", scale)
    assert _fails(TF.test_fp8_and_e5m2_scale_rounding_rows)
    if rounding == "truncate" and fmt == "e5m2":
        assert _fails(TF.test_e5m2_worked_row)      # its quotient's low half is 0xDB6E
