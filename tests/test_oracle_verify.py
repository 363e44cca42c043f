"""Pins of the oracle's multi-query (speculative verification) attention
("KV cache quantization: what FP8/INT8 K and V really give", "How it interacts
with speculative decoding": the target model scores all K+1 proposed positions
in one pass over the quantized cache).

Checked against PyTorch's scaled_dot_product_attention in float64 with an
explicit boolean mask (a library routine), the single-query oracle for
n_query = 1, the last position equal to plain decode over the whole context,
and a planted off-by-one in the causal limit.
"""

import numpy as np
import torch

from oracle import attention as A


def _data(seed, B=2, Hq=4, Hk=2, nq=3, D=16, ctx=(9, 5)):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, nq, D))
    kv = [(rng.standard_normal((c, Hk, D)), rng.standard_normal((c, Hk, D))) for c in ctx]
    return q, kv


def _sdpa(q, kv, sm_scale, Hk):
    B, Hq, nq, D = q.shape
    G = Hq // Hk
    out = np.zeros_like(q)
    for b in range(B):
        K, V = kv[b]
        ctx = K.shape[0]
        pos = torch.arange(ctx)
        lim = torch.tensor([ctx - nq + 1 + j for j in range(nq)])
        mask = pos[None, :] < lim[:, None]                      # [nq][ctx]
        for h in range(Hq):
            qq = torch.from_numpy(q[b, h])[None, None]          # [1][1][nq][D]
            kk = torch.from_numpy(K[:, h // G])[None, None]
            vv = torch.from_numpy(V[:, h // G])[None, None]
            o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask[None, None],
                                                                 scale=sm_scale)
            out[b, h] = o[0, 0].numpy()
    return out


def test_matches_sdpa_with_a_causal_mask():
    q, kv = _data(1)
    got = A.verify_attention(q, kv, 0.25, 2)
    want = _sdpa(q, kv, 0.25, 2)
    assert np.allclose(got, want, atol=1e-12, rtol=1e-12)


def test_one_position_is_plain_decode():
    q, kv = _data(2, nq=1)
    got = A.verify_attention(q, kv, 0.3, 2)[:, :, 0]
    want = A.decode_attention(q[:, :, 0], kv, 0.3, 2)
    assert np.array_equal(got, want)


def test_last_position_sees_the_whole_context_and_the_first_sees_less():
    q, kv = _data(3, nq=4, ctx=(7, 12))
    got = A.verify_attention(q, kv, 0.2, 2)
    whole = A.decode_attention(q[:, :, -1], kv, 0.2, 2)
    assert np.array_equal(got[:, :, -1], whole)
    short = A.decode_attention(q[:, :, 0], [(K[:-3], V[:-3]) for K, V in kv], 0.2, 2)
    assert np.array_equal(got[:, :, 0], short)


def test_positions_without_tokens_are_zero():
    q, kv = _data(4, nq=4, ctx=(2, 4))
    got = A.verify_attention(q, kv, 0.2, 2)
    assert np.all(got[0, :, :2] == 0) and np.all(got[0, :, 2:] != 0)
    assert np.all(got[1] != 0)


def test_an_off_by_one_limit_is_caught():
    q, kv = _data(5)
    B, Hq, nq, D = q.shape
    wrong = np.zeros_like(q)
    for b in range(B):
        K, V = kv[b]
        for h in range(Hq):
            for j in range(nq):
                n = max(0, K.shape[0] - nq + j)                 # misses the position itself
                wrong[b, h, j] = A.attend_one(q[b, h, j], K[:n, h // 2], V[:n, h // 2], 0.25)
    assert not np.allclose(wrong, _sdpa(q, kv, 0.25, 2), atol=1e-6)
