"""FP64 softmax attention for one decode step over the (dequantised) cache —
test oracle.

Test infrastructure (see ``oracle/__init__``).

What the pages fix
------------------
* [GUIDE] "Core concepts 1)": in decode each step attends one new query
  position against the whole cached K/V of the request; the work is bound by
  reading the cache.
* [LIMITS] "What KV cache quantization actually is": the stored K/V are
  dequantised inside the attention kernel right before the matmuls, which run in
  BF16/FP16; the saving is bandwidth, not FLOPs.
* [76X] "4. Precision loss?": storage is 8-bit while the attention dot products
  accumulate in FP32.
* [COMPRESS] "1. The KV cache memory problem" and "6.3": with grouped-query
  attention there are fewer KV heads than query heads.

Readings taken
--------------
* Query head h reads KV head ``h // G`` with G = n_q_heads / n_kv_heads
  (contiguous groups).
* No mask: the step attends every cached position 0..ctx-1, the just-appended
  token included (append first, then attend).
* The oracle computes in float64 (rounding far below the device's), so it is
  the reference both for a quantised cache (fed the dequantised values) and for
  the unquantised BF16 values (the quality number).
* A sequence with ctx == 0 has an all-zero output (nothing to attend).
* Multi-query decode ([LIMITS] "How it interacts with speculative decoding":
  the target model scores the K+1 proposed positions in one pass over the
  quantised cache). Read as: the n_query new tokens are already appended, and
  position j (0-based) sees the cached tokens before it and itself, i.e. the
  first ``ctx - n_query + 1 + j`` positions (causal within the new tokens). A
  position that sees no token has an all-zero output.
"""

from __future__ import annotations

import numpy as np


def attend_one(q, k, v, sm_scale):
    """Single query vector q [D] against keys k [n][D] and values v [n][D]:
    softmax(sm_scale * k q) weighted sum of v, all in float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if k.shape[0] == 0:
        return np.zeros(q.shape[-1], dtype=np.float64)
    scores = (k @ q) * float(sm_scale)
    w = np.exp(scores - scores.max())
    w /= w.sum()
    return w @ v


def decode_attention(q, kv_per_seq, sm_scale, n_kv_heads):
    """Outputs [B][Hq][D] float64.

    q: [B][Hq][D] query vectors (BF16 values).
    kv_per_seq: list of (K, V), each [ctx_b][n_kv_heads][D], in position order.
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    G = Hq // n_kv_heads
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        K, V = kv_per_seq[b]
        for h in range(Hq):
            kh = h // G
            out[b, h] = attend_one(q[b, h], K[:, kh, :], V[:, kh, :], sm_scale)
    return out


def softmax_weights(q, k, sm_scale):
    """The softmax row (float64) of one query against keys k [n][D]."""
    scores = (np.asarray(k, dtype=np.float64) @ np.asarray(q, dtype=np.float64)) * float(sm_scale)
    w = np.exp(scores - scores.max())
    return w / w.sum()


def verify_attention(q, kv_per_seq, sm_scale, n_kv_heads):
    """Multi-query outputs [B][Hq][n_query][D] float64.

    q: [B][Hq][n_query][D]; kv_per_seq: list of (K, V), each [ctx_b][n_kv_heads][D]
    with the n_query new tokens as its last positions. Position j of sequence b
    attends to the first ctx_b - n_query + 1 + j positions."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, nq, D = q.shape
    G = Hq // n_kv_heads
    out = np.zeros((B, Hq, nq, D), dtype=np.float64)
    for b in range(B):
        K, V = kv_per_seq[b]
        ctx = K.shape[0]
        for h in range(Hq):
            kh = h // G
            for j in range(nq):
                n = max(0, ctx - nq + 1 + j)
                out[b, h, j] = attend_one(q[b, h, j], K[:n, kh, :], V[:n, kh, :], sm_scale)
    return out

