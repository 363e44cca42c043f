"""kvq_decode_attn_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plugin inside another framework's step that owns all device
memory; a decode loop that must avoid the synchronisation cudaMalloc/cudaFree
can cause) call this entry point instead of kvq_decode_attn: it takes the
split-K scratch from the library's static device array, so the caller passes
only inputs and outputs. The GPU test calls it through the C ABI twice in a row,
on different inputs, and checks each output against kvq_decode_attn with a
caller workspace, within the attention tolerance of the other parity tests
(max 4e-3, mean 5e-4). The second call must not be disturbed by what the first
left in the shared scratch.

This file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from int8_quantized_paged_quantize_b200 import kvq
from int8_quantized_paged_quantize_b200 import workloads as W

MAX_ABS, MEAN_ABS = 4e-3, 5e-4


def _cache(fmt, ctx, seed):
    w = W.Workload("noalloc", fmt, batch=len(ctx), n_q_heads=16, n_kv_heads=2, head_dim=128,
                   lengths="list", ctx=tuple(ctx), kv_mean=0.3 if fmt == "int8" else 0.0)
    tables, nb = W.block_tables(w, seed)
    d = kvq.dims(nb, w.n_kv_heads, w.n_q_heads, w.head_dim, tables.shape[1])
    c = kvq.LayerCache.allocate(fmt, d)
    for b in range(w.batch):
        k, v = W.kv_history(w, b, seed)
        pos = np.arange(ctx[b])
        sl = tables[b][pos // 16].astype(np.int64) * 16 + pos % 16
        c.append(k.cuda(), v.cuda(), torch.from_numpy(sl).cuda())
    q, _, _ = W.step_inputs(w, 0, seed)
    return w, c, torch.from_numpy(tables).cuda(), torch.from_numpy(np.asarray(ctx, np.int32)).cuda(), q.cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_noalloc_matches_workspace_decode_on_two_calls(fmt):
    L = kvq.lib()
    # call 1: long contexts, many chunks (fills much of the scratch);
    # call 2: short contexts, fewer chunks (stale partials from call 1 remain)
    for call, (ctx, part, seed) in enumerate([([5000, 3100, 777], 128, 1), ([40, 300], 0, 2)]):
        w, c, tables, cl, q = _cache(fmt, ctx, seed)
        max_ctx = int(max(ctx))
        ref = c.decode(q, tables, cl, max_ctx, sm_scale=w.sm_scale, partition_tokens=part,
                       out_dtype=torch.float32)
        out = torch.full_like(ref, float("nan"))
        scales = (ctypes.c_void_p * 2)(c.k_scale.data_ptr(), c.v_scale.data_ptr())
        rc = L.kvq_decode_attn_noalloc(
            ctypes.c_void_p(q.data_ptr()), w.batch, ctypes.c_void_p(c.k.data_ptr()),
            ctypes.c_void_p(c.v.data_ptr()), scales, ctypes.c_void_p(tables.data_ptr()),
            ctypes.c_void_p(cl.data_ptr()), max_ctx, ctypes.c_float(w.sm_scale),
            ctypes.c_void_p(out.data_ptr()), 1, part, kvq.FMT[fmt], ctypes.byref(c.dims),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0, (call, L.kvq_status_string(rc))
        torch.cuda.synchronize()
        err = (out - ref).abs()
        assert torch.isfinite(out).all(), call
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, (call, err.max().item())
        assert kvq.device_error() == 0


def test_noalloc_rejects_plans_beyond_the_scratch():
    """A split plan larger than the static scratch is refused before any device work."""
    L = kvq.lib()
    d = kvq.dims(1 << 20, 8, 64, 128, 1 << 16)
    fake = ctypes.c_void_p(1 << 20)
    scales = (ctypes.c_void_p * 2)(1 << 21, 1 << 22)
    B, max_ctx = 256, 1 << 20                       # 128-token chunks: far above 64 MiB
    need = L.kvq_decode_workspace_bytes(B, max_ctx, 128, 1, ctypes.byref(d))
    assert need > kvq.NOALLOC_SCRATCH_BYTES
    rc = L.kvq_decode_attn_noalloc(fake, B, fake, fake, scales, fake, fake, max_ctx,
                                   ctypes.c_float(0.1), fake, 0, 128, 1, ctypes.byref(d), None)
    assert rc == -3                                  # KVQ_ERR_WORKSPACE
    assert b"workspace" in L.kvq_status_string(rc)


def test_noalloc_limit_is_the_header_constant():
    """A plan of exactly KVQ_NOALLOC_SCRATCH_BYTES is accepted and the next larger
    one refused: with null pointers the first call gets past the size check and
    stops at the pointer check (KVQ_ERR_ARG), the second stops at the size check
    (KVQ_ERR_WORKSPACE). Pins kvq.NOALLOC_SCRATCH_BYTES to the C macro."""
    L = kvq.lib()
    # D = 64, one KV head, one query head, 128-token chunks of max_context_len 384
    # (4 partial slots per row): 63310 sequences need exactly 64 MiB
    d = kvq.dims(1024, 1, 1, 64, 24)
    B, max_ctx, part = 63310, 384, 128
    assert L.kvq_decode_workspace_bytes(B, max_ctx, part, 1, ctypes.byref(d)) == kvq.NOALLOC_SCRATCH_BYTES
    assert L.kvq_decode_workspace_bytes(B + 1, max_ctx, part, 1, ctypes.byref(d)) > kvq.NOALLOC_SCRATCH_BYTES
    null = ctypes.c_void_p(0)
    scales = (ctypes.c_void_p * 2)(0, 0)
    args = (null, null, scales, null, null, max_ctx, ctypes.c_float(0.125), null, 0, part, 1,
            ctypes.byref(d), None)
    assert L.kvq_decode_attn_noalloc(null, B, *args) == -1            # KVQ_ERR_ARG: size accepted
    assert L.kvq_decode_attn_noalloc(null, B + 1, *args) == -3        # KVQ_ERR_WORKSPACE


def test_noalloc_checks_arguments_like_kvq_decode_attn():
    """Batch 0 with a bad format or unsupported dims fails the same way in both
    entry points; a valid batch 0 is a no-op in both."""
    L = kvq.lib()
    null = ctypes.c_void_p(0)
    scales = (ctypes.c_void_p * 2)(0, 0)
    good = kvq.dims(64, 2, 8, 128, 8)
    bad_group = kvq.dims(64, 2, 6, 128, 8)
    for d, fmt in ((good, 99), (bad_group, 1), (good, 1), (good, -1)):
        ws_rc = L.kvq_decode_attn(null, 0, null, null, scales, null, null, 128, ctypes.c_float(0.1),
                                  null, 0, null, 0, 0, fmt, ctypes.byref(d), None)
        na_rc = L.kvq_decode_attn_noalloc(null, 0, null, null, scales, null, null, 128,
                                          ctypes.c_float(0.1), null, 0, 0, fmt, ctypes.byref(d), None)
        assert ws_rc == na_rc, (fmt, ws_rc, na_rc)
    assert L.kvq_decode_attn_noalloc(null, 0, null, null, scales, null, null, 128, ctypes.c_float(0.1),
                                     null, 0, 0, 99, ctypes.byref(good), None) == -1
    # an output dtype outside the enum is refused too
    assert L.kvq_decode_attn_noalloc(null, 0, null, null, scales, null, null, 128, ctypes.c_float(0.1),
                                     null, 7, 0, 1, ctypes.byref(good), None) == -1


@pytest.mark.gpu
def test_noalloc_python_wrapper_matches_workspace_decode():
    """The same through kvq.decode_attn_noalloc, BF16 output, twice in a row."""
    for ctx, seed in (([2000, 129], 3), ([17], 4)):
        w, c, tables, cl, q = _cache("fp8", ctx, seed)
        max_ctx = int(max(ctx))
        ref = c.decode(q, tables, cl, max_ctx, sm_scale=w.sm_scale)
        out = torch.empty_like(ref)
        kvq.decode_attn_noalloc(q, c.k, c.v, c.k_scale, c.v_scale, tables, cl, max_ctx, w.sm_scale,
                                out, "fp8", c.dims)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)             # same kernels, same split plan: same bits
        with pytest.raises(kvq.KvqError):
            kvq.decode_attn_noalloc(q, c.k, c.v, c.k_scale, c.v_scale, tables, cl, max_ctx,
                                    w.sm_scale, out.to(torch.float16), "fp8", c.dims)
