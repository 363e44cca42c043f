"""GPU parity of libkvq against the CPU oracle on small seeded workloads.

Cache codes, BF16 scales and INT8 zero points must be bit-exact; attention
(FP32 output) must be within max |err| 4e-3 and mean |err| 5e-4 of the oracle's
FP64 attention over the same dequantised K/V. Shapes span several 128-token
tiles with ragged tails, every supported head_dim / GQA group / format, split-K
on and off, and the degenerate cases (one token, zero rows, empty calls,
out-of-range slots / blocks / lengths).
"""

import math
from dataclasses import replace

import numpy as np
import pytest
import torch

from int8_quantized_paged_quantize_b200 import kvq
from int8_quantized_paged_quantize_b200 import workloads as W
from tests import gpu_cases as GC

pytestmark = pytest.mark.gpu

FORMATS = ["fp8", "int8", "bf16", "e5m2"]
RAGGED = [1, 15, 16, 17, 127, 128, 129, 300, 555]


def _synthetic(fmt, D, G, Hk=2, ctx=RAGGED, kv_mean=0.0):
    base = W.Workload("synthetic", fmt, batch=len(ctx), n_q_heads=Hk * G, n_kv_heads=Hk,
                      head_dim=D, lengths="list", ctx=tuple(ctx), kv_mean=kv_mean)
    return base


def _check(run, seqs=None, tol=(GC.MAX_ABS, GC.MEAN_ABS)):
    seqs = range(run.w.batch) if seqs is None else seqs
    mx, mean = GC.attention_errors(run, seqs)
    assert mx <= tol[0] and mean <= tol[1], (mx, mean)
    return mx, mean


# ----------------------------------------------------------------------------- the tiny workload
@pytest.mark.parametrize("fmt", FORMATS)
def test_tiny_workload_all_formats(fmt):
    w = W.WORKLOADS["tiny-fp8"]
    run = GC.run_gpu(w, fmt)
    _check(run)


def test_tiny_workload_whole_pool_bit_exact():
    """Every byte of the 16-block pool equals the oracle's logical pool."""
    from oracle import paged as OP
    w = W.WORKLOADS["tiny-fp8"]
    run = GC.run_gpu(w, "fp8")
    tables, nb = W.block_tables(w)
    pool = OP.LogicalPool("fp8", nb, w.n_kv_heads, 16, w.head_dim)
    hist, _, (q, k, v) = GC.inputs(w)
    ctx = W.context_lengths(w)
    for b in range(w.batch):
        pool.append(hist[b][0].float().numpy(), hist[b][1].float().numpy(),
                    GC.slots_for(tables, b, np.arange(ctx[b])))
    pool.append(k.float().numpy(), v.float().numpy(),
                np.array([GC.slots_for(tables, b, [ctx[b]])[0] for b in range(w.batch)]))
    assert np.array_equal(run.cache.k_logical().cpu().numpy(), pool.k)
    assert np.array_equal(run.cache.v_logical().cpu().numpy(), pool.v)
    assert np.array_equal(run.cache.k_scale.float().cpu().numpy(), pool.k_scale)
    assert np.array_equal(run.cache.v_scale.float().cpu().numpy(), pool.v_scale)


# ----------------------------------------------------------------------------- shapes
@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_ragged_shapes(fmt, D, G):
    w = _synthetic(fmt, D, G, kv_mean=0.3 if fmt == "int8" else 0.0)
    _check(GC.run_gpu(w, fmt))


@pytest.mark.parametrize("fmt", FORMATS)
def test_split_k_on_and_off_agree(fmt):
    w = _synthetic(fmt, 128, 8, Hk=2, ctx=[3000, 1, 700, 4097])
    a = GC.run_gpu(w, fmt, partition_tokens=128)            # many chunks + merge
    b = GC.run_gpu(w, fmt, partition_tokens=8192)           # one chunk per sequence
    _check(a)
    _check(b)
    assert (a.out - b.out).abs().max().item() < 1e-3


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("part", [0, 128])
def test_many_short_sequences_split_across_ctas(fmt, part):
    """The persistent kernel's work split: 120 sequences shorter than a few
    tiles around the 128-token boundary, two long ones, GQA group 4. With
    partition 128 every CTA's share crosses many (sequence, head) runs, and
    some shares end inside a run's opening cost, so they hold no tile of it."""
    rng = np.random.default_rng(7)
    ctx = [int(c) for c in rng.integers(0, 300, size=120)] + [0, 126, 127, 128, 255, 3000, 5000]
    w = _synthetic(fmt, 128, 4, Hk=2, ctx=ctx, kv_mean=0.3 if fmt == "int8" else 0.0)
    run = GC.run_gpu(w, fmt, partition_tokens=part)
    _check(run)


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_history_appended_in_chunks_is_identical(fmt):
    w = _synthetic(fmt, 128, 4, ctx=[100, 777, 31])
    a = GC.run_gpu(w, fmt, history_chunks=1)
    b = GC.run_gpu(w, fmt, history_chunks=5)
    assert torch.equal(a.cache.k, b.cache.k) and torch.equal(a.cache.v, b.cache.v)
    assert torch.equal(a.cache.k_scale, b.cache.k_scale)
    assert torch.equal(a.out, b.out)


@pytest.mark.parametrize("fmt", FORMATS)
def test_bf16_output_is_rounded_f32_output(fmt):
    w = _synthetic(fmt, 128, 4, ctx=[50, 1000])
    a = GC.run_gpu(w, fmt, out_dtype=torch.float32)
    b = GC.run_gpu(w, fmt, out_dtype=torch.bfloat16)
    assert torch.equal(a.out.to(torch.bfloat16), b.out)


# ----------------------------------------------------------------------------- edge cases
def _fresh(fmt, nb=8, Hk=2, G=2, D=64, W_=4):
    d = kvq.dims(nb, Hk, Hk * G, D, W_)
    return d, kvq.LayerCache.allocate(fmt, d)


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_zero_rows_store_zero_scale(fmt):
    """All-zero K rows store scale 0 and zero codes; attending them is a plain
    mean of the (dequantised) values."""
    from oracle import formats as OF
    d, c = _fresh(fmt)
    k = torch.zeros(3, 2, 64, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros(3, 2, 64, dtype=torch.bfloat16, device="cuda")
    v[1] = 1.0
    c.append(k, v, torch.tensor([0, 1, 2], dtype=torch.int64, device="cuda"))
    torch.cuda.synchronize()
    assert torch.all(c.k_scale.float().cpu() == 0) and torch.all(c.k_logical().cpu() == 0)
    q = torch.randn(1, 4, 64, device="cuda").to(torch.bfloat16)
    tbl = torch.tensor([[0, -1, -1, -1]], dtype=torch.int32, device="cuda")
    cl = torch.tensor([3], dtype=torch.int32, device="cuda")
    out = c.decode(q, tbl, cl, 3, out_dtype=torch.float32).cpu()[0]
    vr = v.float().cpu().numpy()                                   # [3][Hk][D]
    deq = OF.fp8_dequantize(*OF.fp8_quantize(vr)) if fmt == "fp8" else \
        OF.int8_dequantize(*OF.int8_quantize(vr))
    want = deq.mean(axis=0)                                        # [Hk][D]
    for h in range(4):
        np.testing.assert_allclose(out[h].numpy(), want[h // 2], atol=1e-6, rtol=0)


def test_single_token_context_returns_value():
    w = _synthetic("fp8", 128, 4, ctx=[0, 0])
    run = GC.run_gpu(w, "fp8")                                 # one appended token each
    ref = GC.oracle_sequence(run, 0)
    np.testing.assert_allclose(run.out[0].numpy()[0], ref["V"][0, 0], atol=1e-6, rtol=0)
    _check(run)


def test_empty_calls_are_noops():
    d, c = _fresh("fp8")
    e = torch.zeros(0, 2, 64, dtype=torch.bfloat16, device="cuda")
    c.append(e, e, torch.zeros(0, dtype=torch.int64, device="cuda"))
    q = torch.zeros(0, 4, 64, dtype=torch.bfloat16, device="cuda")
    tbl = torch.zeros(0, 4, dtype=torch.int32, device="cuda")
    cl = torch.zeros(0, dtype=torch.int32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    kvq.decode_attn(q, c.k, c.v, c.k_scale, c.v_scale, tbl, cl, 0, 0.125,
                    torch.zeros(0, 4, 64, dtype=torch.bfloat16, device="cuda"), ws, "fp8", d)
    torch.cuda.synchronize()
    assert kvq.device_error() == 0


def test_zero_context_sequence_outputs_zero():
    d, c = _fresh("int8")
    k = torch.randn(5, 2, 64, device="cuda").to(torch.bfloat16)
    c.append(k, k, torch.arange(5, dtype=torch.int64, device="cuda"))
    q = torch.randn(2, 4, 64, device="cuda").to(torch.bfloat16)
    tbl = torch.tensor([[0, -1, -1, -1], [0, -1, -1, -1]], dtype=torch.int32, device="cuda")
    cl = torch.tensor([0, 5], dtype=torch.int32, device="cuda")
    out = c.decode(q, tbl, cl, 5, out_dtype=torch.float32)
    assert torch.all(out[0] == 0) and torch.all(torch.isfinite(out[1]))
    assert kvq.device_error() == 0


def test_negative_slots_are_skipped_and_bad_slots_flagged():
    d, c = _fresh("fp8", nb=2)
    k = torch.randn(3, 2, 64, device="cuda").to(torch.bfloat16)
    c.append(k, k, torch.tensor([-1, 5, 40], dtype=torch.int64, device="cuda"))  # 40 >= 2*16
    torch.cuda.synchronize()
    assert kvq.device_error() == kvq.DEVERR_SLOT
    written = (c.k_logical().cpu() != 0).any(-1).any(1)          # [blocks][offsets]
    assert written.sum().item() == 1 and bool(written[0, 5])


def test_bad_block_and_context_are_flagged():
    d, c = _fresh("fp8", nb=4, W_=2)
    k = torch.randn(20, 2, 64, device="cuda").to(torch.bfloat16)
    c.append(k, k, torch.arange(20, dtype=torch.int64, device="cuda"))
    q = torch.randn(1, 4, 64, device="cuda").to(torch.bfloat16)
    cl = torch.tensor([20], dtype=torch.int32, device="cuda")
    tbl = torch.tensor([[0, 99]], dtype=torch.int32, device="cuda")       # 99 >= num_blocks
    out = c.decode(q, tbl, cl, 20, out_dtype=torch.float32)
    assert kvq.device_error() == kvq.DEVERR_BLOCK
    assert torch.all(torch.isfinite(out))
    tbl = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    cl = torch.tensor([25], dtype=torch.int32, device="cuda")              # > max_context_len
    out = c.decode(q, tbl, cl, 20, out_dtype=torch.float32)
    assert kvq.device_error() == kvq.DEVERR_CONTEXT
    assert torch.all(out == 0)


def test_host_argument_checks():
    d, c = _fresh("fp8")
    k = torch.randn(2, 2, 64, device="cuda").to(torch.bfloat16)
    sl = torch.tensor([0, 1], dtype=torch.int64, device="cuda")
    with pytest.raises(kvq.KvqError, match="invalid argument"):
        kvq.append(k, k, sl, c.k, c.v, None, c.v_scale, "fp8", d)       # missing scale
    bad = kvq.dims(8, 2, 6, 64, 4)                                       # G = 3
    with pytest.raises(kvq.KvqError, match="unsupported"):
        kvq.append(k, k, sl, c.k, c.v, c.k_scale, c.v_scale, "fp8", bad)
    q = torch.randn(1, 4, 64, device="cuda").to(torch.bfloat16)
    tbl = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    cl = torch.ones(1, dtype=torch.int32, device="cuda")
    tiny = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(kvq.KvqError, match="workspace"):
        kvq.decode_attn(q, c.k, c.v, c.k_scale, c.v_scale, tbl, cl, 64, 0.125,
                        torch.empty_like(q), tiny, "fp8", d)
    assert kvq.device_error() == 0


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_multiple_decode_steps_track_the_oracle(fmt):
    """Three steps of (append one token per sequence, decode) on one cache, each
    checked against an oracle pool that receives the same appends."""
    from oracle import attention as OA
    from oracle import paged as OP
    w = replace(_synthetic(fmt, 128, 8, ctx=[40, 200], kv_mean=0.3), decode_steps=3)
    tables, nb = W.block_tables(w)
    ctx = W.context_lengths(w)
    d = kvq.dims(nb, w.n_kv_heads, w.n_q_heads, w.head_dim, tables.shape[1])
    c = kvq.LayerCache.allocate(fmt, d)
    pool = OP.LogicalPool(fmt, nb, w.n_kv_heads, 16, w.head_dim)
    for b in range(w.batch):
        kh, vh = W.kv_history(w, b)
        sl = GC.slots_for(tables, b, np.arange(ctx[b]))
        c.append(kh.cuda(), vh.cuda(), torch.from_numpy(sl).cuda())
        pool.append(kh.float().numpy(), vh.float().numpy(), sl)
    tbl = torch.from_numpy(tables).cuda()
    for step in range(3):
        q, k, v = W.step_inputs(w, step)
        sl = np.array([GC.slots_for(tables, b, [ctx[b]])[0] for b in range(w.batch)])
        c.append(k.cuda(), v.cuda(), torch.from_numpy(sl).cuda())
        pool.append(k.float().numpy(), v.float().numpy(), sl)
        ctx = ctx + 1
        cl = torch.from_numpy(ctx.astype(np.int32)).cuda()
        out = c.decode(q.cuda(), tbl, cl, int(ctx.max()), sm_scale=w.sm_scale,
                       out_dtype=torch.float32).cpu().numpy()
        kv = [pool.gather(tables[b], ctx[b]) for b in range(w.batch)]
        ref = OA.decode_attention(q.float().numpy(), kv, w.sm_scale, w.n_kv_heads)
        err = np.abs(out - ref)
        assert err.max() <= GC.MAX_ABS and err.mean() <= GC.MEAN_ABS, (step, err.max())
    assert np.array_equal(c.k_logical().cpu().numpy().view(np.int8 if fmt == "int8" else np.uint8),
                          pool.k)
    assert kvq.device_error() == 0


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("D", [64, 128])
def test_bulk_and_per_row_append_write_the_same_bytes(fmt, D):
    """Whole pages appended in order take the staged bulk path; the same tokens in
    a shuffled order take the per-row path. Both must leave identical caches."""
    d = kvq.dims(12, 2, 4, D, 12)
    n = 16 * 10 + 5
    g = torch.Generator().manual_seed(3)
    k = (torch.randn(n, 2, D, generator=g) * 2 + 0.3).to(torch.bfloat16).cuda()
    v = torch.randn(n, 2, D, generator=g).to(torch.bfloat16).cuda()
    slots = torch.arange(n, dtype=torch.int64).cuda() + 16          # pages 1..11, in order
    a = kvq.LayerCache.allocate(fmt, d)
    a.append(k, v, slots)
    perm = torch.randperm(n, generator=g).cuda()
    b = kvq.LayerCache.allocate(fmt, d)
    b.append(k[perm].contiguous(), v[perm].contiguous(), slots[perm].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    if fmt != "bf16":
        assert torch.equal(a.k_scale, b.k_scale) and torch.equal(a.v_scale, b.v_scale)
    assert kvq.device_error() == 0


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("D", [64, 128])
def test_segmented_windows_write_the_same_bytes(fmt, D):
    """Windows of 16 input tokens whose slots form runs inside pages (a page
    continued from an offset, runs crossing a page edge, holes of skipped tokens,
    runs of one token) are stored per run; a fully shuffled order stores every
    token on its own. The caches must be identical byte for byte."""
    d = kvq.dims(24, 2, 4, D, 24)
    g = torch.Generator().manual_seed(11)
    runs = [(16 + 5, 40), (16 * 6 + 15, 1), (16 * 8 + 3, 9), (16 * 10, 16), (16 * 12 + 7, 30),
            (16 * 15 + 1, 2), (16 * 16 + 9, 7), (16 * 18, 5), (16 * 19 + 11, 21)]
    parts = [torch.arange(s, s + n, dtype=torch.int64) for s, n in runs]
    slots = torch.cat(parts)
    skip = torch.randperm(slots.numel(), generator=g)[:7]
    slots[skip] = -1
    n = slots.numel()
    k = (torch.randn(n, 2, D, generator=g) * 2 + 0.3).to(torch.bfloat16).cuda()
    v = torch.randn(n, 2, D, generator=g).to(torch.bfloat16).cuda()
    slots = slots.cuda()
    a = kvq.LayerCache.allocate(fmt, d)
    a.append(k, v, slots)
    perm = torch.randperm(n, generator=g).cuda()
    b = kvq.LayerCache.allocate(fmt, d)
    b.append(k[perm].contiguous(), v[perm].contiguous(), slots[perm].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    if fmt != "bf16":
        assert torch.equal(a.k_scale, b.k_scale) and torch.equal(a.v_scale, b.v_scale)
    assert kvq.device_error() == 0
