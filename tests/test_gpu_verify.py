"""GPU parity of multi-query decode (speculative verification) against the CPU
oracle ("KV cache quantization: what FP8/INT8 K and V really give", "How it
interacts with speculative decoding": the target model scores the K+1 proposed
positions in one pass over the quantized cache).

The n_query new tokens are appended first; position j sees the first
ctx - n_query + 1 + j tokens. Every position's output (FP32) must be within max
|err| 4e-3 and mean |err| 5e-4 of the oracle's FP64 attention over the same
dequantized K/V, across formats, GQA groups, head_dims, ragged contexts
(including contexts shorter than n_query, whose first positions see nothing)
and split-K partitions that end inside the new tokens. More query rows per KV
head than one row group of the kernel holds (G * n_query > 8: 2 or 4 positions
at the 70B-shaped G = 8) are checked the same way. Chunked prefill ("From FP8
KV cache to INT4 weight-only", Core concepts 1): a chunk's queries attend to the
cached prefix and, causally, to the chunk) runs its own kernel (128 query rows
per tensor-core product): 64-token chunks at G = 4 and 8 in every format,
row counts that leave a 128-row block partly empty, long prefixes split across
CTAs, and agreement with the verification kernel on the same positions.
"""

import numpy as np
import pytest
import torch

from int8_quantized_paged_quantize_b200 import kvq
from int8_quantized_paged_quantize_b200 import workloads as W
from oracle import attention as OA
from oracle import formats as OF
from oracle import paged as OP
from tests import gpu_cases as GC

pytestmark = pytest.mark.gpu

CTX = [1, 2, 3, 15, 16, 17, 127, 128, 129, 300, 1000]


def _run(fmt, D, G, nq, ctx=CTX, Hk=2, partition=0, seed=0, call="verify", transform=None):
    w = W.Workload("synthetic", fmt, batch=len(ctx), n_q_heads=Hk * G, n_kv_heads=Hk, head_dim=D,
                   lengths="list", ctx=tuple(ctx), kv_mean=0.3 if fmt == "int8" else 0.0)
    tables, nb = W.block_tables(w, seed)
    lens = W.context_lengths(w, seed)
    hist = [W.kv_history(w, b, seed) for b in range(w.batch)]
    d = kvq.dims(nb, Hk, Hk * G, D, tables.shape[1])
    K = torch.cat([h[0] for h in hist])
    V = torch.cat([h[1] for h in hist])
    if transform is not None:
        K, V = transform(K, V, lens)
    S = torch.cat([torch.from_numpy(GC.slots_for(tables, b, np.arange(lens[b]))) for b in range(w.batch)])
    static = {}
    if fmt in ("int8c", "int8t"):
        pc = fmt == "int8c"
        static = {"k_static": OF.int8_static_calibrate(K.float().numpy(), pc),
                  "v_static": OF.int8_static_calibrate(V.float().numpy(), pc)}
        cache = kvq.LayerCache.allocate(fmt, d, **{k: torch.from_numpy(v).to(torch.bfloat16).cuda()
                                                   for k, v in static.items()})
    else:
        cache = kvq.LayerCache.allocate(fmt, d)
    cache.append(K.cuda(), V.cuda(), S.cuda())
    g = torch.Generator().manual_seed(100 + seed)
    q = torch.randn(w.batch, Hk * G, nq, D, generator=g).to(torch.bfloat16)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    fn = kvq.decode_verify if call == "verify" else kvq.prefill_attn
    fn(q.cuda(), cache.k, cache.v, cache.k_scale, cache.v_scale,
       torch.from_numpy(tables).cuda(), torch.from_numpy(lens.astype(np.int32)).cuda(),
       int(lens.max()), w.sm_scale, out, fmt, d, partition_tokens=partition)
    torch.cuda.synchronize()
    assert kvq.device_error() == 0
    # oracle: the same tokens through the oracle's pool, then FP64 attention
    pool = OP.LogicalPool(fmt, nb, Hk, 16, D, **static)
    pool.append(K.float().numpy(), V.float().numpy(), S.numpy())
    kv = [pool.gather(tables[b], lens[b]) for b in range(w.batch)]
    ref = OA.verify_attention(q.float().numpy(), kv, w.sm_scale, Hk)
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref)
    return err, out.cpu(), ref, lens


def _check(err):
    assert err.max() <= GC.MAX_ABS and err.mean() <= GC.MEAN_ABS, (err.max(), err.mean())


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G,nq", [(1, 2), (1, 4), (1, 8), (2, 2), (2, 4), (4, 2)])
def test_verify_shapes(fmt, D, G, nq):
    err, out, ref, lens = _run(fmt, D, G, nq)
    _check(err)
    # positions that see no token are exact zeros
    for b, c in enumerate(lens):
        for j in range(nq):
            if c - nq + 1 + j <= 0:
                assert torch.count_nonzero(out[b, :, j]) == 0


@pytest.mark.parametrize("fmt", ["e5m2", "bf16", "int8c", "int8t"])
def test_verify_other_formats(fmt):
    _check(_run(fmt, 128, 2, 4)[0])


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_verify_split_inside_the_new_tokens(fmt):
    """Partitions of one tile: a sequence of 129 tokens ends in a piece of one
    token, which the first positions do not see at all (an empty partial)."""
    _check(_run(fmt, 128, 2, 4, ctx=[129, 130, 256, 257, 1000, 3], partition=128)[0])


def test_one_position_equals_plain_decode():
    fmt, D, G, Hk = "fp8", 128, 4, 2
    ctx = [50, 700, 129]
    w = W.Workload("synthetic", fmt, batch=len(ctx), n_q_heads=Hk * G, n_kv_heads=Hk, head_dim=D,
                   lengths="list", ctx=tuple(ctx))
    tables, nb = W.block_tables(w)
    lens = W.context_lengths(w)
    hist = [W.kv_history(w, b) for b in range(w.batch)]
    d = kvq.dims(nb, Hk, Hk * G, D, tables.shape[1])
    cache = kvq.LayerCache.allocate(fmt, d)
    S = torch.cat([torch.from_numpy(GC.slots_for(tables, b, np.arange(lens[b]))) for b in range(w.batch)])
    cache.append(torch.cat([h[0] for h in hist]).cuda(), torch.cat([h[1] for h in hist]).cuda(), S.cuda())
    q = torch.randn(w.batch, Hk * G, 1, D, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16).cuda()
    tb = torch.from_numpy(tables).cuda()
    cl = torch.from_numpy(lens.astype(np.int32)).cuda()
    out_v = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    kvq.decode_verify(q, cache.k, cache.v, cache.k_scale, cache.v_scale, tb, cl, int(lens.max()),
                      w.sm_scale, out_v, fmt, d)
    out_d = cache.decode(q[:, :, 0].contiguous(), tb, cl, int(lens.max()), sm_scale=w.sm_scale,
                         out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(out_v[:, :, 0], out_d)


def _zero_rows(out, lens, nq):
    for b, c in enumerate(lens):
        for j in range(nq):
            if c - nq + 1 + j <= 0:
                assert torch.count_nonzero(out[b, :, j]) == 0


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
@pytest.mark.parametrize("G,nq", [(8, 2), (8, 4), (4, 4), (2, 8), (1, 16), (4, 3), (8, 5)])
def test_verify_rows_beyond_one_group(fmt, G, nq):
    """G * n_query > 8: the rows of a KV head span several row groups (3 and 5
    positions give groups of 4 and 8 rows that split query heads apart)."""
    err, out, ref, lens = _run(fmt, 128, G, nq)
    _check(err)
    _zero_rows(out, lens, nq)


@pytest.mark.parametrize("fmt", ["fp8", "int8", "bf16", "e5m2", "int8c", "int8t"])
def test_prefill_chunk_of_64_at_group_4(fmt):
    """A 64-token prefill chunk at G = 4 (256 query rows per KV head, two
    128-row blocks of the prefill kernel): contexts that are exactly the chunk,
    one token more, and long cached prefixes."""
    err, out, ref, lens = _run(fmt, 128, 4, 64, ctx=[64, 65, 200, 1000, 4000], call="prefill")
    _check(err)


@pytest.mark.parametrize("fmt", ["fp8", "int8", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
def test_prefill_chunk_of_64_at_group_8(fmt, D):
    """The 70B-shaped group: 512 query rows per KV head (four row blocks)."""
    err, out, ref, lens = _run(fmt, D, 8, 64, ctx=[64, 129, 700, 2500], call="prefill")
    _check(err)


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
@pytest.mark.parametrize("G,nq", [(1, 1), (2, 100), (8, 17), (4, 3), (1, 200)])
def test_prefill_ragged_row_blocks(fmt, G, nq):
    """Row counts that leave the last 128-row block partly empty (200 rows: 72
    in the second block; 136 rows: 8), a single row, and contexts shorter than
    the chunk, whose first positions see nothing (zero rows)."""
    err, out, ref, lens = _run(fmt, 128, G, nq, ctx=[1, 5, 130, 333, 1000], call="prefill")
    _check(err)
    _zero_rows(out, lens, nq)


@pytest.mark.parametrize("fmt", ["fp8", "int8", "bf16"])
def test_prefill_split_across_ctas(fmt):
    """Long prefixes cut into 256-token partitions: a row's partials come from
    several CTAs and the merge combines them."""
    err, out, ref, lens = _run(fmt, 128, 4, 32, ctx=[5000, 3100, 777], partition=256, call="prefill")
    _check(err)


def test_prefill_agrees_with_verify_on_the_same_positions():
    """The same positions through the two kernels (query rows as the M
    dimension against query rows as the N dimension of the products): both
    within tolerance of the oracle and close to each other."""
    e1, o1, _, _ = _run("fp8", 64, 2, 16, ctx=[40, 300], call="prefill")
    e2, o2, _, _ = _run("fp8", 64, 2, 16, ctx=[40, 300], call="verify")
    _check(e1)
    _check(e2)
    assert (o1 - o2).abs().max().item() <= 2e-3


def _positions(lens):
    """Each token's position inside its sequence, for the concatenated history."""
    return torch.from_numpy(np.concatenate([np.arange(n) for n in lens]))


def _check_scaled(err, ref):
    """The attention tolerance relative to the outputs' magnitude."""
    scale = max(1.0, float(np.abs(ref).max()))
    assert err.max() <= GC.MAX_ABS * scale and err.mean() <= GC.MEAN_ABS * scale, (err.max(), scale)


@pytest.mark.parametrize("fmt", ["fp8", "int8", "bf16"])
def test_prefill_scores_that_grow_along_the_context(fmt):
    """K grows 4x in the second half of every sequence, so the row maxima jump
    by more than 2^8 after the first tiles: the prefill kernel's lazily moved
    reference must rescale O in TMEM mid-piece (and more than once across the
    split pieces of a long prefix)."""
    def grow(K, V, lens):
        pos = _positions(lens)
        half = torch.from_numpy(np.concatenate([np.full(n, n // 2) for n in lens]))
        f = torch.where(pos >= half, 4.0, 1.0).to(torch.float32)[:, None, None]
        return (K.float() * f).to(torch.bfloat16), V
    err, out, ref, lens = _run(fmt, 128, 4, 32, ctx=[600, 2500, 5000], partition=1024, call="prefill",
                               transform=grow)
    _check_scaled(err, ref)


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_prefill_v_scales_far_apart(fmt):
    """V magnitudes that differ by 2^8 between the two halves of every sequence
    (and so do the per-token V scales): the reference follows the half tiles'
    largest V scale, so the f16 parts of P' neither overflow nor lose precision."""
    def spread(K, V, lens):
        pos = _positions(lens)
        half = torch.from_numpy(np.concatenate([np.full(n, n // 2) for n in lens]))
        f = torch.where(pos >= half, 16.0, 1.0 / 16.0).to(torch.float32)[:, None, None]
        return K, (V.float() * f).to(torch.bfloat16)
    err, out, ref, lens = _run(fmt, 128, 4, 32, ctx=[300, 2100, 4100], call="prefill", transform=spread)
    _check_scaled(err, ref)
