"""Helpers for the GPU parity tests: run one workload through libkvq (append of the
cached history, append of the step's tokens, decode) and through the CPU oracle
on the same seeded inputs, then compare.

Comparison rules:
  * cache codes and BF16 scales/zero points: bit-exact;
  * attention output (FP32 out of the kernel) vs the oracle's FP64 attention
    over the same dequantised K/V: max |err| <= 4e-3 and mean |err| <= 5e-4.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch

from int8_quantized_paged_quantize_b200 import kvq
from int8_quantized_paged_quantize_b200 import paging
from int8_quantized_paged_quantize_b200 import workloads as W
from oracle import attention as OA
from oracle import formats as OF

MAX_ABS = 4e-3
MEAN_ABS = 5e-4


@dataclass
class DeviceRun:
    w: W.Workload
    fmt: str
    cache: kvq.LayerCache
    tables: np.ndarray          # [B][W] int32
    ctx_before: np.ndarray      # cached tokens before the step (history + bulk append)
    ctx_after: np.ndarray       # attended tokens (step token included)
    q: torch.Tensor             # [B][Hq][D] bf16 (CPU)
    k_new: torch.Tensor
    v_new: torch.Tensor
    out: torch.Tensor           # [B][Hq][D] (CPU, dtype of the run)
    seed: int = 0
    k_static: np.ndarray | None = None   # static INT8 scales (int8c [Hk][D], int8t [1])
    v_static: np.ndarray | None = None


def slots_for(tables, b, positions, bs=16):
    positions = np.asarray(positions, dtype=np.int64)
    return tables[b][positions // bs].astype(np.int64) * bs + positions % bs


def with_lengths(w: W.Workload, ctx_list):
    """The same shapes with an explicit list of cached lengths (no bulk append)."""
    return replace(w, lengths="list", ctx=tuple(int(c) for c in ctx_list),
                   batch=len(ctx_list), bulk_append=0, decode_steps=1)


_INPUTS = {}
STATIC = ("int8c", "int8t")


def static_scales(w: W.Workload, fmt: str, seed=0):
    """Static INT8 scales for a run, fixed by the oracle's calibration rule from
    the workload's cached history (the sample a caller would calibrate on)."""
    hist, _, (_, k_new, v_new) = inputs(w, seed)
    ks = [h[0] for h in hist] + [k_new]
    vs = [h[1] for h in hist] + [v_new]
    K = torch.cat(ks).float().numpy()
    V = torch.cat(vs).float().numpy()
    per_channel = fmt == "int8c"
    return OF.int8_static_calibrate(K, per_channel), OF.int8_static_calibrate(V, per_channel)


def inputs(w: W.Workload, seed=0):
    """Seeded inputs of one workload, generated once per process: per-sequence
    history and bulk-append K/V (BF16, CPU) and the first step's q/k/v."""
    key = (w, seed)
    if key not in _INPUTS:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(16) as ex:                  # numpy draws release the GIL
            hist = list(ex.map(lambda b: W.kv_history(w, b, seed), range(w.batch)))
            bulk = (list(ex.map(lambda b: W.kv_bulk(w, b, seed), range(w.batch)))
                    if w.bulk_append else None)
        _INPUTS.clear()                      # keep one workload's data at a time
        _INPUTS[key] = (hist, bulk, W.step_inputs(w, 0, seed))
    return _INPUTS[key]


def run_gpu(w: W.Workload, fmt: str, seed=0, partition_tokens=0, out_dtype=torch.float32,
            history_chunks=1, static=None):
    """Append every sequence's cached history (in `history_chunks` calls), then the
    bulk append if the workload has one, then one token per sequence, and run one
    decode step over ctx + 1 tokens. Returns a DeviceRun."""
    ctx = W.context_lengths(w, seed)
    hist, bulk, (q, k_new, v_new) = inputs(w, seed)
    if w.pool == "fragmented":
        # a shared pool fragmented by other requests: tables and slots come
        # from the library's block allocator as the sequences grow
        pb = paging.paged_batch(w, seed, fmt)
        hist_slots = [pb.extend(b, int(ctx[b])) for b in range(w.batch)]
        bulk_slots = [pb.extend(b, w.bulk_append) for b in range(w.batch)] if bulk is not None else None
        step_np = np.array([pb.extend(b, 1)[0] for b in range(w.batch)], dtype=np.int64)
        tables, nb = pb.tables.copy(), pb.dims.num_blocks
        pb.close()
    else:
        tables, nb = W.block_tables(w, seed)
        hist_slots = [slots_for(tables, b, np.arange(ctx[b])) for b in range(w.batch)]
        bulk_slots = ([slots_for(tables, b, ctx[b] + np.arange(w.bulk_append)) for b in range(w.batch)]
                      if bulk is not None else None)
        c1 = ctx + w.bulk_append
        step_np = np.array([slots_for(tables, b, [c1[b]])[0] for b in range(w.batch)], dtype=np.int64)
    d = kvq.dims(nb, w.n_kv_heads, w.n_q_heads, w.head_dim, tables.shape[1])
    dev = torch.device("cuda")
    kst = vst = None
    if fmt in STATIC:
        kst, vst = static if static is not None else static_scales(w, fmt, seed)
        kst = np.asarray(kst, dtype=np.float32)
        vst = np.asarray(vst, dtype=np.float32)
        cache = kvq.LayerCache.allocate(fmt, d, k_static=torch.from_numpy(kst).to(torch.bfloat16).to(dev),
                                        v_static=torch.from_numpy(vst).to(torch.bfloat16).to(dev))
    else:
        cache = kvq.LayerCache.allocate(fmt, d)
    S = [torch.from_numpy(x) for x in hist_slots]
    S = torch.cat(S) if S else torch.zeros(0, dtype=torch.int64)
    n = S.numel()
    if n:
        K = torch.cat([h[0] for h in hist])
        V = torch.cat([h[1] for h in hist])
        bounds = np.linspace(0, n, history_chunks + 1).astype(int)
        for a, z in zip(bounds[:-1], bounds[1:]):
            if z > a:
                cache.append(K[a:z].to(dev), V[a:z].to(dev), S[a:z].to(dev))
        del K, V
    if bulk is not None:
        nb_tok = w.bulk_append
        K = torch.cat([x[0] for x in bulk]).to(dev)
        V = torch.cat([x[1] for x in bulk]).to(dev)
        S = torch.cat([torch.from_numpy(x) for x in bulk_slots]).to(dev)
        cache.append(K, V, S)
        del K, V
        ctx = ctx + nb_tok
    step_slots = torch.from_numpy(step_np)
    cache.append(k_new.to(dev), v_new.to(dev), step_slots.to(dev))
    ctx_after = ctx + 1
    tbl = torch.from_numpy(tables).to(dev)
    cl = torch.from_numpy(ctx_after.astype(np.int32)).to(dev)
    out = cache.decode(q.to(dev), tbl, cl, int(ctx_after.max()), sm_scale=w.sm_scale,
                       partition_tokens=partition_tokens, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert kvq.device_error(clear=True) == 0
    return DeviceRun(w, fmt, cache, tables, ctx, ctx_after, q, k_new, v_new, out.cpu(), seed, kst, vst)


# ----------------------------------------------------------------------------- oracle side
def oracle_sequence(run: DeviceRun, b: int):
    """Oracle codes/scales and dequantised K/V of sequence b's ctx_after tokens,
    quantised by the oracle from the same seeded BF16 inputs.

    Returns dict with 'k_codes','v_codes' [n][Hk][D], 'k_scale','v_scale' [n][Hk],
    'k_zp','v_zp', 'K','V' float64 [n][Hk][D] and the raw BF16 'Kraw','Vraw'."""
    w = run.w
    hist, bulk, _ = inputs(w, run.seed)
    parts_k, parts_v = [hist[b][0]], [hist[b][1]]
    if bulk is not None:
        parts_k.append(bulk[b][0])
        parts_v.append(bulk[b][1])
    k = torch.cat(parts_k + [run.k_new[b:b + 1]]).float().numpy()
    v = torch.cat(parts_v + [run.v_new[b:b + 1]]).float().numpy()
    res = {"Kraw": k.astype(np.float64), "Vraw": v.astype(np.float64)}
    for name, x in (("k", k), ("v", v)):
        if run.fmt == "fp8":
            c, s = OF.fp8_quantize(x)
            res[name + "_codes"], res[name + "_scale"] = c, s
            res[name.upper()] = OF.fp8_dequantize(c, s)
        elif run.fmt == "e5m2":
            c, s = OF.e5m2_quantize(x)
            res[name + "_codes"], res[name + "_scale"] = c, s
            res[name.upper()] = OF.e5m2_dequantize(c, s)
        elif run.fmt in STATIC:
            st = run.k_static if name == "k" else run.v_static
            c = OF.int8_static_quantize(x, st)
            res[name + "_codes"] = c
            res[name.upper()] = OF.int8_static_dequantize(c, st)
        elif run.fmt == "int8":
            c, s, z = OF.int8_quantize(x)
            res[name + "_codes"], res[name + "_scale"], res[name + "_zp"] = c, s, z
            res[name.upper()] = OF.int8_dequantize(c, s, z)
        else:
            res[name + "_codes"] = OF.bf16_round(x)
            res[name.upper()] = x.astype(np.float64)
    return res


def gpu_sequence(run: DeviceRun, b: int):
    """The GPU cache contents of sequence b's ctx_after tokens in logical order:
    codes [n][Hk][D] and metadata [n][Hk] (scale, zero point)."""
    n = int(run.ctx_after[b])
    pages = int(math.ceil(n / 16))
    ids = torch.from_numpy(run.tables[b][:pages].astype(np.int64)).to(run.cache.k.device)
    kl = run.cache.k_logical(ids)                        # [pages][Hk][16][D]
    vl = run.cache.v_logical(ids)
    kl = kl.permute(0, 2, 1, 3).reshape(pages * 16, kl.shape[1], kl.shape[3])[:n].cpu()
    vl = vl.permute(0, 2, 1, 3).reshape(pages * 16, vl.shape[1], vl.shape[3])[:n].cpu()
    out = {"k_codes": kl, "v_codes": vl}
    if run.fmt not in ("bf16",) + STATIC:
        for name, t in (("k", run.cache.k_scale), ("v", run.cache.v_scale)):
            m = t[ids]                                       # [pages][Hk][16](,2)
            if run.fmt in ("fp8", "e5m2"):
                m = m.permute(0, 2, 1).reshape(pages * 16, -1)[:n].float().cpu().numpy()
                out[name + "_scale"] = m
            else:
                m = m.permute(0, 2, 1, 3).reshape(pages * 16, m.shape[1], 2)[:n].float().cpu().numpy()
                out[name + "_scale"] = m[..., 0]
                out[name + "_zp"] = m[..., 1]
    return out


def assert_codes_equal(run: DeviceRun, b: int, ref: dict):
    g = gpu_sequence(run, b)
    for name in ("k", "v"):
        gc = g[name + "_codes"]
        if run.fmt == "bf16":
            assert torch.equal(gc.float(), torch.from_numpy(ref[name + "_codes"])), name
        elif run.fmt in ("fp8", "e5m2"):
            assert np.array_equal(gc.numpy(), ref[name + "_codes"]), f"{name} codes b={b}"
        else:
            assert np.array_equal(gc.numpy().view(np.int8), ref[name + "_codes"]), f"{name} codes b={b}"
        if run.fmt not in ("bf16",) + STATIC:
            assert np.array_equal(OF.bf16_bits(g[name + "_scale"]), OF.bf16_bits(ref[name + "_scale"])), \
                f"{name} scales b={b}"
        if run.fmt == "int8":
            assert np.array_equal(g[name + "_zp"], ref[name + "_zp"].astype(np.float32)), f"{name} zp b={b}"


def oracle_attention(run: DeviceRun, b: int, ref: dict, raw=False):
    """FP64 attention of sequence b, [Hq][D]: over the dequantised cache, or with
    raw=True over the unquantised BF16 values (the quality reference)."""
    K, V = (ref["Kraw"], ref["Vraw"]) if raw else (ref["K"], ref["V"])
    q = run.q[b:b + 1].float().numpy().astype(np.float64)
    return OA.decode_attention(q, [(K, V)], run.w.sm_scale, run.w.n_kv_heads)[0]


def attention_errors(run: DeviceRun, seqs, check_codes=True):
    """(max abs err, mean abs err) of the GPU output vs the oracle over `seqs`."""
    errs = []
    for b in seqs:
        ref = oracle_sequence(run, b)
        if check_codes:
            assert_codes_equal(run, b, ref)
        o = oracle_attention(run, b, ref)
        errs.append(np.abs(run.out[b].float().numpy().astype(np.float64) - o).ravel())
    e = np.concatenate(errs) if errs else np.zeros(1)
    return float(e.max()), float(e.mean())


# ----------------------------------------------------------------------------- many decode steps
@dataclass
class StepsRun:
    w: W.Workload
    fmt: str
    cache: kvq.LayerCache
    tables: np.ndarray
    ctx_hist: np.ndarray        # cached tokens before the bulk append
    steps: int
    outs: list                  # per step: [B][Hq][D] FP32 (CPU)
    q: list                     # per step: [B][Hq][D] BF16 (CPU)
    k_new: list                 # per step: [B][Hk][D] BF16
    v_new: list
    seed: int = 0


def run_gpu_steps(w: W.Workload, fmt: str, n_steps: int, seed=0):
    """The workload as specified for long contexts: the cached history in one
    append call per sequence, then ONE bulk append of every sequence's bulk
    tokens (all sequences in one call), then n_steps decode steps, each
    appending one token per sequence and decoding over the grown context
    (automatic split plan, FP32 output). Returns a StepsRun."""
    tables, nb = W.block_tables(w, seed)
    ctx = W.context_lengths(w, seed)
    hist, bulk, _ = inputs(w, seed)
    d = kvq.dims(nb, w.n_kv_heads, w.n_q_heads, w.head_dim, tables.shape[1])
    dev = torch.device("cuda")
    cache = kvq.LayerCache.allocate(fmt, d)
    for b in range(w.batch):
        cache.append(hist[b][0].to(dev), hist[b][1].to(dev),
                     torch.from_numpy(slots_for(tables, b, np.arange(ctx[b]))).to(dev))
    if bulk is not None:
        K = torch.cat([x[0] for x in bulk]).to(dev)
        V = torch.cat([x[1] for x in bulk]).to(dev)
        S = torch.cat([torch.from_numpy(slots_for(tables, b, ctx[b] + np.arange(w.bulk_append)))
                       for b in range(w.batch)]).to(dev)
        cache.append(K, V, S)
        del K, V
    c = ctx + w.bulk_append
    tbl = torch.from_numpy(tables).to(dev)
    max_ctx = int((c + n_steps).max())
    ws = cache.workspace(w.batch, max_ctx)
    outs, qs, ks, vs = [], [], [], []
    for s in range(n_steps):
        q, k, v = W.step_inputs(w, s, seed)
        sl = np.array([slots_for(tables, b, [c[b]])[0] for b in range(w.batch)], dtype=np.int64)
        cache.append(k.to(dev), v.to(dev), torch.from_numpy(sl).to(dev))
        c = c + 1
        cl = torch.from_numpy(c.astype(np.int32)).to(dev)
        outs.append(cache.decode(q.to(dev), tbl, cl, max_ctx, sm_scale=w.sm_scale, workspace=ws,
                                 out_dtype=torch.float32).cpu())
        qs.append(q)
        ks.append(k)
        vs.append(v)
    torch.cuda.synchronize()
    assert kvq.device_error(clear=True) == 0
    return StepsRun(w, fmt, cache, tables, ctx, n_steps, outs, qs, ks, vs, seed)


def check_steps_run(run: StepsRun, b: int, steps):
    """Codes and scales of sequence b after every step bit-exact against the
    oracle's, and its attention output at each of `steps` within tolerance.
    Returns (max err, mean err) over the checked steps."""
    w = run.w
    hist, bulk, _ = inputs(w, run.seed)
    k = torch.cat([hist[b][0]] + ([bulk[b][0]] if bulk is not None else []) +
                  [x[b:b + 1] for x in run.k_new]).float().numpy()
    v = torch.cat([hist[b][1]] + ([bulk[b][1]] if bulk is not None else []) +
                  [x[b:b + 1] for x in run.v_new]).float().numpy()
    n = k.shape[0]
    # the cache view of assert_codes_equal: every sequence's tokens after the last step
    one = DeviceRun(w, run.fmt, run.cache, run.tables, run.ctx_hist,
                 run.ctx_hist + w.bulk_append + run.steps, None, None, None, None, run.seed)
    assert int(one.ctx_after[b]) == n
    res = {"Kraw": k.astype(np.float64), "Vraw": v.astype(np.float64)}
    for name, x in (("k", k), ("v", v)):
        if run.fmt == "fp8":
            c, s = OF.fp8_quantize(x)
            res[name + "_codes"], res[name + "_scale"] = c, s
            res[name.upper()] = OF.fp8_dequantize(c, s)
        elif run.fmt == "int8":
            c, s, z = OF.int8_quantize(x)
            res[name + "_codes"], res[name + "_scale"], res[name + "_zp"] = c, s, z
            res[name.upper()] = OF.int8_dequantize(c, s, z)
        else:
            res[name + "_codes"] = OF.bf16_round(x)
            res[name.upper()] = x.astype(np.float64)
    assert_codes_equal(one, b, res)
    errs = []
    base = n - run.steps
    for s in steps:
        L = base + s + 1
        q = run.q[s][b:b + 1].float().numpy().astype(np.float64)
        o = OA.decode_attention(q, [(res["K"][:L], res["V"][:L])], w.sm_scale, w.n_kv_heads)[0]
        errs.append(np.abs(run.outs[s][b].numpy().astype(np.float64) - o).ravel())
    e = np.concatenate(errs)
    return float(e.max()), float(e.mean())
