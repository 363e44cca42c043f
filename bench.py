#!/usr/bin/env python
"""Benchmark of the quantized paged KV-cache decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--fmt F]
    python bench.py --impl reference ...        # the CPU oracle, same metric

One step = the whole hot path for one decode step of the workload: append one
new token per sequence into the quantized paged cache (kvq_append), paged GQA
decode attention split into chunk partials (kvq_decode_partial) and the
log-sum-exp merge into the BF16 output (kvq_decode_merge).

Headline `value`: decode KV bytes read per step (all ranks) / step time, GB/s.
Inputs live in HBM before timing; L2 is flushed (a 256 MB write) before every
timed step and each step is timed on its stream with CUDA events. A timed step
is one CUDA graph replay of its three launches; the per-phase times come from
the same steps launched one by one with events between the phases. K steps are
bracketed by a barrier and a device synchronize; the max over ranks is taken.
Multi-GPU runs are weak-scaled replicas: each rank holds its own batch of
sequences (the path has no exchange step), so `value` sums all ranks' bytes.
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int8_quantized_paged_quantize_b200 import workloads as WL  # noqa: E402

DEFAULT_WORKLOAD = "llama3-8b-fp8"
# per (token, KV head): K and V metadata (the static INT8 formats keep one
# fixed scale per channel or per cache instead)
META_BYTES = {"fp8": 4, "int8": 8, "bf16": 0, "e5m2": 4, "int8c": 0, "int8t": 0}
ELEM = {"fp8": 1, "int8": 1, "bf16": 2, "e5m2": 1, "int8c": 1, "int8t": 1}
DTYPE_TAG = {"fp8": "e4m3 cache / f32 accumulate", "int8": "s8 cache / f32 accumulate",
             "bf16": "bf16 cache / f32 accumulate", "e5m2": "e5m2 cache / f32 accumulate",
             "int8c": "s8 cache, static per-channel scales / f32 accumulate",
             "int8t": "s8 cache, static per-tensor scales / f32 accumulate"}
STATIC = ("int8c", "int8t")


# ----------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kv_bytes_per_step(ctx, w, fmt):
    """Algorithmic bytes one decode step reads: the K and V codes plus their
    per-token metadata for every attended token and KV head, the queries and
    the block-table entries."""
    ctx = np.asarray(ctx, dtype=np.int64)
    kv = int(ctx.sum()) * w.n_kv_heads * (2 * w.head_dim * ELEM[fmt] + META_BYTES[fmt])
    q = w.batch * w.n_q_heads * w.head_dim * 2
    tables = 4 * int(((ctx + 15) // 16).sum())
    return kv, kv + q + tables


def append_bytes_per_token(w, fmt):
    """Append: read K and V BF16 rows, write codes and metadata."""
    return w.n_kv_heads * (2 * w.head_dim * 2 + 2 * w.head_dim * ELEM[fmt] + META_BYTES[fmt])


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.proc, self.path = None, None
        try:
            self.id = "GPU-" + str(torch.cuda.get_device_properties(index).uuid)
        except Exception:
            self.id = str(index)

    def start(self):
        try:
            import tempfile
            self.path = tempfile.mktemp(suffix=".csv")
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.id}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "10"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # the timed region is short: wait until the sampler is producing lines
        t0 = time.time()
        while time.time() - t0 < 5.0 and os.path.getsize(self.path) == 0:
            time.sleep(0.02)

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            c = [x.strip() for x in line.split(",")]
            if len(c) < 9:
                continue
            try:
                sm.append(float(c[1]))
                mx.append(float(c[2]))
            except ValueError:
                continue
            for n, v in zip(names, c[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_traffic(workload, fmt):
    """DRAM bytes per decode launch from the committed ncu capture of this
    workload, or None when there is none or the kernel sources changed since."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    csrc = os.path.join(ROOT, "int8_quantized_paged_quantize_b200", "csrc")
    for name, sha in rec.get("kernel_sha256", {}).items():
        path = os.path.join(csrc, name)
        if not os.path.exists(path):
            return None
        with open(path, "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != sha:
                return None
    v = rec.get("bytes_per_launch", {}).get(f"{workload}/{fmt}")
    return float(v) if v is not None else None


# ----------------------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()



def max_over_ranks(x, world, device="cuda"):
    """Max of a float over all ranks (identity on one rank)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world, device="cuda"):
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# ----------------------------------------------------------------------------- GPU setup
class Setup:
    """Device-resident state of one workload in one format: the filled cache,
    per-step inputs, slots, context lengths, workspace and output."""

    def __init__(self, w, fmt, steps, seed, hist=None):
        from int8_quantized_paged_quantize_b200 import kvq
        self.kvq = kvq
        self.w, self.fmt, self.steps = w, fmt, steps
        self.tables_np, nb = WL.block_tables(w, seed)
        self.ctx0 = WL.context_lengths(w, seed) + w.bulk_append
        d = kvq.dims(nb, w.n_kv_heads, w.n_q_heads, w.head_dim, self.tables_np.shape[1])
        self.dims = d
        dev = torch.device("cuda")
        self.hist = hist if hist is not None else self.make_history(w, seed)
        if fmt in STATIC:
            ks, vs = self.static_scales(self.hist, fmt == "int8c")
            self.cache = kvq.LayerCache.allocate(fmt, d, k_static=ks.to(dev), v_static=vs.to(dev))
        else:
            self.cache = kvq.LayerCache.allocate(fmt, d)
        self.tables = torch.from_numpy(self.tables_np).to(dev)
        self.fill()
        # per-step inputs, resident in HBM
        self.q, self.k, self.v, self.slots, self.ctx = [], [], [], [], []
        ctx = self.ctx0.copy()
        for s in range(steps):
            q, k, v = WL.step_inputs(w, s, seed)
            self.q.append(q.to(dev))
            self.k.append(k.to(dev))
            self.v.append(v.to(dev))
            sl = self.tables_np[np.arange(w.batch), ctx // 16].astype(np.int64) * 16 + ctx % 16
            self.slots.append(torch.from_numpy(sl).to(dev))
            ctx = ctx + 1
            self.ctx.append(torch.from_numpy(ctx.astype(np.int32)).to(dev))
        self.ctx_np = [self.ctx0 + s + 1 for s in range(steps)]
        self.max_ctx = int(self.ctx_np[-1].max())
        self.ws = self.cache.workspace(w.batch, self.max_ctx)
        self.out = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device=dev)

    @staticmethod
    def static_scales(hist, per_channel):
        """Static INT8 scales, calibrated on the cached history before anything is
        timed (the caller's job in a deployment): bf16(max |x| / 127) per (KV
        head, channel) or over the whole cache, for K and for V."""
        out = []
        for x in hist[:2]:
            a = x.abs().amax(dim=0).float() if per_channel else x.abs().amax().float().reshape(1)
            out.append((a / 127.0).to(torch.bfloat16).contiguous())
        return out

    @staticmethod
    def make_history(w, seed):
        """BF16 K/V of every sequence's cached tokens (history + bulk append),
        concatenated, with their slots."""
        tables, _ = WL.block_tables(w, seed)
        ctx = WL.context_lengths(w, seed)
        ks, vs, ss = [], [], []
        for b in range(w.batch):
            k, v = WL.kv_history(w, b, seed)
            ks.append(k)
            vs.append(v)
            pos = np.arange(ctx[b])
            if w.bulk_append:
                kb, vb = WL.kv_bulk(w, b, seed)
                ks.append(kb)
                vs.append(vb)
                pos = np.arange(ctx[b] + w.bulk_append)
            ss.append(torch.from_numpy(tables[b][pos // 16].astype(np.int64) * 16 + pos % 16))
        return torch.cat(ks), torch.cat(vs), torch.cat(ss)

    def fill(self, chunk=1 << 16):
        K, V, S = self.hist
        dev = torch.device("cuda")
        for a in range(0, S.numel(), chunk):
            self.cache.append(K[a:a + chunk].to(dev), V[a:a + chunk].to(dev), S[a:a + chunk].to(dev))
        torch.cuda.synchronize()

    def reset_tail(self):
        """Nothing to undo: step s appends at position ctx0 + s, so re-running the
        steps overwrites the same slots with the same values."""

    # one step of the hot path, with events between its phases
    def step(self, s, ev=None):
        kvq, c = self.kvq, self.cache
        w = self.w
        c.append(self.k[s], self.v[s], self.slots[s])
        if ev is not None:
            ev[1].record()
        kvq.decode_partial(self.q[s], c.k, c.v, c.k_scale, c.v_scale, self.tables, self.ctx[s],
                           self.max_ctx, w.sm_scale, self.ws, self.fmt, self.dims)
        if ev is not None:
            ev[2].record()
        kvq.decode_merge(w.batch, self.ctx[s], self.max_ctx, self.out, self.ws, self.fmt, self.dims)


def timed_loop(st, steps, warmup, world, flush):
    """Run warmup + steps; returns per-phase mean milliseconds over the timed steps."""
    for s in range(warmup):
        st.step(s % st.steps)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev = evs[i]
        ev[0].record()
        st.step(i % st.steps, ev)
        ev[3].record()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    step_ms = [e[0].elapsed_time(e[3]) for e in evs]
    app_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[1].elapsed_time(e[2]) for e in evs]
    mrg_ms = [e[2].elapsed_time(e[3]) for e in evs]
    return {"step": float(np.mean(step_ms)), "append": float(np.mean(app_ms)),
            "decode": float(np.mean(dec_ms)), "merge": float(np.mean(mrg_ms)),
            "launches": 3 * steps}


def graph_loop(st, steps, warmup, world, flush):
    """The same steps, each replayed as one CUDA graph of its three launches
    (append, decode partials, merge), as a serving loop that captures its
    decode step runs them; the graph removes the host launch gaps between the
    kernels, not any of their work. One graph per step index (the step's
    inputs differ); L2 flushed before every timed replay. Returns the mean
    step milliseconds."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                 # eager warm-up before capture
        for s in range(min(3, st.steps)):
            st.step(s)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graphs = {}

    def graph_of(s):
        if s not in graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                st.step(s)
            graphs[s] = g
        return graphs[s]

    for s in range(warmup):
        graph_of(s % st.steps).replay()
    for i in range(steps):
        graph_of(i % st.steps)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        evs[i][0].record()
        graphs[i % st.steps].replay()
        evs[i][1].record()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in evs]
    graphs.clear()
    return float(np.mean(ms))


def e2e_loop(st, steps, warmup, world, flush):
    """The same step through the public API with host inputs: per step the
    step's inputs (q, k, v, slots, context lengths, the block tables) are copied
    from pinned host memory and the output is read back, inside the timing. The
    inputs of a step are packed into one pinned buffer (each at a 256-byte
    aligned offset) and cross in one copy; the kernels take views into it."""
    w = st.w

    def layout(tensors):
        offs, o = [], 0
        for t in tensors:
            offs.append(o)
            o += (t.numel() * t.element_size() + 255) // 256 * 256
        return offs, o

    def step_tensors(s):
        return [st.q[s], st.k[s], st.v[s], st.slots[s], st.ctx[s], st.tables]

    offs, nbytes = layout(step_tensors(0))
    host = []
    for s in range(st.steps):
        hb = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
        for t, o in zip(step_tensors(s), offs):
            n = t.numel() * t.element_size()
            hb[o:o + n].copy_(t.contiguous().view(-1).view(torch.uint8).cpu())
        host.append(hb)
    dbuf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    views = []
    for t, o in zip(step_tensors(0), offs):
        n = t.numel() * t.element_size()
        views.append(dbuf[o:o + n].view(t.dtype).view(t.shape))
    out_h = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()
    h2d = nbytes
    d2h = out_h.numel() * out_h.element_size()

    def one(s):
        dbuf.copy_(host[s], non_blocking=True)
        q, k, v, sl, cl, tables_d = views
        st.cache.append(k, v, sl)
        st.cache.decode(q, tables_d, cl, st.max_ctx, sm_scale=w.sm_scale, out=st.out,
                        workspace=st.ws)
        out_h.copy_(st.out, non_blocking=True)

    for s in range(warmup):
        one(s % st.steps)
    torch.cuda.synchronize()
    barrier(world)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        evs[i][0].record()
        one(i % st.steps)
        evs[i][1].record()
    torch.cuda.synchronize()
    barrier(world)
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    return ms, h2d, d2h


def verify_rate(st, flush, n_query=2, reps=10, warmup=3):
    """Multi-query decode (speculative verification, kvq_decode_verify) over the
    cache as the first timed step leaves it: the last n_query cached tokens of
    every sequence are the positions being verified. L2 flushed before every
    timed call. None when the GQA group times n_query exceeds 8."""
    w, kvq, c = st.w, st.kvq, st.cache
    if w.group * n_query > 8:
        return None
    g = torch.Generator(device="cuda").manual_seed(7)
    q = torch.randn(w.batch, w.n_q_heads, n_query, w.head_dim, generator=g,
                    device="cuda").to(torch.bfloat16)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    import ctypes
    n = kvq.lib().kvq_decode_verify_workspace_bytes(w.batch, n_query, st.max_ctx, 0,
                                                    kvq.FMT[st.fmt], ctypes.byref(st.dims))
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")

    def call():
        kvq.decode_verify(q, c.k, c.v, c.k_scale, c.v_scale, st.tables, st.ctx[0], st.max_ctx,
                          w.sm_scale, out, st.fmt, st.dims, workspace=ws)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for a, b in evs:
        flush.zero_()
        a.record()
        call()
        b.record()
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    kv, alg = kv_bytes_per_step(st.ctx_np[0], w, st.fmt)
    hbm, _ = peaks()
    return {"n_query": n_query, "ms": ms, "kv_gbs": kv / (ms * 1e-3) / 1e9,
            "frac_of_peak": kv / (ms * 1e-3) / 1e9 / hbm,
            "positions_per_s": w.batch * n_query / (ms * 1e-3),
            "what": "decode partials + merge for n_query positions per sequence, pages read once"}


def bulk_append_rate(st, tokens=32768, reps=5):
    """Append throughput for one bulk call of `tokens` tokens (prefill-style)."""
    K, V, S = st.hist
    n = min(tokens, S.numel())
    dev = torch.device("cuda")
    k, v, s = K[:n].to(dev), V[:n].to(dev), S[:n].to(dev)
    for _ in range(2):
        st.cache.append(k, v, s)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        st.cache.append(k, v, s)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    return n / (ms * 1e-3), ms, n


def bulk_append_probe(fmt, mode, reps=5, T=32768, Hk=8, D=128):
    """One bulk append of T tokens (all Hk heads) into a fresh cache, timed with
    CUDA events over `reps` calls after two untimed ones. `aligned`: 4 sequences
    of T/4 tokens, so every 16-token window is one whole page. `continued`:
    sequences of seeded lengths in [17, 3000) laid end to end in the input, so
    most windows straddle two pages of two sequences. Returns one JSON-ready dict."""
    from int8_quantized_paged_quantize_b200 import kvq
    rng = np.random.default_rng(0)
    if mode == "aligned":
        lens = [T // 4] * 4
    else:
        lens = []
        while sum(lens) < T:
            lens.append(int(rng.integers(17, 3000)))
        lens[-1] -= sum(lens) - T
    nb = sum((n + 15) // 16 for n in lens) + 8
    perm = rng.permutation(nb)
    slots, p = [], 0
    for n in lens:
        npg = (n + 15) // 16
        blocks = perm[p:p + npg]
        p += npg
        pos = np.arange(n)
        slots.append(blocks[pos // 16].astype(np.int64) * 16 + pos % 16)
    slots = torch.from_numpy(np.concatenate(slots)).cuda()
    d = kvq.dims(nb, Hk, Hk * 4, D, max((n + 15) // 16 for n in lens))
    g = torch.Generator(device="cuda").manual_seed(0)
    k = torch.randn(T, Hk, D, dtype=torch.bfloat16, device="cuda", generator=g)
    v = torch.randn(T, Hk, D, dtype=torch.bfloat16, device="cuda", generator=g)
    if fmt in STATIC:
        ks, vs = Setup.static_scales((k, v), fmt == "int8c")
        cache = kvq.LayerCache.allocate(fmt, d, k_static=ks, v_static=vs)
    else:
        cache = kvq.LayerCache.allocate(fmt, d)
    for _ in range(2):
        cache.append(k, v, slots)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        cache.append(k, v, slots)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    by = T * append_bytes_per_token(dataclasses.replace(WL.WORKLOADS[DEFAULT_WORKLOAD],
                                                        n_kv_heads=Hk, head_dim=D), fmt)
    hbm, kind = peaks()
    return {"bulk_append": mode, "fmt": fmt, "tokens": T, "sequences": len(lens), "us": ms * 1e3,
            "tok_per_s": T / (ms * 1e-3), "gbs": by / (ms * 1e6), "frac": by / (ms * 1e6) / hbm,
            "peak_kind": kind, "bytes": by}


# ----------------------------------------------------------------------------- CPU oracle
def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def oracle_decode_sample(w, fmt, seed, budget_s=12.0):
    """Time the CPU oracle on a bounded sample of the workload: for sequences in
    order until the time budget is spent, quantize the sequence's cached K/V into
    an oracle pool (append) and run the decode step's attention over it for all
    query heads (dequantising gather + FP64 softmax attention). Returns
    (decode KV GB/s, append tok/s, sample description, threads)."""
    from oracle import attention as OA
    from oracle import paged as OP
    tables, nb = WL.block_tables(w, seed)
    ctx = WL.context_lengths(w, seed)
    q, kn, vn = WL.step_inputs(w, 0, seed)
    t_app = t_dec = 0.0
    n_tok = 0
    kv_bytes = 0
    done = []
    t_start = time.perf_counter()
    for b in range(w.batch):
        if time.perf_counter() - t_start > budget_s and done:
            break
        k, v = WL.kv_history(w, b, seed)
        k = torch.cat([k, kn[b:b + 1]]).float().numpy()
        v = torch.cat([v, vn[b:b + 1]]).float().numpy()
        n = k.shape[0]
        pages = (n + 15) // 16
        if fmt in STATIC:
            from oracle import formats as OF
            per_channel = fmt == "int8c"
            pool = OP.LogicalPool(fmt, pages, w.n_kv_heads, 16, w.head_dim,
                                  k_static=OF.int8_static_calibrate(k, per_channel),
                                  v_static=OF.int8_static_calibrate(v, per_channel))
        else:
            pool = OP.LogicalPool(fmt, pages, w.n_kv_heads, 16, w.head_dim)
        row = np.arange(pages)
        t0 = time.perf_counter()
        pool.append(k, v, OP.slot_of(row, np.arange(n), 16))
        t1 = time.perf_counter()
        K, V = pool.gather(row, n)
        OA.decode_attention(q[b:b + 1].float().numpy(), [(K, V)], w.sm_scale, w.n_kv_heads)
        t2 = time.perf_counter()
        t_app += t1 - t0
        t_dec += t2 - t1
        n_tok += n
        kv_bytes += n * w.n_kv_heads * (2 * w.head_dim * ELEM[fmt] + META_BYTES[fmt])
        done.append(b)
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = 1
    desc = (f"{len(done)} of {w.batch} sequences ({n_tok} tokens, all {w.n_q_heads} query heads): "
            f"oracle append of their cached tokens + one decode step")
    return kv_bytes / t_dec / 1e9, n_tok / t_app, desc, threads


def run_reference(args):
    """The oracle as the reference arm: same metric/unit/config, each step a
    bounded sample of the workload on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = WL.WORKLOADS[args.workload]
    fmt = args.fmt or w.fmt
    vals = []
    t0 = time.perf_counter()
    # each step samples the workload for a bounded time so that the whole run
    # stays near two minutes whatever --steps / --warmup are
    budget = min(args.ref_budget, 120.0 / max(1, args.warmup + args.steps))
    for s in range(args.warmup + args.steps):
        gbs, tok_s, desc, threads = oracle_decode_sample(w, fmt, seed=0, budget_s=budget)
        if s >= args.warmup:
            vals.append(gbs)
    value = float(np.mean(vals))
    line = {"impl": "reference", "metric": metric_name(fmt), "value": value, "unit": "GB/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * (time.perf_counter() - t0) / max(1, args.warmup + args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded)",
            "config": config_block(w, fmt, l2="host run (no GPU)"),
            "cpu_baseline": {"kind": "oracle", "value": value, "unit": "GB/s", "cores": threads,
                             "sample": desc, "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def metric_name(fmt):
    return f"paged decode-attn KV GB/s ({fmt.upper()} cache; step = append + decode + merge)"


def config_block(w, fmt, l2):
    if w.lengths == "fixed":
        lens = f"{w.ctx[0]}"
    elif w.lengths == "uniform":
        lens = f"U[{w.ctx[0]},{w.ctx[1]}]"
    elif w.lengths == "lognormal_mix":
        lens = "lognormal(1500, 1) + 4x30000"
    else:
        lens = "list"
    return {"workload": f"{w.name}: B={w.batch} Hq={w.n_q_heads} Hk={w.n_kv_heads} D={w.head_dim} "
                        f"bs=16 ctx={lens}" + (f" +{w.bulk_append} bulk" if w.bulk_append else ""),
            "fmt": fmt, "batch": w.batch, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim, "block_size": 16, "l2": l2}


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(WL.WORKLOADS))
    ap.add_argument("--fmt", default=None, choices=["fp8", "int8", "bf16", "e5m2", "int8c", "int8t"])
    ap.add_argument("--no-formats", action="store_true", help="skip the per-format comparison")
    ap.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline leg")
    ap.add_argument("--ref-budget", type=float, default=10.0)
    ap.add_argument("--bulk-append", choices=["aligned", "continued"], default=None,
                    help="only time one bulk append of 32,768 tokens and print its line")
    ap.add_argument("--reps", type=int, default=5, help="timed calls of --bulk-append")
    args = ap.parse_args()
    if args.bulk_append:
        print(json.dumps(bulk_append_probe(args.fmt or "fp8", args.bulk_append, args.reps)))
        return 0
    if args.impl == "reference":
        return run_reference(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    rank, world, local = dist_setup(args.gpus)
    w = WL.WORKLOADS[args.workload]
    fmt = args.fmt or w.fmt
    steps_needed = args.warmup + args.steps
    wb = dataclasses.replace(w, decode_steps=max(w.decode_steps, steps_needed))
    seed = rank
    hbm_peak, peak_kind = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    hist = Setup.make_history(wb, seed)
    st = Setup(wb, fmt, steps_needed, seed, hist=hist)
    clocks = ClockSampler(local)
    clocks.start()
    t = timed_loop(st, args.steps, args.warmup, world, flush)        # per-phase events
    tg = graph_loop(st, args.steps, args.warmup, world, flush)        # the step as one graph
    clk = clocks.stop()

    step_ms = max_over_ranks(tg, world)
    dec_ms = max_over_ranks(t["decode"], world)
    # bytes of the timed steps (contexts grow by one per step)
    kv_list, all_list = zip(*[kv_bytes_per_step(st.ctx_np[i % st.steps], wb, fmt)
                              for i in range(args.steps)])
    kv_step = float(np.mean(kv_list))
    alg_step = float(np.mean(all_list))
    kv_total = sum_over_ranks(kv_step, world)
    value = kv_total / (step_ms * 1e-3) / 1e9
    achieved = alg_step / (t["decode"] * 1e-3) / 1e9
    seqs_s = sum_over_ranks(wb.batch, world) / (step_ms * 1e-3)
    app_tok_s = sum_over_ranks(wb.batch, world) / (max_over_ranks(t["append"], world) * 1e-3)
    bulk_tok_s, bulk_ms, bulk_n = bulk_append_rate(st)
    try:
        verify = verify_rate(st, flush)
    except Exception as e:                        # reported, never fatal to the main line
        verify = {"error": f"{type(e).__name__}: {e}"[:200]}

    e2e_ms, h2d, d2h = e2e_loop(st, args.steps, args.warmup, world, flush)
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e_val = kv_total / (e2e_ms * 1e-3) / 1e9

    formats = {}
    outs = {}
    if not args.no_formats:
        for f in ("fp8", "int8", "e5m2", "int8c", "int8t", "bf16"):
            if f == fmt:
                tf, stf = t, st
            else:
                del st
                torch.cuda.empty_cache()
                stf = Setup(wb, f, steps_needed, seed, hist=hist)
                tf = timed_loop(stf, args.steps, args.warmup, world, flush)
            kvf = float(np.mean([kv_bytes_per_step(stf.ctx_np[i % stf.steps], wb, f)[0]
                                 for i in range(args.steps)]))
            algf = float(np.mean([kv_bytes_per_step(stf.ctx_np[i % stf.steps], wb, f)[1]
                                  for i in range(args.steps)]))
            bt, _, _ = bulk_append_rate(stf)
            smax = max_over_ranks(tf["step"], world)
            formats[f] = {
                "kv_gbs_step": sum_over_ranks(kvf, world) / (smax * 1e-3) / 1e9,
                "decode_kernel_gbs": algf / (tf["decode"] * 1e-3) / 1e9,
                "decode_frac_of_peak": algf / (tf["decode"] * 1e-3) / 1e9 / hbm_peak,
                "decode_seqs_per_s": sum_over_ranks(wb.batch, world) / (smax * 1e-3),
                "append_tok_per_s_step": sum_over_ranks(wb.batch, world) / (tf["append"] * 1e-3),
                "append_tok_per_s_bulk": bt,
                "ms": {k: round(v, 5) for k, v in tf.items() if k != "launches"},
                "kv_bytes_per_step": kvf,
            }
            # step 0's attention again, in FP32: every format holds the same tokens
            # up to that context, so the outputs compare directly
            outs[f] = stf.cache.decode(stf.q[0], stf.tables, stf.ctx[0], stf.max_ctx,
                                       sm_scale=wb.sm_scale, workspace=stf.ws,
                                       out_dtype=torch.float32).cpu()
            st = stf
        # quality number (reported, not a pass criterion): the quantized cache's
        # attention output against the same kernel on the unquantized BF16 cache
        for f in ("fp8", "int8", "e5m2", "int8c", "int8t"):
            dev = (outs[f] - outs["bf16"]).abs()
            ref = outs["bf16"].abs()
            formats[f]["quality_vs_bf16_cache"] = {
                "max_abs": float(dev.max()), "mean_abs": float(dev.mean()),
                "rel_l2": float((outs[f] - outs["bf16"]).norm() / max(float(outs["bf16"].norm()), 1e-30)),
                "mean_abs_ref": float(ref.mean()), "step": 0}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        gbs, tok_s, desc, threads = oracle_decode_sample(wb, fmt, seed=0)
        cpu = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc,
               "append_tok_per_s": tok_s, "cpu_model": cpu_model()}

    line = {
        "metric": metric_name(fmt), "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DTYPE_TAG[fmt], "data": "synthetic (seeded; no dataset or weights)",
        "config": dict(config_block(wb, fmt, l2="flushed before every timed step (256 MB write)"),
                       launch="each timed step is one CUDA graph replay of its append, decode "
                              "and merge launches; phase_ms and the per-format table time the "
                              "same steps launched one by one with events between the phases"),
        "decode_seqs_per_s": seqs_s, "append_tok_per_s_step": app_tok_s,
        "append_tok_per_s_bulk": bulk_tok_s, "kv_frac_of_peak_step": value / world / hbm_peak,
        "phase_ms": {k: round(v, 5) for k, v in t.items() if k != "launches"},
        "ms_per_step_eager": t["step"],
        "roofline": {"bound": "hbm", "kernel": "decode partial (kvq_decode_partial)",
                     "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_kind": peak_kind,
                     "alg_bytes_per_launch": alg_step,
                     "traffic": measured_traffic(w.name, fmt)},
        "e2e": {"value": e2e_val, "unit": "GB/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": t["launches"],
        "verify": verify,
        "clocks": clk,
        "formats": formats,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
