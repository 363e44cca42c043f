#!/usr/bin/env python
"""Benchmark of the quantized paged KV-cache decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--fmt F]
    python bench.py --impl reference ...        # the CPU oracle, same metric

One step = the whole hot path for one decode step of the workload: append one
new token per sequence into the quantized paged cache (kvq_append), paged GQA
decode attention split into chunk partials (kvq_decode_partial) and the
log-sum-exp merge into the BF16 output (kvq_decode_merge).

The default workload is the 70B-shaped layer at 32k context with the INT8
cache (B=32, 64 query / 8 KV heads, head_dim 128), the largest single-GPU
configuration; FP8, E5M2, static INT8 and a BF16 cache of the same kernels are
timed beside it. A `configs` block adds the long-context workload as its
specification runs it (4 sequences: a bulk append of 8,192 tokens each, then
64 decode steps with one append each, for FP8, INT8 and BF16) and the mixed
serving batch (256 sequences, block tables from the library's allocator after
allocate/free churn).

Headline `value`: decode KV bytes read per step (all ranks) / step time, GB/s.
Inputs live in HBM before timing. Every step reads the whole cache (2.2 GB
for the headline workload, 0.6-2.2 GB for the others), far more than the
126 MB L2, so steps run back to back without an L2 flush between them (a
flush by a large write would leave the next step to write back 126 MB of dirty
lines). A timed step is one CUDA graph replay of its three launches; K replays
are timed as one region on the stream with CUDA events, bracketed by a
barrier and a device synchronize, and the max over ranks is taken. The
per-phase times come from the same steps launched one by one with events
between the phases.
The roofline fraction is the decode attention's (partials + merge) algorithmic
bytes over their event time, against the measured HBM copy peak.
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

DEFAULT_WORKLOAD = "70b-32k-int8"
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
    """DRAM bytes (read + write) of one decode step's attention launches
    (partials + merge) from the committed ncu capture of this workload, or None
    when there is none or the kernel sources changed since."""
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
class Layout:
    """Block tables and slots of one workload run, fixed on the host before
    anything is timed: the cached history's slots per sequence, the bulk
    append's (if the workload has one) and every decode step's. The fragmented
    shared pool is grown through the library's block allocator (kvq_pool_*,
    paging.py) after allocate/free churn; the other pools are laid out
    directly by workloads.block_tables."""

    def __init__(self, w, seed, fmt):
        from int8_quantized_paged_quantize_b200 import paging
        ctx = WL.context_lengths(w, seed)
        if w.pool == "fragmented":
            pb = paging.paged_batch(w, seed, fmt)
            self.hist = [pb.extend(b, int(ctx[b])) for b in range(w.batch)]
            self.bulk = [pb.extend(b, w.bulk_append) for b in range(w.batch)]
            self.steps = [pb.extend_all(1) for _ in range(w.decode_steps)]
            self.tables, self.num_blocks = pb.tables.copy(), pb.dims.num_blocks
            self.source = "kvq_pool allocator after seeded allocate/free churn"
            pb.close()
            return
        tables, nb = WL.block_tables(w, seed)

        def slots(b, pos):
            return tables[b][pos // 16].astype(np.int64) * 16 + pos % 16
        self.hist = [slots(b, np.arange(ctx[b])) for b in range(w.batch)]
        self.bulk = [slots(b, ctx[b] + np.arange(w.bulk_append)) for b in range(w.batch)]
        c1 = ctx + w.bulk_append
        self.steps = [np.array([slots(b, np.array([c1[b] + s]))[0] for b in range(w.batch)])
                      for s in range(w.decode_steps)]
        self.tables, self.num_blocks = tables, nb
        self.source = f"workloads.block_tables ({w.pool})"


def history(w, seed, bulk=True):
    """BF16 K/V of every sequence's cached tokens (and its bulk append, when
    `bulk`), concatenated sequence by sequence, drawn on host threads."""
    from concurrent.futures import ThreadPoolExecutor

    def one(b):
        k, v = WL.kv_history(w, b, seed)
        if bulk and w.bulk_append:
            kb, vb = WL.kv_bulk(w, b, seed)
            k, v = torch.cat([k, kb]), torch.cat([v, vb])
        return k, v
    with ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
        parts = list(ex.map(one, range(w.batch)))
    return torch.cat([p[0] for p in parts]), torch.cat([p[1] for p in parts])


class Setup:
    """Device-resident state of one workload in one format: the filled cache,
    per-step inputs, slots, context lengths, workspace and output. `with_bulk`
    False leaves the workload's bulk append out of the fill (it is timed on its
    own)."""

    def __init__(self, w, fmt, steps, seed, hist=None, layout=None, with_bulk=True):
        from int8_quantized_paged_quantize_b200 import kvq
        self.kvq = kvq
        self.w, self.fmt, self.steps = w, fmt, steps
        self.layout = layout if layout is not None else Layout(w, seed, fmt)
        lay = self.layout
        self.tables_np, nb = lay.tables, lay.num_blocks
        bulk = w.bulk_append if with_bulk else 0
        self.ctx0 = WL.context_lengths(w, seed) + bulk
        d = kvq.dims(nb, w.n_kv_heads, w.n_q_heads, w.head_dim, self.tables_np.shape[1])
        self.dims = d
        dev = torch.device("cuda")
        self.hist = hist if hist is not None else history(w, seed, bulk=with_bulk)
        if with_bulk:
            hs = [np.concatenate([lay.hist[b], lay.bulk[b]]) for b in range(w.batch)]
        else:
            hs = lay.hist
        self.hist_slots = torch.from_numpy(np.concatenate(hs).astype(np.int64))
        if fmt in STATIC:
            ks, vs = self.static_scales(self.hist, fmt == "int8c")
            self.cache = kvq.LayerCache.allocate(fmt, d, k_static=ks.to(dev), v_static=vs.to(dev))
        else:
            self.cache = kvq.LayerCache.allocate(fmt, d)
        self.tables = torch.from_numpy(self.tables_np).to(dev)
        self.fill()
        # per-step inputs, resident in HBM; the steps follow the bulk append
        # whether or not the fill holds it
        self.q, self.k, self.v, self.slots, self.ctx = [], [], [], [], []
        for s in range(steps):
            q, k, v = WL.step_inputs(w, s, seed)
            self.q.append(q.to(dev))
            self.k.append(k.to(dev))
            self.v.append(v.to(dev))
            self.slots.append(torch.from_numpy(np.asarray(lay.steps[s], dtype=np.int64)).to(dev))
        self.ctx_np = [self.ctx0 + (0 if with_bulk else w.bulk_append) + s + 1 for s in range(steps)]
        for c in self.ctx_np:
            self.ctx.append(torch.from_numpy(c.astype(np.int32)).to(dev))
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

    def fill(self, chunk=1 << 16):
        K, V = self.hist
        S = self.hist_slots
        dev = torch.device("cuda")
        for a in range(0, S.numel(), chunk):
            self.cache.append(K[a:a + chunk].to(dev), V[a:a + chunk].to(dev), S[a:a + chunk].to(dev))
        torch.cuda.synchronize()

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
    for i in range(steps):                        # back to back: each step reads > L2
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
    inputs differ). The K replays run back to back (each reads more than L2
    holds) and are timed as one region. Returns the mean step milliseconds."""
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
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(steps):
        graphs[i % st.steps].replay()
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    graphs.clear()
    return float(ms)


def e2e_loop(st, steps, warmup, world, flush):
    """The same step through the public API with host inputs: per step the
    step's inputs (q, k, v, slots, context lengths, the block tables) are copied
    from pinned host memory and the output is read back into pinned host
    memory, inside the timing. The inputs of a step are packed into one pinned
    buffer (each at a 256-byte aligned offset) and cross in one copy; the
    kernels take views into it. As a serving loop that prefetches its next step
    does, the copies run on a copy stream: step i+1's inputs go in while step
    i computes (two device input buffers, two output buffers), and step i's
    output comes back while step i+1 computes. The timed region runs from the
    first input copy to the last output copy; the step time is its K-th part.
    L2 is not flushed between these overlapped steps: every step reads a cache
    larger than L2."""
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
    dbuf = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    views = []
    for d in dbuf:
        vv = []
        for t, o in zip(step_tensors(0), offs):
            n = t.numel() * t.element_size()
            vv.append(d[o:o + n].view(t.dtype).view(t.shape))
        views.append(vv)
    outs = [torch.empty_like(st.out) for _ in range(2)]
    out_h = [torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory() for _ in range(2)]
    h2d = nbytes
    d2h = out_h[0].numel() * out_h[0].element_size()
    comp = torch.cuda.current_stream()
    cp = torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]     # input buffer b holds its step
    ev_used = [torch.cuda.Event() for _ in range(2)]   # the step using buffer b is done
    ev_out = [torch.cuda.Event() for _ in range(2)]    # output b is back on the host

    def run(idx):
        n = len(idx)
        cp.wait_stream(comp)
        with torch.cuda.stream(cp):
            dbuf[0].copy_(host[idx[0]], non_blocking=True)
            ev_in[0].record(cp)
        for i in range(n):
            b = i & 1
            if i + 1 < n:
                with torch.cuda.stream(cp):
                    if i >= 1:
                        cp.wait_event(ev_used[b ^ 1])
                    dbuf[b ^ 1].copy_(host[idx[i + 1]], non_blocking=True)
                    ev_in[b ^ 1].record(cp)
            comp.wait_event(ev_in[b])
            if i >= 2:
                comp.wait_event(ev_out[b])
            q, k, v, sl, cl, tables_d = views[b]
            st.cache.append(k, v, sl)
            st.cache.decode(q, tables_d, cl, st.max_ctx, sm_scale=w.sm_scale, out=outs[b],
                            workspace=st.ws)
            ev_used[b].record(comp)
            with torch.cuda.stream(cp):
                cp.wait_event(ev_used[b])
                out_h[b].copy_(outs[b], non_blocking=True)
                ev_out[b].record(cp)
        comp.wait_stream(cp)

    run([s % st.steps for s in range(warmup)])
    torch.cuda.synchronize()
    barrier(world)
    flush.zero_()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(cp)
    run([i % st.steps for i in range(steps)])
    t1.record(cp)
    torch.cuda.synchronize()
    barrier(world)
    ms = t0.elapsed_time(t1) / steps
    return ms, h2d, d2h


def multi_query_rate(st, flush, n_query, call="verify", reps=10, warmup=3):
    """Multi-query attention over the cache as the first timed step leaves it:
    the last n_query cached tokens of every sequence are the positions
    (speculative verification, kvq_decode_verify) or the prefill chunk
    (kvq_prefill_attn). Calls run back to back (each reads the whole cache,
    more than L2 holds). Reports KV bytes
    over time (the pages are read from HBM once per KV head; row groups beyond
    the first re-read them, mostly from L2) and the attention FLOPs."""
    w, kvq, c = st.w, st.kvq, st.cache
    g = torch.Generator(device="cuda").manual_seed(7)
    q = torch.randn(w.batch, w.n_q_heads, n_query, w.head_dim, generator=g,
                    device="cuda").to(torch.bfloat16)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    import ctypes
    size_fn = (kvq.lib().kvq_decode_verify_workspace_bytes if call == "verify"
               else kvq.lib().kvq_prefill_attn_workspace_bytes)
    n = size_fn(w.batch, n_query, st.max_ctx, 0, kvq.FMT[st.fmt], ctypes.byref(st.dims))
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    fn = kvq.decode_verify if call == "verify" else kvq.prefill_attn

    def run():
        fn(q, c.k, c.v, c.k_scale, c.v_scale, st.tables, st.ctx[0], st.max_ctx, w.sm_scale, out,
           st.fmt, st.dims, workspace=ws)

    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for a, b in evs:
        a.record()
        run()
        b.record()
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    kv, alg = kv_bytes_per_step(st.ctx_np[0], w, st.fmt)
    hbm, _ = peaks()
    ctx = np.asarray(st.ctx_np[0], dtype=np.float64)
    # causal: position j sees ctx - n_query + 1 + j tokens
    seen = float(np.sum(np.maximum(0, ctx[:, None] - n_query + 1 + np.arange(n_query)[None, :])))
    flops = 4.0 * w.n_q_heads * w.head_dim * seen
    return {"n_query": n_query, "ms": ms, "kv_gbs": kv / (ms * 1e-3) / 1e9,
            "kv_frac_of_peak": kv / (ms * 1e-3) / 1e9 / hbm,
            "positions_per_s": w.batch * n_query / (ms * 1e-3),
            "attention_tflops": flops / (ms * 1e-3) / 1e12,
            **({"row_groups_per_kv_head": (w.group * n_query) // max(
                g_ for g_ in (8, 4, 2, 1) if (w.group * n_query) % g_ == 0),
                "what": "speculative verification: decode partials (at most 8 query rows per "
                        "tensor-core product) + merge for n_query causal positions per sequence"}
               if call == "verify" else
               {"row_blocks_per_kv_head": -(-w.group * n_query // 128),
                "what": "prefill chunk: prefill partials (128 query rows per tensor-core "
                        "product) + merge for n_query causal positions per sequence"})}


def bulk_append_rate(st, tokens=32768, reps=5):
    """Append throughput for one bulk call of the first `tokens` cached tokens
    (prefill-style, re-appended to their own slots)."""
    K, V = st.hist
    S = st.hist_slots
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


def kivi_probe(fmt, B=32, Hk=8, G=8, D=128, ctx=8192, reps=5):
    """One KIVI-style decode (kvq_kivi_decode_attn) on a mid-size case: B
    sequences of ctx tokens in complete 128-token groups plus one residual
    token each, random BF16 K/V and queries. Timed with CUDA events over
    `reps` calls after three untimed ones. Returns one JSON-ready dict."""
    from int8_quantized_paged_quantize_b200 import kvq
    dev = torch.device("cuda")
    g = torch.Generator(device="cuda").manual_seed(0)
    groups = ctx // 128
    nq = B * groups * 8
    qt = torch.randperm(nq, device=dev, generator=g).to(torch.int32).reshape(B, groups * 8)
    rt = torch.arange(B, device=dev, dtype=torch.int32).reshape(B, 1)
    cache = kvq.KiviCache.allocate(fmt, kvq.dims(nq, Hk, Hk * G, D, groups * 8),
                                   kvq.dims(B, Hk, Hk * G, D, 1))
    pos = torch.arange(groups * 128, device=dev)
    for b in range(B):
        k = torch.randn(groups * 128, Hk, D, device=dev, generator=g).to(torch.bfloat16)
        v = torch.randn(groups * 128, Hk, D, device=dev, generator=g).to(torch.bfloat16)
        cache.append_groups(k, v, qt[b][pos // 16].to(torch.int64) * 16 + pos % 16)
    kr = torch.randn(B, Hk, D, device=dev, generator=g).to(torch.bfloat16)
    cache.residual.append(kr, kr, torch.arange(B, device=dev, dtype=torch.int64) * 16)
    q = torch.randn(B, Hk * G, D, device=dev, generator=g).to(torch.bfloat16)
    ql = torch.full((B,), groups * 128, dtype=torch.int32, device=dev)
    rl = torch.ones(B, dtype=torch.int32, device=dev)
    ws = cache.workspace(B, groups * 128, 1)

    def call():
        cache.decode(q, qt, ql, groups * 128, rt, rl, 1, workspace=ws)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        call()
    e.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(e) / reps
    bits = kvq.KIVI_BITS[fmt]
    by = B * groups * 128 * Hk * (2 * D * bits / 8 + 4 + D * 4 / 128)
    return {"kivi_probe": fmt, "batch": B, "context": groups * 128, "n_kv_heads": Hk, "group": G,
            "head_dim": D, "ms": ms, "kv_gbs": by / (ms * 1e6), "tokens_per_s": B * groups * 128 / (ms * 1e-3),
            "device_error": kvq.device_error()}


def prefill_probe(fmt, B=8, Hk=8, G=8, D=128, ctx=8192, n_query=64, reps=5, call="prefill"):
    """One chunked-prefill (kvq_prefill_attn) or verification (kvq_decode_verify)
    call on a mid-size case: B sequences of ctx cached tokens (random BF16 K/V
    appended through kvq_append, shuffled pages), the last n_query of them the
    chunk. Timed with CUDA events over `reps` calls after three untimed ones.
    Returns one JSON-ready dict (KV bytes read once per call, attention FLOPs
    of the causal chunk)."""
    from int8_quantized_paged_quantize_b200 import kvq
    dev = torch.device("cuda")
    g = torch.Generator(device="cuda").manual_seed(0)
    npg = (ctx + 15) // 16
    nb = B * npg
    tables = torch.randperm(nb, device=dev, generator=g).to(torch.int32).reshape(B, npg)
    d = kvq.dims(nb, Hk, Hk * G, D, npg)
    k = torch.randn(B * ctx, Hk, D, device=dev, generator=g).to(torch.bfloat16)
    v = torch.randn(B * ctx, Hk, D, device=dev, generator=g).to(torch.bfloat16)
    pos = torch.arange(ctx, device=dev)
    slots = torch.cat([tables[b][pos // 16].to(torch.int64) * 16 + pos % 16 for b in range(B)])
    if fmt in STATIC:
        ks, vs = Setup.static_scales((k, v), fmt == "int8c")
        cache = kvq.LayerCache.allocate(fmt, d, k_static=ks, v_static=vs)
    else:
        cache = kvq.LayerCache.allocate(fmt, d)
    cache.append(k, v, slots)
    del k, v
    q = torch.randn(B, Hk * G, n_query, D, device=dev, generator=g).to(torch.bfloat16)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lens = torch.full((B,), ctx, dtype=torch.int32, device=dev)
    import ctypes
    size_fn = (kvq.lib().kvq_prefill_attn_workspace_bytes if call == "prefill"
               else kvq.lib().kvq_decode_verify_workspace_bytes)
    n = size_fn(B, n_query, ctx, 0, kvq.FMT[fmt], ctypes.byref(d))
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
    fn = kvq.prefill_attn if call == "prefill" else kvq.decode_verify

    def run():
        fn(q, cache.k, cache.v, cache.k_scale, cache.v_scale, tables, lens, ctx, D ** -0.5, out,
           fmt, d, workspace=ws)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        run()
    e.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(e) / reps
    seen = float(B * sum(ctx - n_query + 1 + j for j in range(n_query)))
    flops = 4.0 * Hk * G * D * seen
    kv = B * ctx * Hk * (2 * D * ELEM[fmt] + META_BYTES[fmt])
    return {"probe": call, "fmt": fmt, "batch": B, "context": ctx, "n_query": n_query,
            "n_kv_heads": Hk, "group": G, "head_dim": D, "ms": ms,
            "attention_tflops": flops / (ms * 1e-3) / 1e12, "kv_gbs": kv / (ms * 1e6),
            "device_error": kvq.device_error()}


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


ORACLE_SAMPLE_TOKENS = 65536
_SAMPLE_INPUTS = {}


def oracle_sample(w, seed):
    """The fixed CPU sample of a workload: its first sequences, in order, until
    they hold ORACLE_SAMPLE_TOKENS cached tokens (at least one sequence)."""
    ctx = WL.context_lengths(w, seed) + w.bulk_append
    n, tok = 0, 0
    while n < w.batch and (n == 0 or tok < ORACLE_SAMPLE_TOKENS):
        tok += int(ctx[n])
        n += 1
    return n


def oracle_decode_sample(w, fmt, seed, threads=None):
    """Time the CPU oracle on the fixed sample of the workload (oracle_sample):
    for each sampled sequence, quantize its cached K/V and the step token into
    an oracle pool (append) and run the decode step's attention over it for all
    query heads (dequantising gather + FP64 softmax attention). `threads` caps
    the BLAS / OpenMP threads (None: all the host's). Returns (decode KV GB/s,
    append tok/s, sample description, threads used)."""
    from threadpoolctl import threadpool_info, threadpool_limits

    from oracle import attention as OA
    from oracle import paged as OP
    key = (w.name, seed)
    if key not in _SAMPLE_INPUTS:                 # drawn once, outside the timing
        q, kn, vn = WL.step_inputs(w, 0, seed)
        n_seq = oracle_sample(w, seed)
        seqs = []
        for b in range(n_seq):
            k, v = WL.kv_history(w, b, seed)
            if w.bulk_append:
                kb, vb = WL.kv_bulk(w, b, seed)
                k, v = torch.cat([k, kb]), torch.cat([v, vb])
            seqs.append((torch.cat([k, kn[b:b + 1]]).float().numpy(),
                         torch.cat([v, vn[b:b + 1]]).float().numpy()))
        _SAMPLE_INPUTS.clear()
        _SAMPLE_INPUTS[key] = (q, seqs)
    q, seqs = _SAMPLE_INPUTS[key]
    n_seq = len(seqs)
    t_app = t_dec = 0.0
    n_tok = 0
    kv_bytes = 0
    with threadpool_limits(limits=threads):
        used = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        for b in range(n_seq):
            k, v = seqs[b]
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
    desc = (f"{n_seq} of {w.batch} sequences ({n_tok} tokens, all {w.n_q_heads} query heads): "
            f"oracle append of their cached tokens + one decode step")
    return kv_bytes / t_dec / 1e9, n_tok / t_app, desc, used


def run_reference(args):
    """The oracle as the reference arm: same metric/unit/config, each step the
    workload's fixed CPU sample (oracle_sample) on all the host's cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = WL.WORKLOADS[args.workload]
    fmt = args.fmt or w.fmt
    vals, tok = [], []
    t0 = time.perf_counter()
    desc, threads = "", 1
    for s in range(args.warmup + args.steps):
        gbs, tok_s, desc, threads = oracle_decode_sample(w, fmt, seed=0)
        if s >= args.warmup:
            vals.append(gbs)
            tok.append(tok_s)
    value = float(np.mean(vals))
    line = {"impl": "reference", "metric": metric_name(fmt), "value": value, "unit": "GB/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * (time.perf_counter() - t0) / max(1, args.warmup + args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded)",
            "config": config_block(w, fmt, l2="host run (no GPU)"),
            "cpu_baseline": {"kind": "oracle", "value": value, "unit": "GB/s", "cores": threads,
                             "sample": desc, "append_tok_per_s": float(np.mean(tok)),
                             "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def step_metrics(st, t, fmt, world, hbm_peak, steps):
    """The per-format numbers of one Setup timed by timed_loop: step and decode
    throughput, fractions of the HBM peak (decode = partials + merge, as the
    roofline counts it; the partials alone beside it), append rates."""
    w = st.w
    kv = float(np.mean([kv_bytes_per_step(st.ctx_np[i % st.steps], w, fmt)[0] for i in range(steps)]))
    alg = float(np.mean([kv_bytes_per_step(st.ctx_np[i % st.steps], w, fmt)[1] for i in range(steps)]))
    smax = max_over_ranks(t["step"], world)
    dec = t["decode"] + t["merge"]
    return {
        "kv_gbs_step": sum_over_ranks(kv, world) / (smax * 1e-3) / 1e9,
        "kv_frac_of_peak_step": kv / (smax * 1e-3) / 1e9 / hbm_peak,
        "decode_gbs": alg / (dec * 1e-3) / 1e9,
        "decode_frac_of_peak": alg / (dec * 1e-3) / 1e9 / hbm_peak,
        "decode_partial_frac_of_peak": alg / (t["decode"] * 1e-3) / 1e9 / hbm_peak,
        "decode_seqs_per_s": sum_over_ranks(w.batch, world) / (dec * 1e-3),
        "step_seqs_per_s": sum_over_ranks(w.batch, world) / (smax * 1e-3),
        "append_tok_per_s_step": sum_over_ranks(w.batch, world) / (t["append"] * 1e-3),
        "ms": {k: round(v, 5) for k, v in t.items() if k != "launches"},
        "kv_bytes_per_step": kv,
        "alg_bytes_per_step": alg,
    }


def long_context_run(w, fmt, seed, hist, bulk_kv, layout, hbm_peak, flush):
    """The long-context workload as specified: the cached history is filled
    untimed; then ONE timed bulk append of every sequence's bulk tokens (w.batch
    x w.bulk_append tokens in one call, slots in all sequences, prefill-style
    quantize), then w.decode_steps timed decode steps, each appending one token
    per sequence before its decode partials and merge. Both are first run once
    untimed with the same values into the same slots, so each step sees the same
    cache. L2 is flushed before the bulk append; each decode step reads far more
    than L2 holds (no flush between steps)."""
    st = Setup(w, fmt, w.decode_steps, seed, hist=hist, layout=layout, with_bulk=False)
    dev = torch.device("cuda")
    kb, vb = bulk_kv[0].to(dev), bulk_kv[1].to(dev)
    sb = torch.from_numpy(np.concatenate(layout.bulk).astype(np.int64)).to(dev)
    st.cache.append(kb, vb, sb)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush.zero_()
    e0.record()
    st.cache.append(kb, vb, sb)
    e1.record()
    torch.cuda.synchronize()
    bulk_ms = e0.elapsed_time(e1)
    n_bulk = sb.numel()
    del kb, vb
    for s in range(w.decode_steps):                    # untimed pass
        st.step(s)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(w.decode_steps)]
    for s in range(w.decode_steps):
        evs[s][0].record()
        st.step(s, evs[s])
        evs[s][3].record()
    torch.cuda.synchronize()
    t = {"step": float(np.mean([e[0].elapsed_time(e[3]) for e in evs])),
         "append": float(np.mean([e[0].elapsed_time(e[1]) for e in evs])),
         "decode": float(np.mean([e[1].elapsed_time(e[2]) for e in evs])),
         "merge": float(np.mean([e[2].elapsed_time(e[3]) for e in evs]))}
    r = step_metrics(st, t, fmt, 1, hbm_peak, w.decode_steps)
    by = n_bulk * append_bytes_per_token(w, fmt)
    r["bulk_append"] = {"tokens": n_bulk, "sequences": w.batch, "ms": bulk_ms,
                        "tok_per_s": n_bulk / (bulk_ms * 1e-3), "gbs": by / (bulk_ms * 1e6),
                        "frac_of_peak": by / (bulk_ms * 1e6) / hbm_peak}
    r["decode_steps"] = w.decode_steps
    r["context"] = [int(st.ctx_np[0].min()), int(st.ctx_np[-1].max())]
    r["l2"] = "flushed before the bulk append; each step reads > L2"
    del st
    torch.cuda.empty_cache()
    return r


def kivi_rate(w, hist, fmt, seed, hbm_peak, flush, reps=10, warmup=3):
    """Decode over the KIVI-style cache (kvq_kivi_decode_attn) for the workload:
    every sequence's complete 128-token groups quantized by kvq_kivi_append, the
    rest (and one step token) in a BF16 residual cache. Calls run back to back
    (each reads more than L2 holds). Algorithmic bytes per token and KV head: the 2b-bit K and V
    codes, V's (s, z) and K's (s, z) spread over its group."""
    from int8_quantized_paged_quantize_b200 import kvq
    bits = kvq.KIVI_BITS[fmt]
    dev = torch.device("cuda")
    ctx = WL.context_lengths(w, seed) + w.bulk_append
    groups = ctx // 128
    res = ctx % 128 + 1                               # + this step's token
    rng = np.random.default_rng(seed)
    nq = int(groups.sum()) * 8
    perm = rng.permutation(max(nq, 1))
    Wq = max(1, int(groups.max()) * 8)
    qt = np.full((w.batch, Wq), -1, dtype=np.int32)
    nr = int(((res + 15) // 16).sum())
    rperm = rng.permutation(nr)
    Wr = int(((res + 15) // 16).max())
    rt = np.full((w.batch, Wr), -1, dtype=np.int32)
    a = r = 0
    for b in range(w.batch):
        qt[b, :8 * groups[b]] = perm[a:a + 8 * groups[b]]
        a += 8 * groups[b]
        n = (res[b] + 15) // 16
        rt[b, :n] = rperm[r:r + n]
        r += n
    d = kvq.dims(max(nq, 1), w.n_kv_heads, w.n_q_heads, w.head_dim, Wq)
    rd = kvq.dims(nr, w.n_kv_heads, w.n_q_heads, w.head_dim, Wr)
    cache = kvq.KiviCache.allocate(fmt, d, rd)
    K, V = hist
    q0, kn, vn = WL.step_inputs(w, 0, seed)
    at = 0
    for b in range(w.batch):
        m = int(groups[b]) * 128
        pos = np.arange(m)
        if m:
            sl = torch.from_numpy(qt[b][pos // 16].astype(np.int64) * 16 + pos % 16)
            cache.append_groups(K[at:at + m].to(dev), V[at:at + m].to(dev), sl.to(dev))
        rest = int(ctx[b]) - m
        kr = torch.cat([K[at + m:at + m + rest], kn[b:b + 1]])
        vr = torch.cat([V[at + m:at + m + rest], vn[b:b + 1]])
        pos = np.arange(rest + 1)
        sl = torch.from_numpy(rt[b][pos // 16].astype(np.int64) * 16 + pos % 16)
        cache.residual.append(kr.to(dev), vr.to(dev), sl.to(dev))
        at += int(ctx[b])
    torch.cuda.synchronize()
    q = q0.to(dev)
    qtd, rtd = torch.from_numpy(qt).to(dev), torch.from_numpy(rt).to(dev)
    qld = torch.from_numpy((groups * 128).astype(np.int32)).to(dev)
    rld = torch.from_numpy(res.astype(np.int32)).to(dev)
    maxq, maxr = int(groups.max()) * 128, int(res.max())
    ws = cache.workspace(w.batch, maxq, maxr)
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device=dev)

    def call():
        cache.decode(q, qtd, qld, maxq, rtd, rld, maxr, sm_scale=w.sm_scale, out=out, workspace=ws)
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for e0, e1 in evs:
        e0.record()
        call()
        e1.record()
    torch.cuda.synchronize()
    ms = float(np.mean([e0.elapsed_time(e1) for e0, e1 in evs]))
    out32 = cache.decode(q, qtd, qld, maxq, rtd, rld, maxr, sm_scale=w.sm_scale, workspace=ws,
                         out_dtype=torch.float32).cpu()
    per_tok = w.n_kv_heads * (2 * w.head_dim * bits / 8 + 4 + w.head_dim * 4 / 128)
    qbytes = float(groups.sum()) * 128 * per_tok
    rbytes = float(res.sum()) * w.n_kv_heads * 2 * w.head_dim * 2
    kv = qbytes + rbytes
    del cache
    torch.cuda.empty_cache()
    return {"bits": bits, "ms": ms, "kv_gbs": kv / (ms * 1e-3) / 1e9,
            "kv_frac_of_peak": kv / (ms * 1e-3) / 1e9 / hbm_peak,
            "decode_seqs_per_s": w.batch / (ms * 1e-3),
            "tokens_per_s": float(ctx.sum() + w.batch) / (ms * 1e-3),
            "kv_bytes": kv, "bytes_per_token_head": per_tok / w.n_kv_heads,
            "what": "groups on the tensor cores from the packed codes + BF16 residual + merge",
            "out": out32}


def configs_block(args, seed, hbm_peak, flush):
    """Workloads beside the headline, each as its specification runs it."""
    out = {}
    w = WL.WORKLOADS["long-128k"]
    hist = history(w, seed, bulk=False)
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
        parts = list(ex.map(lambda b: WL.kv_bulk(w, b, seed), range(w.batch)))
    bulk_kv = (torch.cat([p[0] for p in parts]), torch.cat([p[1] for p in parts]))
    lay = Layout(w, seed, "fp8")
    long_res = {}
    for f in ("fp8", "int8", "bf16"):
        long_res[f] = long_context_run(w, f, seed, hist, bulk_kv, lay, hbm_peak, flush)
    out["long-128k"] = dict(long_res, workload=config_block(w, "fp8", "")["workload"])
    del hist, bulk_kv
    steps = min(args.steps, 10)
    for name in ("mixed-serving-fp8", "llama3-8b-fp8"):
        w = WL.WORKLOADS[name]
        wb = dataclasses.replace(w, decode_steps=max(w.decode_steps, steps + args.warmup))
        st = Setup(wb, "fp8", steps + args.warmup, seed)
        t = timed_loop(st, steps, args.warmup, 1, flush)
        r = step_metrics(st, t, "fp8", 1, hbm_peak, steps)
        # the same steps as one CUDA graph each, back to back (the headline's timing)
        g_ms = graph_loop(st, steps, args.warmup, 1, flush)
        r["ms_step_graph"] = g_ms
        r["kv_gbs_step_graph"] = r["kv_bytes_per_step"] / (g_ms * 1e-3) / 1e9
        r["tables"] = st.layout.source
        out[name] = {"fp8": r, "workload": config_block(w, "fp8", "")["workload"]}
        del st
        torch.cuda.empty_cache()
    return out


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
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' block")
    ap.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline leg")
    ap.add_argument("--no-multiquery", action="store_true", help="skip the verify / prefill entries")
    ap.add_argument("--bulk-append", choices=["aligned", "continued"], default=None,
                    help="only time one bulk append of 32,768 tokens and print its line")
    ap.add_argument("--reps", type=int, default=5, help="timed calls of --bulk-append")
    ap.add_argument("--kivi-probe", choices=["kivi2", "kivi4"], default=None,
                    help="only time one KIVI-style decode on a mid-size case and print its line")
    ap.add_argument("--prefill-probe", choices=["prefill", "verify"], default=None,
                    help="only time one chunked-prefill (or verification) call on a mid-size case")
    ap.add_argument("--n-query", type=int, default=64, help="chunk length of --prefill-probe")
    args = ap.parse_args()
    if args.bulk_append:
        print(json.dumps(bulk_append_probe(args.fmt or "fp8", args.bulk_append, args.reps)))
        return 0
    if args.kivi_probe:
        print(json.dumps(kivi_probe(args.kivi_probe)))
        return 0
    if args.prefill_probe:
        print(json.dumps(prefill_probe(args.fmt or "fp8", n_query=args.n_query, reps=args.reps,
                                       call=args.prefill_probe)))
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

    hist = history(wb, seed)
    lay = Layout(wb, seed, fmt)
    st = Setup(wb, fmt, steps_needed, seed, hist=hist, layout=lay)
    clocks = ClockSampler(local)
    clocks.start()
    t = timed_loop(st, args.steps, args.warmup, world, flush)        # per-phase events
    tg = graph_loop(st, args.steps, args.warmup, world, flush)        # the step as one graph
    clk = clocks.stop()

    step_ms = max_over_ranks(tg, world)
    head = step_metrics(st, t, fmt, world, hbm_peak, args.steps)
    kv_step = head["kv_bytes_per_step"]
    alg_step = head["alg_bytes_per_step"]
    kv_total = sum_over_ranks(kv_step, world)
    value = kv_total / (step_ms * 1e-3) / 1e9
    dec_ms = max_over_ranks(t["decode"] + t["merge"], world)
    achieved = alg_step / (dec_ms * 1e-3) / 1e9
    seqs_s = sum_over_ranks(wb.batch, world) / (step_ms * 1e-3)
    app_tok_s = sum_over_ranks(wb.batch, world) / (max_over_ranks(t["append"], world) * 1e-3)
    bulk_tok_s, bulk_ms, bulk_n = bulk_append_rate(st)
    verify, prefill = {}, {}
    if not args.no_multiquery:
        try:
            verify = multi_query_rate(st, flush, 4, "verify")
        except Exception as e:                    # reported, never fatal to the main line
            verify = {"error": f"{type(e).__name__}: {e}"[:200]}
        try:
            prefill = multi_query_rate(st, flush, 64, "prefill", reps=3, warmup=1)
        except Exception as e:
            prefill = {"error": f"{type(e).__name__}: {e}"[:200]}

    e2e_ms, h2d, d2h = e2e_loop(st, args.steps, args.warmup, world, flush)
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e_val = kv_total / (e2e_ms * 1e-3) / 1e9

    formats = {}
    outs = {}
    if not args.no_formats:
        # the headline format first: its Setup and timings are the ones above
        order = (fmt,) + tuple(f for f in ("fp8", "int8", "e5m2", "int8c", "int8t", "bf16") if f != fmt)
        for f in order:
            if f == fmt:
                tf, stf = t, st
            else:
                del st
                torch.cuda.empty_cache()
                stf = Setup(wb, f, steps_needed, seed, hist=hist, layout=lay)
                tf = timed_loop(stf, args.steps, args.warmup, world, flush)
            bt, _, _ = bulk_append_rate(stf)
            formats[f] = dict(step_metrics(stf, tf, f, world, hbm_peak, args.steps),
                              append_tok_per_s_bulk=bt)
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
    kivi = {}
    if not args.no_formats:
        for f in ("kivi2", "kivi4"):
            try:
                kivi[f] = kivi_rate(wb, hist, f, seed, hbm_peak, flush)
                o = kivi[f].pop("out")
                if "bf16" in outs:                # the same step-0 tokens as the formats
                    ref = outs["bf16"]
                    kivi[f]["quality_vs_bf16_cache"] = {
                        "max_abs": float((o - ref).abs().max()),
                        "mean_abs": float((o - ref).abs().mean()),
                        "rel_l2": float((o - ref).norm() / max(float(ref.norm()), 1e-30)), "step": 0}
            except Exception as e:                # reported, never fatal to the main line
                kivi[f] = {"error": f"{type(e).__name__}: {e}"[:200]}
    del st, hist
    torch.cuda.empty_cache()

    configs = None
    if world == 1 and not args.no_configs:
        configs = configs_block(args, seed, hbm_peak, flush)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        gbs, tok_s, desc, threads = oracle_decode_sample(wb, fmt, seed=0)
        gbs1, tok1, _, _ = oracle_decode_sample(wb, fmt, seed=0, threads=1)
        cpu = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc,
               "append_tok_per_s": tok_s, "cpu_model": cpu_model(),
               "single_thread": {"value": gbs1, "append_tok_per_s": tok1, "cores": 1}}

    line = {
        "metric": metric_name(fmt), "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DTYPE_TAG[fmt], "data": "synthetic (seeded; no dataset or weights)",
        "config": dict(config_block(wb, fmt, l2="not flushed: every step reads the whole cache "
                                                 "(far more than the 126 MB L2); steps back to back"),
                       launch="each timed step is one CUDA graph replay of its append, decode "
                              "and merge launches; phase_ms and the per-format table time the "
                              "same steps launched one by one with events between the phases",
                       tables=lay.source),
        "decode_seqs_per_s": seqs_s, "append_tok_per_s_step": app_tok_s,
        "append_tok_per_s_bulk": bulk_tok_s, "kv_frac_of_peak_step": value / world / hbm_peak,
        "phase_ms": {k: round(v, 5) for k, v in t.items() if k != "launches"},
        "ms_per_step_eager": t["step"],
        "roofline": {"bound": "hbm", "kernel": "decode attention: partials + merge "
                                               "(kvq_decode_partial + kvq_decode_merge)",
                     "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_kind": peak_kind,
                     "partial_only_frac": head["decode_partial_frac_of_peak"],
                     "alg_bytes_per_launch": alg_step,
                     "traffic": measured_traffic(w.name, fmt)},
        "e2e": {"value": e2e_val, "unit": "GB/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "how": "kvq.LayerCache append + decode per step, inputs copied from pinned host "
                       "memory and the output read back on a copy stream overlapped with the "
                       "neighbouring steps' kernels; timed from the first copy to the last"},
        "gpu_launches": t["launches"],
        "verify": verify,
        "prefill": prefill,
        "clocks": clk,
        "formats": formats,
        "kivi": kivi,
        "configs": configs,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
