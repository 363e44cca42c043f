"""Seeded synthetic workloads for the quantized paged KV-cache decode path.

This module only draws inputs: context lengths, block tables, BF16 Q/K/V.
It holds none of the method's arithmetic (no quantisation, no attention), so
both the CUDA library's tests/bench and the CPU oracle can consume the same
inputs without sharing code.

Every random stream is keyed by (seed, stream name, index) through numpy's
SeedSequence/PCG64, so one sequence's history can be regenerated on its own
(the oracle checks sampled sequences of the large workloads that way).

The five workloads stand in for the shapes the pages talk about (a 70B-class
GQA model at 32k context, an 8B-class model at 1-8k, a mixed-length serving
batch, 128K-class contexts); no dataset or model weights are involved.
"""

from __future__ import annotations

import math
import zlib
from dataclasses import dataclass

import numpy as np
import torch

BLOCK_SIZE = 16


@dataclass(frozen=True)
class Workload:
    name: str
    fmt: str                      # format the workload is specified with: fp8 | int8 | bf16
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    block_size: int = BLOCK_SIZE
    lengths: str = "fixed"        # fixed | uniform | lognormal_mix | list
    ctx: tuple = ()               # fixed: (ctx,), uniform: (lo, hi), list: explicit
    kv_mean: float = 0.0          # mean of K and V (std 1)
    k_outlier_channels: int = 0   # number of fixed K channels scaled by k_outlier_gain
    k_outlier_gain: float = 1.0
    kv_outlier_rate: float = 0.0  # fraction of K/V values scaled by kv_outlier_gain
    kv_outlier_gain: float = 1.0
    pool: str = "shuffled"        # shuffled | permutation16 | fragmented
    bulk_append: int = 0          # tokens appended per sequence in one bulk call before decode
    decode_steps: int = 1

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


WORKLOADS = {
    # 1 layer, 2 sequences (37 and 129 cached tokens), GQA group 2, head_dim 64,
    # block tables drawn from a seeded permutation of a 16-block pool.
    "tiny-fp8": Workload("tiny-fp8", "fp8", batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64,
                         lengths="list", ctx=(37, 129), pool="permutation16"),
    # Llama-3-8B-shaped decode layer: 32 q / 8 kv heads, batch 64, ctx U[1024, 8192],
    # K with 4 fixed outlier channels x20, shuffled block tables.
    "llama3-8b-fp8": Workload("llama3-8b-fp8", "fp8", batch=64, n_q_heads=32, n_kv_heads=8,
                              head_dim=128, lengths="uniform", ctx=(1024, 8192),
                              k_outlier_channels=4, k_outlier_gain=20.0),
    # 70B-shaped decode layer: 64 q / 8 kv heads, batch 32, every sequence at 32768,
    # K/V ~ N(0.3, 1) so the INT8 zero point is exercised.
    "70b-32k-int8": Workload("70b-32k-int8", "int8", batch=32, n_q_heads=64, n_kv_heads=8,
                             head_dim=128, lengths="fixed", ctx=(32768,), kv_mean=0.3),
    # Mixed-length serving batch: 252 lognormal lengths (median 1500, sigma 1,
    # clipped to [16, 32768]) + 4 at 30000, from a fragmented shared pool.
    "mixed-serving-fp8": Workload("mixed-serving-fp8", "fp8", batch=256, n_q_heads=32,
                                  n_kv_heads=8, head_dim=128, lengths="lognormal_mix",
                                  ctx=(1500, 1.0, 16, 32768, 30000, 4), pool="fragmented"),
    # Long context: 4 x 131072 tokens reached by a bulk append of 8192 per sequence
    # onto 122880 cached tokens, then 64 decode steps; rare outliers (0.1% x50).
    "long-128k": Workload("long-128k", "fp8", batch=4, n_q_heads=64, n_kv_heads=8,
                          head_dim=128, lengths="fixed", ctx=(131072 - 8192,),
                          kv_outlier_rate=0.001, kv_outlier_gain=50.0,
                          bulk_append=8192, decode_steps=64),
}


# --------------------------------------------------------------------------- rng
def _rng(seed: int, stream: str, index: int = 0) -> np.random.Generator:
    key = zlib.crc32(stream.encode())
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, key, index])))


def _to_bf16(x: np.ndarray) -> torch.Tensor:
    """float32 draws -> BF16 tensor (the inputs are defined as these BF16 values)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


# --------------------------------------------------------------------------- lengths
def context_lengths(w: Workload, seed: int = 0) -> np.ndarray:
    """Cached tokens per sequence before the bulk append / decode steps (int64 [B])."""
    if w.lengths == "fixed":
        return np.full(w.batch, w.ctx[0], dtype=np.int64)
    if w.lengths == "list":
        return np.asarray(w.ctx, dtype=np.int64)
    rng = _rng(seed, "ctx")
    if w.lengths == "uniform":
        lo, hi = w.ctx
        return rng.integers(lo, hi + 1, size=w.batch).astype(np.int64)
    if w.lengths == "lognormal_mix":
        median, sigma, lo, hi, fixed_len, n_fixed = w.ctx
        n_ln = w.batch - n_fixed
        draw = np.exp(rng.normal(math.log(median), sigma, size=n_ln))
        ln = np.clip(np.rint(draw), lo, hi).astype(np.int64)
        return np.concatenate([ln, np.full(n_fixed, fixed_len, dtype=np.int64)])
    raise ValueError(w.lengths)


def final_lengths(w: Workload, seed: int = 0) -> np.ndarray:
    """Tokens per sequence once the bulk append and every decode step's append are done."""
    return context_lengths(w, seed) + w.bulk_append + w.decode_steps


# --------------------------------------------------------------------------- block tables
def pool_blocks(w: Workload, seed: int = 0) -> int:
    """Blocks in the pool of a workload: exactly what the sequences need for
    their final lengths, except the fragmented shared pool (about 1.25x)."""
    need = int(((final_lengths(w, seed) + w.block_size - 1) // w.block_size).sum())
    if w.pool == "permutation16":
        return 16
    if w.pool == "fragmented":
        return int(math.ceil(1.25 * need))
    return need


def block_tables(w: Workload, seed: int = 0):
    """(block_tables int32 [B][W], num_blocks) covering final_lengths(), for the
    pools laid out directly (not through an allocator).

    Entries past a sequence's last block are -1.
      shuffled:      the pool holds exactly the blocks needed, handed out in a
                     seeded random order;
      permutation16: a 16-block pool, sequences take consecutive runs of one
                     seeded permutation of 0..15.
    The fragmented shared pool is built by the library's block allocator
    instead (paging.paged_batch plays pool_churn() on it).
    """
    bs = w.block_size
    need = (final_lengths(w, seed) + bs - 1) // bs
    W = int(need.max()) if need.size else 0
    tables = np.full((w.batch, max(W, 1)), -1, dtype=np.int32)
    rng = _rng(seed, "blocks")
    num_blocks = pool_blocks(w, seed)
    if w.pool == "permutation16":
        if need.sum() > num_blocks:
            raise ValueError("permutation16 pool too small")
        order = rng.permutation(num_blocks)
    elif w.pool == "shuffled":
        order = rng.permutation(num_blocks)
    elif w.pool == "fragmented":
        raise ValueError("the fragmented pool comes from the block allocator: use paging.paged_batch")
    else:
        raise ValueError(w.pool)
    at = 0
    for b in range(w.batch):
        n = int(need[b])
        tables[b, :n] = order[at:at + n]
        at += n
    return tables, num_blocks


@dataclass(frozen=True)
class ChurnRound:
    take: int                     # blocks allocated in this round
    give_back: tuple              # positions, in the list of held blocks, freed afterwards


def pool_churn(w: Workload, seed: int = 0, rounds: int = 64):
    """Seeded allocate/free schedule that fragments a shared pool before the
    workload's sequences take their blocks (what other requests coming and
    going leave behind). Only counts and positions are drawn here; the block
    ids are whatever the allocator hands out. The first round fills the pool
    but for one block (earlier requests holding it); every later round
    allocates a run of 1 .. pool/16 blocks (never the last free one). After
    each allocation a random half of all blocks held so far is freed, named by
    their positions in the held list (held blocks in allocation order, freed
    ones removed)."""
    num_blocks = pool_blocks(w, seed)
    rng = _rng(seed, "churn")
    free, held = num_blocks, 0
    out = []
    for r in range(rounds):
        take = num_blocks - 1 if r == 0 else int(rng.integers(1, max(2, num_blocks // 16)))
        take = max(0, min(take, free - 1))
        free -= take
        held += take
        idx = rng.permutation(held)[:held // 2] if held else np.zeros(0, dtype=np.int64)
        out.append(ChurnRound(take, tuple(int(i) for i in idx)))
        free += len(idx)
        held -= len(idx)
    return out


# --------------------------------------------------------------------------- values
def _k_outlier_channels(w: Workload, seed: int) -> np.ndarray:
    if w.k_outlier_channels == 0:
        return np.zeros(0, dtype=np.int64)
    return np.sort(_rng(seed, "k_outlier_channels").choice(w.head_dim, w.k_outlier_channels,
                                                           replace=False))


def _kv_draw(w: Workload, seed: int, stream: str, index: int, n_tokens: int, is_k: bool):
    rng = _rng(seed, stream, index)
    x = rng.standard_normal((n_tokens, w.n_kv_heads, w.head_dim), dtype=np.float32)
    if w.kv_mean:
        x += np.float32(w.kv_mean)
    if is_k and w.k_outlier_channels:
        x[..., _k_outlier_channels(w, seed)] *= np.float32(w.k_outlier_gain)
    if w.kv_outlier_rate:
        hit = rng.random(x.shape, dtype=np.float32) < w.kv_outlier_rate
        x[hit] *= np.float32(w.kv_outlier_gain)
    return _to_bf16(x)


def kv_history(w: Workload, b: int, seed: int = 0, ctx: int | None = None):
    """BF16 (K, V) [ctx_b][n_kv_heads][head_dim] cached for sequence b before the run."""
    n = int(context_lengths(w, seed)[b]) if ctx is None else int(ctx)
    return (_kv_draw(w, seed, "k_hist", b, n, True), _kv_draw(w, seed, "v_hist", b, n, False))


def kv_bulk(w: Workload, b: int, seed: int = 0):
    """BF16 (K, V) [bulk_append][n_kv_heads][head_dim] of sequence b's bulk append."""
    n = w.bulk_append
    return (_kv_draw(w, seed, "k_bulk", b, n, True), _kv_draw(w, seed, "v_bulk", b, n, False))


def step_inputs(w: Workload, step: int, seed: int = 0):
    """BF16 inputs of decode step `step`: q [B][Hq][D], k and v [B][Hk][D]
    (one new token per sequence)."""
    rng = _rng(seed, "q", step)
    q = _to_bf16(rng.standard_normal((w.batch, w.n_q_heads, w.head_dim), dtype=np.float32))
    k = torch.cat([_kv_draw(w, seed, "k_step", step * w.batch + b, 1, True)
                   for b in range(w.batch)]) if w.batch else torch.zeros(0)
    v = torch.cat([_kv_draw(w, seed, "v_step", step * w.batch + b, 1, False)
                   for b in range(w.batch)]) if w.batch else torch.zeros(0)
    return q, k, v
