"""Block tables and slot mappings of a batch of sequences, taken from the
library's host block allocator (kvq_pool_*).

"From FP8 KV cache to INT4 weight-only", Core concepts 2) (PagedAttention): the
KV cache is a pool of fixed-size blocks shared by all requests, and each
request is mapped to just the blocks it needs. A serving loop grows each
sequence through the allocator: kvq_pool_extend_seq takes the blocks a new run
of tokens needs and returns their slots, which become kvq_append's
slot_mapping; the block-table rows it fills are what kvq_decode_attn reads.
This module is that loop's bookkeeping, on the host and off the timed path.
"""

from __future__ import annotations

import numpy as np

from . import kvq
from . import workloads as W


class PagedBatch:
    """A pool and the block tables of a batch of sequences growing in it."""

    def __init__(self, pool: kvq.Pool, dims: kvq.Dims, batch: int):
        self.pool = pool
        self.dims = dims
        self.tables = np.full((batch, dims.max_blocks_per_seq), -1, dtype=np.int32)
        self.lens = np.zeros(batch, dtype=np.int64)

    def extend(self, b: int, n: int) -> np.ndarray:
        """Grow sequence b by n tokens; returns their slots (int64 [n])."""
        row = self.tables[b].tolist()
        slots = self.pool.extend_seq(row, int(self.lens[b]), int(n))
        self.tables[b] = np.asarray(row, dtype=np.int32)
        self.lens[b] += n
        return np.asarray(slots, dtype=np.int64)

    def extend_all(self, n) -> np.ndarray:
        """Grow every sequence b by n[b] tokens (or n each), in order of b;
        returns the slots of all new tokens, sequence by sequence."""
        n = np.broadcast_to(np.asarray(n, dtype=np.int64), self.lens.shape)
        parts = [self.extend(b, int(n[b])) for b in range(len(self.lens))]
        return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)

    def close(self):
        self.pool.close()


def play_churn(pool: kvq.Pool, schedule) -> None:
    """Run an allocate/free schedule (workloads.pool_churn) on the pool, then
    free what it still holds: the pool's free list is left in the order the
    churn produced."""
    held = []
    for rnd in schedule:
        if rnd.take:
            held.extend(pool.alloc(rnd.take))
        if rnd.give_back:
            back = set(rnd.give_back)
            pool.free([held[i] for i in rnd.give_back])
            held = [x for i, x in enumerate(held) if i not in back]
    if held:
        pool.free(held)


def paged_batch(w: W.Workload, seed: int = 0, fmt: str | None = None) -> PagedBatch:
    """An empty batch of w.batch sequences over a pool of
    workloads.pool_blocks(w) blocks, sized for the workload's final lengths;
    the fragmented shared pool first goes through workloads.pool_churn."""
    need = (W.final_lengths(w, seed) + w.block_size - 1) // w.block_size
    nb = W.pool_blocks(w, seed)
    d = kvq.dims(nb, w.n_kv_heads, w.n_q_heads, w.head_dim, max(1, int(need.max())))
    pool = kvq.Pool(d, fmt or w.fmt)
    if w.pool == "fragmented":
        play_churn(pool, W.pool_churn(w, seed))
    return PagedBatch(pool, d, w.batch)
