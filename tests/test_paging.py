"""Host checks of the allocator-driven block tables (paging.py over kvq_pool_*):
the fragmented shared pool of the mixed serving batch, grown sequence by
sequence through kvq_pool_extend_seq, gives valid tables whose slots are the
ones the page formula of the block table names, with the pool's accounting
intact. No GPU: the allocator is host code."""

import numpy as np
import pytest

from int8_quantized_paged_quantize_b200 import paging
from int8_quantized_paged_quantize_b200 import workloads as W


@pytest.fixture(scope="module")
def built():
    from int8_quantized_paged_quantize_b200 import build
    build.build()


def _slots_of(tables, b, pos):
    pos = np.asarray(pos, dtype=np.int64)
    return tables[b][pos // 16].astype(np.int64) * 16 + pos % 16


def test_fragmented_pool_tables_from_the_allocator(built):
    w = W.WORKLOADS["mixed-serving-fp8"]
    ctx = W.context_lengths(w)
    pb = paging.paged_batch(w)
    nb = pb.dims.num_blocks
    assert nb == W.pool_blocks(w) and pb.pool.num_free() == nb      # churn returned everything
    hist = [pb.extend(b, int(ctx[b])) for b in range(w.batch)]
    steps = [pb.extend_all(1) for _ in range(w.decode_steps)]
    fin = W.final_lengths(w)
    need = (fin + 15) // 16
    used = []
    for b in range(w.batch):
        row = pb.tables[b]
        assert np.all(row[:need[b]] >= 0) and np.all(row[:need[b]] < nb)
        assert np.all(row[need[b]:] == -1)
        used.extend(row[:need[b]].tolist())
        # the slots the allocator returned are the block-table slots of those positions
        assert np.array_equal(hist[b], _slots_of(pb.tables, b, np.arange(ctx[b])))
        for s, st in enumerate(steps):
            assert st[b] == _slots_of(pb.tables, b, [ctx[b] + s])[0]
    assert len(used) == len(set(used))
    assert pb.pool.num_free() == nb - len(used)
    # fragmented: a sequence's blocks are not one ascending run
    gaps = [np.any(np.diff(pb.tables[b][:need[b]]) != 1) for b in range(w.batch) if need[b] > 4]
    assert np.mean(gaps) > 0.9
    pb.close()


def test_same_seed_same_tables(built):
    w = W.WORKLOADS["mixed-serving-fp8"]
    ctx = W.context_lengths(w)
    a, b = paging.paged_batch(w), paging.paged_batch(w)
    a.extend_all(ctx)
    b.extend_all(ctx)
    assert np.array_equal(a.tables, b.tables)
    a.close()
    b.close()
