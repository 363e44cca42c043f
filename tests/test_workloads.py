"""Host-side checks of the seeded synthetic workloads (shapes, determinism, block tables)."""

import numpy as np
import pytest

from int8_quantized_paged_quantize_b200 import workloads as W


@pytest.mark.parametrize("name", [n for n, w in W.WORKLOADS.items() if w.pool != "fragmented"])
def test_block_tables_are_valid(name):
    w = W.WORKLOADS[name]
    tables, nb = W.block_tables(w, seed=0)
    fin = W.final_lengths(w, seed=0)
    need = (fin + w.block_size - 1) // w.block_size
    used = []
    for b in range(w.batch):
        row = tables[b]
        assert np.all(row[:need[b]] >= 0) and np.all(row[:need[b]] < nb)
        assert np.all(row[need[b]:] == -1)
        used.extend(row[:need[b]].tolist())
    assert len(used) == len(set(used))          # no block shared by two positions
    assert nb >= len(used)


def test_determinism_and_independent_streams():
    w = W.WORKLOADS["tiny-fp8"]
    k1, v1 = W.kv_history(w, 1, seed=0)
    k2, v2 = W.kv_history(w, 1, seed=0)
    assert k1.equal(k2) and v1.equal(v2)
    assert not k1[:10].equal(W.kv_history(w, 0, seed=0)[0][:10])
    assert tuple(k1.shape) == (129, 2, 64)
    q, k, v = W.step_inputs(w, 0)
    assert tuple(q.shape) == (2, 4, 64) and tuple(k.shape) == (2, 2, 64)


def test_tiny_uses_16_block_permutation():
    w = W.WORKLOADS["tiny-fp8"]
    tables, nb = W.block_tables(w)
    assert nb == 16
    assert (tables[0] >= 0).sum() == 3 and (tables[1] >= 0).sum() == 9   # 38 and 130 tokens


def test_length_distributions():
    w = W.WORKLOADS["llama3-8b-fp8"]
    c = W.context_lengths(w)
    assert c.min() >= 1024 and c.max() <= 8192 and len(c) == 64
    w = W.WORKLOADS["mixed-serving-fp8"]
    c = W.context_lengths(w)
    assert len(c) == 256 and np.sum(c == 30000) >= 4
    assert c.min() >= 16 and c.max() <= 32768
    assert 800 < np.median(c) < 2500
    need = ((W.final_lengths(w) + 15) // 16).sum()
    assert W.pool_blocks(w) == int(np.ceil(1.25 * need))
    with pytest.raises(ValueError):
        W.block_tables(w)                      # comes from the allocator instead


def test_outlier_structure():
    w = W.WORKLOADS["llama3-8b-fp8"]
    k, v = W.kv_history(w, 0, ctx=2000)
    ch = W._k_outlier_channels(w, 0)
    assert len(ch) == 4
    std = k.float().std(dim=(0, 1)).numpy()
    assert np.all(std[ch] > 10) and np.median(std) < 1.5
    assert v.float().std() < 1.5
    w = W.WORKLOADS["long-128k"]
    k, _ = W.kv_history(w, 0, ctx=4000)
    frac = (k.float().abs() > 8).float().mean().item()
    assert 0.0003 < frac < 0.003


def test_pool_churn_schedule_is_feasible_and_seeded():
    w = W.WORKLOADS["mixed-serving-fp8"]
    sched = W.pool_churn(w, seed=0)
    assert sched == W.pool_churn(w, seed=0) and sched != W.pool_churn(w, seed=1)
    nb, held = W.pool_blocks(w), 0
    for rnd in sched:
        assert 0 <= rnd.take and held + rnd.take < nb          # never the last free block
        held += rnd.take
        assert len(set(rnd.give_back)) == len(rnd.give_back) == held // 2
        assert all(0 <= i < held for i in rnd.give_back)
        held -= len(rnd.give_back)
