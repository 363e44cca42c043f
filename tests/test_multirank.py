"""The multi-GPU path of bench.py on CPU: two gloo ranks check the reductions
that turn per-rank step times into the job's time (max over ranks) and per-rank
bytes into the job's bytes (sum over ranks), and that ranks draw independent
sequences (weak scaling by sequence, no collective on the data path)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from int8_quantized_paged_quantize_b200 import workloads as W
    t = bench.max_over_ranks(1.5 + rank, world, device="cpu")
    s = bench.sum_over_ranks(10.0 * (rank + 1), world, device="cpu")
    bench.barrier(world)
    k, _ = W.kv_history(W.WORKLOADS["tiny-fp8"], 0, seed=rank)
    q.put((rank, t, s, float(k.float().sum())))
    dist.destroy_process_group()


def test_two_rank_reductions_and_independent_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]           # max of 1.5, 2.5
    assert [r[2] for r in res] == [30.0, 30.0]         # 10 + 20
    assert res[0][3] != res[1][3]                       # rank seeds give different data
