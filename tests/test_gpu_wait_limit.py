"""The decode kernels' bounded waits, made to run out on purpose.

Every wait inside the decode kernel gives up after a bounded number of SM clock
cycles (kvq_set_wait_limit). A limit of a few hundred cycles is far shorter than
loading a page from HBM, so the first waits run out: each CTA must stop issuing,
drain the copies and MMAs it issued, write NaN markers for its partials, free
its tensor memory and return, with KVQ_DEVERR_TIMEOUT set. The GPU must still
answer afterwards, and the next call at the default limit must pass parity
against the oracle. No GPU fault is involved: the failure is a wait that runs
out and is reported through the error word.
"""

import numpy as np
import pytest
import torch

from int8_quantized_paged_quantize_b200 import kvq
from int8_quantized_paged_quantize_b200 import workloads as W
from tests import gpu_cases as GC


def test_wait_limit_setting_on_the_host():
    L = kvq.lib()
    default = kvq.wait_limit()
    assert default == 2_000_000_000
    try:
        kvq.set_wait_limit(300)
        assert kvq.wait_limit() == 300
        assert L.kvq_set_wait_limit(-1) == -1              # KVQ_ERR_ARG, nothing changed
        assert kvq.wait_limit() == 300
    finally:
        kvq.set_wait_limit(0)
    assert kvq.wait_limit() == default


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_waits_run_out_cleanly_and_the_next_call_is_correct(fmt):
    w = GC.with_lengths(W.Workload("timeout", fmt, batch=3, n_q_heads=16, n_kv_heads=2,
                                   head_dim=128, kv_mean=0.3 if fmt == "int8" else 0.0),
                        [700, 2100, 90])
    run = GC.run_gpu(w, fmt)                              # normal call: parity below
    assert kvq.device_error(clear=True) == 0
    dev = torch.device("cuda")
    tables = torch.from_numpy(run.tables).to(dev)
    cl = torch.from_numpy(run.ctx_after.astype(np.int32)).to(dev)
    max_ctx = int(run.ctx_after.max())
    q = run.q.to(dev)
    try:
        kvq.set_wait_limit(300)
        timed_out = run.cache.decode(q, tables, cl, max_ctx, sm_scale=w.sm_scale,
                                     partition_tokens=256, out_dtype=torch.float32)
        torch.cuda.synchronize()
    finally:
        kvq.set_wait_limit(0)
    flags = kvq.device_error(clear=True)
    assert flags & kvq.DEVERR_TIMEOUT, hex(flags)
    assert flags & ~kvq.DEVERR_TIMEOUT == 0, hex(flags)
    assert torch.isnan(timed_out).any()                   # marked, not plausible values
    # the context still works: the same decode at the default limit passes parity
    again = run.cache.decode(q, tables, cl, max_ctx, sm_scale=w.sm_scale, partition_tokens=256,
                             out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kvq.device_error(clear=True) == 0
    run.out = again.cpu()
    mx, mean = GC.attention_errors(run, range(w.batch))
    assert mx <= GC.MAX_ABS and mean <= GC.MEAN_ABS, (mx, mean)
