"""GPU parity at the workloads' full sizes, in the launch configuration bench.py
times (automatic split-K plan), on sampled sequences the oracle recomputes one
by one from the same seeded inputs: the sampled sequences' cache codes and
scales bit-exact, their attention outputs within 4e-3 max / 5e-4 mean.
"""

import numpy as np
import pytest
import torch

from int8_quantized_paged_quantize_b200 import workloads as W
from tests import gpu_cases as GC

pytestmark = pytest.mark.gpu


def _sampled(w, extra=()):
    B = w.batch
    return sorted(set([0, B // 2, B - 1, *extra]))


def _run_and_check(name, fmt, extra=()):
    w = W.WORKLOADS[name]
    run = GC.run_gpu(w, fmt)
    mx, mean = GC.attention_errors(run, _sampled(w, extra))
    assert mx <= GC.MAX_ABS and mean <= GC.MEAN_ABS, (name, fmt, mx, mean)
    out = run.out.float()
    assert torch.isfinite(out).all()
    return run


def test_llama3_8b_fp8_full():
    _run_and_check("llama3-8b-fp8", "fp8", extra=(7, 41))


def test_llama3_8b_e5m2_full():
    """The same workload on an E5M2 cache (the wider-range FP8 variant)."""
    _run_and_check("llama3-8b-fp8", "e5m2", extra=(7, 41))


def test_70b_32k_int8_full():
    _run_and_check("70b-32k-int8", "int8", extra=(9,))


def test_mixed_serving_fp8_full():
    w = W.WORKLOADS["mixed-serving-fp8"]
    ctx = W.context_lengths(w)
    longest = np.argsort(ctx)[-4:]
    shortest = np.argsort(ctx)[:2]
    _run_and_check("mixed-serving-fp8", "fp8", extra=tuple(int(i) for i in [*longest, *shortest]))


@pytest.mark.parametrize("fmt", ["fp8", "int8", "bf16"])
def test_long_128k_full(fmt):
    _run_and_check("long-128k", fmt)


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_long_128k_bulk_then_64_steps(fmt):
    """The long-context workload as specified: one bulk append of 8,192 tokens
    into each of the 4 sequences (one call), then 64 decode steps of one append
    each. After step 64 every sequence's codes and scales are bit-exact and its
    attention at the last step is within tolerance; sequence 0 is also checked
    at steps 1 and 32 (the contexts grow by one token per step)."""
    w = W.WORKLOADS["long-128k"]
    run = GC.run_gpu_steps(w, fmt, w.decode_steps)
    for b in range(w.batch):
        steps = [0, 31, 63] if b == 0 else [63]
        mx, mean = GC.check_steps_run(run, b, steps)
        assert mx <= GC.MAX_ABS and mean <= GC.MEAN_ABS, (fmt, b, mx, mean)
