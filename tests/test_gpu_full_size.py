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
