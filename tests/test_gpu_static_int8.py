"""GPU parity of the static-scale INT8 cache formats against the CPU oracle.

Per-channel (one BF16 scale per KV head and channel) and per-tensor (one per
cache) symmetric INT8, as "KV cache quantization: what FP8/INT8 K and V really
give" ("Formats you will actually meet") lists them beside per-token INT8. The
scales are inputs fixed before the tokens arrive (here by the oracle's
calibration over the run's tokens, or given outright). Codes must be
bit-exact; attention within max |err| 4e-3 and mean |err| 5e-4 of the oracle's
FP64 attention over the same dequantised K/V.
"""

import numpy as np
import pytest
import torch

from int8_quantized_paged_quantize_b200 import kvq
from int8_quantized_paged_quantize_b200 import workloads as W
from oracle import formats as OF
from tests import gpu_cases as GC

pytestmark = pytest.mark.gpu

STATIC = ["int8c", "int8t"]
RAGGED = [1, 15, 16, 17, 127, 128, 129, 300, 555]


def _synthetic(fmt, D, G, Hk=2, ctx=RAGGED, kv_mean=0.0):
    return W.Workload("synthetic", fmt, batch=len(ctx), n_q_heads=Hk * G, n_kv_heads=Hk,
                      head_dim=D, lengths="list", ctx=tuple(ctx), kv_mean=kv_mean)


def _check(run):
    mx, mean = GC.attention_errors(run, range(run.w.batch))
    assert mx <= GC.MAX_ABS and mean <= GC.MEAN_ABS, (mx, mean)
    return mx, mean


@pytest.mark.parametrize("fmt", STATIC)
def test_tiny_workload(fmt):
    _check(GC.run_gpu(W.WORKLOADS["tiny-fp8"], fmt))


@pytest.mark.parametrize("fmt", STATIC)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_ragged_shapes(fmt, D, G):
    _check(GC.run_gpu(_synthetic(fmt, D, G, kv_mean=0.3), fmt))


@pytest.mark.parametrize("fmt", STATIC)
def test_split_k_on_and_off_agree(fmt):
    w = _synthetic(fmt, 128, 8, ctx=[3000, 1, 700, 4097])
    a = GC.run_gpu(w, fmt, partition_tokens=128)
    b = GC.run_gpu(w, fmt, partition_tokens=8192)
    _check(a)
    _check(b)
    assert (a.out - b.out).abs().max().item() < 1e-3


@pytest.mark.parametrize("part", [0, 128])
def test_many_short_sequences(part):
    rng = np.random.default_rng(7)
    ctx = [int(c) for c in rng.integers(0, 300, size=120)] + [0, 126, 127, 128, 255, 3000, 5000]
    _check(GC.run_gpu(_synthetic("int8c", 128, 4, ctx=ctx, kv_mean=0.3), "int8c", partition_tokens=part))


def test_outlier_channels_and_saturation():
    """K with four channels x20; scales calibrated on a quarter of the values'
    range, so many codes saturate at +-127; one channel's scale is 0 (code 0);
    one channel's scale is subnormal in BF16 (the IEEE division path)."""
    from dataclasses import replace
    w = replace(_synthetic("int8c", 128, 4, ctx=[200, 900]), k_outlier_channels=4, k_outlier_gain=20.0)
    kst, vst = GC.static_scales(w, "int8c")
    kst = kst.copy() / 4
    vst = vst.copy() / 4
    kst = OF.bf16_round(kst)
    vst = OF.bf16_round(vst)
    kst[0, 5] = 0.0
    vst[1, 7] = 0.0
    kst[1, 9] = np.float32(2.0 ** -130)                       # BF16 subnormal
    run = GC.run_gpu(w, "int8c", static=(kst, vst))
    mx, mean = GC.attention_errors(run, range(w.batch))
    assert mx <= GC.MAX_ABS and mean <= GC.MEAN_ABS, (mx, mean)
    codes = run.cache.k_logical().cpu().numpy().view(np.int8)
    assert (np.abs(codes) == 127).sum() > 1000


def test_per_tensor_equals_per_channel_with_equal_scales():
    w = _synthetic("int8t", 128, 4, ctx=[333, 1200])
    kt, vt = GC.static_scales(w, "int8t")
    a = GC.run_gpu(w, "int8t", static=(kt, vt))
    kc = np.full((w.n_kv_heads, w.head_dim), kt[0], dtype=np.float32)
    vc = np.full((w.n_kv_heads, w.head_dim), vt[0], dtype=np.float32)
    b = GC.run_gpu(w, "int8c", static=(kc, vc))
    assert torch.equal(a.cache.k, b.cache.k) and torch.equal(a.cache.v, b.cache.v)
    assert torch.equal(a.out, b.out)
    _check(a)


@pytest.mark.parametrize("fmt", STATIC)
def test_segmented_windows_write_the_same_bytes(fmt):
    D = 128
    d = kvq.dims(24, 2, 4, D, 24)
    g = torch.Generator().manual_seed(5)
    runs = [(16 + 5, 40), (16 * 6 + 15, 1), (16 * 8 + 3, 9), (16 * 10, 16), (16 * 12 + 7, 30)]
    slots = torch.cat([torch.arange(s, s + n, dtype=torch.int64) for s, n in runs])
    n = slots.numel()
    k = (torch.randn(n, 2, D, generator=g) * 2 + 0.3).to(torch.bfloat16)
    v = torch.randn(n, 2, D, generator=g).to(torch.bfloat16)
    per_channel = fmt == "int8c"
    kst = torch.from_numpy(OF.int8_static_calibrate(k.float().numpy(), per_channel)).to(torch.bfloat16).cuda()
    vst = torch.from_numpy(OF.int8_static_calibrate(v.float().numpy(), per_channel)).to(torch.bfloat16).cuda()
    a = kvq.LayerCache.allocate(fmt, d, k_static=kst, v_static=vst)
    a.append(k.cuda(), v.cuda(), slots.cuda())
    perm = torch.randperm(n, generator=g)
    b = kvq.LayerCache.allocate(fmt, d, k_static=kst, v_static=vst)
    b.append(k[perm].contiguous().cuda(), v[perm].contiguous().cuda(), slots[perm].contiguous().cuda())
    torch.cuda.synchronize()
    assert torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    # and the codes are the oracle's
    want = OF.int8_static_quantize(k.float().numpy(), kst.float().cpu().numpy())
    got = a.k_logical().cpu().numpy().view(np.int8)
    s = slots.numpy()
    assert np.array_equal(got[s // 16, :, s % 16, :], want)
    assert kvq.device_error() == 0
