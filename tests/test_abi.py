"""CPU tests of the C ABI: the library loads and exports every function
include/kvq.h declares; host-only calls (sizes, allocator, argument checks)
behave as documented without touching a GPU; the allocator's byte counts
reproduce the pages' worked KV sizes exactly.
"""

import ctypes
import os
import re
from fractions import Fraction

import numpy as np
import pytest

from tests.conftest import ROOT, read_golden


@pytest.fixture(scope="module")
def kvq():
    from int8_quantized_paged_quantize_b200 import build, kvq as K
    build.build()
    return K


def _declared():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(kvq):
    names = _declared()
    assert "kvq_append" in names and "kvq_decode_attn" in names
    L = ctypes.CDLL(kvq.lib_path())
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    bound = {n for n, _, _ in kvq._SIGNATURES}
    assert set(names) == bound, set(names) ^ bound


def test_status_strings(kvq):
    L = kvq.lib()
    for rc in (0, -1, -2, -3, -4, -5, -6):
        assert L.kvq_status_string(rc)
    assert L.kvq_version() >= 100


def test_cache_bytes(kvq):
    d = kvq.dims(100, 8, 64, 128, 10)
    assert kvq.cache_bytes(d, "fp8") == (100 * 8 * 16 * 128, 100 * 8 * 16 * 2)
    assert kvq.cache_bytes(d, "int8") == (100 * 8 * 16 * 128, 100 * 8 * 16 * 4)
    assert kvq.cache_bytes(d, "bf16") == (100 * 8 * 16 * 128 * 2, 0)
    assert kvq.cache_bytes(d, "e5m2") == (100 * 8 * 16 * 128, 100 * 8 * 16 * 2)
    # static INT8: the scales do not grow with the tokens
    assert kvq.cache_bytes(d, "int8c") == (100 * 8 * 16 * 128, 8 * 128 * 2)
    assert kvq.cache_bytes(d, "int8t") == (100 * 8 * 16 * 128, 16)


def test_allocator_reproduces_printed_sizes(kvq):
    """Element bytes of a pool sized for the pages' worked examples equal the
    closed form exactly; 8-bit formats halve them; INT8 metadata > FP8 metadata."""
    for name, L, hk, hd, n, b, bpe, _p, _u, _src in read_golden("kv_size_examples.txt"):
        L, hk, hd, n, b = int(L), int(hk), int(hd), int(n), int(b)
        tokens = n * b
        blocks = max(1, tokens // 16)
        scale = Fraction(tokens, blocks * 16)           # per-token case: one 16-token block
        want = 2 * L * hk * hd * tokens * int(bpe)
        pool = kvq.Pool(kvq.dims(blocks, hk, hk, hd, 1), "bf16", L)
        eb, mb = pool.bytes()
        assert eb * scale == want and mb == 0, name
        e8, m8 = kvq.Pool(kvq.dims(blocks, hk, hk, hd, 1), "fp8", L).bytes()
        ei, mi = kvq.Pool(kvq.dims(blocks, hk, hk, hd, 1), "int8", L).bytes()
        assert 2 * e8 == eb and e8 == ei and mi > m8 > 0, name
    # the pages' 70B / 4096-token figure, literally
    pool = kvq.Pool(kvq.dims(4096 // 16, 8, 64, 128, 256), "bf16", 80)
    assert pool.bytes()[0] == 1_342_177_280


def test_pool_alloc_free_and_exhaustion(kvq):
    p = kvq.Pool(kvq.dims(8, 1, 1, 64, 8), "fp8")
    assert p.num_free() == 8
    a = p.alloc(5)
    assert len(set(a)) == 5 and all(0 <= i < 8 for i in a) and p.num_free() == 3
    with pytest.raises(kvq.KvqError, match="exhausted"):
        p.alloc(4)
    assert p.num_free() == 3                                   # all or nothing
    with pytest.raises(kvq.KvqError):
        p.free([a[0], a[0]])                                   # repeated id
    with pytest.raises(kvq.KvqError):
        p.free([99])                                           # out of range
    p.free(a[:2])
    with pytest.raises(kvq.KvqError):
        p.free([a[0]])                                         # already free
    assert p.num_free() == 5


def test_pool_extend_seq_slots(kvq):
    p = kvq.Pool(kvq.dims(10, 1, 1, 64, 4), "int8")
    row = [-1] * 4
    s1 = p.extend_seq(row, 0, 20)                              # needs 2 blocks
    assert row[2:] == [-1, -1] and p.num_free() == 8
    assert s1 == [row[i // 16] * 16 + i % 16 for i in range(20)]
    s2 = p.extend_seq(row, 20, 13)                             # 33 tokens -> 3 blocks
    assert s2 == [row[i // 16] * 16 + i % 16 for i in range(20, 33)]
    before = list(row)
    with pytest.raises(kvq.KvqError):
        p.extend_seq(row, 33, 40)                              # beyond max_blocks_per_seq
    assert row == before and p.num_free() == 7


def test_host_checks_need_no_gpu(kvq):
    """Argument checks run before any launch: fake but aligned pointers reach the
    workspace check; null / misaligned pointers and bad shapes fail first."""
    L = kvq.lib()
    d = kvq.dims(64, 2, 4, 64, 8)
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    scales = (ctypes.c_void_p * 2)(1 << 21, 1 << 22)
    args = lambda q, ws, n: (q, 1, fake, fake, scales, fake, fake, 100, ctypes.c_float(0.1), fake,
                             0, ws, n, 0, 1, ctypes.byref(d), None)
    assert L.kvq_decode_attn(*args(fake, fake, 0)) == -3          # workspace too small
    assert L.kvq_decode_attn(*args(None, fake, 1 << 30)) == -1    # null q
    assert L.kvq_decode_attn(*args(odd, fake, 1 << 30)) == -1     # misaligned q
    bad = kvq.dims(64, 2, 6, 64, 8)                               # G = 3
    assert L.kvq_append(fake, fake, fake, 4, fake, fake, fake, fake, 1, ctypes.byref(bad), None) == -2
    assert L.kvq_append(fake, fake, fake, 4, fake, fake, None, fake, 1, ctypes.byref(d), None) == -1
    assert L.kvq_append(fake, fake, fake, 0, None, None, None, None, 1, ctypes.byref(d), None) == 0
    # the static INT8 formats need their scale arrays too; an unknown format is refused
    for fmt in (4, 5):
        assert L.kvq_append(fake, fake, fake, 4, fake, fake, fake, None, fmt, ctypes.byref(d), None) == -1
        none = (ctypes.c_void_p * 2)(1 << 21, 0)
        assert L.kvq_decode_attn(fake, 1, fake, fake, none, fake, fake, 100, ctypes.c_float(0.1), fake,
                                 0, fake, 1 << 30, 0, fmt, ctypes.byref(d), None) == -1
    assert L.kvq_append(fake, fake, fake, 4, fake, fake, fake, fake, 6, ctypes.byref(d), None) == -1
    # multi-query decode: n_query in 1..1024; a workspace that is too small is
    # refused before any launch (so these fake pointers never reach a kernel)
    vargs = lambda nq, ws: (fake, 1, nq, fake, fake, scales, fake, fake, 100, ctypes.c_float(0.1),
                            fake, 0, fake, ws, 0, 1, ctypes.byref(d), None)
    assert L.kvq_decode_verify(*vargs(8, 0)) == -3                # G = 2: 16 rows, two groups
    assert L.kvq_decode_verify(*vargs(0, 1 << 30)) == -1
    assert L.kvq_decode_verify(*vargs(1025, 1 << 30)) == -1
    assert L.kvq_decode_verify_workspace_bytes(1, 4, 100, 0, 1, ctypes.byref(d)) == \
        L.kvq_decode_workspace_bytes(1, 100, 0, 1, ctypes.byref(kvq.dims(64, 2, 16, 64, 8)))
    # max_context_len beyond what the block table can hold
    assert kvq.lib().kvq_decode_workspace_bytes(1, 8 * 16 + 1, 0, 1, ctypes.byref(d)) == 0
    # partition must be a multiple of 128
    assert kvq.lib().kvq_decode_workspace_bytes(1, 100, 100, 1, ctypes.byref(d)) == 0


def test_workspace_plan_scales_with_splits(kvq):
    d = kvq.dims(65568, 8, 64, 128, 2049)
    one = kvq.decode_workspace_bytes(32, 32769, "int8", d, partition_tokens=32768 + 128)
    many = kvq.decode_workspace_bytes(32, 32769, "int8", d, partition_tokens=128)
    assert many > one >= 32 * 64 * (128 + 2) * 4


def test_multi_query_workspace_and_limits(kvq):
    """Host checks of kvq_decode_verify / kvq_prefill_attn: any n_query in
    1..1024 has a split plan (more query rows than one group of 8 included),
    the plan grows with the positions, and out-of-range counts are refused
    before any device work."""
    import ctypes as C
    L = kvq.lib()
    d = kvq.dims(4096, 8, 64, 128, 256)            # G = 8
    sizes = [L.kvq_decode_verify_workspace_bytes(4, nq, 4096, 0, 1, C.byref(d))
             for nq in (1, 2, 4, 64, 1024)]
    assert all(x > 0 for x in sizes) and sizes == sorted(sizes)
    assert L.kvq_decode_verify_workspace_bytes(4, 1, 4096, 0, 1, C.byref(d)) == \
        L.kvq_decode_workspace_bytes(4, 4096, 0, 1, C.byref(d))
    assert L.kvq_prefill_attn_workspace_bytes(4, 64, 4096, 0, 1, C.byref(d)) == \
        L.kvq_decode_verify_workspace_bytes(4, 64, 4096, 0, 1, C.byref(d))
    for nq in (0, -1, 1025):
        assert L.kvq_decode_verify_workspace_bytes(4, nq, 4096, 0, 1, C.byref(d)) == 0
    null = C.c_void_p(0)
    scales = (C.c_void_p * 2)(0, 0)
    for fn in (L.kvq_decode_verify, L.kvq_prefill_attn):
        assert fn(null, 1, 1025, null, null, scales, null, null, 64, C.c_float(0.1), null, 0,
                  null, 0, 0, 1, C.byref(d), None) == -1
        # a valid count with null device pointers stops at the pointer checks
        assert fn(null, 1, 64, null, null, scales, null, null, 64, C.c_float(0.1), null, 0,
                  null, 0, 0, 1, C.byref(d), None) == -1
        assert fn(null, 0, 64, null, null, scales, null, null, 64, C.c_float(0.1), null, 0,
                  null, 0, 0, 1, C.byref(d), None) == 0


def test_kivi_host_checks(kvq):
    """kvq_kivi_*: token counts and lengths in whole groups, matching residual
    dims, workspace sizes; refused before any device work."""
    import ctypes as C
    L = kvq.lib()
    d = kvq.dims(1024, 2, 8, 128, 64)
    rd = kvq.dims(64, 2, 8, 128, 8)
    null = C.c_void_p(0)
    assert L.kvq_kivi_append(null, null, null, 100, null, null, null, null, 6, C.byref(d), None) == -1
    assert L.kvq_kivi_append(null, null, null, 0, null, null, null, null, 6, C.byref(d), None) == 0
    assert L.kvq_kivi_append(null, null, null, 128, null, null, null, null, 1, C.byref(d), None) == -1
    assert L.kvq_kivi_append(null, null, null, 128, null, null, null, null, 7, C.byref(d), None) == -1
    ws = L.kvq_kivi_decode_workspace_bytes(4, 1024, 100, 6, C.byref(d), C.byref(rd))
    assert ws == L.kvq_decode_workspace_bytes(4, 1024, 0, 1, C.byref(d)) + \
        L.kvq_decode_workspace_bytes(4, 100, 0, 0, C.byref(rd))
    assert L.kvq_kivi_decode_workspace_bytes(4, 1000, 100, 6, C.byref(d), C.byref(rd)) == 0   # not whole groups
    bad = kvq.dims(64, 2, 16, 128, 8)                                                           # other heads
    assert L.kvq_kivi_decode_workspace_bytes(4, 1024, 100, 6, C.byref(d), C.byref(bad)) == 0
    assert L.kvq_kivi_decode_workspace_bytes(4, 1024, 100, 2, C.byref(d), C.byref(rd)) == 0     # not KIVI
    # sizes: 2-bit codes are a quarter of the 8-bit formats' bytes
    assert kvq.cache_bytes(d, "kivi2")[0] * 4 == kvq.cache_bytes(d, "int8")[0]
    assert kvq.cache_bytes(d, "kivi4")[0] * 2 == kvq.cache_bytes(d, "int8")[0]
