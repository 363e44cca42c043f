"""Host model of the decode kernel's work split, checked on random batches.

The persistent decode kernel (csrc/kvq_decode_mma.cuh) shares the work list of
every (sequence b, KV head h, 128-token tile) among N CTAs by cost: each
(b, h) run costs its tiles plus one unit in front of them (opening and closing
a piece). CTA c takes the cost range [c*T/N, (c+1)*T/N); its pieces are the
runs it meets, and a piece writes its online-softmax partial to workspace slot
c - cta_of(first tile of the run), where cta_of(x) = ((x+1)*N - 1) // T is the
CTA holding cost position x. The piece holding a run's last tile writes the
run's partial count. The merge reads slots 0 .. count-1.

This file restates that arithmetic on the host and checks, for thousands of
random batches (empty, one-token, over-long and ordinary contexts, several
head counts and partitions), the invariants the kernel relies on:
  * every tile of every (b, h) is taken by exactly one piece;
  * slots are in [0, ceil(max_ctx / partition) + 1), the workspace's size;
  * the slots of one (b, h) are exactly 0 .. count-1, each written once.
It also checks the automatic partition (the smallest 128-token multiple that
cuts the longest sequence into at most 15 runs) through the library's
workspace size, which is host-only.
"""

import ctypes
import math
import random

import pytest

PIECE_COST = 1          # virtual cost units in front of every (b, h) run
TILE = 128


def _legal(c, max_ctx, W):
    return 0 if (c < 0 or c > max_ctx or c > W * 16) else c


def _split(ctxs, Hk, max_ctx, partition, grid):
    """Pieces (c, b, h, lo, hi, slot) of the cost-weighted split, in CTA order."""
    B = len(ctxs)
    W = (max_ctx + 15) // 16
    tiles = [(_legal(c, max_ctx, W) + TILE - 1) // TILE for c in ctxs]
    cost = [t + PIECE_COST if t else 0 for t in tiles]
    T = Hk * sum(cost)
    if T == 0:
        return [], tiles
    N = min(grid, max(1, T // max(1, partition // TILE)))
    run_start = []                 # cost position of (b, h)'s run: Hk * (cost of b' < b) + h * cost[b]
    acc = 0
    for b in range(B):
        run_start.append([Hk * acc + h * cost[b] for h in range(Hk)])
        acc += cost[b]

    def cta_of(x):
        return ((x + 1) * N - 1) // T

    pieces = []
    for c in range(N):
        start, end = c * T // N, (c + 1) * T // N
        for b in range(B):
            if not cost[b]:
                continue
            for h in range(Hk):
                r0 = run_start[b][h]
                r1 = r0 + cost[b]
                a, z = max(start, r0), min(end, r1)
                if a >= z:
                    continue
                lo = max(0, a - r0 - PIECE_COST)
                hi = max(0, z - r0 - PIECE_COST)
                if hi <= lo:
                    continue                   # the share holds only the run's virtual unit
                slot = c - cta_of(r0 + PIECE_COST)
                pieces.append((c, b, h, lo, hi, slot))
    return pieces, tiles


def _check(ctxs, Hk, max_ctx, partition, grid):
    pieces, tiles = _split(ctxs, Hk, max_ctx, partition, grid)
    slots = max(1, math.ceil(max_ctx / partition)) + 1
    taken = {}
    by_run = {}
    count = {}
    for c, b, h, lo, hi, slot in pieces:
        assert 0 <= slot < slots, (slot, slots)
        for t in range(lo, hi):
            assert (b, h, t) not in taken
            taken[(b, h, t)] = c
        by_run.setdefault((b, h), []).append(slot)
        if hi == tiles[b]:
            count[(b, h)] = slot + 1
    for b, nt in enumerate(tiles):
        for h in range(Hk):
            assert all((b, h, t) in taken for t in range(nt))
            if nt:
                assert sorted(by_run[(b, h)]) == list(range(count[(b, h)]))
    assert len(taken) == Hk * sum(tiles)


def test_random_batches():
    rng = random.Random(2)
    for _ in range(1500):
        B = rng.choice([1, 2, 3, 7, 16, 64, 200])
        Hk = rng.choice([1, 2, 8])
        max_ctx = rng.choice([1, 16, 129, 1000, 4096, 33000])
        ctxs = [rng.choice([0, 1, rng.randint(0, max_ctx), max_ctx,
                            max_ctx + 5 if rng.random() < 0.05 else max_ctx]) for _ in range(B)]
        tiles = max(1, (max_ctx + TILE - 1) // TILE)
        partition = rng.choice([128, 256, 1024, 4096, TILE * ((tiles + 14) // 15)])
        grid = rng.choice([1, 5, 148, 296])
        _check(ctxs, Hk, max_ctx, partition, grid)


def test_long_contexts_keep_every_resident_cta_busy():
    # four sequences of 128k tokens with the automatic partition (69 tiles):
    # every one of the 296 resident CTAs takes at least one piece
    part = TILE * ((1024 + 14) // 15)
    pieces, _ = _split([131072] * 4, 8, 131072, part, 296)
    assert {p[0] for p in pieces} == set(range(296))
    _check([131072] * 4, 8, 131072, part, 296)
    # one such sequence: a share holds at least a partition's tiles, so fewer
    # CTAs work (8 heads x 1025 units / 69 = 118)
    pieces, _ = _split([131072], 8, 131072, part, 296)
    assert len({p[0] for p in pieces}) == 8 * 1025 // 69


@pytest.mark.parametrize("max_ctx", [1, 128, 129, 1920, 1921, 8192, 32769, 131072])
def test_automatic_partition_through_the_library(max_ctx):
    """The workspace of the automatic plan equals the one of an explicit
    partition of 128 * ceil(tiles / 15) tokens."""
    from int8_quantized_paged_quantize_b200 import kvq
    W = (max_ctx + 15) // 16
    d = kvq.dims(W, 8, 32, 128, W)
    L = kvq.lib()
    tiles = max(1, (max_ctx + TILE - 1) // TILE)
    part = TILE * ((tiles + 14) // 15)
    auto = L.kvq_decode_workspace_bytes(4, max_ctx, 0, 1, ctypes.byref(d))
    explicit = L.kvq_decode_workspace_bytes(4, max_ctx, part, 1, ctypes.byref(d))
    assert auto == explicit > 0
    splits = max(1, math.ceil(max_ctx / part))
    assert splits <= 15
