"""Paged KV block pool, quantize-on-append and paged gather — test oracle.

Test infrastructure (see ``oracle/__init__``).

What the pages fix
------------------
* [GUIDE] "Core concepts 2) PagedAttention": the cache is cut into fixed-size
  blocks (pages) held in one pool; each request is mapped only to the blocks it
  needs, which avoids fragmentation and over-allocation.
* [COMPRESS] "6.2 Combining with other techniques": with low-bit K/V a block
  holds more tokens for the same bytes.
* [COMPRESS] "5.1 Quantization pipeline" and "6.3 Implementation
  considerations": a new token's K and V are computed in high precision,
  quantised right after, stored in GPU memory, and dequantised right before
  attention.

Readings taken
--------------
* Logical layout of one cache: ``[num_blocks][n_kv_heads][block_size][head_dim]``
  codes, with scales (and INT8 zero points) ``[num_blocks][n_kv_heads][block_size]``,
  separately for K and for V. The physical device layout is the library's
  business; tests map it to this logical one.
* Token position p of a sequence lives at
  ``slot = block_table[p // block_size] * block_size + p % block_size``.
* A slot below zero means "do not store this token". Slots in one append are
  distinct.
"""

from __future__ import annotations

import numpy as np

from . import formats

FORMATS = ("bf16", "fp8", "int8", "e5m2", "int8c", "int8t")
STATIC_FORMATS = ("int8c", "int8t")


def slot_of(block_table_row, pos, block_size):
    """Flat slot index of token position(s) ``pos`` of one sequence."""
    row = np.asarray(block_table_row, dtype=np.int64)
    p = np.asarray(pos, dtype=np.int64)
    return row[p // block_size] * block_size + p % block_size


class LogicalPool:
    """One layer's K and V caches in the logical layout, for one format.

    bf16: codes hold the BF16 values themselves (as f32).
    fp8:  uint8 E4M3 codes + f32 scales (BF16 values).
    e5m2: uint8 E5M2 codes + f32 scales (BF16 values).
    int8: int8 codes + f32 scales (BF16 values) + int64 zero points.
    int8c / int8t: int8 codes under static scales given here (BF16 values):
    [n_kv_heads][head_dim] per channel or [1] per tensor, for K and for V.
    """

    def __init__(self, fmt, num_blocks, n_kv_heads, block_size, head_dim, k_static=None,
                 v_static=None):
        if fmt not in FORMATS:
            raise ValueError(fmt)
        if fmt in STATIC_FORMATS:
            shape = (n_kv_heads, head_dim) if fmt == "int8c" else (1,)
            self.k_static = np.asarray(k_static, dtype=np.float32).reshape(shape)
            self.v_static = np.asarray(v_static, dtype=np.float32).reshape(shape)
        self.fmt = fmt
        self.num_blocks, self.n_kv_heads = num_blocks, n_kv_heads
        self.block_size, self.head_dim = block_size, head_dim
        shape = (num_blocks, n_kv_heads, block_size, head_dim)
        dtype = {"bf16": np.float32, "fp8": np.uint8, "int8": np.int8, "e5m2": np.uint8,
                 "int8c": np.int8, "int8t": np.int8}[fmt]
        self.k = np.zeros(shape, dtype=dtype)
        self.v = np.zeros(shape, dtype=dtype)
        mshape = shape[:3]
        self.k_scale = np.zeros(mshape, dtype=np.float32)
        self.v_scale = np.zeros(mshape, dtype=np.float32)
        self.k_zp = np.zeros(mshape, dtype=np.int64)
        self.v_zp = np.zeros(mshape, dtype=np.int64)

    # ------------------------------------------------------------------ append
    def append(self, k, v, slot_mapping):
        """Quantise and store new tokens.

        k, v: [T][n_kv_heads][head_dim] BF16 values (given as f32).
        slot_mapping: [T] int; token t goes to slot slot_mapping[t], i.e. block
        slot // block_size, offset slot % block_size; negative slots are skipped.
        Each (token, KV head) row of K and of V gets its own scale (and zero
        point), computed from that row's full BF16 values."""
        k = np.asarray(k, dtype=np.float32)
        v = np.asarray(v, dtype=np.float32)
        slots = np.asarray(slot_mapping, dtype=np.int64)
        keep = slots >= 0
        if not np.any(keep):
            return
        if np.any(slots[keep] >= self.num_blocks * self.block_size):
            raise IndexError("slot beyond the pool")
        blk = slots[keep] // self.block_size
        off = slots[keep] % self.block_size
        for which, src, codes, scale, zp in (("k", k[keep], self.k, self.k_scale, self.k_zp),
                                             ("v", v[keep], self.v, self.v_scale, self.v_zp)):
            # src: [n][Hk][D]; codes[blk, :, off, :] is [n][Hk][D]
            if self.fmt in STATIC_FORMATS:
                st = self.k_static if which == "k" else self.v_static
                codes[blk, :, off, :] = formats.int8_static_quantize(src, st)
            elif self.fmt == "bf16":
                codes[blk, :, off, :] = formats.bf16_round(src)
            elif self.fmt == "fp8":
                c, s = formats.fp8_quantize(src)
                codes[blk, :, off, :] = c
                scale[blk, :, off] = s
            elif self.fmt == "e5m2":
                c, s = formats.e5m2_quantize(src)
                codes[blk, :, off, :] = c
                scale[blk, :, off] = s
            else:
                c, s, z = formats.int8_quantize(src)
                codes[blk, :, off, :] = c
                scale[blk, :, off] = s
                zp[blk, :, off] = z

    # ------------------------------------------------------------------ gather
    def dequantized(self, which, blk, off):
        """float64 [n][Hk][D] values stored at (blk[i], off[i]) of cache 'k' or 'v'."""
        codes = (self.k if which == "k" else self.v)[blk, :, off, :]
        scale = (self.k_scale if which == "k" else self.v_scale)[blk, :, off]
        zp = (self.k_zp if which == "k" else self.v_zp)[blk, :, off]
        if self.fmt == "bf16":
            return codes.astype(np.float64)
        if self.fmt in STATIC_FORMATS:
            return formats.int8_static_dequantize(codes, self.k_static if which == "k" else self.v_static)
        if self.fmt == "fp8":
            return formats.fp8_dequantize(codes, scale)
        if self.fmt == "e5m2":
            return formats.e5m2_dequantize(codes, scale)
        return formats.int8_dequantize(codes, scale, zp)

    def gather(self, block_table_row, ctx):
        """Dequantised K and V of positions 0..ctx-1 of one sequence, each
        float64 [ctx][n_kv_heads][head_dim], read through its block table."""
        pos = np.arange(int(ctx), dtype=np.int64)
        slots = slot_of(block_table_row, pos, self.block_size)
        blk, off = slots // self.block_size, slots % self.block_size
        return self.dequantized("k", blk, off), self.dequantized("v", blk, off)
