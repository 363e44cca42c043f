"""Thin ctypes binding of libkvq (include/kvq.h).

Argument marshalling only: PyTorch tensors supply device pointers, the current
CUDA stream supplies the stream; every computation runs in the library's CUDA
kernels. If ``libkvq.so`` is missing or a call fails, a ``KvqError`` is raised;
there is no CPU path.
"""

from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkvq.so")

# int8c / int8t: symmetric INT8 with static BF16 scales given by the caller,
# one per (KV head, channel) or one per cache (K and V separately)
FMT = {"bf16": 0, "fp8": 1, "int8": 2, "e5m2": 3, "int8c": 4, "int8t": 5, "kivi2": 6, "kivi4": 7}
KIVI_BITS = {"kivi2": 2, "kivi4": 4}
KIVI_GROUP = 128
ELEM_BYTES = {"bf16": 2, "fp8": 1, "int8": 1, "e5m2": 1, "int8c": 1, "int8t": 1}
META_VALUES = {"bf16": 0, "fp8": 1, "int8": 2, "e5m2": 1, "int8c": 0, "int8t": 0}   # per token
STATIC_FORMATS = ("int8c", "int8t")
BLOCK_SIZE = 16

DEVERR_SLOT, DEVERR_BLOCK, DEVERR_CONTEXT, DEVERR_TIMEOUT = 0x1, 0x2, 0x4, 0x8

# Every function the header declares: (name, restype, argtypes)
_c = ctypes
_P = _c.c_void_p
_SIGNATURES = [
    ("kvq_version", _c.c_int, []),
    ("kvq_status_string", _c.c_char_p, [_c.c_int]),
    ("kvq_cache_bytes", _c.c_int, [_P, _c.c_int, _c.POINTER(_c.c_size_t), _c.POINTER(_c.c_size_t)]),
    ("kvq_pool_create", _c.c_int, [_P, _c.c_int, _c.c_int32, _c.POINTER(_P)]),
    ("kvq_pool_destroy", None, [_P]),
    ("kvq_pool_bytes", _c.c_int, [_P, _c.POINTER(_c.c_size_t), _c.POINTER(_c.c_size_t)]),
    ("kvq_pool_num_free", _c.c_int, [_P, _c.POINTER(_c.c_int32)]),
    ("kvq_pool_alloc", _c.c_int, [_P, _c.c_int32, _P]),
    ("kvq_pool_free", _c.c_int, [_P, _c.c_int32, _P]),
    ("kvq_pool_extend_seq", _c.c_int, [_P, _P, _c.c_int32, _c.c_int32, _P]),
    ("kvq_append", _c.c_int, [_P, _P, _P, _c.c_int32, _P, _P, _P, _P, _c.c_int, _P, _P]),
    ("kvq_decode_workspace_bytes", _c.c_size_t, [_c.c_int32, _c.c_int32, _c.c_int32, _c.c_int, _P]),
    ("kvq_decode_attn", _c.c_int, [_P, _c.c_int32, _P, _P, _P, _P, _P, _c.c_int32, _c.c_float, _P,
                                   _c.c_int, _P, _c.c_size_t, _c.c_int32, _c.c_int, _P, _P]),
    ("kvq_decode_partial", _c.c_int, [_P, _c.c_int32, _P, _P, _P, _P, _P, _c.c_int32, _c.c_float,
                                      _P, _c.c_size_t, _c.c_int32, _c.c_int, _P, _P]),
    ("kvq_decode_merge", _c.c_int, [_c.c_int32, _P, _c.c_int32, _P, _c.c_int, _P, _c.c_size_t,
                                    _c.c_int32, _c.c_int, _P, _P]),
    ("kvq_device_error", _c.c_int, [_c.POINTER(_c.c_uint32), _c.c_int]),
    ("kvq_set_wait_limit", _c.c_int, [_c.c_int64]),
    ("kvq_get_wait_limit", _c.c_int64, []),
    ("kvq_decode_attn_noalloc", _c.c_int, [_P, _c.c_int32, _P, _P, _P, _P, _P, _c.c_int32,
                                           _c.c_float, _P, _c.c_int, _c.c_int32, _c.c_int, _P,
                                           _P]),
    ("kvq_decode_verify_workspace_bytes", _c.c_size_t, [_c.c_int32, _c.c_int32, _c.c_int32,
                                                        _c.c_int32, _c.c_int, _P]),
    ("kvq_decode_verify", _c.c_int, [_P, _c.c_int32, _c.c_int32, _P, _P, _P, _P, _P, _c.c_int32,
                                     _c.c_float, _P, _c.c_int, _P, _c.c_size_t, _c.c_int32, _c.c_int,
                                     _P, _P]),
    ("kvq_kivi_append", _c.c_int, [_P, _P, _P, _c.c_int32, _P, _P, _P, _P, _c.c_int, _P, _P]),
    ("kvq_kivi_decode_workspace_bytes", _c.c_size_t, [_c.c_int32, _c.c_int32, _c.c_int32, _c.c_int,
                                                      _P, _P]),
    ("kvq_kivi_decode_attn", _c.c_int, [_P, _c.c_int32, _P, _P, _P, _P, _P, _c.c_int32, _P, _P, _P,
                                        _P, _c.c_int32, _c.c_float, _P, _c.c_int, _P, _c.c_size_t,
                                        _c.c_int, _P, _P, _P]),
    ("kvq_prefill_attn_workspace_bytes", _c.c_size_t, [_c.c_int32, _c.c_int32, _c.c_int32,
                                                       _c.c_int32, _c.c_int, _P]),
    ("kvq_prefill_attn", _c.c_int, [_P, _c.c_int32, _c.c_int32, _P, _P, _P, _P, _P, _c.c_int32,
                                    _c.c_float, _P, _c.c_int, _P, _c.c_size_t, _c.c_int32, _c.c_int,
                                    _P, _P]),
]

NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024

_lib = None


class KvqError(RuntimeError):
    pass


def lib():
    """The loaded libkvq (raises KvqError if the library has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise KvqError(f"libkvq.so not built (expected at {_LIB_PATH}); "
                           "run python -m int8_quantized_paged_quantize_b200.build")
        L = ctypes.CDLL(_LIB_PATH)
        for name, res, args in _SIGNATURES:
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def lib_path() -> str:
    return _LIB_PATH


def _check(rc: int, what: str):
    if rc != 0:
        msg = lib().kvq_status_string(rc).decode()
        raise KvqError(f"{what}: {msg} (status {rc})")


class Dims(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("max_blocks_per_seq", ctypes.c_int32)]


def dims(num_blocks, n_kv_heads, n_q_heads, head_dim, max_blocks_per_seq, block_size=BLOCK_SIZE):
    return Dims(num_blocks, block_size, n_kv_heads, n_q_heads, head_dim, max_blocks_per_seq)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _out_dtype(out):
    if out.dtype == torch.bfloat16:
        return 0
    if out.dtype == torch.float32:
        return 1
    raise KvqError("out must be bfloat16 or float32")


def _need(t, dtype, name):
    if not t.is_cuda or not t.is_contiguous() or t.dtype != dtype:
        raise KvqError(f"{name} must be a contiguous CUDA {dtype} tensor")


def _need_out(out):
    """Decode outputs: a contiguous CUDA bfloat16 or float32 tensor."""
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise KvqError("out must be bfloat16 or float32")
    _need(out, out.dtype, "out")


# --------------------------------------------------------------------------- sizes / allocator
def cache_bytes(d: Dims, fmt: str):
    cb, mb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().kvq_cache_bytes(ctypes.byref(d), FMT[fmt], ctypes.byref(cb), ctypes.byref(mb)),
           "kvq_cache_bytes")
    return cb.value, mb.value


class Pool:
    """Host block allocator (kvq_pool_*)."""

    def __init__(self, d: Dims, fmt: str, n_layers: int = 1):
        self._d = d
        h = ctypes.c_void_p()
        _check(lib().kvq_pool_create(ctypes.byref(d), FMT[fmt], n_layers, ctypes.byref(h)),
               "kvq_pool_create")
        self._h = h

    def close(self):
        if self._h:
            lib().kvq_pool_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def bytes(self):
        eb, mb = ctypes.c_size_t(), ctypes.c_size_t()
        _check(lib().kvq_pool_bytes(self._h, ctypes.byref(eb), ctypes.byref(mb)), "kvq_pool_bytes")
        return eb.value, mb.value

    def num_free(self):
        n = ctypes.c_int32()
        _check(lib().kvq_pool_num_free(self._h, ctypes.byref(n)), "kvq_pool_num_free")
        return n.value

    def alloc(self, n):
        ids = (ctypes.c_int32 * max(n, 1))()
        _check(lib().kvq_pool_alloc(self._h, n, ids), "kvq_pool_alloc")
        return list(ids[:n])

    def free(self, ids):
        arr = (ctypes.c_int32 * max(len(ids), 1))(*ids)
        _check(lib().kvq_pool_free(self._h, len(ids), arr), "kvq_pool_free")

    def extend_seq(self, row, cur_len, n_new):
        """row: a mutable list of max_blocks_per_seq ints (updated in place); returns slots."""
        arr = (ctypes.c_int32 * len(row))(*row)
        slots = (ctypes.c_int64 * max(n_new, 1))()
        _check(lib().kvq_pool_extend_seq(self._h, arr, cur_len, n_new, slots), "kvq_pool_extend_seq")
        row[:] = list(arr)
        return list(slots[:n_new])


# --------------------------------------------------------------------------- hot calls
def append(k, v, slot_mapping, k_cache, v_cache, k_scale, v_scale, fmt: str, d: Dims, stream=None):
    """Quantize-on-append (kvq_append). k, v: [T][Hk][D] bf16; slot_mapping [T] int64."""
    _need(k, torch.bfloat16, "k")
    _need(v, torch.bfloat16, "v")
    _need(slot_mapping, torch.int64, "slot_mapping")
    T = slot_mapping.numel()
    _check(lib().kvq_append(_ptr(k), _ptr(v), _ptr(slot_mapping), T, _ptr(k_cache), _ptr(v_cache),
                            _ptr(k_scale), _ptr(v_scale), FMT[fmt], ctypes.byref(d),
                            _stream(stream)), "kvq_append")


def decode_workspace_bytes(batch, max_context_len, fmt, d: Dims, partition_tokens=0):
    n = lib().kvq_decode_workspace_bytes(batch, max_context_len, partition_tokens, FMT[fmt],
                                         ctypes.byref(d))
    if n == 0 and batch > 0:
        raise KvqError("kvq_decode_workspace_bytes: invalid arguments")
    return n


def _scales(k_scale, v_scale):
    arr = (ctypes.c_void_p * 2)(k_scale.data_ptr() if k_scale is not None else 0,
                                v_scale.data_ptr() if v_scale is not None else 0)
    return arr


def decode_attn(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                max_context_len, sm_scale, out, workspace, fmt: str, d: Dims,
                partition_tokens=0, stream=None):
    """Paged GQA decode attention (kvq_decode_attn): partials + merge into out."""
    _need(q, torch.bfloat16, "q")
    _need_out(out)
    _need(block_tables, torch.int32, "block_tables")
    _need(context_lens, torch.int32, "context_lens")
    B = q.shape[0]
    _check(lib().kvq_decode_attn(_ptr(q), B, _ptr(k_cache), _ptr(v_cache), _scales(k_scale, v_scale),
                                 _ptr(block_tables), _ptr(context_lens), int(max_context_len),
                                 float(sm_scale), _ptr(out), _out_dtype(out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), partition_tokens,
                                 FMT[fmt], ctypes.byref(d), _stream(stream)), "kvq_decode_attn")


def decode_partial(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                   max_context_len, sm_scale, workspace, fmt: str, d: Dims, partition_tokens=0,
                   stream=None):
    B = q.shape[0]
    _check(lib().kvq_decode_partial(_ptr(q), B, _ptr(k_cache), _ptr(v_cache),
                                    _scales(k_scale, v_scale), _ptr(block_tables),
                                    _ptr(context_lens), int(max_context_len), float(sm_scale),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    partition_tokens, FMT[fmt], ctypes.byref(d), _stream(stream)),
           "kvq_decode_partial")


def decode_merge(batch, context_lens, max_context_len, out, workspace, fmt: str, d: Dims,
                 partition_tokens=0, stream=None):
    _check(lib().kvq_decode_merge(batch, _ptr(context_lens), int(max_context_len), _ptr(out),
                                  _out_dtype(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  partition_tokens, FMT[fmt], ctypes.byref(d), _stream(stream)),
           "kvq_decode_merge")


def decode_attn_noalloc(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                        max_context_len, sm_scale, out, fmt: str, d: Dims, partition_tokens=0,
                        stream=None):
    """kvq_decode_attn_noalloc: decode attention with the library's own static
    scratch instead of a caller workspace (for callers that cannot allocate)."""
    _need(q, torch.bfloat16, "q")
    _need_out(out)
    _need(block_tables, torch.int32, "block_tables")
    _need(context_lens, torch.int32, "context_lens")
    B = q.shape[0]
    _check(lib().kvq_decode_attn_noalloc(_ptr(q), B, _ptr(k_cache), _ptr(v_cache),
                                         _scales(k_scale, v_scale), _ptr(block_tables),
                                         _ptr(context_lens), int(max_context_len), float(sm_scale),
                                         _ptr(out), _out_dtype(out), partition_tokens, FMT[fmt],
                                         ctypes.byref(d), _stream(stream)),
           "kvq_decode_attn_noalloc")


def decode_verify(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                  max_context_len, sm_scale, out, fmt: str, d: Dims, workspace=None,
                  partition_tokens=0, stream=None):
    """Multi-query decode for speculative verification (kvq_decode_verify).
    q, out: [B][Hq][n_query][D]; position j of sequence b sees the tokens before
    the last n_query - 1 - j of its context."""
    _need(q, torch.bfloat16, "q")
    _need_out(out)
    _need(block_tables, torch.int32, "block_tables")
    _need(context_lens, torch.int32, "context_lens")
    if q.dim() != 4 or tuple(out.shape) != tuple(q.shape):
        raise KvqError("q and out must be [batch][n_q_heads][n_query][head_dim]")
    B, nq = q.shape[0], q.shape[2]
    if workspace is None:
        n = lib().kvq_decode_verify_workspace_bytes(B, nq, int(max_context_len), partition_tokens,
                                                    FMT[fmt], ctypes.byref(d))
        if n == 0 and B > 0:
            raise KvqError("kvq_decode_verify_workspace_bytes: invalid arguments")
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    _check(lib().kvq_decode_verify(_ptr(q), B, nq, _ptr(k_cache), _ptr(v_cache),
                                   _scales(k_scale, v_scale), _ptr(block_tables),
                                   _ptr(context_lens), int(max_context_len), float(sm_scale),
                                   _ptr(out), _out_dtype(out), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), partition_tokens,
                                   FMT[fmt], ctypes.byref(d), _stream(stream)), "kvq_decode_verify")
    return out


def set_wait_limit(cycles: int):
    """Bound, in SM clock cycles, on each pipeline wait of later decode launches
    (kvq_set_wait_limit); 0 restores the default of about one second."""
    _check(lib().kvq_set_wait_limit(int(cycles)), "kvq_set_wait_limit")


def wait_limit() -> int:
    return int(lib().kvq_get_wait_limit())


def prefill_attn(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                 max_context_len, sm_scale, out, fmt: str, d: Dims, workspace=None,
                 partition_tokens=0, stream=None):
    """Chunked-prefill attention over the quantized cache (kvq_prefill_attn).
    q, out: [B][Hq][chunk_len][D]; the chunk's tokens are the last chunk_len
    cached tokens of each sequence and attend causally."""
    _need(q, torch.bfloat16, "q")
    _need_out(out)
    _need(block_tables, torch.int32, "block_tables")
    _need(context_lens, torch.int32, "context_lens")
    if q.dim() != 4 or tuple(out.shape) != tuple(q.shape):
        raise KvqError("q and out must be [batch][n_q_heads][chunk_len][head_dim]")
    B, n = q.shape[0], q.shape[2]
    if workspace is None:
        nb = lib().kvq_prefill_attn_workspace_bytes(B, n, int(max_context_len), partition_tokens,
                                                    FMT[fmt], ctypes.byref(d))
        if nb == 0 and B > 0:
            raise KvqError("kvq_prefill_attn_workspace_bytes: invalid arguments")
        workspace = torch.empty(max(nb, 16), dtype=torch.uint8, device=q.device)
    _check(lib().kvq_prefill_attn(_ptr(q), B, n, _ptr(k_cache), _ptr(v_cache),
                                  _scales(k_scale, v_scale), _ptr(block_tables),
                                  _ptr(context_lens), int(max_context_len), float(sm_scale),
                                  _ptr(out), _out_dtype(out), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), partition_tokens,
                                  FMT[fmt], ctypes.byref(d), _stream(stream)), "kvq_prefill_attn")
    return out


def device_error(clear=True) -> int:
    """KVQ_DEVERR_* bits flagged by kernels on the current device (synchronizes)."""
    f = ctypes.c_uint32()
    rc = lib().kvq_device_error(ctypes.byref(f), 1 if clear else 0)
    if rc not in (0, -6):
        _check(rc, "kvq_device_error")
    return f.value


# --------------------------------------------------------------------------- convenience
@dataclass
class LayerCache:
    """Device buffers of one layer's quantized K/V cache (torch-owned memory)."""
    fmt: str
    dims: Dims
    k: torch.Tensor
    v: torch.Tensor
    k_scale: torch.Tensor | None
    v_scale: torch.Tensor | None

    @staticmethod
    def allocate(fmt, d: Dims, device="cuda", k_static=None, v_static=None):
        """Zeroed K/V caches and scales in the library's page layout (include/kvq.h).
        The static formats take their scales here: BF16 [Hk][D] (int8c) or [1]
        (int8t) tensors, kept by reference."""
        nb, hk, D = d.num_blocks, d.n_kv_heads, d.head_dim
        E = ELEM_BYTES[fmt]
        edt = torch.bfloat16 if fmt == "bf16" else torch.uint8
        k = torch.zeros((nb, hk, 2, D * E // 16, 8, 16 // E), dtype=edt, device=device)
        v = torch.zeros((nb, hk, E, D, 16 // E), dtype=edt, device=device)
        mv = META_VALUES[fmt]
        if fmt in STATIC_FORMATS:
            shape = (hk, D) if fmt == "int8c" else (1,)
            for name, t in (("k_static", k_static), ("v_static", v_static)):
                if t is None or tuple(t.shape) != shape:
                    raise KvqError(f"{fmt} needs {name} of shape {shape}")
                _need(t, torch.bfloat16, name)
            ks, vs = k_static, v_static
        elif mv:
            shape = (nb, hk, BLOCK_SIZE) if mv == 1 else (nb, hk, BLOCK_SIZE, 2)
            ks = torch.zeros(shape, dtype=torch.bfloat16, device=device)
            vs = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        else:
            ks = vs = None
        return LayerCache(fmt, d, k, v, ks, vs)

    def append(self, k, v, slot_mapping, stream=None):
        append(k, v, slot_mapping, self.k, self.v, self.k_scale, self.v_scale, self.fmt, self.dims,
               stream)

    def workspace(self, batch, max_context_len, partition_tokens=0, device="cuda"):
        n = decode_workspace_bytes(batch, max_context_len, self.fmt, self.dims, partition_tokens)
        return torch.empty(max(n, 16), dtype=torch.uint8, device=device)

    def decode(self, q, block_tables, context_lens, max_context_len, sm_scale=None, out=None,
               workspace=None, partition_tokens=0, stream=None, out_dtype=torch.bfloat16):
        if sm_scale is None:
            sm_scale = 1.0 / math.sqrt(self.dims.head_dim)
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        if workspace is None:
            workspace = self.workspace(q.shape[0], max_context_len, partition_tokens, q.device)
        decode_attn(q, self.k, self.v, self.k_scale, self.v_scale, block_tables, context_lens,
                    max_context_len, sm_scale, out, workspace, self.fmt, self.dims,
                    partition_tokens, stream)
        return out

    def verify(self, q, block_tables, context_lens, max_context_len, sm_scale=None, out=None,
               workspace=None, partition_tokens=0, stream=None, out_dtype=torch.bfloat16):
        """Multi-query decode (kvq_decode_verify): q [B][Hq][n_query][D], the
        n_query newest cached tokens of each sequence being the positions."""
        if sm_scale is None:
            sm_scale = 1.0 / math.sqrt(self.dims.head_dim)
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        return decode_verify(q, self.k, self.v, self.k_scale, self.v_scale, block_tables,
                             context_lens, max_context_len, sm_scale, out, self.fmt, self.dims,
                             workspace=workspace, partition_tokens=partition_tokens, stream=stream)

    def prefill(self, q, block_tables, context_lens, max_context_len, sm_scale=None, out=None,
                workspace=None, partition_tokens=0, stream=None, out_dtype=torch.bfloat16):
        """Chunked-prefill attention (kvq_prefill_attn): q [B][Hq][chunk][D], the
        chunk being the newest cached tokens of each sequence."""
        if sm_scale is None:
            sm_scale = 1.0 / math.sqrt(self.dims.head_dim)
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        return prefill_attn(q, self.k, self.v, self.k_scale, self.v_scale, block_tables,
                            context_lens, max_context_len, sm_scale, out, self.fmt, self.dims,
                            workspace=workspace, partition_tokens=partition_tokens, stream=stream)

    # ---- copies in the logical layout [NB][Hk][block_size][D] (for inspection and tests)
    def k_logical(self, blocks=None):
        """K of all blocks (or of the block ids `blocks`) as [n][Hk][block_size][D]."""
        k = self.k if blocks is None else self.k[blocks]
        return k.permute(0, 1, 2, 4, 3, 5).reshape(k.shape[0], k.shape[1], BLOCK_SIZE,
                                                   self.dims.head_dim)

    def v_logical(self, blocks=None):
        """V of all blocks (or of the block ids `blocks`) as [n][Hk][block_size][D]."""
        v = self.v if blocks is None else self.v[blocks]
        return v.permute(0, 1, 2, 4, 3).reshape(v.shape[0], v.shape[1], BLOCK_SIZE,
                                                self.dims.head_dim)


# --------------------------------------------------------------------------- KIVI-style cache
@dataclass
class KiviCache:
    """One layer's KIVI-style low-bit cache (torch-owned device memory): packed
    b-bit K and V pages, their BF16 (scale, minimum) arrays, and a BF16 cache
    of its own for each sequence's residual tokens (those after its last
    complete 128-token group)."""
    fmt: str
    dims: Dims
    k: torch.Tensor            # [NB][Hk][16 * D * b / 8] uint8, packed K pages
    v: torch.Tensor            # [NB][Hk][16 * D * b / 8] uint8, packed V pages
    k_meta: torch.Tensor       # [NB][Hk][16][2] bf16: page i of a group holds channels i*D/8..
    v_meta: torch.Tensor       # [NB][Hk][16][2] bf16: per token
    residual: LayerCache       # BF16 cache of the residual tokens

    @staticmethod
    def allocate(fmt, d: Dims, res_dims: Dims, device="cuda"):
        if fmt not in KIVI_BITS:
            raise KvqError("KIVI formats: kivi2, kivi4")
        nb, hk, D = d.num_blocks, d.n_kv_heads, d.head_dim
        pb = BLOCK_SIZE * D * KIVI_BITS[fmt] // 8
        k = torch.zeros((nb, hk, pb), dtype=torch.uint8, device=device)
        v = torch.zeros((nb, hk, pb), dtype=torch.uint8, device=device)
        km = torch.zeros((nb, hk, BLOCK_SIZE, 2), dtype=torch.bfloat16, device=device)
        vm = torch.zeros((nb, hk, BLOCK_SIZE, 2), dtype=torch.bfloat16, device=device)
        return KiviCache(fmt, d, k, v, km, vm, LayerCache.allocate("bf16", res_dims, device))

    def append_groups(self, k, v, slot_mapping, stream=None):
        """Quantize whole 128-token groups (kvq_kivi_append): k, v [T][Hk][D] bf16
        with T a multiple of 128, each run of 128 tokens one group whose slots fill
        eight pages in order."""
        _need(k, torch.bfloat16, "k")
        _need(v, torch.bfloat16, "v")
        _need(slot_mapping, torch.int64, "slot_mapping")
        _check(lib().kvq_kivi_append(_ptr(k), _ptr(v), _ptr(slot_mapping), slot_mapping.numel(),
                                     _ptr(self.k), _ptr(self.v), _ptr(self.k_meta), _ptr(self.v_meta),
                                     FMT[self.fmt], ctypes.byref(self.dims), _stream(stream)),
               "kvq_kivi_append")

    def workspace(self, batch, max_quant_len, max_res_len, device="cuda"):
        n = lib().kvq_kivi_decode_workspace_bytes(batch, int(max_quant_len), int(max_res_len),
                                                  FMT[self.fmt], ctypes.byref(self.dims),
                                                  ctypes.byref(self.residual.dims))
        if n == 0 and batch > 0:
            raise KvqError("kvq_kivi_decode_workspace_bytes: invalid arguments")
        return torch.empty(max(n, 16), dtype=torch.uint8, device=device)

    def decode(self, q, block_tables, quant_lens, max_quant_len, res_tables, res_lens, max_res_len,
               sm_scale=None, out=None, workspace=None, stream=None, out_dtype=torch.bfloat16):
        """Decode attention over each sequence's quantized groups (quant_lens[b]
        tokens, a multiple of 128) and its residual tokens (res_lens[b])."""
        if sm_scale is None:
            sm_scale = 1.0 / math.sqrt(self.dims.head_dim)
        _need(q, torch.bfloat16, "q")
        for t, name in ((block_tables, "block_tables"), (quant_lens, "quant_lens"),
                        (res_tables, "res_tables"), (res_lens, "res_lens")):
            _need(t, torch.int32, name)
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        _need_out(out)
        B = q.shape[0]
        if workspace is None:
            workspace = self.workspace(B, max_quant_len, max_res_len, q.device)
        meta = (ctypes.c_void_p * 2)(self.k_meta.data_ptr(), self.v_meta.data_ptr())
        r = self.residual
        _check(lib().kvq_kivi_decode_attn(_ptr(q), B, _ptr(self.k), _ptr(self.v), meta,
                                          _ptr(block_tables), _ptr(quant_lens), int(max_quant_len),
                                          _ptr(r.k), _ptr(r.v), _ptr(res_tables), _ptr(res_lens),
                                          int(max_res_len), float(sm_scale), _ptr(out),
                                          _out_dtype(out), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          FMT[self.fmt], ctypes.byref(self.dims),
                                          ctypes.byref(r.dims), _stream(stream)),
               "kvq_kivi_decode_attn")
        return out
