"""Quantized paged KV cache (FP8 E4M3 / INT8 asymmetric) for LLM decode on B200.

Two hot operations, both hand-written CUDA for sm_100a behind the C-ABI library
``libkvq.so`` (declared in ``include/kvq.h``):

* ``append``      quantize-on-append of new tokens' K/V into a paged block pool;
* ``decode_attn`` paged GQA decode attention that dequantises the cache in
                  registers, with an online-softmax split-K and a merge kernel.

The Python layer (``kvq``) only marshals arguments: PyTorch tensors supply device
pointers and the current CUDA stream. Nothing here computes on the CPU; if the
library is missing, every call raises.
"""

from . import workloads  # noqa: F401  (seeded input generators; no method arithmetic)

__all__ = ["workloads", "kvq"]


def __getattr__(name):
    if name == "kvq":
        import importlib
        return importlib.import_module(__name__ + ".kvq")
    raise AttributeError(name)
