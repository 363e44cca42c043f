"""CPU oracle for the quantized paged KV cache — TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, obviously-correct restatement of what the
quantized KV-cache decode path computes. Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it. The product path (the CUDA library and its
Python binding) never imports, calls or links anything here, and nothing here
imports the product. The two share no code; they meet only through the seeded
input generators of ``int8_quantized_paged_quantize_b200.workloads``, which hold
none of the method's arithmetic.

Sources (web pages; cited by title and section):

* [LIMITS] "KV cache quantization: what FP8/INT8 K and V really give, and their
  limits" (molayo1419.me) — sections "What KV cache quantization actually is",
  "Formats you will actually meet" (the notes under the formats table), "TL;DR".
* [76X] "Fitting 76x concurrent requests with an FP8 KV cache" (storycompiler,
  tistory 431) — "2. How much memory the KV cache takes", "4. Precision loss?".
* [COMPRESS] "KV Cache compression" (ryotta.opik.net) — "1. The KV cache memory
  problem", "3.1 Quantization techniques", "5.1 Quantization pipeline",
  "6.2 Combining with other techniques", "6.3 Implementation considerations".
* [GUIDE] "From FP8 KV cache to INT4 weight-only: GPU LLM serving optimisation
  guide (May 2026)" (daewooki.github.io) — "Core concepts" 1) prefill vs decode,
  2) PagedAttention, 3) KV cache quantization.

Modules
-------
``formats``   E4M3 and INT8 codecs, BF16 rounding, the per-token scale rules.
``paged``     slot arithmetic, quantize-on-append into a logical block pool,
              paged gather + dequantisation.
``attention`` FP64 softmax attention over the gathered K/V (GQA head mapping).
``sizes``     the closed-form KV-cache byte count.
``kivi``      KIVI-style low-bit codes (K per channel, V per token, BF16
              residual); the CUDA path for it is not built.

Parity status of each function is given in its docstring; the one result with
no pin is the quality number (deviation from a BF16-cache attention), which is
reported, not checked: "parity unpinned".
"""

from . import formats, paged, attention, sizes, kivi  # noqa: F401
