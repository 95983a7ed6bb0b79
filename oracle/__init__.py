"""CPU oracle for the WUSH-KV append + decode-attention path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or run
anything in this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

It is a plain, slow restatement of what the method computes, written from the
WUSH-KV pages ("WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms"
and the cnshai.top post "kv-cache-quantization-fp8-training"), in numpy:
float64 everywhere, except the per-token quantizer, whose fp32 decisions
(percentile, scale, code rounding) are part of its definition and are taken in
fp32 exactly, operation by operation.  It shares no code with the CUDA library.

Modules:
  quantizer  -- per-token percentile-clipped asymmetric affine quantizer, packing
  cache      -- the cache with full-precision sink / recent windows (Alg. 2 prose)
  attention  -- query compensation and exact-softmax decode attention
  footprint  -- the pages' cache-size arithmetic
  rope       -- per-head RMSNorm and rotate-half RoPE of the path's raw inputs
  transform  -- the normalised Walsh-Hadamard key transform
  quest      -- the RMS-scaled symmetric (QuEST-style) alternative quantizer
  calibration -- per-KV-head Gram matrices of cached vectors (calibration statistics)

Parity status: every function is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_pins.py``, ``tests/test_oracle_rope.py``,
``tests/test_oracle_transform.py``, ``tests/test_oracle_quest.py`` and
``tests/test_oracle_calibration.py``; none is "parity
unpinned" (the QuEST-style quantizer's reading of the lost Eq. 5 is pinned by the Gaussian
optimum and its grid, not by the pages' equation).
"""
from . import quantizer, cache, attention, footprint, rope, transform, quest, calibration  # noqa: F401
