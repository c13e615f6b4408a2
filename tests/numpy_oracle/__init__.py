"""A second restatement of the oracle in numpy -- TEST INFRASTRUCTURE ONLY.

The oracle proper is the C++ library under ``oracle/`` (quantizers in IEEE
binary32 without fused operations, attention in binary64).  This package is an
earlier restatement of the same definitions in numpy, written independently of
the C++ code and of the CUDA library.  Only ``tests/test_oracle_cross.py``
imports it: it checks that both restatements produce the same quantized bytes
bit for bit and the same dequantized values and attention outputs to binary64
rounding, which catches a porting slip in either.  Nothing else uses it.

Precision:
  * quantizers run in IEEE binary32 exactly as the block formats state them
    (numpy float32 element-wise arithmetic: one rounding per operation, no
    fused multiply-add), so their bytes are unique and must match bit for bit;
  * dequantization and attention run in binary64.

Modules:
  blocks      q8_0 / q4_0 / f16 cache rows (quantize, pack, dequantize)
  turbo3      seeded sign vector (splitmix64), Sylvester Hadamard, fast
              Walsh-Hadamard transform, Lloyd-Max codebook, turbo3 rows
  turbo       the same rows at 2 and 4 bits per value (turbo2, turbo4)
  qjl         turbo3_qjl key rows: the 2-bit row plus 1-bit QJL signs of its
              residual and the residual's norm
  attention   decode attention (plain softmax definition), split partials
              and their combine
  cache_model bytes per cache row / per cache, the nominal-size model
"""

from . import blocks, turbo3, turbo, qjl, attention, cache_model  # noqa: F401
