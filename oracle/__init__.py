"""CPU oracle for quantized-KV decode attention -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, obviously-correct restatement of what the
quantized-KV decode path computes.  It exists to check the CUDA library and
nothing else: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
and ``--impl reference`` legs of ``bench.py`` may import it.  The product path
(``decode_attention_q8_b200``) never imports, calls or falls back to it, and it
imports nothing from the product path.

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

Pins (what each function is checked against, in ``tests/test_oracle_*.py``):
  blocks      brute-force nearest-grid-point search, round-trip bounds,
              hand-worked blocks, the pages' KV-cache byte counts
  turbo3      published splitmix64 vectors, H*H = d*I, FWHT(e_k) = column k,
              Max (1960) 8-level Gaussian quantizer table, centroid and
              midpoint conditions, round-trip MSE of the Gaussian quantizer
  turbo       2-level closed form +-sqrt(2/pi), Max (1960) 4- and 16-level
              tables, hand-packed 2- and 4-bit bytes, the turbo3 oracle at 3
              bits, round-trip error = the quantizer's distortion
  qjl         unbiased inner products over the projection's draw and the QJL
              variance bound, residual norm and signs formed in the original
              domain, the turbo2 row as its 2-bit stage, no residual = turbo2,
              hand-packed bytes
  attention   brute-force full-matrix softmax(Q K^T) V, closed forms
              (ctx=1, identical keys, q=0), rows summing to 1, split/combine
              identity
No oracle function is left unpinned.
"""

from . import blocks, turbo3, turbo, qjl, attention, cache_model  # noqa: F401
