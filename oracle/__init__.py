"""CPU oracle for quantized-KV decode attention -- TEST INFRASTRUCTURE ONLY.

The oracle is a plain, slow C++ library (``oracle/*.cc``, built into
``oracle/liboracle.so`` with ``-O2 -ffp-contract=off -fno-fast-math``) that
restates what the quantized-KV decode path computes, to check the CUDA library
and nothing else.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline and ``--impl reference`` legs of ``bench.py`` may import it.  The
product path (``decode_attention_q8_b200``) never imports, calls, links or
falls back to it, and it includes nothing from the product's sources or
headers.  The modules here only marshal numpy arrays to its C entry points
(``oracle/oracle.h``); every step of the arithmetic runs in the C++ code.

Precision:
  * quantizers run in IEEE binary32 exactly as the block formats state them
    (one rounding per operation, no fused multiply-add), so their bytes are
    unique and must match bit for bit;
  * dequantization and attention run in binary64.

Modules:
  blocks      q8_0 / q4_0 / q5_0 / f16 cache rows (quantize, pack, dequantize)
  turbo3      seeded sign vector (splitmix64), Sylvester Hadamard, fast
              Walsh-Hadamard transform, Lloyd-Max codebook, turbo3 rows
  turbo       the same rows at 2 and 4 bits per value (turbo2, turbo4)
  qjl         turbo3_qjl key rows: the 2-bit row plus 1-bit QJL signs of its
              residual and the residual's norm
  attention   decode attention (plain softmax definition), split partials
              and their combine, one decode over a stored cache
  cache_model bytes per cache row / per cache

Pins (what each function is checked against, in ``tests/test_oracle_*.py``):
  blocks      hand-worked single blocks and multi-block rows (quantized bytes
              and dequantized values), brute-force nearest-grid-point search,
              round-trip bounds through the dequantizers, the pages' KV-cache
              byte counts
  turbo3      published splitmix64 vectors, H*H = d*I, FWHT(e_k) = column k,
              Max (1960) 8-level Gaussian quantizer table, centroid and
              midpoint conditions, closed-form rows, round-trip MSE of the
              Gaussian quantizer
  turbo       2-level closed form +-sqrt(2/pi), Max (1960) 4- and 16-level
              tables, hand-packed 2- and 4-bit bytes, the 3-bit rows equal to
              turbo3's, round-trip error = the quantizer's distortion
  qjl         unbiased inner products over the projection's draw and the QJL
              variance bound, residual norm and signs formed in the original
              domain, the turbo2 row as its 2-bit stage, no residual = turbo2,
              hand-packed bytes
  attention   torch's scaled_dot_product_attention, brute-force full-matrix
              softmax(Q K^T) V, closed forms (ctx = 1, identical keys, q = 0),
              rows summing to 1, split/combine identity, the stored-cache
              decode equal to dequantize-then-attend
No oracle function is left unpinned.
"""

from . import blocks, turbo3, turbo, qjl, attention, cache_model  # noqa: F401
