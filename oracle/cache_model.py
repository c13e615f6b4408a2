"""Oracle byte model of the KV cache: bytes per cached row and per cache --
TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Per 32 elements: f16 64 bytes, q8_0 34 bytes (fp16 scale + 32 int8), q4_0 18
bytes (fp16 scale + 16 bytes of nibbles), q5_0 22 bytes (fp16 scale, 16 bytes
of nibbles, a 32-bit word of fifth bits).  turbo2 / turbo3 / turbo4 per row of
d elements: 2d/8, 3d/8, 4d/8 bytes of codes + an fp16 norm; turbo3_qjl 3d/8
bytes of codes (2-bit levels, 1-bit residual signs) + two fp16 norms
(``orc_row_bytes`` in ``oracle/blocks.cc``).  Nominal costs are on
``llama.cpp für Geschwindigkeit und Speicher optimieren``, section
"KV-Cache-Präzision" (2 / 1 / 0.5 bytes per element); the exact block sizes
are pinned by the cache sizes the KVSplit page and the llama.cpp issue print
(``tests/golden/kv_cache_bytes.txt``).
"""

from . import _lib


def row_bytes(kind, d):
    """Bytes one cached row of d elements takes."""
    n = int(_lib.lib.orc_row_bytes(_lib.TYPES[kind], d))
    if n == 0:
        raise ValueError(f"{kind} has no row of {d} elements")
    return n


def cache_bytes(kind, n_layers, n_kv_heads, head_dim, n_cells):
    """Bytes of one tensor (K or V) of a cache over all layers."""
    return n_layers * n_kv_heads * n_cells * row_bytes(kind, head_dim)
