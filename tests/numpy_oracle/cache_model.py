"""Oracle byte model of the KV cache: bytes per cached row and per cache.

Test infrastructure only (see ``oracle/__init__.py``).

Per 32 elements: f16 64 bytes, q8_0 34 bytes (fp16 scale + 32 int8),
q4_0 18 bytes (fp16 scale + 16 bytes of nibbles), q5_0 22 bytes (fp16 scale, 16 bytes of
nibbles, a 32-bit word of fifth bits).  turbo2 / turbo3 / turbo4
per row of d elements: 2d/8, 3d/8, 4d/8 bytes of codes + an fp16 norm; turbo3_qjl
3d/8 bytes of codes (2-bit levels, 1-bit residual signs) + two fp16 norms.  Nominal costs are on
``llama.cpp für Geschwindigkeit und Speicher optimieren``, section
"KV-Cache-Präzision" (2 / 1 / 0.5 bytes per element); the exact block sizes
are pinned by the cache sizes the KVSplit page and the llama.cpp issue print
(see ``tests/golden/kv_cache_bytes.txt``).
"""

BYTES_PER_32 = {"f16": 64, "q8_0": 34, "q4_0": 18, "q5_0": 22}


def row_bytes(kind, d):
    """Bytes one cached row of d elements takes."""
    if kind in ("turbo2", "turbo3", "turbo4"):
        return int(kind[-1]) * d // 8 + 2
    if kind == "turbo3_qjl":
        return 3 * d // 8 + 4
    if d % 32:
        raise ValueError("head_dim must be a multiple of 32")
    return BYTES_PER_32[kind] * d // 32


def cache_bytes(kind, n_layers, n_kv_heads, head_dim, n_cells):
    """Bytes of one tensor (K or V) of a cache over all layers."""
    return n_layers * n_kv_heads * n_cells * row_bytes(kind, head_dim)
