"""Oracle for the 32-element block cache formats q8_0, q4_0 and q5_0, and the
f16 row -- TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

numpy marshalling around ``oracle/blocks.cc``, where the arithmetic and its
citations live ("llama.cpp für Geschwindigkeit und Speicher optimieren",
section "KV-Cache-Präzision"; the block formats' definitions):

  q8_0: d = amax / 127; q_j = round-half-away(x_j / d); fp16 d stored.
  q4_0: m = the signed x_j of largest magnitude (lowest index on ties);
        d = m / -8; q_j = min(15, trunc(x_j * (1/d) + 8.5)) with two binary32
        roundings; element j -> low nibble of byte j, j+16 -> high nibble.
  q5_0: d = m / -16; q_j = min(31, trunc(x_j * (1/d) + 16.5)); low four bits
        packed as q4_0's nibbles, bit 4 of q_j in bit j of a 32-bit word qh.

Every quantizer takes fp16 input (numpy float16, last axis a multiple of 32).
Dequantizers return float64.
"""

import numpy as np

from . import _lib

QK = 32  # elements per block


def _rows(x_f16):
    bits = _lib.f16_bits(x_f16)
    n = bits.shape[-1]
    if n % QK:
        raise ValueError("last axis must be a multiple of 32")
    return bits.reshape(-1, n), bits.shape[:-1], n


def quantize_q8_0(x_f16):
    """Rows -> ``(d, qs)``: ``d`` float16 ``[..., n/32]``, ``qs`` int8 ``[..., n]``."""
    x, lead, n = _rows(x_f16)
    d = np.empty((x.shape[0], n // QK), np.uint16)
    q = np.empty(x.shape, np.int8)
    _lib.check(_lib.lib.orc_quantize_q8_0(_lib.ptr(x), x.shape[0], n, _lib.ptr(d), _lib.ptr(q)), "q8_0")
    return d.view(np.float16).reshape(*lead, n // QK), q.reshape(*lead, n)


def dequantize_q8_0(d_f16, qs):
    """x_hat_j = double(d_h) * q_j, float64 ``[..., n]``."""
    q = _lib.arr(qs, np.int8)
    n = q.shape[-1]
    d = _lib.f16_bits(_lib.arr(d_f16, np.float16))
    out = np.empty(q.shape, np.float64)
    rows = q.size // n
    assert d.size == rows * (n // QK)
    _lib.check(_lib.lib.orc_dequantize_q8_0(_lib.ptr(d), _lib.ptr(q), rows, n, _lib.ptr(out)), "q8_0 dequantize")
    return out


def quantize_q4_0_codes(x_f16):
    """Rows -> ``(d, codes)``: ``d`` float16 ``[..., n/32]``, codes uint8 0..15 ``[..., n]``."""
    x, lead, n = _rows(x_f16)
    d = np.empty((x.shape[0], n // QK), np.uint16)
    c = np.empty(x.shape, np.uint8)
    _lib.check(_lib.lib.orc_quantize_q4_0_codes(_lib.ptr(x), x.shape[0], n, _lib.ptr(d), _lib.ptr(c)), "q4_0")
    return d.view(np.float16).reshape(*lead, n // QK), c.reshape(*lead, n)


def pack_q4_0(codes):
    """Element j of a block -> low nibble of byte j, element j+16 -> high nibble."""
    c = _lib.arr(codes, np.uint8)
    n = c.shape[-1]
    out = np.empty((*c.shape[:-1], n // 2), np.uint8)
    _lib.check(_lib.lib.orc_pack_q4_0(_lib.ptr(c), c.size // n, n, _lib.ptr(out)), "q4_0 pack")
    return out


def unpack_q4_0(qs):
    p = _lib.arr(qs, np.uint8)
    n = 2 * p.shape[-1]
    out = np.empty((*p.shape[:-1], n), np.uint8)
    _lib.check(_lib.lib.orc_unpack_q4_0(_lib.ptr(p), p.size * 2 // n, n, _lib.ptr(out)), "q4_0 unpack")
    return out


def quantize_q4_0(x_f16):
    """Rows -> ``(d, qs)`` with ``qs`` packed uint8 ``[..., n/2]``."""
    d, codes = quantize_q4_0_codes(x_f16)
    return d, pack_q4_0(codes)


def dequantize_q4_0(d_f16, qs):
    """x_hat_j = double(d_h) * (q_j - 8), float64 ``[..., n]``."""
    p = _lib.arr(qs, np.uint8)
    n = 2 * p.shape[-1]
    d = _lib.f16_bits(_lib.arr(d_f16, np.float16))
    rows = p.size * 2 // n
    assert d.size == rows * (n // QK)
    out = np.empty((*p.shape[:-1], n), np.float64)
    _lib.check(_lib.lib.orc_dequantize_q4_0(_lib.ptr(d), _lib.ptr(p), rows, n, _lib.ptr(out)), "q4_0 dequantize")
    return out


def quantize_q5_0_codes(x_f16):
    """Rows -> ``(d, codes)``: ``d`` float16 ``[..., n/32]``, codes uint8 0..31 ``[..., n]``."""
    x, lead, n = _rows(x_f16)
    d = np.empty((x.shape[0], n // QK), np.uint16)
    c = np.empty(x.shape, np.uint8)
    _lib.check(_lib.lib.orc_quantize_q5_0_codes(_lib.ptr(x), x.shape[0], n, _lib.ptr(d), _lib.ptr(c)), "q5_0")
    return d.view(np.float16).reshape(*lead, n // QK), c.reshape(*lead, n)


def pack_q5_0(codes):
    """``(qs, qh)``: the low four bits as q4_0's nibbles ``[..., n/2]`` and bit 4 of
    element j as bit j of a uint32 per block ``[..., n/32]``."""
    c = _lib.arr(codes, np.uint8)
    n = c.shape[-1]
    qs = np.empty((*c.shape[:-1], n // 2), np.uint8)
    qh = np.empty((*c.shape[:-1], n // QK), np.uint32)
    _lib.check(_lib.lib.orc_pack_q5_0(_lib.ptr(c), c.size // n, n, _lib.ptr(qs), _lib.ptr(qh)), "q5_0 pack")
    return qs, qh


def unpack_q5_0(qs, qh):
    p = _lib.arr(qs, np.uint8)
    h = _lib.arr(qh, np.uint32)
    n = 2 * p.shape[-1]
    out = np.empty((*p.shape[:-1], n), np.uint8)
    _lib.check(_lib.lib.orc_unpack_q5_0(_lib.ptr(p), _lib.ptr(h), p.size * 2 // n, n, _lib.ptr(out)), "q5_0 unpack")
    return out


def quantize_q5_0(x_f16):
    """Rows -> ``(d, qs, qh)``."""
    d, codes = quantize_q5_0_codes(x_f16)
    qs, qh = pack_q5_0(codes)
    return d, qs, qh


def dequantize_q5_0(d_f16, qs, qh):
    """x_hat_j = double(d_h) * (q_j - 16), float64 ``[..., n]``."""
    p = _lib.arr(qs, np.uint8)
    h = _lib.arr(qh, np.uint32)
    n = 2 * p.shape[-1]
    d = _lib.f16_bits(_lib.arr(d_f16, np.float16))
    rows = p.size * 2 // n
    assert d.size == rows * (n // QK) and h.size == rows * (n // QK)
    out = np.empty((*p.shape[:-1], n), np.float64)
    _lib.check(_lib.lib.orc_dequantize_q5_0(_lib.ptr(d), _lib.ptr(p), _lib.ptr(h), rows, n, _lib.ptr(out)),
               "q5_0 dequantize")
    return out


def dequantize_f16(x_f16):
    """The f16 cache stores the input unchanged; x_hat = double(x)."""
    x = _lib.f16_bits(_lib.arr(x_f16, np.float16))
    out = np.empty(x.shape, np.float64)
    _lib.lib.orc_dequantize_f16(_lib.ptr(x), x.size, _lib.ptr(out))
    return out


def f32_to_f16(x):
    """binary32 -> binary16 (round to nearest even), the rounding the quantizers'
    stored scales and norms use."""
    a = _lib.arr(x, np.float32)
    out = np.empty(a.shape, np.uint16)
    _lib.lib.orc_f32_to_f16(_lib.ptr(a), a.size, _lib.ptr(out))
    return out.view(np.float16)
