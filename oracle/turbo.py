"""Oracle for the turbo value-cache rows at b = 2, 3 or 4 bits per value
("turbo2", "turbo3", "turbo4") -- TEST INFRASTRUCTURE ONLY (see
``oracle/__init__.py``).

numpy marshalling around ``oracle/turbo.cc``.  The TurboQuant page
("Benchmark TurboQuant en Apple Silicon", section "¿Qué es TurboQuant?")
describes a random Walsh-Hadamard rotation followed by an optimal scalar
quantizer; its FAQ ("¿Qué formato TurboQuant debería usar?") puts values at 2
to 3 bits.  The widths other than 3 are the same construction with another
level count: the 2^b-level Lloyd-Max quantizer of N(0,1), codes packed b bits
each, little-endian.  Dequantization: x_hat = (norm_h / d) * D * H_un *
c[code] (float64).
"""

import numpy as np

from . import _lib

BITS = {"turbo2": 2, "turbo3": 3, "turbo4": 4}


def lloyd_max_gaussian(n_levels):
    """n-level Lloyd-Max quantizer for N(0,1) (n even), float64, by Lloyd's
    iteration: ``(levels[n], thresholds[n-1])`` ascending."""
    lv = np.empty(n_levels, np.float64)
    th = np.empty(n_levels - 1, np.float64)
    if _lib.lib.orc_lloyd_max_gaussian(n_levels, _lib.ptr(lv), _lib.ptr(th)) < 0:
        raise RuntimeError("Lloyd iteration did not converge")
    return lv, th


def codebook_f32(bits):
    """(levels, thresholds) of the 2^bits-level quantizer rounded to binary32."""
    lv, th = lloyd_max_gaussian(1 << bits)
    return lv.astype(np.float32), th.astype(np.float32)


def code_bytes(bits, d):
    return bits * d // 8


def _rows(x_f16):
    bits = _lib.f16_bits(x_f16)
    d = bits.shape[-1]
    return bits.reshape(-1, d), bits.shape[:-1], d


def quantize_indices(x_f16, seed, bits):
    """(norm_h float16 ``[...]``, codes uint8 ``[..., d]``) of rows x_f16 ``[..., d]``."""
    x, lead, d = _rows(x_f16)
    norm = np.empty(x.shape[0], np.uint16)
    idx = np.empty(x.shape, np.uint8)
    _lib.check(_lib.lib.orc_turbo_quantize_indices(_lib.ptr(x), x.shape[0], d, seed, bits, _lib.ptr(norm),
                                                   _lib.ptr(idx)), "turbo quantize")
    return norm.view(np.float16).reshape(lead), idx.reshape(*lead, d)


def pack(idx, bits):
    """b-bit little-endian bit stream: code i in bits b*i .. b*i+b-1."""
    c = _lib.arr(idx, np.uint8)
    d = c.shape[-1]
    out = np.empty((*c.shape[:-1], bits * d // 8), np.uint8)
    _lib.check(_lib.lib.orc_turbo_pack(_lib.ptr(c), c.size // d, d, bits, _lib.ptr(out)), "pack")
    return out


def unpack(codes, d, bits):
    c = _lib.arr(codes, np.uint8)
    nb = c.shape[-1]
    out = np.empty((*c.shape[:-1], d), np.uint8)
    _lib.check(_lib.lib.orc_turbo_unpack(_lib.ptr(c), c.size // nb, d, bits, _lib.ptr(out)), "unpack")
    return out


def quantize(x_f16, seed, bits):
    """Rows ``[..., d]`` -> (norm_h float16 ``[...]``, packed codes uint8 ``[..., b*d/8]``)."""
    x, lead, d = _rows(x_f16)
    norm = np.empty(x.shape[0], np.uint16)
    codes = np.empty((x.shape[0], bits * d // 8), np.uint8)
    _lib.check(_lib.lib.orc_turbo_quantize(_lib.ptr(x), x.shape[0], d, seed, bits, _lib.ptr(norm),
                                           _lib.ptr(codes)), "turbo quantize")
    return norm.view(np.float16).reshape(lead), codes.reshape(*lead, bits * d // 8)


def dequantize(norm_h, codes, seed, d, bits):
    """x_hat = (norm_h / d) * D * H_un * c[code], float64 ``[..., d]``."""
    c = _lib.arr(codes, np.uint8)
    n = _lib.f16_bits(_lib.arr(norm_h, np.float16))
    rows = c.size // c.shape[-1]
    assert n.size == rows
    out = np.empty((*c.shape[:-1], d), np.float64)
    _lib.check(_lib.lib.orc_turbo_dequantize(_lib.ptr(n), _lib.ptr(c), rows, d, seed, bits, _lib.ptr(out)),
               "turbo dequantize")
    return out
