"""Oracle for "turbo3_qjl" key rows: a 2-bit turbo row plus a 1-bit Quantized
Johnson-Lindenstrauss (QJL) code of its residual, 3 bits per value in all --
TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

numpy marshalling around ``oracle/turbo.cc``, where the steps are stated.  The
TurboQuant page ("Benchmark TurboQuant en Apple Silicon", section
"¿Qué es TurboQuant?") builds its 3-bit cache from a random Walsh-Hadamard
rotation, an optimal scalar quantizer and QJL, which keeps inner products; it
defines none of them.  The reading follows the published constructions (Zandieh
et al., "QJL: 1-Bit Quantized JL Transform for KV Cache Quantization", 2024;
"TurboQuant", 2025): the scalar quantizer takes 2 bits (the turbo2 row), the
residual in the rotated unit domain e = g - c32[code] is projected by the
caller's float32 [d][d] matrix P (u = P e, binary32, left to right), its
signs z = [u < 0] are kept, and gamma = fp16(min(fl(fl(norm * |e|) *
fl32(1/sqrt d)), 65504)) is the residual's norm.  Code row: the 2-bit codes
(d/4 bytes), then the sign bits (d/8 bytes); scale row: (norm, gamma).
Dequantization (float64):
  x_hat = (norm_h/d) D H_un c[code] + sqrt(pi/2)/d * gamma_h * S^T (1 - 2z),
  S^T = D H_un P^T / sqrt(d).
"""

import numpy as np

from . import _lib, turbo

MSE_BITS = 2


def code_bytes(d):
    return MSE_BITS * d // 8 + d // 8


def _rows(x_f16):
    bits = _lib.f16_bits(x_f16)
    d = bits.shape[-1]
    return bits.reshape(-1, d), bits.shape[:-1], d


def residual_f32(x_f16, seed):
    """(norm float32 [n], codes uint8 [n, d], e float32 [n, d]) of rows [n, d]: the
    binary32 norm (before its fp16 rounding), the 2-bit codes and the residual."""
    x, _, d = _rows(x_f16)
    n = x.shape[0]
    norm = np.empty(n, np.float32)
    idx = np.empty((n, d), np.uint8)
    e = np.empty((n, d), np.float32)
    _lib.check(_lib.lib.orc_qjl_residual(_lib.ptr(x), n, d, seed, _lib.ptr(norm), _lib.ptr(idx), _lib.ptr(e)),
               "qjl residual")
    return norm, idx, e


def project_f32(proj, e):
    """u[n, i] = sum_j proj[i][j] * e[n, j] in binary32, left to right."""
    p = _lib.arr(proj, np.float32)
    ee = _lib.arr(e, np.float32)
    d = ee.shape[-1]
    u = np.empty(ee.shape, np.float32)
    _lib.check(_lib.lib.orc_qjl_project(_lib.ptr(p), _lib.ptr(ee), ee.size // d, d, _lib.ptr(u)), "qjl project")
    return u


def quantize_parts(x_f16, seed, proj):
    """(norm_h, gamma_h float16 ``[...]``, codes uint8 ``[..., d]``, z uint8 ``[..., d]``)."""
    x, lead, d = _rows(x_f16)
    n = x.shape[0]
    p = _lib.arr(proj, np.float32)
    norm = np.empty(n, np.uint16)
    gamma = np.empty(n, np.uint16)
    idx = np.empty((n, d), np.uint8)
    z = np.empty((n, d), np.uint8)
    _lib.check(_lib.lib.orc_qjl_quantize_parts(_lib.ptr(x), n, d, seed, _lib.ptr(p), _lib.ptr(norm),
                                               _lib.ptr(gamma), _lib.ptr(idx), _lib.ptr(z)), "qjl quantize")
    return (norm.view(np.float16).reshape(lead), gamma.view(np.float16).reshape(lead), idx.reshape(*lead, d),
            z.reshape(*lead, d))


def quantize(x_f16, seed, proj):
    """Rows ``[..., d]`` -> (scales float16 ``[..., 2]`` = (norm_h, gamma_h), codes
    uint8 ``[..., 3d/8]`` = the 2-bit code field, then the 1-bit z field)."""
    x, lead, d = _rows(x_f16)
    n = x.shape[0]
    p = _lib.arr(proj, np.float32)
    scales = np.empty((n, 2), np.uint16)
    codes = np.empty((n, code_bytes(d)), np.uint8)
    _lib.check(_lib.lib.orc_qjl_quantize(_lib.ptr(x), n, d, seed, _lib.ptr(p), _lib.ptr(scales), _lib.ptr(codes)),
               "qjl quantize")
    return scales.view(np.float16).reshape(*lead, 2), codes.reshape(*lead, code_bytes(d))


def split_codes(codes, d):
    """(codes uint8 ``[..., d]``, z uint8 ``[..., d]``) of stored code rows."""
    c = np.asarray(codes, dtype=np.uint8)
    nb = MSE_BITS * d // 8
    return turbo.unpack(c[..., :nb], d, MSE_BITS), turbo.unpack(c[..., nb:], d, 1)


def dequantize(scales, codes, seed, proj, d):
    """x_hat float64 ``[..., d]`` of stored rows (scales ``[..., 2]``, codes ``[..., 3d/8]``)."""
    c = _lib.arr(codes, np.uint8)
    sc = _lib.f16_bits(_lib.arr(scales, np.float16))
    p = _lib.arr(proj, np.float32)
    rows = c.size // c.shape[-1]
    assert sc.size == 2 * rows
    out = np.empty((*c.shape[:-1], d), np.float64)
    _lib.check(_lib.lib.orc_qjl_dequantize(_lib.ptr(sc), _lib.ptr(c), rows, d, seed, _lib.ptr(p), _lib.ptr(out)),
               "qjl dequantize")
    return out


def projection_matrix(seed, proj, d):
    """S = P H_un D / sqrt(d) in float64: the original-domain QJL matrix that
    coding the rotated residual with P amounts to."""
    p = _lib.arr(proj, np.float32)
    out = np.empty((d, d), np.float64)
    _lib.check(_lib.lib.orc_qjl_projection_matrix(seed, _lib.ptr(p), d, _lib.ptr(out)), "qjl projection")
    return out
