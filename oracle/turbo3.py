"""Oracle for the turbo3 value-cache row: seeded signs, Walsh-Hadamard rotation,
per-vector norm and an 8-level Lloyd-Max scalar code packed at 3 bits --
TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

numpy marshalling around ``oracle/turbo.cc``, where the steps and their
readings are stated ("Benchmark TurboQuant en Apple Silicon", section
"¿Qué es TurboQuant?": a random Walsh-Hadamard rotation, then an optimal
scalar quantizer, at 3 bits per value):

  signs s_i from splitmix64(seed); v = s * x; norm = sqrtf(strided tree sum
  of v_i^2); w = unnormalised FWHT(v) (stages 1, 2, ..., d/2);
  g = fl(w * fl(1/norm)); code_i = #{k : g_i > tau_k} over the 7 binary32
  midpoints of the 8-level Lloyd-Max quantizer of N(0,1); codes packed 3 bits
  each, little-endian; stored norm fp16(min(norm, 65504)).
Dequantization: x_hat = (norm_h / d) * D * H_un * c[code] (float64).
"""

import numpy as np

from . import _lib
from . import turbo

ROW_LEVELS = 8


def splitmix64(seed, n):
    """First n outputs of splitmix64 started at state ``seed`` (Python ints)."""
    out = np.empty(n, np.uint64)
    _lib.lib.orc_splitmix64(seed, n, _lib.ptr(out))
    return [int(v) for v in out]


def signs(seed, d):
    """The +-1 vector D (float32 [d]) for ``seed``."""
    out = np.empty(d, np.float32)
    _lib.check(_lib.lib.orc_signs(seed, d, _lib.ptr(out)), "signs")
    return out


def sylvester(d):
    """Unnormalised Sylvester-Hadamard matrix of order d (float64 [d][d])."""
    out = np.empty((d, d), np.float64)
    _lib.check(_lib.lib.orc_sylvester(d, _lib.ptr(out)), "sylvester")
    return out


def fwht_f32(v):
    """Unnormalised fast Walsh-Hadamard transform over the last axis, binary32."""
    a = _lib.arr(v, np.float32)
    d = a.shape[-1]
    out = np.empty(a.shape, np.float32)
    _lib.check(_lib.lib.orc_fwht_f32(_lib.ptr(a), a.size // d, d, _lib.ptr(out)), "fwht")
    return out


def tree_sum_f32(a):
    """Strided pairwise sum over the last axis in binary32 (stride d/2, ..., 1)."""
    x = _lib.arr(a, np.float32)
    d = x.shape[-1]
    out = np.empty(x.shape[:-1], np.float32)
    _lib.check(_lib.lib.orc_tree_sum_f32(_lib.ptr(x), x.size // d, d, _lib.ptr(out)), "tree sum")
    return out[()] if out.ndim == 0 else out


def lloyd_max_gaussian8():
    """8-level Lloyd-Max quantizer for N(0,1), float64: ``(levels[8], thresholds[7])``."""
    return turbo.lloyd_max_gaussian(ROW_LEVELS)


def codebook_f32():
    """(levels, thresholds) rounded to binary32, the decision values both sides compare."""
    return turbo.codebook_f32(3)


def code_bytes(d):
    return 3 * d // 8


def quantize_turbo3_indices(x_f16, seed):
    """Rows ``[..., d]`` -> (norm_h float16 ``[...]``, codes uint8 0..7 ``[..., d]``)."""
    return turbo.quantize_indices(x_f16, seed, 3)


def quantize_turbo3(x_f16, seed):
    """Rows ``[..., d]`` -> (norm_h float16 ``[...]``, packed codes uint8 ``[..., 3d/8]``)."""
    return turbo.quantize(x_f16, seed, 3)


def pack3(idx):
    """3-bit little-endian bit stream: code i in bits 3i..3i+2."""
    return turbo.pack(idx, 3)


def unpack3(codes, d):
    return turbo.unpack(codes, d, 3)


def dequantize_turbo3(norm_h, codes, seed, d):
    """x_hat = (norm_h / d) * D * H_un * c[code], float64 ``[..., d]``."""
    return turbo.dequantize(norm_h, codes, seed, d, 3)
