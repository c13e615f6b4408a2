"""Loads the C++ oracle (oracle/liboracle.so) -- TEST INFRASTRUCTURE ONLY.

Builds it first when it is missing or older than its sources (g++ is part of
the image, so a fresh checkout needs no separate step), then declares the
argument types of every entry point in ``oracle/oracle.h``.
"""

import ctypes

import numpy as np

from . import build as _build

lib = ctypes.CDLL(_build.build())

_P = ctypes.c_void_p
_I32, _I64, _U64, _F64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double

_SIGS = {
    "orc_f32_to_f16": (None, [_P, _I64, _P]),
    "orc_f16_to_f64": (None, [_P, _I64, _P]),
    "orc_row_bytes": (_I64, [_I32, _I32]),
    "orc_quantize_q8_0": (ctypes.c_int, [_P, _I64, _I32, _P, _P]),
    "orc_quantize_q4_0_codes": (ctypes.c_int, [_P, _I64, _I32, _P, _P]),
    "orc_pack_q4_0": (ctypes.c_int, [_P, _I64, _I32, _P]),
    "orc_unpack_q4_0": (ctypes.c_int, [_P, _I64, _I32, _P]),
    "orc_quantize_q5_0_codes": (ctypes.c_int, [_P, _I64, _I32, _P, _P]),
    "orc_pack_q5_0": (ctypes.c_int, [_P, _I64, _I32, _P, _P]),
    "orc_unpack_q5_0": (ctypes.c_int, [_P, _P, _I64, _I32, _P]),
    "orc_dequantize_q8_0": (ctypes.c_int, [_P, _P, _I64, _I32, _P]),
    "orc_dequantize_q4_0": (ctypes.c_int, [_P, _P, _I64, _I32, _P]),
    "orc_dequantize_q5_0": (ctypes.c_int, [_P, _P, _P, _I64, _I32, _P]),
    "orc_dequantize_f16": (None, [_P, _I64, _P]),
    "orc_splitmix64": (None, [_U64, _I64, _P]),
    "orc_signs": (ctypes.c_int, [_U64, _I32, _P]),
    "orc_sylvester": (ctypes.c_int, [_I32, _P]),
    "orc_fwht_f32": (ctypes.c_int, [_P, _I64, _I32, _P]),
    "orc_tree_sum_f32": (ctypes.c_int, [_P, _I64, _I32, _P]),
    "orc_lloyd_max_gaussian": (ctypes.c_int, [_I32, _P, _P]),
    "orc_turbo_quantize_indices": (ctypes.c_int, [_P, _I64, _I32, _U64, _I32, _P, _P]),
    "orc_turbo_pack": (ctypes.c_int, [_P, _I64, _I32, _I32, _P]),
    "orc_turbo_unpack": (ctypes.c_int, [_P, _I64, _I32, _I32, _P]),
    "orc_turbo_quantize": (ctypes.c_int, [_P, _I64, _I32, _U64, _I32, _P, _P]),
    "orc_turbo_dequantize": (ctypes.c_int, [_P, _P, _I64, _I32, _U64, _I32, _P]),
    "orc_qjl_residual": (ctypes.c_int, [_P, _I64, _I32, _U64, _P, _P, _P]),
    "orc_qjl_project": (ctypes.c_int, [_P, _P, _I64, _I32, _P]),
    "orc_qjl_quantize_parts": (ctypes.c_int, [_P, _I64, _I32, _U64, _P, _P, _P, _P, _P]),
    "orc_qjl_quantize": (ctypes.c_int, [_P, _I64, _I32, _U64, _P, _P, _P]),
    "orc_qjl_dequantize": (ctypes.c_int, [_P, _P, _I64, _I32, _U64, _P, _P]),
    "orc_qjl_projection_matrix": (ctypes.c_int, [_U64, _P, _I32, _P]),
    "orc_decode_attention": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I64, _I32, _F64, _P, _I32]),
    "orc_softmax_weights": (ctypes.c_int, [_P, _P, _I64, _I32, _F64, _P]),
    "orc_partials": (ctypes.c_int, [_P, _P, _P, _I32, _F64, _P, _I32, _P, _P, _P]),
    "orc_combine": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _P]),
    "orc_decode_cache": (ctypes.c_int, [_I32, _I32, _I32, _I32, _I32, _I64, _I32, _P, _P, _P, _P, _U64, _P, _P,
                                        _F64, _P, _I32]),
    "orc_hardware_threads": (_I32, []),
}

for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args

TYPES = {"f16": 0, "q8_0": 1, "q4_0": 2, "turbo3": 3, "turbo2": 4, "turbo4": 5, "q5_0": 6, "turbo3_qjl": 7}


def ptr(a):
    """Address of a C-contiguous numpy array (None -> NULL)."""
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def arr(x, dtype):
    """x as a C-contiguous array of dtype (a copy only when needed)."""
    return np.ascontiguousarray(np.asarray(x), dtype=dtype)


def f16_bits(x):
    """A float16 array's IEEE binary16 bit patterns, as contiguous uint16."""
    x = np.asarray(x)
    if x.dtype != np.float16:
        raise TypeError("oracle quantizers take float16 input")
    return np.ascontiguousarray(x).view(np.uint16)


def check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle: {what} rejected its arguments")
