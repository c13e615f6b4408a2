"""Oracle for the 32-element block cache formats q8_0, q4_0 and q5_0, and the f16 row.

Test infrastructure only (see ``oracle/__init__.py``).

The pages name these cache types and their nominal cost per element --
``llama.cpp für Geschwindigkeit und Speicher optimieren``, section
"KV-Cache-Präzision" (table: f16 2 bytes, q8_0 1 byte, q4_0 0.5 bytes) -- and
the KVSplit page ("Vergleich der Speicherersparnis") and the llama.cpp issue
"Eval bug: Metal fails mixed quantized KV ..." ("Relevant output") print cache
sizes that only a 34-byte q8_0 block and an 18-byte q4_0 block per 32 elements
reproduce.  The arithmetic inside a block is the format definition this
library implements; the pages print none of it:

  q8_0: amax = max |x_j|; d = amax / 127; q_j = round-half-away(x_j / d);
        store d as fp16 and q_j as int8.
  q4_0: m = the signed x_j of largest magnitude; d = m / -8;
        q_j = min(15, trunc(x_j * (1/d) + 8.5)); element j goes to the low
        nibble of byte j and element j+16 to its high nibble; store d as fp16.
  q5_0: q4_0 widened by one bit: d = m / -16; q_j = min(31, trunc(x_j * (1/d)
        + 16.5)); the low four bits of q_j are packed as q4_0's nibbles and bit 4
        of q_j is bit j of a little-endian 32-bit word qh; store d as fp16.  (A
        comment in the llama.cpp issue reports q5_0/q5_0 caches as a usable
        middle ground between q8_0 and q4_0; no page prints q5_0's arithmetic,
        so this widening of q4_0 is a reading.)

Readings taken where the definition is silent:
  * the fp32 d, not its fp16 image, is used to compute q_j;
  * q8_0 divides x_j by d (an IEEE divide per element); q4_0 multiplies by
    the fp32 reciprocal 1/d, then adds 8.5 in a second rounding (no FMA);
  * d == 0 gives q_j = 0 (q8_0) and nibble 8 (q4_0);
  * q4_0 ties in |x_j| (also +a against -a) go to the lowest index j.

Every quantizer takes fp16 input (numpy float16, last axis a multiple of 32)
and works on its exact float32 widening, one IEEE rounding per operation.
"""

import numpy as np

QK = 32  # elements per block

F32 = np.float32


def _blocks_f32(x_f16):
    x = np.asarray(x_f16)
    if x.dtype != np.float16:
        raise TypeError("oracle quantizers take float16 input")
    if x.shape[-1] % QK:
        raise ValueError("last axis must be a multiple of 32")
    return x.astype(np.float32).reshape(-1, QK)


def round_half_away(r):
    """C ``roundf``: nearest integer, halfway cases away from zero.

    Evaluated in float64, where |r| + 0.5 is exact for every float32 |r| < 2^29
    (no double rounding), so the result is the exact rounding of the float32
    value r.
    """
    r64 = np.asarray(r, dtype=np.float64)
    return np.sign(r64) * np.floor(np.abs(r64) + 0.5)


# --------------------------------------------------------------------- q8_0

def quantize_q8_0(x_f16):
    """Quantize rows to q8_0.

    Returns ``(d, qs)``: ``d`` float16 of shape ``[..., n/32]`` (the stored
    scale) and ``qs`` int8 of shape ``[..., n]``.
    """
    lead = np.asarray(x_f16).shape[:-1]
    n = np.asarray(x_f16).shape[-1]
    x = _blocks_f32(x_f16)
    amax = np.max(np.abs(x), axis=1)               # exact
    d = amax / F32(127.0)                          # one IEEE binary32 divide
    q = np.zeros(x.shape, dtype=np.int8)
    nz = d != 0
    r = x[nz] / d[nz, None]                        # IEEE binary32 divide per element
    q[nz] = round_half_away(r).astype(np.int8)     # |q| <= 127 (see test)
    return d.astype(np.float16).reshape(*lead, n // QK), q.reshape(*lead, n)


def dequantize_q8_0(d_f16, qs):
    """x_hat_j = double(d_h) * q_j, in float64."""
    d = np.asarray(d_f16, dtype=np.float16).astype(np.float64)
    q = np.asarray(qs, dtype=np.int8).astype(np.float64)
    n = q.shape[-1]
    return (q.reshape(*q.shape[:-1], n // QK, QK) * d[..., None]).reshape(q.shape)


# --------------------------------------------------------------------- q4_0

def quantize_q4_0_codes(x_f16):
    """Quantize rows to q4_0; returns ``(d, codes)`` before nibble packing.

    ``d`` float16 ``[..., n/32]``; ``codes`` uint8 in 0..15, ``[..., n]``.
    """
    lead = np.asarray(x_f16).shape[:-1]
    n = np.asarray(x_f16).shape[-1]
    x = _blocks_f32(x_f16)
    j = np.argmax(np.abs(x), axis=1)               # first (lowest) index on ties
    m = x[np.arange(x.shape[0]), j]                # signed value of largest magnitude
    d = m / F32(-8.0)
    inv = np.zeros_like(d)
    nz = d != 0
    inv[nz] = F32(1.0) / d[nz]                     # IEEE binary32 reciprocal
    t = (x * inv[:, None]) + F32(8.5)              # two binary32 roundings
    q = np.minimum(15, t.astype(np.int32))         # int conversion truncates; t >= 0.5
    return (d.astype(np.float16).reshape(*lead, n // QK),
            q.astype(np.uint8).reshape(*lead, n))


def pack_q4_0(codes):
    """Element j of a block -> low nibble of byte j, element j+16 -> high nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    n = c.shape[-1]
    b = c.reshape(*c.shape[:-1], n // QK, QK)
    packed = b[..., :16] | (b[..., 16:] << 4)
    return packed.reshape(*c.shape[:-1], n // 2).astype(np.uint8)


def unpack_q4_0(qs):
    p = np.asarray(qs, dtype=np.uint8)
    nb = p.shape[-1] // 16
    b = p.reshape(*p.shape[:-1], nb, 16)
    codes = np.concatenate([b & 0x0F, b >> 4], axis=-1)
    return codes.reshape(*p.shape[:-1], nb * QK)


def quantize_q4_0(x_f16):
    """Quantize rows to q4_0; returns ``(d, qs)`` with ``qs`` packed uint8 ``[..., n/2]``."""
    d, codes = quantize_q4_0_codes(x_f16)
    return d, pack_q4_0(codes)


def dequantize_q4_0(d_f16, qs):
    """x_hat_j = double(d_h) * (q_j - 8), in float64."""
    codes = unpack_q4_0(qs).astype(np.float64) - 8.0
    d = np.asarray(d_f16, dtype=np.float16).astype(np.float64)
    n = codes.shape[-1]
    return (codes.reshape(*codes.shape[:-1], n // QK, QK) * d[..., None]).reshape(codes.shape)


def quantize_q5_0_codes(x_f16):
    """Quantize rows to q5_0; returns ``(d, codes)``: ``d`` float16 ``[..., n/32]``,
    ``codes`` uint8 in 0..31 ``[..., n]`` (the q4_0 steps with -16, 16.5, 31)."""
    lead = np.asarray(x_f16).shape[:-1]
    n = np.asarray(x_f16).shape[-1]
    x = _blocks_f32(x_f16)
    j = np.argmax(np.abs(x), axis=1)               # first (lowest) index on ties
    m = x[np.arange(x.shape[0]), j]
    d = m / F32(-16.0)
    inv = np.zeros_like(d)
    nz = d != 0
    inv[nz] = F32(1.0) / d[nz]
    t = (x * inv[:, None]) + F32(16.5)             # two binary32 roundings
    q = np.minimum(31, t.astype(np.int32))         # truncation; t >= 0.5
    return (d.astype(np.float16).reshape(*lead, n // QK),
            q.astype(np.uint8).reshape(*lead, n))


def pack_q5_0(codes):
    """(qs, qh): the low four bits as q4_0's nibbles ``[..., n/2]`` and bit 4 of
    element j as bit j of a uint32 per block ``[..., n/32]``."""
    c = np.asarray(codes, dtype=np.uint8)
    n = c.shape[-1]
    qs = pack_q4_0(c & 0x0F)
    b = (c.reshape(*c.shape[:-1], n // QK, QK) >> 4).astype(np.uint64) & 1
    qh = np.sum(b << np.arange(QK, dtype=np.uint64), axis=-1).astype(np.uint32)
    return qs, qh


def unpack_q5_0(qs, qh):
    low = unpack_q4_0(qs)
    h = np.asarray(qh, dtype=np.uint32)
    bits = ((h[..., None] >> np.arange(QK, dtype=np.uint32)) & 1).astype(np.uint8)
    return low | (bits.reshape(low.shape) << 4)


def quantize_q5_0(x_f16):
    """Quantize rows to q5_0; returns ``(d, qs, qh)``."""
    d, codes = quantize_q5_0_codes(x_f16)
    qs, qh = pack_q5_0(codes)
    return d, qs, qh


def dequantize_q5_0(d_f16, qs, qh):
    """x_hat_j = double(d_h) * (q_j - 16), in float64."""
    codes = unpack_q5_0(qs, qh).astype(np.float64) - 16.0
    d = np.asarray(d_f16, dtype=np.float16).astype(np.float64)
    n = codes.shape[-1]
    return (codes.reshape(*codes.shape[:-1], n // QK, QK) * d[..., None]).reshape(codes.shape)


# --------------------------------------------------------------------- f16

def dequantize_f16(x_f16):
    """The f16 cache stores the input unchanged; x_hat = double(x)."""
    return np.asarray(x_f16, dtype=np.float16).astype(np.float64)
