"""Oracle for the turbo value-cache rows at b = 2, 3 or 4 bits per value
("turbo2", "turbo3", "turbo4").

Test infrastructure only (see ``oracle/__init__.py``).

The TurboQuant page ("Benchmark TurboQuant en Apple Silicon", section
"¿Qué es TurboQuant?") describes a random Walsh-Hadamard rotation followed by
an optimal scalar quantizer; its FAQ ("¿Qué formato TurboQuant debería usar?")
adds that values take 2 to 3 bits without harming attention.  The widths other
than 3 are therefore the same construction with another level count, which is
the reading taken here: steps 1-5 of ``oracle/turbo3.py`` unchanged (signs,
norm by the strided tree, unnormalised FWHT, g = fl(w * fl(1/norm))), then

  6'. idx_i = #{k : g_i > tau_k} over the 2^b - 1 binary32 midpoints tau_k of
      the 2^b-level Lloyd-Max quantizer of N(0,1) (unit levels c_k);
  7'. idx_i occupies bits b*i .. b*i+b-1 of a little-endian bit stream
      (b*d/8 bytes);
  8.  the stored norm is fp16(min(norm, 65504)).
Dequantization: x_hat = (norm_h / d) * D * H_un * c[idx]  (float64).
"""

import math

import numpy as np

from . import turbo3

F32 = np.float32
BITS = {"turbo2": 2, "turbo3": 3, "turbo4": 4}


def lloyd_max_gaussian(n_levels, tol=1e-15, max_iter=400000):
    """n-level Lloyd-Max quantizer for N(0,1) (n even), float64, by Lloyd's
    iteration on the positive half (middle threshold 0, mirrored exactly):
    thresholds are midpoints of adjacent levels and each level is the mean of
    N(0,1) on its cell, (phi(a) - phi(b)) / (P(Z > a) - P(Z > b)).
    Returns ``(levels[n], thresholds[n-1])`` ascending."""
    if n_levels < 2 or n_levels % 2:
        raise ValueError("an even level count is needed")
    m = n_levels // 2
    pos = [(k + 0.5) * 3.0 / m for k in range(m)]   # spread start over [0, 3]
    for _ in range(max_iter):
        t = [0.0] + [(pos[k] + pos[k + 1]) / 2.0 for k in range(m - 1)] + [math.inf]
        new = []
        for k in range(m):
            a, b = t[k], t[k + 1]
            pb = turbo3._phi(b) if b != math.inf else 0.0
            qb = turbo3._upper_tail(b) if b != math.inf else 0.0
            new.append((turbo3._phi(a) - pb) / (turbo3._upper_tail(a) - qb))
        delta = max(abs(x - y) for x, y in zip(new, pos))
        pos = new
        if delta < tol:
            break
    else:
        raise RuntimeError("Lloyd iteration did not converge")
    levels = [-p for p in reversed(pos)] + pos
    thresholds = [(levels[k] + levels[k + 1]) / 2.0 for k in range(n_levels - 1)]
    return np.array(levels), np.array(thresholds)


def codebook_f32(bits):
    """(levels, thresholds) of the 2^bits-level quantizer rounded to binary32."""
    lv, th = lloyd_max_gaussian(1 << bits)
    return lv.astype(np.float32), th.astype(np.float32)


def code_bytes(bits, d):
    return bits * d // 8


def quantize_indices(x_f16, seed, bits):
    """(norm_h float16 [...], idx uint8 [..., d]) of rows x_f16 [..., d]."""
    x16 = np.asarray(x_f16)
    if x16.dtype != np.float16:
        raise TypeError("oracle quantizers take float16 input")
    d = x16.shape[-1]
    lead = x16.shape[:-1]
    x = x16.astype(np.float32).reshape(-1, d)
    v = x * turbo3.signs(seed, d)                   # exact sign flips
    norm = np.sqrt(turbo3.tree_sum_f32(v * v))      # binary32 sqrt of the tree sum
    w = turbo3.fwht_f32(v)
    r = np.zeros_like(norm)
    nz = norm > 0
    r[nz] = F32(1.0) / norm[nz]
    g = w * r[:, None]
    _, tau = codebook_f32(bits)
    idx = np.zeros(g.shape, dtype=np.uint8)
    for t in tau:
        idx += (g > t).astype(np.uint8)
    norm_h = np.minimum(norm, F32(65504.0)).astype(np.float16)
    return norm_h.reshape(lead), idx.reshape(*lead, d)


def pack(idx, bits):
    """b-bit little-endian bit stream: idx_i in bits b*i .. b*i+b-1."""
    idx = np.asarray(idx, dtype=np.uint8)
    d = idx.shape[-1]
    lead = idx.shape[:-1]
    flat = idx.reshape(-1, d).astype(np.uint32)
    out = np.zeros((flat.shape[0], bits * d // 8), dtype=np.uint8)
    for i in range(d):
        for j in range(bits):
            pos = bits * i + j
            out[:, pos // 8] |= (((flat[:, i] >> j) & 1) << (pos % 8)).astype(np.uint8)
    return out.reshape(*lead, bits * d // 8)


def unpack(codes, d, bits):
    c = np.asarray(codes, dtype=np.uint8)
    lead = c.shape[:-1]
    flat = c.reshape(-1, c.shape[-1])
    idx = np.zeros((flat.shape[0], d), dtype=np.uint8)
    for i in range(d):
        v = np.zeros(flat.shape[0], dtype=np.uint8)
        for j in range(bits):
            pos = bits * i + j
            v |= ((flat[:, pos // 8] >> (pos % 8)) & 1) << j
        idx[:, i] = v
    return idx.reshape(*lead, d)


def quantize(x_f16, seed, bits):
    """Rows [..., d] -> (norm_h float16 [...], packed codes uint8 [..., b*d/8])."""
    norm_h, idx = quantize_indices(x_f16, seed, bits)
    return norm_h, pack(idx, bits)


def dequantize(norm_h, codes, seed, d, bits):
    """x_hat = (norm_h / d) * D * H_un * c[idx], float64 [..., d]."""
    levels, _ = lloyd_max_gaussian(1 << bits)
    y = levels[unpack(codes, d, bits)]
    rot = y @ turbo3.sylvester(d).T
    s = turbo3.signs(seed, d).astype(np.float64)
    n = np.asarray(norm_h, dtype=np.float16).astype(np.float64)
    return (n[..., None] / d) * s * rot
