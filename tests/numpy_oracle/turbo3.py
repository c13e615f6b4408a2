"""Oracle for the turbo3 value-cache row: seeded signs, Walsh-Hadamard rotation,
per-vector norm and an 8-level Lloyd-Max scalar code packed at 3 bits.

Test infrastructure only (see ``oracle/__init__.py``).

The TurboQuant page (``Benchmark TurboQuant en Apple Silicon``, section
"¿Qué es TurboQuant?") outlines the method: a random rotation by a
Walsh-Hadamard transform to make the coordinates Gaussian, then an optimal
scalar quantizer, at 3 bits per value ("turbo3"), about 5x smaller than fp16
(section "Resultados" and the q8_0-vs-turbo3 comparison table).  The format
this library implements fixes: a per-vector L2 norm, a +-1 sign vector drawn
from a seed, an orthonormal Hadamard transform of size head_dim, and a fixed
8-level Lloyd-Max codebook for N(0, 1/head_dim), packed at 3 bits.  Everything
finer is a reading, taken here and mirrored by the CUDA side:

  1. signs: splitmix64 (Steele, Lea & Flood 2014; Vigna's reference code)
     seeded with the 64-bit seed; output i (i = 0..d-1, first output is i=0)
     gives s_i = -1 when its top bit is set, else +1;
  2. v = s * x (exact);
  3. n2 = sum of fl(v_i^2) by the strided pairwise tree a[i] += a[i+h] for
     h = d/2, d/4, ..., 1; norm = sqrtf(n2) (IEEE, correctly rounded);
  4. w = unnormalised fast Walsh-Hadamard transform of v in binary32, stages
     h = 1, 2, 4, ..., d/2 in that order, butterfly (a, b) -> (a+b, a-b);
  5. r = 1/norm (0 when norm == 0); g_i = fl(w_i * r).  Since H = H_un/sqrt(d),
     g = sqrt(d) * H D x/|x|, whose coordinates are ~N(0,1); comparing g with
     the unit-variance Lloyd-Max thresholds is the N(0,1/d) codebook applied to
     H D x/|x|, without an inexact multiply by 1/sqrt(d);
  6. idx_i = #{k in 0..6 : g_i > tau_k}, tau_k = binary32 rounding of the
     midpoint of unit levels c_k, c_k+1;
  7. idx_i occupies bits 3i..3i+2 of a little-endian bit stream (3d/8 bytes);
  8. the stored norm is fp16(min(norm, 65504)).
Dequantization: x_hat = (norm_h / d) * D * H_un * c[idx]  (float64), which is
|x| * D H^T (c/sqrt(d)) with the stored norm.
"""

import math

import numpy as np

F32 = np.float32
MASK64 = (1 << 64) - 1
SPLITMIX_GAMMA = 0x9E3779B97F4A7C15


# ------------------------------------------------------------ sign vector

def splitmix64(seed, n):
    """First n outputs of splitmix64 started at state ``seed``.

    State advances by the golden-ratio increment before each output; the
    output is the state passed through the two xor-shift-multiply rounds and
    a final xor-shift.
    """
    out = []
    s = seed & MASK64
    for _ in range(n):
        s = (s + SPLITMIX_GAMMA) & MASK64
        z = s
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        out.append(z ^ (z >> 31))
    return out


def signs(seed, d):
    """The +-1 vector D (float32 [d]) for ``seed``."""
    return np.array([-1.0 if (z >> 63) else 1.0 for z in splitmix64(seed, d)],
                    dtype=np.float32)


# ---------------------------------------------------------------- Hadamard

def sylvester(d):
    """Unnormalised Sylvester-Hadamard matrix of order d (float64), built by
    the recursion H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]."""
    if d < 1 or d & (d - 1):
        raise ValueError("order must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def fwht_f32(v):
    """Unnormalised fast Walsh-Hadamard transform over the last axis, in
    binary32, stages h = 1, 2, ..., d/2; each pairs index i (bit h clear) with
    i + h and replaces (a, b) by (fl(a + b), fl(a - b))."""
    w = np.array(v, dtype=np.float32, copy=True)
    d = w.shape[-1]
    lead = w.shape[:-1]
    h = 1
    while h < d:
        blk = w.reshape(*lead, d // (2 * h), 2, h)
        a = blk[..., 0, :]
        b = blk[..., 1, :]
        w = np.stack([a + b, a - b], axis=-2).reshape(*lead, d)
        h *= 2
    return w


def tree_sum_f32(a):
    """Strided pairwise sum over the last axis in binary32:
    a[i] <- a[i] + a[i+h] for h = d/2, d/4, ..., 1; returns a[0]."""
    a = np.array(a, dtype=np.float32, copy=True)
    h = a.shape[-1] // 2
    while h >= 1:
        a[..., :h] = a[..., :h] + a[..., h:2 * h]
        h //= 2
    return a[..., 0]


# --------------------------------------------------------------- codebook

def _phi(x):
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _upper_tail(x):
    """P(Z > x) for Z ~ N(0,1), via erfc (no cancellation)."""
    return 0.5 * math.erfc(x / math.sqrt(2.0))


def lloyd_max_gaussian8(tol=1e-15, max_iter=200000):
    """8-level Lloyd-Max quantizer for N(0,1), in float64.

    Lloyd's iteration: thresholds are midpoints of adjacent levels, levels are
    the conditional means of N(0,1) on their cells,
    E[Z | a < Z < b] = (phi(a) - phi(b)) / (P(Z > a) - P(Z > b)).
    The quantizer is symmetric, so the positive half is iterated with the
    middle threshold fixed at 0 and mirrored exactly.
    Returns ``(levels[8], thresholds[7])`` ascending.
    """
    pos = [0.25, 0.75, 1.35, 2.15]              # starting guess, positive levels
    for _ in range(max_iter):
        t = [0.0] + [(pos[k] + pos[k + 1]) / 2.0 for k in range(3)] + [math.inf]
        new = []
        for k in range(4):
            a, b = t[k], t[k + 1]
            pb = _phi(b) if b != math.inf else 0.0
            qb = _upper_tail(b) if b != math.inf else 0.0
            new.append((_phi(a) - pb) / (_upper_tail(a) - qb))
        delta = max(abs(x - y) for x, y in zip(new, pos))
        pos = new
        if delta < tol:
            break
    else:
        raise RuntimeError("Lloyd iteration did not converge")
    levels = [-p for p in reversed(pos)] + pos
    thresholds = [(levels[k] + levels[k + 1]) / 2.0 for k in range(7)]
    return np.array(levels), np.array(thresholds)


def codebook_f32():
    """(levels, thresholds) rounded to binary32, the decision values both
    sides compare against."""
    lv, th = lloyd_max_gaussian8()
    return lv.astype(np.float32), th.astype(np.float32)


# --------------------------------------------------------------- rows

ROW_LEVELS = 8


def code_bytes(d):
    return 3 * d // 8


def quantize_turbo3(x_f16, seed):
    """Quantize rows (float16 ``[..., d]``, d a power of two >= 8) to turbo3.

    Returns ``(norm_h, codes)``: float16 ``[...]`` and packed uint8
    ``[..., 3d/8]``.  Also usable through ``quantize_turbo3_indices``.
    """
    norm_h, idx = quantize_turbo3_indices(x_f16, seed)
    return norm_h, pack3(idx)


def quantize_turbo3_indices(x_f16, seed):
    x16 = np.asarray(x_f16)
    if x16.dtype != np.float16:
        raise TypeError("oracle quantizers take float16 input")
    d = x16.shape[-1]
    lead = x16.shape[:-1]
    x = x16.astype(np.float32).reshape(-1, d)
    s = signs(seed, d)
    v = x * s                                       # exact sign flips
    n2 = tree_sum_f32(v * v)                        # fl(v_i^2), strided tree
    norm = np.sqrt(n2)                              # binary32 sqrt, correctly rounded
    w = fwht_f32(v)
    r = np.zeros_like(norm)
    nz = norm > 0
    r[nz] = F32(1.0) / norm[nz]
    g = w * r[:, None]                              # binary32 multiply
    _, tau = codebook_f32()
    idx = np.zeros(g.shape, dtype=np.uint8)
    for k in range(7):
        idx += (g > tau[k]).astype(np.uint8)
    norm_h = np.minimum(norm, F32(65504.0)).astype(np.float16)
    return norm_h.reshape(lead), idx.reshape(*lead, d)


def pack3(idx):
    """3-bit little-endian bit stream: idx_i in bits 3i..3i+2."""
    idx = np.asarray(idx, dtype=np.uint8)
    d = idx.shape[-1]
    lead = idx.shape[:-1]
    flat = idx.reshape(-1, d).astype(np.uint32)
    out = np.zeros((flat.shape[0], 3 * d // 8), dtype=np.uint8)
    for i in range(d):
        for b in range(3):
            bit = (flat[:, i] >> b) & 1
            pos = 3 * i + b
            out[:, pos // 8] |= (bit << (pos % 8)).astype(np.uint8)
    return out.reshape(*lead, 3 * d // 8)


def unpack3(codes, d):
    c = np.asarray(codes, dtype=np.uint8)
    lead = c.shape[:-1]
    flat = c.reshape(-1, c.shape[-1])
    idx = np.zeros((flat.shape[0], d), dtype=np.uint8)
    for i in range(d):
        v = np.zeros(flat.shape[0], dtype=np.uint8)
        for b in range(3):
            pos = 3 * i + b
            v |= ((flat[:, pos // 8] >> (pos % 8)) & 1) << b
        idx[:, i] = v
    return idx.reshape(*lead, d)


def dequantize_turbo3(norm_h, codes, seed, d):
    """x_hat = (norm_h / d) * D * H_un * c[idx], float64 ``[..., d]``."""
    levels, _ = lloyd_max_gaussian8()
    idx = unpack3(codes, d)
    y = levels[idx]                                 # unit-variance levels
    h = sylvester(d)
    rot = y @ h.T                                   # H_un c  (H_un symmetric)
    s = signs(seed, d).astype(np.float64)
    n = np.asarray(norm_h, dtype=np.float16).astype(np.float64)
    return (n[..., None] / d) * s * rot
