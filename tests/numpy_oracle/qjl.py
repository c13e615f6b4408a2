"""Oracle for "turbo3_qjl" key rows: a 2-bit turbo row plus a 1-bit Quantized
Johnson-Lindenstrauss (QJL) code of its residual, 3 bits per value in all.

Test infrastructure only (see ``oracle/__init__.py``).

The TurboQuant page ("Benchmark TurboQuant en Apple Silicon", section
"¿Qué es TurboQuant?") builds its 3-bit cache from three parts: a random
Walsh-Hadamard rotation, an optimal scalar quantizer, and QJL, whose job is to
keep inner products.  It defines none of them.  The reading taken here follows
the published constructions those names refer to (Zandieh et al., "QJL: 1-Bit
Quantized JL Transform for KV Cache Quantization", 2024; "TurboQuant", 2025):
the scalar quantizer takes b - 1 = 2 bits (the turbo2 row), and QJL codes the
residual r = x - x_hat_mse in one bit per coordinate, the signs of a d x d
projection S with i.i.d. N(0,1) entries, together with the residual's norm.
The inner-product estimate sqrt(pi/2)/d * |r| * <S q, sign(S r)> is then
unbiased for <q, r> over the draw of S, so <q, x_hat> is unbiased for <q, x>.

Steps for one row x (float16 [d], d a power of two) in binary32, one rounding
per operation:
  1-6. the turbo2 row of ``oracle/turbo.py``: signs s, norm by the strided
       tree, unnormalised FWHT w, g = fl(w * fl(1/norm)),
       idx_i = #{k : g_i > tau_k} over the 3 midpoints of the 4-level
       Lloyd-Max quantizer of N(0,1);
  7.   residual in the rotated unit domain: e_i = fl(g_i - c32[idx_i]), c32 the
       binary32 levels;
  8.   u_i = sum_j P[i][j] * e_j, summed left to right (j = 0 .. d-1), and
       z_i = 1 where u_i < 0 (P is the caller's float32 [d][d] projection);
  9.   eps = sqrt(tree sum of fl(e_i^2)) and
       gamma = fp16(min(fl(fl(norm * eps) * fl32(1/sqrt(d))), 65504));
  10.  the code row holds idx at 2 bits each (d/4 bytes, as turbo2), then z at
       1 bit each (d/8 bytes, bit i of the field little-endian); the scale row
       holds (fp16(min(norm, 65504)), gamma).
Why the rotated domain: x = (norm/d) D H_un g, so the residual of the 2-bit
stage is r = (norm/d) D H_un e with |r| = norm |e| / sqrt(d), and
sign(P e) = sign(S r) for S = P H_un D / sqrt(d).  H_un D / sqrt(d) is
orthogonal, so S has i.i.d. N(0,1) entries exactly when P has: coding e with P
is QJL of r with the matrix S.
Dequantization (float64):
  x_hat = (norm_h/d) D H_un c[idx] + sqrt(pi/2)/d * gamma_h * S^T z~,
  z~_i = 1 - 2 z_i,  S^T = D H_un P^T / sqrt(d).
"""

import math

import numpy as np

from . import turbo, turbo3

F32 = np.float32
MSE_BITS = 2


def code_bytes(d):
    return MSE_BITS * d // 8 + d // 8


def _rows(x_f16):
    x16 = np.asarray(x_f16)
    if x16.dtype != np.float16:
        raise TypeError("oracle quantizers take float16 input")
    d = x16.shape[-1]
    return x16.reshape(-1, d), x16.shape[:-1], d


def residual_f32(x_f16, seed):
    """(norm float32 [n], idx uint8 [n, d], e float32 [n, d]) of rows [n, d]:
    steps 1-7 (the fp32 norm, before its fp16 rounding)."""
    x, _, d = _rows(x_f16)
    v = x.astype(np.float32) * turbo3.signs(seed, d)
    norm = np.sqrt(turbo3.tree_sum_f32(v * v))
    w = turbo3.fwht_f32(v)
    r = np.zeros_like(norm)
    nz = norm > 0
    r[nz] = F32(1.0) / norm[nz]
    g = w * r[:, None]
    levels, tau = turbo.codebook_f32(MSE_BITS)
    idx = np.zeros(g.shape, dtype=np.uint8)
    for t in tau:
        idx += (g > t).astype(np.uint8)
    e = g - levels[idx]
    return norm, idx, e


def project_f32(proj, e):
    """u[n, i] = sum_j proj[i][j] * e[n, j] in binary32, left to right."""
    p = np.asarray(proj, dtype=np.float32)
    u = np.zeros(e.shape, dtype=np.float32)
    for j in range(e.shape[-1]):
        u = u + p[None, :, j] * e[:, j:j + 1]
    return u


def quantize_parts(x_f16, seed, proj):
    """(norm_h, gamma_h float16 [...], idx uint8 [..., d], z uint8 [..., d])."""
    _, lead, d = _rows(x_f16)
    norm, idx, e = residual_f32(x_f16, seed)
    z = (project_f32(proj, e) < 0).astype(np.uint8)
    eps = np.sqrt(turbo3.tree_sum_f32(e * e))
    kappa = F32(1.0 / math.sqrt(d))
    gamma = np.minimum((norm * eps) * kappa, F32(65504.0)).astype(np.float16)
    norm_h = np.minimum(norm, F32(65504.0)).astype(np.float16)
    return norm_h.reshape(lead), gamma.reshape(lead), idx.reshape(*lead, d), z.reshape(*lead, d)


def quantize(x_f16, seed, proj):
    """Rows [..., d] -> (scales float16 [..., 2] = (norm_h, gamma_h),
    codes uint8 [..., 3d/8] = 2-bit idx field, then the 1-bit z field)."""
    norm_h, gamma_h, idx, z = quantize_parts(x_f16, seed, proj)
    codes = np.concatenate([turbo.pack(idx, MSE_BITS), turbo.pack(z, 1)], axis=-1)
    return np.stack([norm_h, gamma_h], axis=-1), codes


def split_codes(codes, d):
    """(idx uint8 [..., d], z uint8 [..., d]) of stored code rows."""
    c = np.asarray(codes, dtype=np.uint8)
    nb = MSE_BITS * d // 8
    return turbo.unpack(c[..., :nb], d, MSE_BITS), turbo.unpack(c[..., nb:], d, 1)


def dequantize(scales, codes, seed, proj, d):
    """x_hat float64 [..., d] of stored rows (scales [..., 2], codes [..., 3d/8])."""
    sc = np.asarray(scales, dtype=np.float16).astype(np.float64)
    idx, z = split_codes(codes, d)
    levels, _ = turbo.lloyd_max_gaussian(1 << MSE_BITS)
    h = turbo3.sylvester(d).astype(np.float64)
    s = turbo3.signs(seed, d).astype(np.float64)
    mse = (sc[..., 0:1] / d) * s * (levels[idx] @ h.T)
    zt = 1.0 - 2.0 * z.astype(np.float64)
    st_z = s * ((zt @ np.asarray(proj, dtype=np.float64)) @ h.T) / math.sqrt(d)   # S^T z~ per row
    return mse + math.sqrt(math.pi / 2) / d * sc[..., 1:2] * st_z


def projection_matrix(seed, proj, d):
    """S = P H_un D / sqrt(d) in float64: the original-domain QJL matrix that
    coding the rotated residual with P amounts to."""
    h = turbo3.sylvester(d).astype(np.float64)
    s = turbo3.signs(seed, d).astype(np.float64)
    return (np.asarray(proj, dtype=np.float64) @ h) * s[None, :] / math.sqrt(d)
