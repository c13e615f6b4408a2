"""Pins of the turbo3_qjl oracle (oracle/qjl.py) against what the QJL
construction and plain algebra fix: unbiased inner products over the draw of
the projection, the QJL variance bound, the residual's norm and signs computed
in the original domain, the 2-bit stage equal to the turbo2 row, the case of
no residual, and hand-packed bytes."""

import math

import numpy as np
import pytest

from oracle import qjl, turbo, turbo3


def _x(seed, n, d):
    return np.random.default_rng(seed).standard_normal((n, d)).astype(np.float16)


def _proj(seed, d):
    return np.random.default_rng(seed).standard_normal((d, d)).astype(np.float32)


def test_two_bit_stage_is_the_turbo2_row():
    x = _x(1, 30, 64)
    p = _proj(2, 64)
    norm_h, gamma_h, idx, z = qjl.quantize_parts(x, 99, p)
    n2, i2 = turbo.quantize_indices(x, 99, 2)
    np.testing.assert_array_equal(idx, i2)
    np.testing.assert_array_equal(norm_h.view(np.uint16), n2.view(np.uint16))
    scales, codes = qjl.quantize(x, 99, p)
    np.testing.assert_array_equal(codes[:, :16], turbo.quantize(x, 99, 2)[1])
    assert codes.shape == (30, qjl.code_bytes(64)) == (30, 24)


def test_residual_norm_in_the_original_domain():
    """gamma = |x - x_hat_mse| with the fp32 norm, computed from x directly
    (fp64 Sylvester matrix), to fp16 rounding."""
    d = 128
    x = _x(3, 40, d)
    seed = 1234
    norm, idx, _ = qjl.residual_f32(x, seed)
    _, gamma_h, _, _ = qjl.quantize_parts(x, seed, _proj(4, d))
    levels, _ = turbo.lloyd_max_gaussian(4)
    h = turbo3.sylvester(d).astype(np.float64)
    s = turbo3.signs(seed, d).astype(np.float64)
    xm = (norm.astype(np.float64)[:, None] / d) * s * (levels[idx] @ h.T)
    r = np.linalg.norm(x.astype(np.float64) - xm, axis=1)
    np.testing.assert_allclose(gamma_h.astype(np.float64), r, rtol=2.0 ** -10 + 1e-5)
    # the 2-bit quantizer leaves about its distortion (0.1175) of |x|^2
    rel = (r / np.linalg.norm(x.astype(np.float64), axis=1)) ** 2
    assert 0.09 < rel.mean() < 0.15


def test_signs_are_those_of_the_original_domain_projection():
    """z_i = [ (S r)_i < 0 ] with S = P H_un D / sqrt(d) and r = x - x_hat_mse,
    both formed in fp64 from x; checked where |(S r)_i| clears the fp32 noise."""
    d = 64
    seed = 77
    x = _x(5, 50, d)
    p = _proj(6, d)
    norm, idx, _ = qjl.residual_f32(x, seed)
    _, _, _, z = qjl.quantize_parts(x, seed, p)
    levels, _ = turbo.lloyd_max_gaussian(4)
    h = turbo3.sylvester(d).astype(np.float64)
    s = turbo3.signs(seed, d).astype(np.float64)
    r = x.astype(np.float64) - (norm.astype(np.float64)[:, None] / d) * s * (levels[idx] @ h.T)
    S = qjl.projection_matrix(seed, p, d)
    u = r @ S.T
    clear = np.abs(u) > 1e-3 * np.linalg.norm(S, axis=1)[None, :] * np.linalg.norm(r, axis=1)[:, None]
    assert clear.mean() > 0.95
    np.testing.assert_array_equal(z[clear], (u[clear] < 0).astype(np.uint8))
    # S is P composed with an orthogonal matrix: S S^T = P P^T
    np.testing.assert_allclose(S @ S.T, p.astype(np.float64) @ p.astype(np.float64).T, atol=1e-9)


def test_projection_sum_is_row_times_residual():
    """u = P e within the binary32 bound of a d-term sum (a transposed P or a
    dropped term is far off)."""
    d = 32
    x = _x(7, 20, d)
    p = _proj(8, d)
    _, _, e = qjl.residual_f32(x, 5)
    u = qjl.project_f32(p, e).astype(np.float64)
    exact = e.astype(np.float64) @ p.astype(np.float64).T
    bound = d * 2.0 ** -24 * (np.abs(e.astype(np.float64)) @ np.abs(p.astype(np.float64)).T)
    assert np.all(np.abs(u - exact) <= bound + 1e-30)
    assert not np.allclose(exact, e.astype(np.float64) @ p.astype(np.float64), atol=1e-3)


def _estimates(x, q, seed, draws, d):
    """<q, x_hat> for `draws` independent projections, and the 2-bit part."""
    out = []
    for k in range(draws):
        scales, codes = qjl.quantize(x, seed, _proj(1000 + k, d))
        out.append(float(qjl.dequantize(scales, codes, seed, _proj(1000 + k, d), d)[0] @ q))
    sc = qjl.quantize(x, seed, _proj(0, d))[0]
    mse = float(turbo.dequantize(sc[:, 0], turbo.quantize(x, seed, 2)[1], seed, d, 2)[0] @ q)
    return np.array(out), mse


@pytest.mark.parametrize("along_residual", [True, False])
def test_inner_products_unbiased_over_the_projection(along_residual):
    """E_S <q, x_hat> = <q, x> (QJL is unbiased for <q, r>), and the spread is
    within the QJL bound Var <= pi/(2d) |q|^2 |r|^2.  With q along the residual
    the correction is the whole residual norm, so a wrong constant (sqrt(2/pi)
    for sqrt(pi/2)), a lost norm or a wrong sign fails by many standard errors."""
    d, seed, draws = 32, 21, 1500
    x = _x(11, 1, d)
    x64 = x.astype(np.float64)[0]
    norm, idx, _ = qjl.residual_f32(x, seed)
    levels, _ = turbo.lloyd_max_gaussian(4)
    h = turbo3.sylvester(d).astype(np.float64)
    s = turbo3.signs(seed, d).astype(np.float64)
    r = x64 - (float(norm[0]) / d) * s * (levels[idx[0]] @ h.T)
    q = r / np.linalg.norm(r) if along_residual else np.random.default_rng(12).standard_normal(d)
    est, mse = _estimates(x, q, seed, draws, d)
    truth = float(x64 @ q)
    se = est.std(ddof=1) / math.sqrt(draws)
    # fp16 norms move the mean by ~1e-3 |q||r|, far below 5 standard errors
    assert abs(est.mean() - truth) < 5 * se + 2e-3 * np.linalg.norm(q) * np.linalg.norm(r)
    bound = math.pi / (2 * d) * float(q @ q) * float(r @ r)
    assert est.var(ddof=1) <= 1.15 * bound
    if along_residual:   # the 2-bit part alone misses <q, r> = |r| entirely
        assert abs(mse - truth) > 20 * se


def test_no_residual_reduces_to_turbo2():
    """With gamma = 0 the row decodes exactly as the turbo2 row of the same
    codes; a zero row stores norm 0 and gamma 0 and decodes to 0."""
    d, seed = 64, 3
    x = _x(13, 8, d)
    p = _proj(14, d)
    scales, codes = qjl.quantize(x, seed, p)
    sc0 = scales.copy()
    sc0[:, 1] = 0
    np.testing.assert_array_equal(qjl.dequantize(sc0, codes, seed, p, d),
                                  turbo.dequantize(scales[:, 0], codes[:, :d // 4], seed, d, 2))
    zs, zc = qjl.quantize(np.zeros((1, d), np.float16), seed, p)
    assert zs.tolist() == [[0.0, 0.0]]
    assert not np.any(qjl.dequantize(zs, zc, seed, p, d))


def test_bytes_by_hand():
    """d = 32: idx field 8 bytes (code i in bits 2i, 2i+1), z field 4 bytes
    (bit i), z after idx."""
    d = 32
    idx = np.array([[3, 0, 1, 2] * 8], np.uint8)
    z = np.array([[1, 0, 0, 0, 0, 0, 0, 1] + [0] * 8 + [1] * 8 + [0, 1] * 4], np.uint8)
    row = np.concatenate([turbo.pack(idx, 2), turbo.pack(z, 1)], axis=1)
    assert row.tolist() == [[0b10010011] * 8 + [0b10000001, 0x00, 0xFF, 0b10101010]]
    got_idx, got_z = qjl.split_codes(row, d)
    np.testing.assert_array_equal(got_idx, idx)
    np.testing.assert_array_equal(got_z, z)
