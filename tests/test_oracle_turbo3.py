"""Pins of the turbo3 oracle: generator vectors, Hadamard algebra, the textbook
Gaussian quantizer, closed-form rows and the quantizer's statistical error.  No GPU."""

import math

import numpy as np
import pytest
from scipy import integrate

from oracle import turbo3
from conftest import read_golden


def test_splitmix64_published_vectors():
    for row in read_golden("splitmix64.txt"):
        vals = [int(v) for v in row.split()]
        assert turbo3.splitmix64(vals[0], len(vals) - 1) == vals[1:]


def test_signs_are_top_bits():
    s = turbo3.signs(1234567, 5)
    # top bits of the published outputs for seed 1234567: 0 0 1 0 1
    np.testing.assert_array_equal(s, [1, 1, -1, 1, -1])


@pytest.mark.parametrize("d", [2, 8, 32, 64, 128, 256])
def test_sylvester_orthogonal(d):
    h = turbo3.sylvester(d)
    np.testing.assert_array_equal(h @ h.T, d * np.eye(d))
    np.testing.assert_array_equal(h, h.T)
    i = np.arange(d)
    popc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    np.testing.assert_array_equal(h, (-1.0) ** popc)


@pytest.mark.parametrize("d", [8, 32, 128, 256])
def test_fwht_columns_and_product(d):
    h = turbo3.sylvester(d)
    eye = np.eye(d, dtype=np.float32)
    np.testing.assert_array_equal(turbo3.fwht_f32(eye), h.T.astype(np.float32))
    rng = np.random.default_rng(d)
    v = rng.standard_normal((50, d)).astype(np.float32)
    w = turbo3.fwht_f32(v).astype(np.float64)
    exact = v.astype(np.float64) @ h.T
    scale = np.abs(v.astype(np.float64)) @ np.abs(h.T)
    assert np.all(np.abs(w - exact) <= math.log2(d) * 2.0 ** -23 * scale + 1e-30)
    # orthonormal H = H_un / sqrt(d) preserves the norm
    np.testing.assert_allclose(np.linalg.norm(exact / math.sqrt(d), axis=1),
                               np.linalg.norm(v.astype(np.float64), axis=1), rtol=1e-13)


def test_tree_sum():
    a = np.arange(128, dtype=np.float32)
    assert turbo3.tree_sum_f32(a) == 127 * 128 / 2
    rng = np.random.default_rng(5)
    x = rng.standard_normal((100, 128)).astype(np.float32) ** 2
    np.testing.assert_allclose(turbo3.tree_sum_f32(x), x.astype(np.float64).sum(axis=1), rtol=1e-5)


def test_lloyd_max_matches_max_1960():
    lv, th = turbo3.lloyd_max_gaussian8()
    tab = {r.split()[0]: [float(v) for v in r.split()[1:]] for r in read_golden("max1960_gauss8.txt")}
    np.testing.assert_allclose(lv[4:], tab["levels"], atol=6e-4)
    np.testing.assert_allclose(th[3:], tab["thresholds"], atol=6e-4)
    np.testing.assert_array_equal(lv, -lv[::-1])
    assert th[3] == 0.0

    pdf = lambda z: math.exp(-z * z / 2) / math.sqrt(2 * math.pi)
    edges = [-math.inf] + list(th) + [math.inf]
    mse = 0.0
    for k in range(8):
        a, b = edges[k], edges[k + 1]
        mass = integrate.quad(pdf, a, b, epsabs=1e-15, epsrel=1e-13)[0]
        mean = integrate.quad(lambda z: z * pdf(z), a, b, epsabs=1e-15, epsrel=1e-13)[0] / mass
        assert mean == pytest.approx(lv[k], abs=1e-11)          # centroid condition
        mse += integrate.quad(lambda z: (z - lv[k]) ** 2 * pdf(z), a, b, epsabs=1e-15)[0]
    np.testing.assert_allclose(th, (lv[:-1] + lv[1:]) / 2, atol=0)  # midpoint condition
    assert mse == pytest.approx(tab["mse"][0], abs=5e-5)


def test_pack3_handworked():
    idx = np.array([[1, 2, 3, 4, 5, 6, 7, 0]], np.uint8)
    # sum idx_i << 3i = 0x1F58D1, little-endian bytes d1 58 1f
    np.testing.assert_array_equal(turbo3.pack3(idx)[0], [0xD1, 0x58, 0x1F])
    rng = np.random.default_rng(7)
    r = rng.integers(0, 8, size=(4, 128)).astype(np.uint8)
    np.testing.assert_array_equal(turbo3.unpack3(turbo3.pack3(r), 128), r)


@pytest.mark.parametrize("d", [32, 128, 256])
def test_basis_vector_closed_form(d):
    """x = a e_k: v = a s_k e_k, |x| = |a|, g_i = sign(a) s_k H[i,k] = +-1, so the
    codes are 5 (level +0.756) and 2 (level -0.756), and x_hat = c_5 a e_k."""
    seed = 99
    s = turbo3.signs(seed, d)
    h = turbo3.sylvester(d)
    lv, _ = turbo3.lloyd_max_gaussian8()
    for k, a in [(0, 3.0), (5, -0.5), (d - 1, 1000.0), (d // 2 + 1, -7.25)]:
        x = np.zeros((1, d), np.float16)
        x[0, k] = a
        norm_h, idx = turbo3.quantize_turbo3_indices(x, seed)
        assert float(norm_h[0]) == abs(a)
        sigma = np.sign(a) * s[k] * h[:, k]
        np.testing.assert_array_equal(idx[0], np.where(sigma > 0, 5, 2))
        norm_h, codes = turbo3.quantize_turbo3(x, seed)
        xh = turbo3.dequantize_turbo3(norm_h, codes, seed, d)[0]
        expect = np.zeros(d)
        expect[k] = lv[5] * a
        np.testing.assert_allclose(xh, expect, atol=1e-12 * abs(a))


def test_zero_row():
    x = np.zeros((1, 128), np.float16)
    norm_h, idx = turbo3.quantize_turbo3_indices(x, 1)
    assert float(norm_h[0]) == 0.0
    assert np.all(idx == 3)                     # g = 0 is above tau_0..tau_2 only
    norm_h, codes = turbo3.quantize_turbo3(x, 1)
    np.testing.assert_array_equal(turbo3.dequantize_turbo3(norm_h, codes, 1, 128), 0.0)


def test_norm_saturates():
    x = np.full((1, 128), 60000.0, np.float16)  # |x| = 678822 > fp16 max
    norm_h, _ = turbo3.quantize_turbo3_indices(x, 3)
    assert float(norm_h[0]) == 65504.0


def test_gaussian_round_trip_mse():
    """For x ~ N(0, I), H D x/|x| has ~N(0,1/d) coordinates; the 8-level optimal
    quantizer's relative error is ~0.0345 (its MSE on a unit Gaussian)."""
    d = 128
    rng = np.random.default_rng(11)
    x = rng.standard_normal((10000, d)).astype(np.float16)
    norm_h, codes = turbo3.quantize_turbo3(x, turbo3.splitmix64(0, 1)[0])
    xh = turbo3.dequantize_turbo3(norm_h, codes, turbo3.splitmix64(0, 1)[0], d)
    xd = x.astype(np.float64)
    rel = np.sum((xd - xh) ** 2, axis=1) / np.sum(xd ** 2, axis=1)
    assert 0.032 < rel.mean() < 0.037
    # 3 bits per element + 16-bit norm: 3.125 bits at d = 128, 5.12x under fp16
    assert codes.shape[-1] == 48 and 16 * 128 / (48 * 8 + 16) == pytest.approx(5.12)
