"""Pins of the turbo oracle at 2 and 4 bits (oracle/turbo.py): the codebooks
against closed forms and Max's printed tables, the bit layout against
hand-packed bytes, the 3-bit case against the turbo3 oracle, and the
reconstruction error against the quantizer's distortion."""

import math
import os

import numpy as np
import pytest

from oracle import turbo, turbo3

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "max1960_gauss4_16.txt")


def _printed():
    tab = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        n, what, *vals = line.split()
        tab[(int(n[1:]), what)] = vals
    return tab


def _upper_tail(x):
    """P(Z > x) for Z ~ N(0,1) (math.erfc, no cancellation)."""
    return 0.0 if x == np.inf else 0.5 * math.erfc(x / math.sqrt(2.0))


def _last_digit(text):
    """One unit in the last printed digit (the 1960 table is good to about that)."""
    dec = len(text.split(".")[1]) if "." in text else 0
    return 10.0 ** -dec


def test_two_levels_closed_form():
    """The 2-level optimum for N(0,1) is +-E|Z| = +-sqrt(2/pi), threshold 0."""
    lv, th = turbo.lloyd_max_gaussian(2)
    assert lv == pytest.approx([-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)], abs=1e-12)
    assert th == pytest.approx([0.0], abs=1e-15)


@pytest.mark.parametrize("n", [4, 16])
def test_levels_and_thresholds_match_max_1960(n):
    tab = _printed()
    lv, th = turbo.lloyd_max_gaussian(n)
    pos_lv, pos_th = lv[n // 2:], th[n // 2 - 1:]
    for got, text in zip(pos_lv, tab[(n, "levels")]):
        assert abs(got - float(text)) <= _last_digit(text) + 1e-9, (n, text, got)
    for got, text in zip(pos_th, tab[(n, "thresholds")]):
        assert abs(got - float(text)) <= _last_digit(text) + 1e-9, (n, text, got)
    # symmetric, and the Lloyd conditions: midpoints and centroids
    assert np.allclose(lv, -lv[::-1], atol=0) and np.allclose(th, (lv[:-1] + lv[1:]) / 2)
    # distortion 1 - sum c_k^2 P(cell k) (centroid condition), against the printed value
    edges = np.concatenate([[-np.inf], th, [np.inf]])
    p = [_upper_tail(a) - _upper_tail(b) if a != -np.inf else 1 - _upper_tail(b)
         for a, b in zip(edges[:-1], edges[1:])]
    mse = 1.0 - float(np.sum(lv ** 2 * np.array(p)))
    text = tab[(n, "mse")][0]
    assert abs(mse - float(text)) <= 1e-3 * float(text), (n, mse, text)   # 4 printed digits


def test_three_bits_is_turbo3():
    lv, th = turbo.codebook_f32(3)
    olv, oth = turbo3.codebook_f32()
    np.testing.assert_array_equal(lv, olv)
    np.testing.assert_array_equal(th, oth)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((20, 128)).astype(np.float16)
    n1, c1 = turbo.quantize(x, 77, 3)
    n2, c2 = turbo3.quantize_turbo3(x, 77)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(n1.view(np.uint16), n2.view(np.uint16))


def test_bit_layout_by_hand():
    idx2 = np.array([[1, 2, 3, 0, 3, 3, 0, 1]], np.uint8)
    # b=2: codes 0..3 of byte 0 in bits 0-1, 2-3, 4-5, 6-7
    assert turbo.pack(idx2, 2).tolist() == [[0b00111001, 0b01001111]]
    idx4 = np.array([[0x3, 0xC, 0xF, 0x0]], np.uint8)
    assert turbo.pack(idx4, 4).tolist() == [[0xC3, 0x0F]]
    for bits in (2, 4):
        rng = np.random.default_rng(bits)
        idx = rng.integers(0, 1 << bits, (7, 64)).astype(np.uint8)
        np.testing.assert_array_equal(turbo.unpack(turbo.pack(idx, bits), 64, bits), idx)


@pytest.mark.parametrize("bits,mse", [(2, 0.1175), (4, 0.009497)])
def test_reconstruction_error_is_the_quantizer_distortion(bits, mse):
    """After the rotation the coordinates are near N(0,1), so the mean relative
    squared error of a row is about the quantizer's distortion; a wrong sign,
    transform or codebook index is far off."""
    rng = np.random.default_rng(bits + 10)
    d = 128
    x = rng.standard_normal((400, d)).astype(np.float16)
    norm_h, codes = turbo.quantize(x, 12345, bits)
    xh = turbo.dequantize(norm_h, codes, 12345, d, bits)
    x64 = x.astype(np.float64)
    rel = np.sum((xh - x64) ** 2, axis=1) / np.sum(x64 ** 2, axis=1)
    assert 0.8 * mse < rel.mean() < 1.25 * mse, rel.mean()


def test_codes_follow_the_thresholds():
    """A row whose rotated coordinates sit just above / below each threshold
    gets the counts #{k : g > tau_k}: built by inverting the transform."""
    d = 16
    for bits in (2, 4):
        _, tau = turbo.codebook_f32(bits)
        g = np.concatenate([tau + 0.01, tau - 0.01])[:d]
        g = np.pad(g, (0, d - len(g)), constant_values=0.3).astype(np.float64)
        # x = D H_un^-1 g * |x| / sqrt(d)... choose x so that w / |x| = g: x = s * H_un g / d * c
        h = turbo3.sylvester(d)
        s = turbo3.signs(5, d).astype(np.float64)
        x = (s * (h @ g) / d * 3.0).astype(np.float16)
        _, idx = turbo.quantize_indices(x, 5, bits)
        # recompute g the oracle's way and count
        v = x.astype(np.float32) * turbo3.signs(5, d)
        norm = np.sqrt(turbo3.tree_sum_f32(v * v))
        gg = turbo3.fwht_f32(v) * (np.float32(1.0) / norm)
        expect = np.array([int(np.sum(val > tau)) for val in gg], np.uint8)
        np.testing.assert_array_equal(idx, expect)
        assert idx.max() <= (1 << bits) - 1
