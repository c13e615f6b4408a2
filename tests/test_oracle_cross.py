"""The C++ oracle (oracle/) against the independent numpy restatement of the same
definitions (tests/numpy_oracle/): quantized bytes equal bit for bit, decoded
values and attention equal to binary64 rounding.  No GPU.

Both follow the format definitions step by step in IEEE binary32 with one
rounding per operation; a porting slip in either (a fused multiply-add, a
reordered sum, a wrong stride) shows here as a byte that differs."""

import numpy as np
import pytest

import numpy_oracle as npo
from oracle import attention, blocks, cache_model, qjl, turbo, turbo3


def _rows(seed, n, d, spread=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d))
    if spread:  # block scales from subnormal to large
        x *= np.exp(rng.uniform(-12, 10, size=(n, d // 32 if d >= 32 else 1))).repeat(32 if d >= 32 else d, axis=1)
    x[0, :] = 0.0
    if n > 2:
        x[1, 5] = 60000.0
        x[2, :8] = [0.5, -0.5, 1.5, -1.5, 2.5, 127, -127, 0]
    return np.clip(x, -65504, 65504).astype(np.float16)


def _eq16(a, b):
    np.testing.assert_array_equal(np.asarray(a, np.float16).view(np.uint16), np.asarray(b, np.float16).view(np.uint16))


def test_fp16_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * np.exp(rng.uniform(-20, 12, 20000)),
                        [65504.0, 65519.99, 65520.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 1 + 2.0 ** -11,
                         1 + 3 * 2.0 ** -11, -0.0, 0.0]]).astype(np.float32)
    with np.errstate(over="ignore"):   # 65520 rounds to inf in both
        _eq16(blocks.f32_to_f16(x), x.astype(np.float16))


@pytest.mark.parametrize("d", [32, 128, 256])
def test_block_formats_bit_exact(d):
    x = _rows(d, 600, d)
    for a, b in zip(blocks.quantize_q8_0(x), npo.blocks.quantize_q8_0(x)):
        np.testing.assert_array_equal(np.asarray(a).view(np.uint8), np.asarray(b).view(np.uint8))
    for a, b in zip(blocks.quantize_q4_0(x), npo.blocks.quantize_q4_0(x)):
        np.testing.assert_array_equal(np.asarray(a).view(np.uint8), np.asarray(b).view(np.uint8))
    for a, b in zip(blocks.quantize_q5_0(x), npo.blocks.quantize_q5_0(x)):
        np.testing.assert_array_equal(np.asarray(a).view(np.uint8), np.asarray(b).view(np.uint8))
    d8, q8 = blocks.quantize_q8_0(x)
    np.testing.assert_array_equal(blocks.dequantize_q8_0(d8, q8), npo.blocks.dequantize_q8_0(d8, q8))
    d4, p4 = blocks.quantize_q4_0(x)
    np.testing.assert_array_equal(blocks.dequantize_q4_0(d4, p4), npo.blocks.dequantize_q4_0(d4, p4))
    d5, s5, h5 = blocks.quantize_q5_0(x)
    np.testing.assert_array_equal(blocks.dequantize_q5_0(d5, s5, h5), npo.blocks.dequantize_q5_0(d5, s5, h5))


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [8, 64, 128, 256])
def test_turbo_rows_bit_exact(bits, d):
    x = _rows(bits * 1000 + d, 300, d, spread=False)
    x[3] = (x[3].astype(np.float32) * 1000).clip(-65504, 65504).astype(np.float16)
    n1, c1 = turbo.quantize(x, 0x7475726233, bits)
    n2, c2 = npo.turbo.quantize(x, 0x7475726233, bits)
    _eq16(n1, n2)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_allclose(turbo.dequantize(n1, c1, 0x7475726233, d, bits),
                               npo.turbo.dequantize(n2, c2, 0x7475726233, d, bits), rtol=1e-13, atol=1e-300)


def test_codebooks_and_transforms():
    for n in (2, 4, 8, 16):
        lv, th = turbo.lloyd_max_gaussian(n)
        nlv, nth = npo.turbo.lloyd_max_gaussian(n)
        np.testing.assert_allclose(lv, nlv, rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(th, nth, rtol=1e-14, atol=1e-15)
    for bits in (2, 3, 4):
        for a, b in zip(turbo.codebook_f32(bits), npo.turbo.codebook_f32(bits)):
            np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(turbo3.codebook_f32()[0], npo.turbo3.codebook_f32()[0])
    np.testing.assert_array_equal(turbo3.codebook_f32()[1], npo.turbo3.codebook_f32()[1])
    assert turbo3.splitmix64(99, 40) == npo.turbo3.splitmix64(99, 40)
    np.testing.assert_array_equal(turbo3.signs(2 ** 64 - 1, 256), npo.turbo3.signs(2 ** 64 - 1, 256))
    for d in (2, 16, 128):
        np.testing.assert_array_equal(turbo3.sylvester(d), npo.turbo3.sylvester(d))
    v = np.random.default_rng(1).standard_normal((40, 128)).astype(np.float32)
    np.testing.assert_array_equal(turbo3.fwht_f32(v), npo.turbo3.fwht_f32(v))
    np.testing.assert_array_equal(turbo3.tree_sum_f32(v * v), npo.turbo3.tree_sum_f32(v * v))


@pytest.mark.parametrize("d", [32, 128])
def test_qjl_rows_bit_exact(d):
    x = _rows(d + 7, 200, d, spread=False)
    p = np.random.default_rng(d).standard_normal((d, d)).astype(np.float32)
    s1, c1 = qjl.quantize(x, 4242, p)
    s2, c2 = npo.qjl.quantize(x, 4242, p)
    _eq16(s1, s2)
    np.testing.assert_array_equal(c1, c2)
    r1, r2 = qjl.residual_f32(x, 4242), npo.qjl.residual_f32(x, 4242)
    for a, b in zip(r1, r2):
        np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(qjl.project_f32(p, r1[2]), npo.qjl.project_f32(p, r2[2]))
    np.testing.assert_allclose(qjl.dequantize(s1, c1, 4242, p, d), npo.qjl.dequantize(s2, c2, 4242, p, d),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(qjl.projection_matrix(4242, p, d), npo.qjl.projection_matrix(4242, p, d),
                               rtol=1e-12, atol=1e-12)


def test_attention_and_combine():
    rng = np.random.default_rng(9)
    q = rng.standard_normal((2, 8, 64))
    k = rng.standard_normal((2, 2, 300, 64)) * 3
    v = rng.standard_normal((2, 2, 300, 64))
    for threads in (1, 3):
        np.testing.assert_allclose(attention.decode_attention(q, k, v, 0.125, threads=threads),
                                   npo.attention.decode_attention(q, k, v, 0.125), rtol=0, atol=1e-13)
    b = [0, 33, 34, 200, 300]
    m1, l1, a1 = attention.partials(q[0, 0], k[0, 0], v[0, 0], 0.125, b)
    m2, l2, a2 = npo.attention.partials(q[0, 0], k[0, 0], v[0, 0], 0.125, b)
    np.testing.assert_allclose(m1, m2, rtol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-13)
    np.testing.assert_allclose(np.array(a1), np.array(a2), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(attention.combine(m1, l1, a1), npo.attention.combine(m2, l2, a2), atol=1e-13)


def test_row_bytes():
    for kind in ("f16", "q8_0", "q4_0", "q5_0", "turbo2", "turbo3", "turbo4", "turbo3_qjl"):
        for d in (32, 64, 128, 256):
            assert cache_model.row_bytes(kind, d) == npo.cache_model.row_bytes(kind, d)
