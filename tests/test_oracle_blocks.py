"""Pins of the q8_0 / q4_0 / f16 oracle against what the definitions and the pages fix.

No GPU.  Each check is something other than the oracle's own formula: hand-worked
blocks, rounding and error-bound properties, brute force over the code grid, and
the cache sizes the pages print.
"""

import numpy as np
import pytest

from oracle import blocks, cache_model
from golden_blocks import handworked_blocks
from conftest import read_golden


def _rand_blocks(rng, n_blocks, spread=True):
    x = rng.standard_normal((n_blocks, 32))
    if spread:
        x *= np.exp(rng.uniform(-12, 10, size=(n_blocks, 1)))   # subnormal ... large scales
    return np.clip(x, -65504, 65504).astype(np.float16)


def _adversarial_blocks(rng):
    """Blocks with exact halves, equal +-maxima, zeros and tiny scales."""
    out = []
    for amax in (127.0, 254.0, 63.5, 1.0, 2.0 ** -14, 2.0 ** -20, 1000.0):
        k = rng.integers(-254, 255, size=32).astype(np.float64) / 2.0
        b = np.clip(k / 127.0 * amax, -65504, 65504)
        b[rng.integers(0, 32)] = amax
        b[rng.integers(0, 32)] = -amax
        out.append(b)
    out.append(np.zeros(32))
    z = np.zeros(32)
    z[7] = -3.0
    z[20] = 3.0
    out.append(z)
    return np.array(out).astype(np.float16)


def test_handworked_blocks():
    for blk in handworked_blocks():
        x = blk["x"][None, :]
        if blk["type"] == "q8_0":
            d, q = blocks.quantize_q8_0(x)
            assert int(d.view(np.uint16)[0, 0]) == blk["scale_bits"], blk["name"]
            np.testing.assert_array_equal(q[0], blk["q"], err_msg=blk["name"])
            np.testing.assert_array_equal(blocks.dequantize_q8_0(d, q)[0],
                                          blk["q"].astype(np.float64) * float(d[0, 0]))
        else:
            d, qs = blocks.quantize_q4_0(x)
            assert int(d.view(np.uint16)[0, 0]) == blk["scale_bits"], blk["name"]
            np.testing.assert_array_equal(qs[0], blk["bytes"], err_msg=blk["name"])


def _multiblock_rows():
    rows, cur = [], None
    for line in read_golden("blocks_multiblock_rows.txt"):
        tok = line.split()
        if tok[0] == "row":
            cur = {"name": tok[1], "type": tok[2], "d": int(tok[3])}
            rows.append(cur)
        else:
            cur[tok[0]] = tok[1:]
    return rows


def test_dequantizers_on_handworked_multiblock_rows():
    """Four blocks with four different scales per row: the value of every
    element follows by hand (exact products).  A wrong code offset, swapped
    nibbles, a wrong qh bit or one block's scale used for another block fails."""
    rows = _multiblock_rows()
    assert [r["type"] for r in rows] == ["q8_0", "q4_0", "q5_0"]
    for r in rows:
        d = r["d"]
        scales = np.array([int(v, 16) for v in r["scales"]], np.uint16).view(np.float16)[None]
        expect = np.array([float(v) for v in r["x"]])[None]
        assert expect.shape == (1, d) and scales.shape == (1, d // 32)
        if r["type"] == "q8_0":
            q = np.array([int(v) for v in r["q"]], np.int8)[None]
            got = blocks.dequantize_q8_0(scales, q)
        elif r["type"] == "q4_0":
            qs = np.array([int(v, 16) for v in r["bytes"]], np.uint8)[None]
            got = blocks.dequantize_q4_0(scales, qs)
        else:
            qs = np.array([int(v, 16) for v in r["bytes"]], np.uint8)[None]
            qh = np.array([int(v, 16) for v in r["qh"]], np.uint32)[None]
            got = blocks.dequantize_q5_0(scales, qs, qh)
        np.testing.assert_array_equal(got, expect, err_msg=r["name"])


def test_q8_0_rounding_and_bounds():
    rng = np.random.default_rng(1)
    x16 = np.concatenate([_rand_blocks(rng, 4000), _adversarial_blocks(rng)])
    d_h, q = blocks.quantize_q8_0(x16)
    x = x16.astype(np.float64)
    amax = np.abs(x).max(axis=1)
    assert np.abs(q.astype(np.int32)).max() <= 127
    nz = amax > 0
    # fp32 scale recomputed from the definition's meaning (amax/127), in fp64
    d = amax / 127.0
    r = x[nz] / d[nz, None]
    qq = q[nz].astype(np.float64)
    # nearest grid point: |x/d - q| <= 1/2 (up to binary32 rounding of x/d and d)
    assert np.all(np.abs(r - qq) <= 0.5 + 1e-5)
    # brute force over the grid: no integer in [-127, 127] is strictly closer
    grid = np.arange(-127, 128, dtype=np.float64)
    best = np.abs(r[..., None] - grid).min(axis=-1)
    assert np.all(np.abs(r - qq) <= best + 1e-5)
    # round trip through the dequantizer (stored fp16 scale): |x - x_hat| <= d/2 + 127 |d - d_h|
    dh = d_h[:, 0].astype(np.float64)[nz]
    err = np.abs(x[nz] - blocks.dequantize_q8_0(d_h, q)[nz])
    bound = d[nz] / 2 * (1 + 1e-5) + 127 * np.abs(d[nz] - dh)
    assert np.all(err <= bound[:, None] + 1e-12)
    assert np.all(q[~nz] == 0)
    assert np.all(blocks.dequantize_q8_0(d_h, q)[~nz] == 0)


def test_q8_0_exact_ties_round_away():
    # x/d exactly k + 1/2 (d = 1): round half away from zero, not to even
    x = np.zeros((1, 32), np.float16)
    x[0, 0] = 127
    x[0, 1:9] = [0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, -3.5]
    _, q = blocks.quantize_q8_0(x)
    np.testing.assert_array_equal(q[0, 1:9], [1, 2, 3, 4, -1, -2, -3, -4])


def test_q4_0_codes_and_bounds():
    rng = np.random.default_rng(2)
    x16 = np.concatenate([_rand_blocks(rng, 4000), _adversarial_blocks(rng)])
    d_h, codes = blocks.quantize_q4_0_codes(x16)
    x = x16.astype(np.float64)
    assert codes.max() <= 15
    j = np.argmax(np.abs(x), axis=1)
    m = x[np.arange(len(x)), j]
    nz = m != 0
    # the element of largest magnitude maps to code 0 (value -8 d)
    assert np.all(codes[np.arange(len(x)), j][nz] == 0)
    assert np.all(codes[~nz] == 8)
    d = m[nz] / -8.0
    r = x[nz] / d[:, None]                      # in [-8, 8]
    c = codes[nz].astype(np.float64) - 8.0
    unclamped = r < 7.5 - 1e-5
    # nearest grid point in -8..7 for every unclamped element
    assert np.all(np.abs(r - c)[unclamped] <= 0.5 + 1e-5)
    # clamped elements (opposite sign to m, |x/d| in [7.5, 8]) sit at the top code 7
    assert np.all(c[r > 7.5 + 1e-5] == 7)
    # round trip through the packed bytes and the dequantizer (stored fp16 scale)
    d_p, qs = blocks.quantize_q4_0(x16)
    np.testing.assert_array_equal(d_p.view(np.uint16), d_h.view(np.uint16))
    x_hat = blocks.dequantize_q4_0(d_p, qs)
    dh = d_h[:, 0].astype(np.float64)[nz]
    np.testing.assert_array_equal(x_hat[nz], dh[:, None] * c)      # value = d_h * (code - 8)
    err = np.abs(x[nz] - x_hat[nz])
    bound_un = np.abs(d)[:, None] / 2 * (1 + 1e-5) + 16 * np.abs(d - dh)[:, None]
    bound_cl = np.abs(d)[:, None] * (1 + 1e-5) + 16 * np.abs(d - dh)[:, None]
    assert np.all(np.where(unclamped, err <= bound_un + 1e-12, err <= bound_cl + 1e-12))
    assert np.all(x_hat[~nz] == 0)


def test_q4_0_ties_lowest_index():
    x = np.zeros((2, 32), np.float16)
    x[0, 3], x[0, 9] = 2.0, -2.0      # +2 first -> d = -0.25
    x[1, 3], x[1, 9] = -2.0, 2.0      # -2 first -> d = +0.25
    d, codes = blocks.quantize_q4_0_codes(x)
    assert float(d[0, 0]) == -0.25 and float(d[1, 0]) == 0.25
    assert codes[0, 3] == 0 and codes[0, 9] == 15
    assert codes[1, 3] == 0 and codes[1, 9] == 15


def test_q4_0_pack_roundtrip_and_order():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, size=(5, 128)).astype(np.uint8)
    packed = blocks.pack_q4_0(codes)
    assert packed.shape == (5, 64)
    np.testing.assert_array_equal(blocks.unpack_q4_0(packed), codes)
    # element j of block 1 is the low nibble of byte 16 + j, element j+16 the high one
    assert packed[0, 16 + 5] & 0xF == codes[0, 32 + 5]
    assert packed[0, 16 + 5] >> 4 == codes[0, 32 + 21]


def test_q5_0_codes_and_bounds():
    """Every unclamped element at the nearest point of the grid -16..15 (times
    d = m / -16), the largest-magnitude element at code 0, the opposite extreme
    clamped to 31, and the qualified round-trip bound with the stored fp16 d."""
    rng = np.random.default_rng(5)
    x16 = np.concatenate([_rand_blocks(rng, 4000), _adversarial_blocks(rng)])
    d_h, codes = blocks.quantize_q5_0_codes(x16)
    x = x16.astype(np.float64)
    assert codes.max() <= 31
    j = np.argmax(np.abs(x), axis=1)
    m = x[np.arange(len(x)), j]
    nz = m != 0
    assert np.all(codes[np.arange(len(x)), j][nz] == 0)
    assert np.all(codes[~nz] == 16)
    d = m[nz] / -16.0
    r = x[nz] / d[:, None]                      # in [-16, 16]
    c = codes[nz].astype(np.float64) - 16.0
    unclamped = r < 15.5 - 1e-5
    assert np.all(np.abs(r - c)[unclamped] <= 0.5 + 1e-5)
    assert np.all(c[r > 15.5 + 1e-5] == 15)
    d_p, qs, qh = blocks.quantize_q5_0(x16)
    x_hat = blocks.dequantize_q5_0(d_p, qs, qh)
    dh = d_h[:, 0].astype(np.float64)[nz]
    np.testing.assert_array_equal(x_hat[nz], dh[:, None] * c)      # value = d_h * (code - 16)
    err = np.abs(x[nz] - x_hat[nz])
    bound_un = np.abs(d)[:, None] / 2 * (1 + 1e-5) + 32 * np.abs(d - dh)[:, None]
    bound_cl = np.abs(d)[:, None] * (1 + 1e-5) + 32 * np.abs(d - dh)[:, None]
    assert np.all(np.where(unclamped, err <= bound_un + 1e-12, err <= bound_cl + 1e-12))


def test_q5_0_closed_form_block():
    """x_j = j - 16: m = -16 (index 0), d = 1, q_j = j; the fifth bits are
    those of j >= 16, each byte holds (j, j + 16 mod 16) = j | j << 4, and
    the block dequantizes to x exactly."""
    x = (np.arange(32) - 16).astype(np.float16)[None]
    d, qs, qh = blocks.quantize_q5_0(x)
    assert float(d[0, 0]) == 1.0
    assert int(qh[0, 0]) == 0xFFFF0000
    assert qs[0].tolist() == [j | (j << 4) for j in range(16)]
    np.testing.assert_array_equal(blocks.dequantize_q5_0(d, qs, qh)[0], np.arange(32) - 16.0)
    # and the same block negated: m = +16 at index 0... index 0 holds -16 -> +16, d = -1
    d2, qs2, qh2 = blocks.quantize_q5_0(-x)
    assert float(d2[0, 0]) == -1.0
    np.testing.assert_array_equal(blocks.dequantize_q5_0(d2, qs2, qh2)[0], -(np.arange(32) - 16.0))


def test_q5_0_is_q4_0_widened():
    """q5_0's grid step (|m|/16) is half of q4_0's (|m|/8), so over many blocks
    its largest error per block is about half of q4_0's."""
    rng = np.random.default_rng(6)
    x16 = _rand_blocks(rng, 2000)
    d4, c4 = blocks.quantize_q4_0_codes(x16)
    d5, c5 = blocks.quantize_q5_0_codes(x16)
    x = x16.astype(np.float64)
    e4 = np.abs(x - d4.astype(np.float64) * (c4.astype(np.float64) - 8)).max(axis=1)
    e5 = np.abs(x - d5.astype(np.float64) * (c5.astype(np.float64) - 16)).max(axis=1)
    assert 0.4 < np.mean(e5) / np.mean(e4) < 0.6


def test_q5_0_pack_roundtrip_and_order():
    rng = np.random.default_rng(7)
    codes = rng.integers(0, 32, size=(5, 128)).astype(np.uint8)
    qs, qh = blocks.pack_q5_0(codes)
    assert qs.shape == (5, 64) and qh.shape == (5, 4) and qh.dtype == np.uint32
    np.testing.assert_array_equal(blocks.unpack_q5_0(qs, qh), codes)
    assert (int(qh[0, 1]) >> 7) & 1 == codes[0, 32 + 7] >> 4
    assert qs[0, 16 + 5] & 0xF == codes[0, 32 + 5] & 0xF


def test_f16_identity():
    x = np.array([[1.5, -2.0, 65504.0, 2.0 ** -24]], np.float16)
    np.testing.assert_array_equal(blocks.dequantize_f16(x), x.astype(np.float64))


def test_cache_sizes_match_pages():
    mib = 1024.0 * 1024.0
    rows = read_golden("kv_cache_bytes.txt")
    assert len(rows) == 10
    for row in rows:
        L, H, D, T, kt, vt, exp, which = row.split()
        L, H, D, T, exp = int(L), int(H), int(D), int(T), float(exp)
        k = cache_model.cache_bytes(kt, L, H, D, T)
        v = cache_model.cache_bytes(vt, L, H, D, T)
        got = {"K": k, "V": v, "KV": k + v}[which] / mib
        assert got == pytest.approx(exp, abs=1e-9), row


def test_row_bytes_nominal():
    # per element: f16 2 B, q8_0 8.5 bits, q4_0 4.5 bits, turbo3 3.125 bits at d = 128
    assert cache_model.row_bytes("f16", 128) == 256
    assert cache_model.row_bytes("q8_0", 128) == 136
    assert cache_model.row_bytes("q4_0", 128) == 72
    assert cache_model.row_bytes("turbo3", 128) * 8 / 128 == 3.125


def test_turbo3_qjl_row_bytes():
    """3 bits of codes per value (2-bit levels + 1-bit residual signs, as the
    TurboQuant page's "3 bits per value"), plus two fp16 norms: 52 bytes at
    d = 128, a 4.9x reduction from fp16 (the page: about 5x)."""
    assert cache_model.row_bytes("turbo3_qjl", 128) == 52
    assert cache_model.row_bytes("turbo3_qjl", 64) == 28
    assert abs(cache_model.row_bytes("f16", 128) / cache_model.row_bytes("turbo3_qjl", 128) - 5) < 0.1
