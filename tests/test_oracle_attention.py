"""Pins of the attention oracle: a library attention routine, closed forms and the
split/combine identity.  No GPU."""

import numpy as np
import pytest
import torch

from oracle import attention


def _sdpa_reference(q, k, v, scale):
    """torch's CPU scaled_dot_product_attention in float64, GQA by repeating
    each KV head over its G consecutive query heads."""
    B, n_q, D = q.shape
    n_kv = k.shape[1]
    G = n_q // n_kv
    qt = torch.from_numpy(q)[:, :, None, :]                          # [B, n_q, 1, D]
    kt = torch.from_numpy(k).repeat_interleave(G, dim=1)             # [B, n_q, T, D]
    vt = torch.from_numpy(v).repeat_interleave(G, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return o[:, :, 0, :].numpy()


@pytest.mark.parametrize("B,n_q,n_kv,T,D", [(1, 4, 2, 256, 64), (2, 8, 1, 37, 32), (3, 6, 6, 5, 128)])
def test_matches_library_attention(B, n_q, n_kv, T, D):
    rng = np.random.default_rng(B * 100 + T)
    q = rng.standard_normal((B, n_q, D))
    k = rng.standard_normal((B, n_kv, T, D)) * 2
    v = rng.standard_normal((B, n_kv, T, D))
    scale = 1 / np.sqrt(D)
    np.testing.assert_allclose(attention.decode_attention(q, k, v, scale),
                               _sdpa_reference(q, k, v, scale), atol=1e-12, rtol=0)


def test_full_matrix_brute_force():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 2, 8))
    k = rng.standard_normal((1, 1, 6, 8))
    v = rng.standard_normal((1, 1, 6, 8))
    scores = q[0] @ k[0, 0].T * 0.3                   # [2, 6]
    e = np.exp(scores)
    expect = (e / e.sum(axis=1, keepdims=True)) @ v[0, 0]
    np.testing.assert_allclose(attention.decode_attention(q, k, v, 0.3)[0], expect, atol=1e-13)


def test_closed_forms():
    rng = np.random.default_rng(4)
    D = 16
    q = rng.standard_normal((1, 2, D))
    v = rng.standard_normal((1, 1, 9, D))
    # one cached row: o = v_0
    k1 = rng.standard_normal((1, 1, 1, D))
    np.testing.assert_allclose(attention.decode_attention(q, k1, v[:, :, :1], 0.5)[0, 1], v[0, 0, 0], atol=1e-14)
    # identical keys: uniform weights, o = mean(v)
    k = np.repeat(rng.standard_normal((1, 1, 1, D)), 9, axis=2)
    np.testing.assert_allclose(attention.decode_attention(q, k, v, 0.5)[0, 0], v[0, 0].mean(axis=0), atol=1e-14)
    # q = 0: o = mean(v)
    k = rng.standard_normal((1, 1, 9, D))
    np.testing.assert_allclose(attention.decode_attention(np.zeros_like(q), k, v, 0.5)[0, 0],
                               v[0, 0].mean(axis=0), atol=1e-14)
    # a dominant key takes all the weight
    k = np.zeros((1, 1, 9, D))
    k[0, 0, 4] = 1000 * q[0, 0]
    np.testing.assert_allclose(attention.decode_attention(q, k, v, 1.0)[0, 0], v[0, 0, 4], atol=1e-12)


def test_weights_sum_to_one():
    rng = np.random.default_rng(5)
    w = attention.softmax_weights(rng.standard_normal(32), rng.standard_normal((500, 32)) * 5, 0.2)
    assert abs(w.sum() - 1) < 1e-12 and np.all(w >= 0)


@pytest.mark.parametrize("bounds", [[0, 100], [0, 1, 100], [0, 37, 38, 64, 100], list(range(0, 101, 10))])
def test_split_combine_identity(bounds):
    rng = np.random.default_rng(len(bounds))
    D = 32
    q = rng.standard_normal(D)
    k = rng.standard_normal((100, D)) * 3
    v = rng.standard_normal((100, D))
    ms, ls, accs = attention.partials(q, k, v, 0.25, bounds)
    full = attention.decode_attention(q[None, None], k[None, None], v[None, None], 0.25)[0, 0]
    np.testing.assert_allclose(attention.combine(ms, ls, accs), full, atol=1e-12)


@pytest.mark.parametrize("k_type,v_type", [("q8_0", "q4_0"), ("q4_0", "turbo3"), ("f16", "q5_0"),
                                           ("turbo3_qjl", "turbo2"), ("turbo4", "q8_0")])
def test_decode_over_stored_cache_is_dequantize_then_attend(k_type, v_type):
    """orc_decode_cache (the CPU baseline and the full-size check) equals the
    dequantizers followed by the plain attention, on any thread count."""
    from oracle import blocks, qjl, turbo
    B, n_kv, G, T, D, seed = 2, 2, 3, 70, 64, 99
    rng = np.random.default_rng(hash((k_type, v_type)) % 2 ** 32)
    proj = rng.standard_normal((D, D)).astype(np.float32)

    def store(kind, x):
        if kind == "f16":
            return x.view(np.uint8).reshape(*x.shape[:-1], 2 * D), np.zeros((*x.shape[:-1], 0), np.float16)
        if kind == "q8_0":
            d, q = blocks.quantize_q8_0(x)
            return q.view(np.uint8), d
        if kind == "q4_0":
            d, qs = blocks.quantize_q4_0(x)
            return qs, d
        if kind == "q5_0":
            d, qs, qh = blocks.quantize_q5_0(x)
            return qs, np.concatenate([d, np.ascontiguousarray(qh).view(np.float16)], axis=-1)
        if kind == "turbo3_qjl":
            sc, codes = qjl.quantize(x, seed, proj)
            return codes, sc
        n, codes = turbo.quantize(x, seed, turbo.BITS[kind])
        return codes, n[..., None]

    def dequant(kind, codes, sc):
        if kind == "f16":
            return blocks.dequantize_f16(np.ascontiguousarray(codes).view(np.float16))
        if kind == "q8_0":
            return blocks.dequantize_q8_0(sc, np.ascontiguousarray(codes).view(np.int8))
        if kind == "q4_0":
            return blocks.dequantize_q4_0(sc, codes)
        if kind == "q5_0":
            nb = D // 32
            return blocks.dequantize_q5_0(sc[..., :nb], codes, np.ascontiguousarray(sc[..., nb:]).view(np.uint32))
        if kind == "turbo3_qjl":
            return qjl.dequantize(sc, codes, seed, proj, D)
        return turbo.dequantize(sc[..., 0], codes, seed, D, turbo.BITS[kind])

    k = (rng.standard_normal((B, n_kv, T, D)) * 2).astype(np.float16)
    v = rng.standard_normal((B, n_kv, T, D)).astype(np.float16)
    q = rng.standard_normal((B, n_kv * G, D)).astype(np.float16)
    kc, ks = store(k_type, k)
    vc, vs = store(v_type, v)
    expect = attention.decode_attention(q.astype(np.float64), dequant(k_type, kc, ks), dequant(v_type, vc, vs), 0.125)
    got1 = attention.decode_cache(k_type, v_type, kc, ks, vc, vs, q, 0.125, seed=seed, proj=proj, threads=1)
    got4 = attention.decode_cache(k_type, v_type, kc, ks, vc, vs, q, 0.125, seed=seed, proj=proj, threads=4)
    np.testing.assert_allclose(got1, expect, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(got1, got4)
