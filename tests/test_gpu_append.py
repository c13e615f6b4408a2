"""Quantize-on-append on the GPU against the oracle: stored bytes must match bit
for bit, rows outside [pos, pos + n_tok) must stay untouched."""

import numpy as np
import pytest
import torch

import decode_attention_q8_b200 as kvq
import synth
from golden_blocks import handworked_blocks
from kvq_testlib import SENTINEL, alloc_cache, oracle_rows, rows_of

pytestmark = pytest.mark.gpu


def _adversarial_rows(n, D, rng):
    """fp16 rows mixing hand-worked blocks, exact halves, ties, zeros and a wide
    range of magnitudes (down to fp16 subnormals)."""
    hand = [b["x"] for b in handworked_blocks()]
    out = np.zeros((n, D), np.float16)
    for r in range(n):
        for blk in range(D // 32):
            kind = (r * 7 + blk) % 5
            if kind == 0:
                out[r, blk * 32:(blk + 1) * 32] = hand[(r + blk) % len(hand)]
            elif kind == 1:
                k = rng.integers(-254, 255, size=32) / 2.0
                out[r, blk * 32:(blk + 1) * 32] = k.astype(np.float16)
            elif kind == 2:
                x = rng.standard_normal(32) * np.exp(rng.uniform(-14, 10))
                out[r, blk * 32:(blk + 1) * 32] = np.clip(x, -65504, 65504).astype(np.float16)
            elif kind == 3:
                v = np.zeros(32)
                i, j = rng.integers(0, 32, size=2)
                v[i], v[j] = 3.0, -3.0
                out[r, blk * 32:(blk + 1) * 32] = v.astype(np.float16)
            else:
                out[r, blk * 32:(blk + 1) * 32] = rng.standard_normal(32).astype(np.float16)
    return out


def _check_append(k_type, v_type, D, B, H, max_ctx, pos, n_tok, seed, adversarial=False):
    rng = np.random.default_rng(seed)
    proj = synth.qjl_projection(seed + 5, D) if k_type == "turbo3_qjl" else None
    desc = kvq.make_desc(H, H, D, k_type, v_type, max_ctx, turbo_seed=seed * 7919 + 1,
                         qjl_proj=None if proj is None else proj.cuda())
    if adversarial:
        k_new = _adversarial_rows(B * n_tok * H, D, rng).reshape(B, n_tok, H, D)
        v_new = _adversarial_rows(B * n_tok * H, D, rng).reshape(B, n_tok, H, D)
    else:
        k_new = synth.normal_f16((B, n_tok, H, D), seed, outlier_channels=(3, 17), outlier_scale=10.0).numpy()
        v_new = synth.normal_f16((B, n_tok, H, D), seed + 1).numpy()
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, torch.from_numpy(k_new).cuda(), torch.from_numpy(v_new).cuda(),
                            B, pos, n_tok)
    torch.cuda.synchronize()
    for which, cache, new, kind in ((0, kc, k_new, k_type), (1, vc, v_new, v_type)):
        lay = kvq.kvq_cache_layout(desc, B, which)
        host = cache.cpu().numpy()
        for b in range(B):
            for h in range(H):
                codes, scales = rows_of(host, lay, b, h, H, pos, pos + n_tok)
                ecodes, escales = oracle_rows(kind, new[b, :, h, :], desc.turbo_seed,
                                              None if proj is None else proj.numpy())
                np.testing.assert_array_equal(codes, ecodes, err_msg=f"{kind} codes b{b} h{h}")
                np.testing.assert_array_equal(scales.view(np.uint16), escales.view(np.uint16),
                                              err_msg=f"{kind} scales b{b} h{h}")
                before, sb = rows_of(host, lay, b, h, H, 0, pos)
                after, sa = rows_of(host, lay, b, h, H, pos + n_tok, lay.rows_per_plane)
                assert np.all(before == SENTINEL) and np.all(after == SENTINEL)
                assert np.all(sb.view(np.uint8) == SENTINEL) and np.all(sa.view(np.uint8) == SENTINEL)


@pytest.mark.parametrize("k_type,v_type", [("q8_0", "q4_0"), ("q4_0", "q8_0"), ("f16", "turbo3"),
                                           ("q8_0", "turbo3"), ("f16", "f16"), ("q8_0", "turbo2"),
                                           ("q4_0", "turbo4"), ("q5_0", "q5_0"), ("q8_0", "q5_0"),
                                           ("turbo3", "turbo3"), ("turbo2", "q8_0"), ("turbo4", "turbo4"),
                                           ("turbo3_qjl", "q8_0"), ("turbo3_qjl", "turbo3")])
@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_append_bit_exact(k_type, v_type, D):
    _check_append(k_type, v_type, D, B=2, H=3, max_ctx=100, pos=37, n_tok=21, seed=D)


@pytest.mark.parametrize("k_type,v_type", [("q8_0", "q4_0"), ("q4_0", "turbo3"), ("q8_0", "turbo2"),
                                           ("f16", "turbo4"), ("q5_0", "q5_0"), ("turbo3_qjl", "q4_0")])
def test_append_adversarial_blocks(k_type, v_type):
    _check_append(k_type, v_type, 128, B=1, H=2, max_ctx=64, pos=0, n_tok=64, seed=3, adversarial=True)


def test_append_single_row_at_end():
    # one decode step appends one row at the last cell
    _check_append("q8_0", "q4_0", 128, B=1, H=8, max_ctx=8192, pos=8191, n_tok=1, seed=11)


def test_append_two_calls_compose():
    """Prefill then a single-row append: both ranges hold the oracle's bytes."""
    D, H, B = 128, 2, 1
    desc = kvq.make_desc(H, H, D, "q8_0", "turbo3", 64, turbo_seed=99)
    k = synth.normal_f16((B, 40, H, D), 5).numpy()
    v = synth.normal_f16((B, 40, H, D), 6).numpy()
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, torch.from_numpy(k[:, :39]).cuda(), torch.from_numpy(v[:, :39]).cuda(),
                            B, 0, 39)
    kvq.kvq_append_quantize(desc, kc, vc, torch.from_numpy(k[:, 39:]).cuda(), torch.from_numpy(v[:, 39:]).cuda(),
                            B, 39, 1)
    torch.cuda.synchronize()
    for which, cache, new, kind in ((0, kc, k, "q8_0"), (1, vc, v, "turbo3")):
        lay = kvq.kvq_cache_layout(desc, B, which)
        for h in range(H):
            codes, scales = rows_of(cache.cpu().numpy(), lay, 0, h, H, 0, 40)
            ecodes, escales = oracle_rows(kind, new[0, :, h, :], 99)
            np.testing.assert_array_equal(codes, ecodes)
            np.testing.assert_array_equal(scales.view(np.uint16), escales.view(np.uint16))


def test_append_rejects_out_of_range_without_writing():
    desc = kvq.make_desc(2, 2, 64, "q8_0", "q4_0", 32)
    kc, vc = alloc_cache(desc, 1, 0), alloc_cache(desc, 1, 1)
    rows = torch.zeros((1, 4, 2, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(kvq.KvqError):
        kvq.kvq_append_quantize(desc, kc, vc, rows, rows, 1, 30, 4)
    torch.cuda.synchronize()
    assert bool((kc == SENTINEL).all()) and bool((vc == SENTINEL).all())


@pytest.mark.parametrize("D", [32, 64, 128])
def test_qjl_bulk_append_staged_projection(D):
    """A prefill large enough that every CTA holds many rows: the append kernel
    then reads the projection from a transposed shared-memory copy.  The bytes
    must still match the oracle's left-to-right sums bit for bit."""
    B, H, n_tok = 1, 8, 8192
    proj = synth.qjl_projection(D + 3, D)
    desc = kvq.make_desc(H, H, D, "turbo3_qjl", "q8_0", n_tok, turbo_seed=D * 3 + 1, qjl_proj=proj.cuda())
    k_new = synth.normal_f16((B, n_tok, H, D), D + 100, outlier_channels=(3, 17), outlier_scale=10.0)
    v_new = synth.normal_f16((B, n_tok, H, D), D + 101)
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k_new.cuda(), v_new.cuda(), B, 0, n_tok)
    torch.cuda.synchronize()
    lay = kvq.kvq_cache_layout(desc, B, 0)
    host = kc.cpu().numpy()
    for h in range(H):
        codes, scales = rows_of(host, lay, 0, h, H, 0, n_tok)
        ecodes, escales = oracle_rows("turbo3_qjl", k_new[0, :, h, :].numpy(), desc.turbo_seed, proj.numpy())
        np.testing.assert_array_equal(codes, ecodes, err_msg=f"codes h{h}")
        np.testing.assert_array_equal(scales.view(np.uint16), escales.view(np.uint16), err_msg=f"scales h{h}")
