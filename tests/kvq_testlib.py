"""Helpers shared by the GPU tests: cache allocation, reading rows back out of
the library's layout, and the oracle-side view of the same rows.  The expected
values all come from ``oracle/``; the library only provides the buffers under
test and the documented layout (include/kvq.h) used to read them."""

import numpy as np
import torch

import decode_attention_q8_b200 as kvq
from oracle import attention, blocks, qjl, turbo, turbo3

SENTINEL = 0xA5

ATOL = 2e-3        # max abs error of attention outputs against the fp64 oracle
REL_L2 = 1e-3      # relative L2 error of attention outputs against the fp64 oracle


def alloc_cache(desc, batch, which, device="cuda"):
    n = kvq.kvq_cache_bytes(desc, batch, which)
    assert n > 0
    return torch.full((n,), SENTINEL, dtype=torch.uint8, device=device)


def rows_of(cache_cpu, layout, b, h, n_kv, t0, t1):
    """(codes uint8 [n, code_bytes], scales fp16 [n, n_scales]) of rows t0..t1-1
    of plane (b, h), read by the layout documented in include/kvq.h."""
    c = np.asarray(cache_cpu, dtype=np.uint8)
    T, cb, ns = layout.rows_per_plane, layout.code_bytes, layout.n_scales
    plane = b * n_kv + h
    codes = c[(plane * T + t0) * cb:(plane * T + t1) * cb].reshape(t1 - t0, cb)
    if ns:
        off = layout.scale_offset + (plane * T + t0) * ns * 2
        scales = c[off:off + (t1 - t0) * ns * 2].view(np.float16).reshape(t1 - t0, ns)
    else:
        scales = np.zeros((t1 - t0, 0), np.float16)
    return codes, scales


def oracle_rows(kind, x_f16, seed=0, proj=None):
    """Oracle codes/scales of rows x_f16 [n, D] in the same per-row form
    (proj: the turbo3_qjl projection, float32 [D][D] on the host)."""
    x = np.asarray(x_f16, np.float16)
    n, D = x.shape
    if kind == "f16":
        return x.view(np.uint8).reshape(n, 2 * D), np.zeros((n, 0), np.float16)
    if kind == "q8_0":
        d, q = blocks.quantize_q8_0(x)
        return q.view(np.uint8), d
    if kind == "q4_0":
        d, qs = blocks.quantize_q4_0(x)
        return qs, d
    if kind == "q5_0":  # scale plane row: block scales, then each qh word as two fp16 slots
        d, qs, qh = blocks.quantize_q5_0(x)
        return qs, np.concatenate([d, np.ascontiguousarray(qh).view(np.float16)], axis=1)
    if kind == "turbo3":
        nrm, codes = turbo3.quantize_turbo3(x, seed)
        return codes, nrm.reshape(n, 1)
    if kind in ("turbo2", "turbo4"):
        nrm, codes = turbo.quantize(x, seed, turbo.BITS[kind])
        return codes, nrm.reshape(n, 1)
    if kind == "turbo3_qjl":
        scales, codes = qjl.quantize(x, seed, proj)
        return codes, scales
    raise ValueError(kind)


def oracle_dequant(kind, codes, scales, D, seed=0, proj=None):
    """float64 [n, D] decoded rows (oracle definitions) from stored codes/scales."""
    if kind == "f16":
        return blocks.dequantize_f16(np.ascontiguousarray(codes).view(np.float16))
    if kind == "q8_0":
        return blocks.dequantize_q8_0(scales, np.ascontiguousarray(codes).view(np.int8))
    if kind == "q4_0":
        return blocks.dequantize_q4_0(scales, codes)
    if kind == "q5_0":
        nb = D // 32
        qh = np.ascontiguousarray(scales[:, nb:]).view(np.uint32)
        return blocks.dequantize_q5_0(scales[:, :nb], codes, qh)
    if kind == "turbo3":
        return turbo3.dequantize_turbo3(scales[:, 0], codes, seed, D)
    if kind in ("turbo2", "turbo4"):
        return turbo.dequantize(scales[:, 0], codes, seed, D, turbo.BITS[kind])
    if kind == "turbo3_qjl":
        return qjl.dequantize(scales, codes, seed, proj, D)
    raise ValueError(kind)


def oracle_attention_rows(q_f16, k_hat, v_hat, scale):
    """Oracle attention of the G query heads of one KV head.
    q_f16 [G, D]; k_hat, v_hat float64 [T, D]; returns float64 [G, D]."""
    return attention.decode_attention(np.asarray(q_f16, np.float64)[None], k_hat[None, None],
                                      v_hat[None, None], scale)[0]


def assert_attention_close(got, expect, what=""):
    got = np.asarray(got, np.float64)
    expect = np.asarray(expect, np.float64)
    err = np.abs(got - expect)
    rel = np.linalg.norm(got - expect) / max(np.linalg.norm(expect), 1e-30)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err.max() <= ATOL, f"{what}: max abs err {err.max():.3e} > {ATOL}"
    assert rel <= REL_L2, f"{what}: rel L2 err {rel:.3e} > {REL_L2}"
    return err.max(), rel


def decode(desc, k_cache, v_cache, q, batch, ctx, scale, n_splits=0, stream=None):
    """Runs decode + combine through the C ABI; returns fp32 [B, n_q, D] (device)."""
    ws_bytes = kvq.kvq_workspace_bytes(desc, batch, n_splits)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    out = torch.empty((batch, desc.n_q_heads, desc.head_dim), dtype=torch.float32, device=q.device)
    kvq.kvq_decode_attention(desc, k_cache, v_cache, q, batch, ctx, scale, n_splits, ws, stream=stream)
    kvq.kvq_combine(desc, ws, batch, ctx, n_splits, out, stream=stream)
    return out
