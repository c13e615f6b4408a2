"""Decode attention (split-KV decode + combine) on the GPU against the fp64 oracle.

Tolerance: max abs error 2e-3 and relative L2 error 1e-3 of the fp32 output
against the oracle's fp64 attention over the oracle's own dequantization of the
same fp16 inputs (the stored bytes are checked bit-exact in test_gpu_append)."""

import math

import numpy as np
import pytest
import torch

import decode_attention_q8_b200 as kvq
import synth
from kvq_testlib import (alloc_cache, assert_attention_close, decode, oracle_attention_rows, oracle_dequant,
                         oracle_rows, rows_of)

pytestmark = pytest.mark.gpu


def _setup(k_type, v_type, B, n_q, n_kv, D, ctx, seed, max_ctx=None, outliers=(3, 17), oscale=10.0,
           turbo_seed=None):
    max_ctx = max_ctx or ctx
    proj = synth.qjl_projection(seed + 11, D) if k_type == "turbo3_qjl" else None
    desc = kvq.make_desc(n_q, n_kv, D, k_type, v_type, max_ctx,
                         turbo_seed=(seed * 31 + 7) if turbo_seed is None else turbo_seed,
                         qjl_proj=None if proj is None else proj.cuda())
    desc.qjl_host = None if proj is None else proj.numpy()
    w = synth.Workload("case", B, 1, n_q, n_kv, D, ctx, k_type, v_type, outliers, oscale, seed)
    q, k, v = synth.layer_inputs(w, device="cuda")
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k, v, B, 0, ctx)
    return desc, q, k, v, kc, vc


def _oracle_out(desc, q, k, v, b, g, ctx, scale):
    """Oracle outputs [G, D] of the query heads of KV head g in batch row b."""
    G = desc.n_q_heads // desc.n_kv_heads
    names = {0: "f16", 1: "q8_0", 2: "q4_0", 3: "turbo3", 4: "turbo2", 5: "turbo4", 6: "q5_0", 7: "turbo3_qjl"}
    kt, vt = names[desc.k_type], names[desc.v_type]
    kx = k[b, :ctx, g, :].cpu().numpy()
    vx = v[b, :ctx, g, :].cpu().numpy()
    proj = getattr(desc, "qjl_host", None)
    kh = oracle_dequant(kt, *oracle_rows(kt, kx, desc.turbo_seed, proj), desc.head_dim, desc.turbo_seed, proj)
    vh = oracle_dequant(vt, *oracle_rows(vt, vx, desc.turbo_seed), desc.head_dim, desc.turbo_seed)
    return oracle_attention_rows(q[b, g * G:(g + 1) * G].cpu().numpy(), kh, vh, scale)


def _check_all(desc, q, k, v, out, ctx, scale, what):
    G = desc.n_q_heads // desc.n_kv_heads
    o = out.cpu().numpy()
    for b in range(q.shape[0]):
        for g in range(desc.n_kv_heads):
            exp = _oracle_out(desc, q, k, v, b, g, ctx, scale)
            assert_attention_close(o[b, g * G:(g + 1) * G], exp, f"{what} b{b} g{g}")


def test_tiny_workload():
    """Batch 1, 4 query / 2 KV heads, head_dim 64, context 256, K q8_0 / V q4_0,
    K channels 3 and 17 x10, scale 1/sqrt(64); all 256 rows appended."""
    w = synth.WORKLOADS["tiny"]
    desc = kvq.make_desc(w.n_q, w.n_kv, w.head_dim, w.k_type, w.v_type, w.ctx)
    q, k, v = synth.layer_inputs(w, device="cuda")
    kc, vc = alloc_cache(desc, 1, 0), alloc_cache(desc, 1, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k, v, 1, 0, w.ctx)
    out = decode(desc, kc, vc, q, 1, w.ctx, w.scale)
    _check_all(desc, q, k, v, out, w.ctx, w.scale, "tiny")


@pytest.mark.parametrize("k_type", ["f16", "q8_0", "q4_0", "q5_0"])
@pytest.mark.parametrize("v_type", ["f16", "q8_0", "q4_0", "turbo3", "turbo2", "turbo4", "q5_0"])
def test_type_matrix(k_type, v_type):
    B, n_q, n_kv, D, ctx = 2, 16, 4, 128, 1000
    desc, q, k, v, kc, vc = _setup(k_type, v_type, B, n_q, n_kv, D, ctx, seed=41, max_ctx=1100)
    scale = 1 / math.sqrt(D)
    for S in (0, 3):
        out = decode(desc, kc, vc, q, B, ctx, scale, S)
        _check_all(desc, q, k, v, out, ctx, scale, f"{k_type}/{v_type} S={S}")


@pytest.mark.parametrize("ctx", [1, 2, 15, 16, 17, 33, 129, 777])
def test_ragged_context_lengths(ctx):
    desc, q, k, v, kc, vc = _setup("q8_0", "q4_0", 1, 8, 2, 128, ctx, seed=ctx, max_ctx=800)
    for S in (0, 1, 5):
        out = decode(desc, kc, vc, q, 1, ctx, 0.09, S)
        _check_all(desc, q, k, v, out, ctx, 0.09, f"ctx={ctx} S={S}")


@pytest.mark.parametrize("k_type,v_type", [("turbo3", "turbo3"), ("turbo2", "turbo2"), ("turbo4", "turbo4"),
                                           ("turbo3", "q8_0"), ("turbo2", "q4_0")])
@pytest.mark.parametrize("G", [1, 8, 16])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_turbo_keys(k_type, v_type, G, D):
    """Turbo keys: each query is rotated once in the kernel (H_un (s * q)) and
    scored against the level table, scaled by norm / D per row."""
    n_kv = 2
    desc, q, k, v, kc, vc = _setup(k_type, v_type, 2, n_kv * G, n_kv, D, 400, seed=G * 3 + D + 5)
    for S in (0, 3):
        out = decode(desc, kc, vc, q, 2, 400, 1 / math.sqrt(D), S)
        _check_all(desc, q, k, v, out, 400, 1 / math.sqrt(D), f"{k_type}/{v_type} G={G} D={D} S={S}")


@pytest.mark.parametrize("v_type", ["q8_0", "q4_0", "turbo3"])
@pytest.mark.parametrize("G", [1, 8, 16])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_qjl_keys(v_type, G, D):
    """turbo3_qjl keys: the rotated query scores the 2-bit levels (scaled by
    norm / D) and, projected once by P, the QJL sign bits (scaled by
    gamma * sqrt(pi/2) / D^1.5)."""
    n_kv = 2
    desc, q, k, v, kc, vc = _setup("turbo3_qjl", v_type, 2, n_kv * G, n_kv, D, 400, seed=G * 5 + D + 1)
    for S in (0, 3):
        out = decode(desc, kc, vc, q, 2, 400, 1 / math.sqrt(D), S)
        _check_all(desc, q, k, v, out, 400, 1 / math.sqrt(D), f"qjl/{v_type} G={G} D={D} S={S}")


@pytest.mark.parametrize("k_type,v_type", [("q5_0", "q5_0"), ("q5_0", "q8_0"), ("q8_0", "q5_0")])
@pytest.mark.parametrize("G", [1, 8])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_q5_0_head_dims_and_groups(k_type, v_type, G, D):
    """q5_0 keys and values (the fifth bit spliced into the subnormal codes)
    at every head dim: the scale-plane rows (scales + qh words) are 12, 24 and
    48 bytes, the last loaded row-wise."""
    n_kv = 2
    desc, q, k, v, kc, vc = _setup(k_type, v_type, 2, n_kv * G, n_kv, D, 300, seed=G * 7 + D)
    out = decode(desc, kc, vc, q, 2, 300, 1 / math.sqrt(D))
    _check_all(desc, q, k, v, out, 300, 1 / math.sqrt(D), f"{k_type}/{v_type} G={G} D={D}")


@pytest.mark.parametrize("v_type", ["turbo2", "turbo4"])
@pytest.mark.parametrize("G", [1, 8, 16])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_turbo_widths_group_sizes_and_head_dims(v_type, G, D):
    """2- and 4-bit values at every head dim (one or two 64-bit code windows
    per lane group) and group size."""
    n_kv = 2
    desc, q, k, v, kc, vc = _setup("q8_0", v_type, 2, n_kv * G, n_kv, D, 300, seed=G * 10 + D + 1)
    out = decode(desc, kc, vc, q, 2, 300, 1 / math.sqrt(D))
    _check_all(desc, q, k, v, out, 300, 1 / math.sqrt(D), f"{v_type} G={G} D={D}")


@pytest.mark.parametrize("G", [1, 2, 3, 4, 8, 12, 16])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_group_sizes_and_head_dims(G, D):
    n_kv = 2
    desc, q, k, v, kc, vc = _setup("q8_0", "turbo3", 2, n_kv * G, n_kv, D, 300, seed=G * 10 + D)
    out = decode(desc, kc, vc, q, 2, 300, 1 / math.sqrt(D))
    _check_all(desc, q, k, v, out, 300, 1 / math.sqrt(D), f"G={G} D={D}")


@pytest.mark.parametrize("k_type", ["f16", "q8_0", "q4_0", "q5_0"])
@pytest.mark.parametrize("v_type", ["f16", "q8_0", "q4_0", "turbo3", "turbo2", "turbo4", "q5_0"])
def test_type_matrix_head_dim_256(k_type, v_type):
    B, n_q, n_kv, D, ctx = 1, 8, 2, 256, 333
    desc, q, k, v, kc, vc = _setup(k_type, v_type, B, n_q, n_kv, D, ctx, seed=77)
    if k_type == "f16" and v_type == "f16":
        # a 16-row f16/f16 stage at head_dim 256 does not fit the shared-memory budget
        with pytest.raises(kvq.KvqError) as e:
            decode(desc, kc, vc, q, B, ctx, 0.06)
        assert e.value.status == kvq.KVQ_ERR_UNSUPPORTED
        return
    out = decode(desc, kc, vc, q, B, ctx, 0.06)
    _check_all(desc, q, k, v, out, ctx, 0.06, f"D=256 {k_type}/{v_type}")


def test_split_invariance_and_empty_splits():
    """S = 1, 2, 7, auto and S larger than ctx/16 (trailing splits empty) agree.

    The kernel rounds each softmax weight, scaled to its split's running max,
    to fp16 (relative error <= 2^-11 after the value-scale product) before the
    PV product, so two partitions round differently: their outputs may differ
    by up to 2 * 2^-11 * max|v_hat| (each is a convex combination of the rows)."""
    ctx = 520
    desc, q, k, v, kc, vc = _setup("q4_0", "q4_0", 1, 8, 2, 128, ctx, seed=5)
    outs = [decode(desc, kc, vc, q, 1, ctx, 0.1, S).cpu().numpy() for S in (1, 2, 7, 0, 40)]
    vmax = max(np.abs(oracle_dequant("q4_0", *oracle_rows("q4_0", v[0, :ctx, g, :].cpu().numpy()), 128)).max()
               for g in range(2))
    bound = 2 * 2.0 ** -11 * vmax
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= bound
    for o in outs:
        _check_all(desc, q, k, v, torch.from_numpy(o), ctx, 0.1, "split count")


def test_prefix_of_a_longer_cache():
    """ctx_len < max_ctx: rows past ctx_len (here filled with other data) are ignored."""
    desc, q, k, v, kc, vc = _setup("q8_0", "q4_0", 1, 8, 2, 128, 600, seed=9, max_ctx=600)
    out = decode(desc, kc, vc, q, 1, 333, 0.1)
    _check_all(desc, q, k, v, out, 333, 0.1, "prefix")


def test_decode_leaves_cache_untouched():
    desc, q, k, v, kc, vc = _setup("q8_0", "turbo3", 1, 8, 2, 128, 200, seed=2)
    k0, v0 = kc.clone(), vc.clone()
    decode(desc, kc, vc, q, 1, 200, 0.1)
    torch.cuda.synchronize()
    assert torch.equal(k0, kc) and torch.equal(v0, vc)


def test_llama8b_layer_with_controls():
    """Llama-3.1-8B-shaped layer (32/8 heads, head_dim 128, ctx 8192): K8V4 and the
    f16/f16 and q8_0/q8_0 controls on the same fp16 inputs, every output checked."""
    w = synth.WORKLOADS["llama8b_ctx8k"]
    q, k, v = synth.layer_inputs(w, device="cuda")
    for kt, vt in ((w.k_type, w.v_type),) + w.controls:
        desc = kvq.make_desc(w.n_q, w.n_kv, w.head_dim, kt, vt, w.ctx)
        kc, vc = alloc_cache(desc, 1, 0), alloc_cache(desc, 1, 1)
        kvq.kvq_append_quantize(desc, kc, vc, k, v, 1, 0, w.ctx)
        out = decode(desc, kc, vc, q, 1, w.ctx, w.scale)
        _check_all(desc, q, k, v, out, w.ctx, w.scale, f"8B {kt}/{vt}")


@pytest.mark.parametrize("name", ["llama70b_ctx32k_b4", "turbo3_ctx32k", "k4v4_ctx128k_b1",
                                  "k4v4_ctx128k_b4", "k4v4_ctx128k_b16"])
def test_full_size_sampled(name):
    """One layer at full size in the benchmark's launch configuration (automatic
    splits); every output of sampled (batch row, KV head) groups is checked, plus
    the stored bytes of sampled rows."""
    w = synth.WORKLOADS[name]
    desc = kvq.make_desc(w.n_q, w.n_kv, w.head_dim, w.k_type, w.v_type, w.ctx, turbo_seed=w.turbo_seed)
    q, k, v = synth.layer_inputs(w, layer=0, device="cuda")
    kc, vc = alloc_cache(desc, w.batch, 0), alloc_cache(desc, w.batch, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k, v, w.batch, 0, w.ctx)
    out = decode(desc, kc, vc, q, w.batch, w.ctx, w.scale).cpu().numpy()
    G = w.n_q // w.n_kv
    samples = {(0, 0), (w.batch - 1, w.n_kv - 1), (w.batch // 2, w.n_kv // 2)}
    for b, g in sorted(samples):
        exp = _oracle_out(desc, q, k, v, b, g, w.ctx, w.scale)
        assert_attention_close(out[b, g * G:(g + 1) * G], exp, f"{name} b{b} g{g}")
    # stored bytes of a few rows per sampled plane
    for which, cache, new, kind in ((0, kc, k, w.k_type), (1, vc, v, w.v_type)):
        lay = kvq.kvq_cache_layout(desc, w.batch, which)
        host = cache.cpu().numpy()
        for b, g in sorted(samples):
            for t0 in (0, w.ctx // 2 + 3, w.ctx - 5):
                codes, scales = rows_of(host, lay, b, g, w.n_kv, t0, t0 + 5)
                ec, es = oracle_rows(kind, new[b, t0:t0 + 5, g, :].cpu().numpy(), w.turbo_seed)
                np.testing.assert_array_equal(codes, ec)
                np.testing.assert_array_equal(scales.view(np.uint16), es.view(np.uint16))
    del kc, vc, k, v
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["llama70b_ctx32k_b4", "turbo3_ctx32k"])
def test_full_size_layer_every_byte_and_output(name):
    """One full-size layer in the benchmark's launch configuration: rows
    0 .. ctx-2 by the bulk append, the last row by the fused decode step
    (automatic splits).  Every stored byte of both caches (70B: 1 M rows per
    tensor) equals the oracle's quantization of the same fp16 rows, and every
    output equals the oracle's decode over the oracle's own cache."""
    from oracle import attention
    w = synth.WORKLOADS[name]
    B, ctx, D, n_kv = w.batch, w.ctx, w.head_dim, w.n_kv
    desc = kvq.make_desc(w.n_q, n_kv, D, w.k_type, w.v_type, ctx, turbo_seed=w.turbo_seed)
    q, k, v = synth.layer_inputs(w, layer=0, device="cuda")
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k[:, :ctx - 1].contiguous(), v[:, :ctx - 1].contiguous(), B, 0, ctx - 1)
    ws = torch.zeros(kvq.kvq_workspace_bytes(desc, B, 0), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, w.n_q, D), dtype=torch.float32, device="cuda")
    kvq.kvq_decode_step(desc, kc, vc, q, k[:, ctx - 1].contiguous(), v[:, ctx - 1].contiguous(), B, ctx, w.scale,
                        0, ws, out)
    torch.cuda.synchronize()
    stored = {}
    for which, cache, x, kind in ((0, kc, k, w.k_type), (1, vc, v, w.v_type)):
        lay = kvq.kvq_cache_layout(desc, B, which)
        host = cache.cpu().numpy()
        T, cb, ns = lay.rows_per_plane, lay.code_bytes, lay.n_scales
        rows = x.cpu().numpy().transpose(0, 2, 1, 3).reshape(-1, D)           # [B * n_kv * ctx, D]
        ec, es = oracle_rows(kind, rows, w.turbo_seed)
        got_c = host[:B * n_kv * T * cb].reshape(B * n_kv, T, cb)[:, :ctx]
        got_s = host[lay.scale_offset:lay.scale_offset + B * n_kv * T * ns * 2].view(np.float16)
        got_s = got_s.reshape(B * n_kv, T, ns)[:, :ctx]
        np.testing.assert_array_equal(got_c, ec.reshape(B * n_kv, ctx, cb), err_msg=f"{name} codes {which}")
        np.testing.assert_array_equal(got_s.view(np.uint16), es.reshape(B * n_kv, ctx, ns).view(np.uint16),
                                      err_msg=f"{name} scales {which}")
        stored[which] = (ec.reshape(B, n_kv, ctx, cb), es.reshape(B, n_kv, ctx, ns))
    del kc, vc, k, v
    expect = attention.decode_cache(w.k_type, w.v_type, *stored[0], *stored[1], q.cpu().numpy(), w.scale,
                                    seed=w.turbo_seed, threads=0)
    assert_attention_close(out.cpu().numpy(), expect, f"{name} every output")
    torch.cuda.empty_cache()
