"""Per-sequence context lengths (kvq_decode_attention_varlen,
kvq_decode_step_varlen, kvq_append_quantize_varlen) on the GPU against the
oracle: batch row b attends its own first ctx_lens[b] rows, each output within
the attention tolerance of the fp64 oracle over exactly those rows; appended
bytes bit-exact at each row's own position; a length out of range touches no
cache byte and yields NaN; a captured graph replayed after the lengths change
on the device follows the new lengths."""

import math

import numpy as np
import pytest
import torch

import decode_attention_q8_b200 as kvq
import synth
from kvq_testlib import alloc_cache, assert_attention_close, oracle_attention_rows, oracle_dequant, oracle_rows, rows_of

pytestmark = pytest.mark.gpu

NAMES = {0: "f16", 1: "q8_0", 2: "q4_0", 3: "turbo3"}


def _inputs(k_type, v_type, B, n_q, n_kv, D, rows, max_ctx, seed):
    desc = kvq.make_desc(n_q, n_kv, D, k_type, v_type, max_ctx, turbo_seed=seed * 31 + 7)
    w = synth.Workload("varlen", B, 1, n_q, n_kv, D, rows, k_type, v_type, (3, 17), 10.0, seed)
    q, k, v = synth.layer_inputs(w, device="cuda")
    return desc, q, k, v


def _oracle(desc, q, k, v, b, g, n):
    """Oracle output of group (b, g) over rows 0 .. n-1 of the fp16 inputs k, v."""
    G = desc.n_q_heads // desc.n_kv_heads
    kt, vt = NAMES[desc.k_type], NAMES[desc.v_type]
    kh = oracle_dequant(kt, *oracle_rows(kt, k[b, :n, g, :].cpu().numpy(), desc.turbo_seed), desc.head_dim,
                        desc.turbo_seed)
    vh = oracle_dequant(vt, *oracle_rows(vt, v[b, :n, g, :].cpu().numpy(), desc.turbo_seed), desc.head_dim,
                        desc.turbo_seed)
    return oracle_attention_rows(q[b, g * G:(g + 1) * G].cpu().numpy(), kh, vh, 1 / math.sqrt(desc.head_dim))


def _check_out(desc, q, k, v, out, lens, max_len, what):
    """Rows with a length in [1, max_len] match the oracle; the others are NaN."""
    G = desc.n_q_heads // desc.n_kv_heads
    o = out.cpu().numpy()
    for b, n in enumerate(lens):
        for g in range(desc.n_kv_heads):
            got = o[b, g * G:(g + 1) * G]
            if 1 <= n <= max_len:
                assert_attention_close(got, _oracle(desc, q, k, v, b, g, n), f"{what} b{b} len {n} g{g}")
            else:
                assert np.isnan(got).all(), f"{what} b{b} len {n}: expected NaN"


def _decode_varlen(desc, kc, vc, q, lens_dev, max_len, S, B):
    ws = torch.zeros(kvq.kvq_workspace_bytes(desc, B, S), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, desc.n_q_heads, desc.head_dim), dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attention_varlen(desc, kc, vc, q, B, lens_dev, max_len, 1 / math.sqrt(desc.head_dim), S, ws)
    kvq.kvq_combine(desc, ws, B, max_len, S, out)
    return out


@pytest.mark.parametrize("k_type,v_type", [("q8_0", "q4_0"), ("q4_0", "q4_0"), ("q8_0", "turbo3"),
                                           ("f16", "f16"), ("q8_0", "q8_0")])
def test_decode_varlen_matches_oracle_per_row(k_type, v_type):
    """Ragged lengths across several 32-row tiles and splits: 1 row, a partial
    tile, a split boundary, the bound itself; automatic and explicit splits."""
    B, n_q, n_kv, D, max_len = 5, 16, 4, 128, 1200
    desc, q, k, v = _inputs(k_type, v_type, B, n_q, n_kv, D, max_len, max_ctx=1300, seed=71)
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k, v, B, 0, max_len)
    lens = [1, 37, 300, 1200, 817]
    lens_dev = torch.tensor(lens, dtype=torch.int32, device="cuda")
    for S in (0, 1, 7, 40):
        out = _decode_varlen(desc, kc, vc, q, lens_dev, max_len, S, B)
        _check_out(desc, q, k, v, out, lens, max_len, f"{k_type}/{v_type} S={S}")


def test_decode_varlen_equal_lengths_equal_uniform_decode():
    """Every length = ctx: the same splits and chunks as kvq_decode_attention,
    so the outputs agree bit for bit."""
    B, n_q, n_kv, D, ctx = 3, 64, 8, 128, 2000
    desc, q, k, v = _inputs("q8_0", "q4_0", B, n_q, n_kv, D, ctx, max_ctx=2048, seed=5)
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k, v, B, 0, ctx)
    for S in (0, 6):
        ws = torch.zeros(kvq.kvq_workspace_bytes(desc, B, S), dtype=torch.uint8, device="cuda")
        ref = torch.empty((B, n_q, D), dtype=torch.float32, device="cuda")
        kvq.kvq_decode_attention(desc, kc, vc, q, B, ctx, 1 / math.sqrt(D), S, ws)
        kvq.kvq_combine(desc, ws, B, ctx, S, ref)
        got = _decode_varlen(desc, kc, vc, q, torch.full((B,), ctx, dtype=torch.int32, device="cuda"), ctx, S, B)
        assert torch.equal(got, ref), f"S={S}"


def test_decode_varlen_out_of_range_lengths_give_nan_and_leave_others_alone():
    B, n_q, n_kv, D, max_len = 4, 8, 2, 64, 500
    desc, q, k, v = _inputs("q8_0", "q4_0", B, n_q, n_kv, D, max_len, max_ctx=512, seed=9)
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k, v, B, 0, max_len)
    lens = [0, 250, max_len + 1, -3]
    out = _decode_varlen(desc, kc, vc, q, torch.tensor(lens, dtype=torch.int32, device="cuda"), max_len, 0, B)
    _check_out(desc, q, k, v, out, lens, max_len, "out of range")


def test_append_varlen_writes_each_row_at_its_own_position():
    """n_tok = 3 rows per sequence at lens[b] - 3 .. lens[b] - 1; bytes equal
    the oracle's; a sequence whose length is below n_tok or above max_ctx is
    not written (its sentinel bytes stay)."""
    B, n_q, n_kv, D, max_ctx, n_tok = 5, 8, 2, 128, 256, 3
    for k_type, v_type in (("q8_0", "q4_0"), ("f16", "turbo3"), ("q4_0", "q8_0")):
        desc, q, k, v = _inputs(k_type, v_type, B, n_q, n_kv, D, n_tok, max_ctx=max_ctx, seed=13)
        kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
        lens = [3, 100, 256, 2, 257]
        kvq.kvq_append_quantize_varlen(desc, kc, vc, k, v, B, torch.tensor(lens, dtype=torch.int32, device="cuda"),
                                       n_tok)
        for which, cache, x, kind in ((0, kc, k, k_type), (1, vc, v, v_type)):
            lay = kvq.kvq_cache_layout(desc, B, which)
            host = cache.cpu().numpy()
            written = np.zeros(host.shape, bool)
            for b, n in enumerate(lens):
                for g in range(n_kv):
                    if not (n_tok <= n <= max_ctx):
                        continue
                    codes, scales = rows_of(host, lay, b, g, n_kv, n - n_tok, n)
                    ec, es = oracle_rows(kind, x[b, :, g, :].cpu().numpy(), desc.turbo_seed)
                    np.testing.assert_array_equal(codes, ec, err_msg=f"{kind} codes b{b} g{g}")
                    np.testing.assert_array_equal(scales.view(np.uint16), es.view(np.uint16),
                                                  err_msg=f"{kind} scales b{b} g{g}")
                    plane = b * n_kv + g
                    T, cb, ns = lay.rows_per_plane, lay.code_bytes, lay.n_scales
                    written[(plane * T + n - n_tok) * cb:(plane * T + n) * cb] = True
                    so = lay.scale_offset + (plane * T + n - n_tok) * ns * 2
                    written[so:so + n_tok * ns * 2] = True
            assert (host[~written] == 0xA5).all(), f"{kind}: bytes outside the appended rows changed"


def test_step_varlen_appends_and_attends_per_row():
    """Each sequence has rows 0 .. lens[b]-2 cached; the fused step writes row
    lens[b]-1 from k_new / v_new and attends rows 0 .. lens[b]-1."""
    B, n_q, n_kv, D, max_len = 4, 64, 8, 128, 3000
    for k_type, v_type in (("q8_0", "q4_0"), ("q8_0", "turbo3"), ("q4_0", "q4_0")):
        desc, q, k, v = _inputs(k_type, v_type, B, n_q, n_kv, D, max_len, max_ctx=3072, seed=29)
        lens = [1, 33, 3000, 1500]
        kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
        kvq.kvq_append_quantize(desc, kc, vc, k, v, B, 0, max_len)  # rows 0 .. max_len-1 of k, v
        # the new rows: row lens[b]-1 of each sequence, written over by the step
        k2, v2 = k.clone(), v.clone()
        k_new = torch.empty((B, n_kv, D), dtype=torch.float16, device="cuda")
        v_new = torch.empty_like(k_new)
        for b, n in enumerate(lens):
            k_new[b] = -k[b, (n * 7) % max_len]
            v_new[b] = v[b, (n * 11) % max_len] * 0.5
            k2[b, n - 1], v2[b, n - 1] = k_new[b], v_new[b]
        for S in (0, 5):
            ws = torch.zeros(kvq.kvq_workspace_bytes(desc, B, S), dtype=torch.uint8, device="cuda")
            out = torch.empty((B, n_q, D), dtype=torch.float32, device="cuda")
            kvq.kvq_decode_step_varlen(desc, kc, vc, q, k_new, v_new, B,
                                       torch.tensor(lens, dtype=torch.int32, device="cuda"), max_len,
                                       1 / math.sqrt(D), S, ws, out)
            _check_out(desc, q, k2, v2, out, lens, max_len, f"{k_type}/{v_type} S={S}")
            assert not ws[:4 * B * n_kv].cpu().numpy().any()
        # the cache now holds k2 / v2: the same bytes a uniform append of them writes
        kr, vr = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
        kvq.kvq_append_quantize(desc, kr, vr, k2, v2, B, 0, max_len)
        assert torch.equal(kc, kr) and torch.equal(vc, vr)


def test_step_varlen_out_of_range_length_writes_nothing():
    B, n_q, n_kv, D, max_len = 3, 8, 2, 128, 400
    desc, q, k, v = _inputs("q8_0", "q4_0", B, n_q, n_kv, D, max_len, max_ctx=400, seed=3)
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k, v, B, 0, max_len)
    k_ref, v_ref = kc.clone(), vc.clone()
    lens = [0, 401, 200]
    k_new = torch.zeros((B, n_kv, D), dtype=torch.float16, device="cuda")
    ws = torch.zeros(kvq.kvq_workspace_bytes(desc, B, 0), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, n_q, D), dtype=torch.float32, device="cuda")
    kvq.kvq_decode_step_varlen(desc, kc, vc, q, k_new, k_new, B, torch.tensor(lens, dtype=torch.int32, device="cuda"),
                               max_len, 1 / math.sqrt(D), 0, ws, out)
    k2, v2 = k.clone(), v.clone()
    k2[2, 199], v2[2, 199] = 0, 0
    _check_out(desc, q, k2, v2, out, lens, max_len, "step out of range")
    # only sequence 2's row 199 changed
    kvq.kvq_append_quantize_varlen(desc, k_ref, v_ref, k_new[:, None], k_new[:, None], B,
                                   torch.tensor([0, 0, 200], dtype=torch.int32, device="cuda"), 1)
    assert torch.equal(kc, k_ref) and torch.equal(vc, v_ref)


def test_graph_replay_follows_device_lengths():
    """One captured graph of the fused step, replayed three times while a
    device-side increment grows every length by one: each replay appends at
    the new end and attends the new length."""
    B, n_q, n_kv, D, max_len = 3, 32, 8, 128, 2048
    desc, q, k, v = _inputs("q8_0", "q4_0", B, n_q, n_kv, D, max_len, max_ctx=max_len, seed=17)
    start = [100, 1000, 1900]
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k, v, B, 0, max_len)
    lens = torch.tensor(start, dtype=torch.int32, device="cuda")
    k_new = torch.empty((B, n_kv, D), dtype=torch.float16, device="cuda")
    v_new = torch.empty_like(k_new)
    ws = torch.zeros(kvq.kvq_workspace_bytes(desc, B, 0), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, n_q, D), dtype=torch.float32, device="cuda")
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        kvq.kvq_decode_step_varlen(desc, kc, vc, q, k_new, v_new, B, lens, max_len, 1 / math.sqrt(D), 0, ws, out,
                                   stream=stream)
    k2, v2 = k.clone(), v.clone()
    for step in range(3):
        cur = [n + step for n in start]
        lens.copy_(torch.tensor(cur, dtype=torch.int32))
        for b, n in enumerate(cur):
            k_new[b] = k[b, n - 1] * -1.0
            v_new[b] = v[b, (n + 5) % max_len]
            k2[b, n - 1], v2[b, n - 1] = k_new[b], v_new[b]
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        _check_out(desc, q, k2, v2, out, cur, max_len, f"replay {step}")
    del g
