"""Fused decode step (kvq_decode_step: append one row, decode, combine in one
launch) on the GPU against the oracle: the appended row's bytes bit-exact, the
other rows untouched, the output within the attention tolerance of the fp64
oracle over all ctx_len rows (the new one included)."""

import math

import numpy as np
import pytest
import torch

import decode_attention_q8_b200 as kvq
import synth
from kvq_testlib import (alloc_cache, assert_attention_close, decode, oracle_attention_rows, oracle_dequant,
                         oracle_rows, rows_of)

pytestmark = pytest.mark.gpu

NAMES = {0: "f16", 1: "q8_0", 2: "q4_0", 3: "turbo3", 4: "turbo2", 5: "turbo4", 6: "q5_0", 7: "turbo3_qjl"}


def _inputs(k_type, v_type, B, n_q, n_kv, D, ctx, seed, max_ctx=None, turbo_seed=None):
    proj = synth.qjl_projection(seed + 13, D) if k_type == "turbo3_qjl" else None
    desc = kvq.make_desc(n_q, n_kv, D, k_type, v_type, max_ctx or ctx,
                         turbo_seed=(seed * 31 + 7) if turbo_seed is None else turbo_seed,
                         qjl_proj=None if proj is None else proj.cuda())
    desc.qjl_host = None if proj is None else proj.numpy()
    w = synth.Workload("case", B, 1, n_q, n_kv, D, ctx, k_type, v_type, (3, 17), 10.0, seed)
    q, k, v = synth.layer_inputs(w, device="cuda")
    return desc, q, k, v


def _workspace(desc, B, S):
    # the counter words must be zero before the first fused call with this workspace
    return torch.zeros(kvq.kvq_workspace_bytes(desc, B, S), dtype=torch.uint8, device="cuda")


def _step(desc, kc, vc, q, k, v, B, ctx, scale, S, ws):
    """Fused step appending row ctx-1 (taken from k, v) and attending over ctx rows."""
    out = torch.empty((B, desc.n_q_heads, desc.head_dim), dtype=torch.float32, device="cuda")
    k_new = k[:, ctx - 1].contiguous()
    v_new = v[:, ctx - 1].contiguous()
    kvq.kvq_decode_step(desc, kc, vc, q, k_new, v_new, B, ctx, scale, S, ws, out)
    return out


def _oracle(desc, q, k, v, b, g, ctx, scale):
    G = desc.n_q_heads // desc.n_kv_heads
    kt, vt = NAMES[desc.k_type], NAMES[desc.v_type]
    proj = getattr(desc, "qjl_host", None)
    kh = oracle_dequant(kt, *oracle_rows(kt, k[b, :ctx, g, :].cpu().numpy(), desc.turbo_seed, proj),
                        desc.head_dim, desc.turbo_seed, proj)
    vh = oracle_dequant(vt, *oracle_rows(vt, v[b, :ctx, g, :].cpu().numpy(), desc.turbo_seed), desc.head_dim,
                        desc.turbo_seed)
    return oracle_attention_rows(q[b, g * G:(g + 1) * G].cpu().numpy(), kh, vh, scale)


def _check_out(desc, q, k, v, out, ctx, scale, what, groups=None):
    G = desc.n_q_heads // desc.n_kv_heads
    o = out.cpu().numpy()
    groups = groups or [(b, g) for b in range(q.shape[0]) for g in range(desc.n_kv_heads)]
    for b, g in groups:
        assert_attention_close(o[b, g * G:(g + 1) * G], _oracle(desc, q, k, v, b, g, ctx, scale), f"{what} b{b} g{g}")


def _check_row_bytes(desc, kc, vc, k, v, B, row, what):
    for which, cache, x, kind in ((0, kc, k, NAMES[desc.k_type]), (1, vc, v, NAMES[desc.v_type])):
        lay = kvq.kvq_cache_layout(desc, B, which)
        host = cache.cpu().numpy()
        for b in range(B):
            for g in range(desc.n_kv_heads):
                codes, scales = rows_of(host, lay, b, g, desc.n_kv_heads, row, row + 1)
                ec, es = oracle_rows(kind, x[b, row:row + 1, g, :].cpu().numpy(), desc.turbo_seed,
                                     getattr(desc, "qjl_host", None))
                np.testing.assert_array_equal(codes, ec, err_msg=f"{what} {kind} codes b{b} g{g}")
                np.testing.assert_array_equal(scales.view(np.uint16), es.view(np.uint16),
                                              err_msg=f"{what} {kind} scales b{b} g{g}")


def _pairs():
    plain = [(k, v) for k in ("f16", "q8_0", "q4_0", "q5_0")
             for v in ("f16", "q8_0", "q4_0", "turbo3", "turbo2", "turbo4", "q5_0")]
    turbo_keys = [(k, v) for k in ("turbo2", "turbo3", "turbo4") for v in ("q8_0", "q4_0", k)]
    qjl_keys = [("turbo3_qjl", v) for v in ("q8_0", "q4_0", "turbo3")]
    return plain + turbo_keys + qjl_keys


@pytest.mark.parametrize("k_type,v_type", _pairs())
def test_type_matrix(k_type, v_type):
    """Rows 0 .. ctx-2 prefilled by kvq_append_quantize; the step writes row
    ctx-1 (over sentinel bytes) and attends over all ctx rows."""
    B, n_q, n_kv, D, ctx = 2, 16, 4, 128, 1000
    desc, q, k, v = _inputs(k_type, v_type, B, n_q, n_kv, D, ctx, seed=43, max_ctx=1100)
    scale = 1 / math.sqrt(D)
    for S in (0, 3):
        kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
        kvq.kvq_append_quantize(desc, kc, vc, k[:, :ctx - 1].contiguous(), v[:, :ctx - 1].contiguous(), B, 0, ctx - 1)
        k_ref, v_ref = kc.clone(), vc.clone()
        ws = _workspace(desc, B, S)
        out = _step(desc, kc, vc, q, k, v, B, ctx, scale, S, ws)
        _check_row_bytes(desc, kc, vc, k, v, B, ctx - 1, f"{k_type}/{v_type} S={S}")
        # every other byte is as the plain append left it: the same as appending row ctx-1 there
        kvq.kvq_append_quantize(desc, k_ref, v_ref, k[:, ctx - 1:ctx].contiguous(), v[:, ctx - 1:ctx].contiguous(),
                                B, ctx - 1, 1)
        assert torch.equal(kc, k_ref) and torch.equal(vc, v_ref)
        _check_out(desc, q, k, v, out, ctx, scale, f"{k_type}/{v_type} S={S}")
        # the arrival counters (the workspace's first B * n_kv words) are back to zero
        assert not ws[:4 * B * n_kv].cpu().numpy().any()


def test_new_row_is_read_in_the_same_launch():
    """The new key is twice the first query head of each group (score about
    2 |q|^2 / sqrt(D), some 22 above the rest), so that head's output is the
    new value row: a decode that read the row's previous (sentinel) bytes
    would miss it."""
    B, n_q, n_kv, D, ctx = 2, 8, 2, 128, 700
    desc, q, k, v = _inputs("q8_0", "q4_0", B, n_q, n_kv, D, ctx, seed=11)
    G = n_q // n_kv
    for b in range(B):
        for g in range(n_kv):
            k[b, ctx - 1, g] = (q[b, g * G].float() * 2.0).half()
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k[:, :ctx - 1].contiguous(), v[:, :ctx - 1].contiguous(), B, 0, ctx - 1)
    scale = 1 / math.sqrt(D)
    for S in (0, 1, 5):
        ws = _workspace(desc, B, S)
        out = _step(desc, kc, vc, q, k, v, B, ctx, scale, S, ws)
        _check_out(desc, q, k, v, out, ctx, scale, f"dominant new row S={S}")
        vh = oracle_dequant("q4_0", *oracle_rows("q4_0", v[:, ctx - 1].reshape(-1, D).cpu().numpy()), D)
        o = out.cpu().numpy()
        for b in range(B):
            for g in range(n_kv):
                assert np.abs(o[b, g * G] - vh[b * n_kv + g]).max() < 2e-3


@pytest.mark.parametrize("ctx", [1, 2, 17, 33, 257])
def test_short_contexts(ctx):
    """ctx_len = 1: the new row is the whole context (output = its value row)."""
    desc, q, k, v = _inputs("q8_0", "turbo3", 1, 8, 2, 128, ctx, seed=ctx + 100, max_ctx=300)
    kc, vc = alloc_cache(desc, 1, 0), alloc_cache(desc, 1, 1)
    if ctx > 1:
        kvq.kvq_append_quantize(desc, kc, vc, k[:, :ctx - 1].contiguous(), v[:, :ctx - 1].contiguous(), 1, 0, ctx - 1)
    ws = _workspace(desc, 1, 0)
    out = _step(desc, kc, vc, q, k, v, 1, ctx, 0.09, 0, ws)
    _check_row_bytes(desc, kc, vc, k, v, 1, ctx - 1, f"ctx={ctx}")
    _check_out(desc, q, k, v, out, ctx, 0.09, f"ctx={ctx}")


@pytest.mark.parametrize("G", [1, 3, 8, 16])
@pytest.mark.parametrize("D", [64, 256])
def test_group_sizes_and_head_dims(G, D):
    desc, q, k, v = _inputs("q4_0", "q8_0", 2, 2 * G, 2, D, 300, seed=G + D)
    kc, vc = alloc_cache(desc, 2, 0), alloc_cache(desc, 2, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k[:, :299].contiguous(), v[:, :299].contiguous(), 2, 0, 299)
    ws = _workspace(desc, 2, 0)
    out = _step(desc, kc, vc, q, k, v, 2, 300, 1 / math.sqrt(D), 0, ws)
    _check_row_bytes(desc, kc, vc, k, v, 2, 299, f"G={G} D={D}")
    _check_out(desc, q, k, v, out, 300, 1 / math.sqrt(D), f"G={G} D={D}")


def test_consecutive_steps_share_a_workspace():
    """Token after token on one stream: each step appends its row and sees all
    earlier ones; the arrival counters return to zero after every call, also
    when the split count changes from one call to the next."""
    B, n_q, n_kv, D, ctx0 = 1, 16, 4, 128, 500
    desc, q, k, v = _inputs("q8_0", "q4_0", B, n_q, n_kv, D, ctx0 + 40, seed=5)
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k[:, :ctx0].contiguous(), v[:, :ctx0].contiguous(), B, 0, ctx0)
    ws = _workspace(desc, B, 7)  # large enough for every split count used below
    scale = 1 / math.sqrt(D)
    outs = []
    for i, S in enumerate((0, 0, 2, 7, 0)):
        ctx = ctx0 + 1 + i
        outs.append((ctx, _step(desc, kc, vc, q, k, v, B, ctx, scale, S, ws)))
    torch.cuda.synchronize()
    for ctx, out in outs[::2]:
        _check_out(desc, q, k, v, out, ctx, scale, f"step ctx={ctx}")
    assert not ws[:4 * B * n_kv].cpu().numpy().any()  # the counters: the first B * n_kv words
    # the same rows through the separate calls give the same output within fp32 rounding
    ctx, out = outs[-1]
    ref = decode(desc, kc, vc, q, B, ctx, scale)
    assert torch.allclose(out, ref, atol=2e-4, rtol=0)


@pytest.mark.parametrize("name", ["llama70b_ctx32k_b4", "turbo3_ctx32k", "k4v4_ctx128k_b1"])
def test_full_size_sampled(name):
    """One layer at full size in the benchmark's launch configuration: the step
    appends the last row over a cache holding the first ctx-1; sampled
    (batch row, KV head) groups are checked against the oracle."""
    w = synth.WORKLOADS[name]
    desc = kvq.make_desc(w.n_q, w.n_kv, w.head_dim, w.k_type, w.v_type, w.ctx, turbo_seed=w.turbo_seed)
    q, k, v = synth.layer_inputs(w, layer=0, device="cuda")
    kc, vc = alloc_cache(desc, w.batch, 0), alloc_cache(desc, w.batch, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k[:, :w.ctx - 1].contiguous(), v[:, :w.ctx - 1].contiguous(), w.batch, 0,
                            w.ctx - 1)
    ws = _workspace(desc, w.batch, 0)
    out = _step(desc, kc, vc, q, k, v, w.batch, w.ctx, w.scale, 0, ws)
    samples = sorted({(0, 0), (w.batch - 1, w.n_kv - 1), (w.batch // 2, w.n_kv // 2)})
    _check_out(desc, q, k, v, out, w.ctx, w.scale, name, groups=samples)
    for which, cache, x, kind in ((0, kc, k, w.k_type), (1, vc, v, w.v_type)):
        lay = kvq.kvq_cache_layout(desc, w.batch, which)
        host = cache.cpu().numpy()
        for b, g in samples:
            codes, scales = rows_of(host, lay, b, g, w.n_kv, w.ctx - 1, w.ctx)
            ec, es = oracle_rows(kind, x[b, w.ctx - 1:w.ctx, g, :].cpu().numpy(), w.turbo_seed)
            np.testing.assert_array_equal(codes, ec)
            np.testing.assert_array_equal(scales.view(np.uint16), es.view(np.uint16))
    del kc, vc, k, v
    torch.cuda.empty_cache()


@pytest.mark.parametrize("S", [33, 100, 300])
def test_many_splits_and_empty_ones(S):
    """More than 32 splits (the in-kernel combine takes the weights 32 at a
    time) and, at S = 300 over 3000 rows, trailing splits left empty by the
    32-row chunk rounding (weight 0)."""
    B, n_q, n_kv, D, ctx = 1, 8, 2, 128, 3000
    desc, q, k, v = _inputs("q8_0", "turbo3", B, n_q, n_kv, D, ctx, seed=S)
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k[:, :ctx - 1].contiguous(), v[:, :ctx - 1].contiguous(), B, 0, ctx - 1)
    ws = _workspace(desc, B, S)
    out = _step(desc, kc, vc, q, k, v, B, ctx, 0.09, S, ws)
    _check_out(desc, q, k, v, out, ctx, 0.09, f"S={S}")
    assert not ws[:4 * B * n_kv].cpu().numpy().any()


@pytest.mark.parametrize("B,n_q,n_kv", [(1, 64, 8), (1, 16, 1), (2, 48, 4), (64, 32, 8)])
def test_combine_shared_by_the_last_arrivals(B, n_q, n_kv):
    """With many (head, split) partials per group the last arrivals share the
    combine, a share of the G heads each (at batch 64 the waiting CTAs would
    hold too many slots, so one CTA combines): every head matches the oracle,
    whatever value the epoch words held before, over consecutive calls on one
    workspace, with automatic and with 40 explicit splits."""
    D, ctx = 128, 16384
    desc, q, k, v = _inputs("q8_0", "q4_0", B, n_q, n_kv, D, ctx, seed=B + n_q)
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k[:, :ctx - 1].contiguous(), v[:, :ctx - 1].contiguous(), B, 0, ctx - 1)
    scale = 1 / math.sqrt(D)
    groups = [(b, g) for b in range(B) for g in range(n_kv)]
    if B > 4:
        groups = [(0, 0), (B // 2, 3), (B - 1, n_kv - 1)]
    for S in (0, 40):
        ws = _workspace(desc, B, S)
        words = ws.view(torch.int32)
        words[B * n_kv:2 * B * n_kv] = torch.randint(-2**31, 2**31 - 1, (B * n_kv,), dtype=torch.int32,
                                                     device="cuda")
        for call in range(2):
            out = _step(desc, kc, vc, q, k, v, B, ctx, scale, S, ws)
            _check_out(desc, q, k, v, out, ctx, scale, f"B{B} G{n_q // n_kv} S={S} call {call}", groups=groups)
            assert not ws[:4 * B * n_kv].cpu().numpy().any()


def test_missing_arrival_times_out_to_nan():
    """Failure detection without a fault: group 0's arrival counter is left
    outside [0, S) (the contract asks for 0), so no CTA of that group becomes
    its last arrival.  The CTAs that would share its combine wait for an epoch
    bump that never comes; each wait gives up after its bound (about 2 s) and
    writes NaN for its heads and sets the combine-wait bit of the workspace's
    status word.  The other groups are unaffected, and the GPU context stays
    usable: the next call on a zeroed workspace is correct, with status 0."""
    import time
    B, n_q, n_kv, D, ctx, S = 1, 64, 8, 128, 16384, 40   # 8 heads x 40 splits: several CTAs combine
    desc, q, k, v = _inputs("q8_0", "q4_0", B, n_q, n_kv, D, ctx, seed=17)
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k[:, :ctx - 1].contiguous(), v[:, :ctx - 1].contiguous(), B, 0, ctx - 1)
    scale = 1 / math.sqrt(D)
    good = _step(desc, kc, vc, q, k, v, B, ctx, scale, S, _workspace(desc, B, S))
    ws = _workspace(desc, B, S)
    ws.view(torch.int32)[0] = -1                      # group (0, 0): counter 0xffffffff
    out = torch.full((B, n_q, D), 12345.0, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.time()
    kvq.kvq_decode_step(desc, kc, vc, q, k[:, ctx - 1].contiguous(), v[:, ctx - 1].contiguous(), B, ctx, scale, S,
                        ws, out)
    torch.cuda.synchronize()
    waited = time.time() - t0
    G = n_q // n_kv
    o = out.cpu().numpy()
    g0 = o[0, :G]
    nan_heads = [h for h in range(G) if np.isnan(g0[h]).all()]
    untouched = [h for h in range(G) if (g0[h] == 12345.0).all()]
    assert nan_heads and sorted(nan_heads + untouched) == list(range(G)), (nan_heads, untouched)
    assert waited > 1.0, waited
    assert torch.equal(out[:, G:], good[:, G:])       # the other groups
    off = kvq.kvq_workspace_status_offset(desc, B)
    assert int(ws[off:off + 4].view(torch.int32).item()) == kvq.STATUS_COMBINE_WAIT
    # the context is usable: a fresh workspace gives the right output again
    ws2 = _workspace(desc, B, S)
    again = _step(desc, kc, vc, q, k, v, B, ctx, scale, S, ws2)
    assert torch.equal(again, good)
    assert int(ws2[off:off + 4].view(torch.int32).item()) == 0
