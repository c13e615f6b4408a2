"""Context split across ranks (kvq_partials_region, kvq_combine_ranks) on one
GPU: the ranks are emulated in one process, each with a cache holding only its
slice of the rows, decoding it with the same split count; their partial regions
are laid back to back as an all-gather leaves them, and the combine of all of
them is checked against the oracle over every row and against one decode of
the whole cache."""

import math

import numpy as np
import pytest
import torch

import decode_attention_q8_b200 as kvq
import synth
from kvq_testlib import alloc_cache, assert_attention_close, decode, oracle_attention_rows, oracle_dequant, oracle_rows

pytestmark = pytest.mark.gpu

NAMES = {0: "f16", 1: "q8_0", 2: "q4_0", 3: "turbo3", 4: "turbo2", 5: "turbo4", 6: "q5_0"}


def _inputs(k_type, v_type, B, n_q, n_kv, D, ctx, seed):
    desc = kvq.make_desc(n_q, n_kv, D, k_type, v_type, ctx, turbo_seed=seed * 13 + 5)
    w = synth.Workload("split", B, 1, n_q, n_kv, D, ctx, k_type, v_type, (3, 17), 10.0, seed)
    q, k, v = synth.layer_inputs(w, device="cuda")
    return desc, q, k, v


def _rank_partials(desc, q, k, v, B, bounds, S, scale, lens=None):
    """Each rank's partial region after decoding rows [lo, hi) of every sequence
    (or, with lens, rows [lo, min(hi, lens[b])) of sequence b), back to back."""
    off, n = kvq.kvq_partials_region(desc, B, S)
    regions = []
    for lo, hi in bounds:
        local = kvq.make_desc(desc.n_q_heads, desc.n_kv_heads, desc.head_dim, desc.k_type, desc.v_type, hi - lo,
                              turbo_seed=desc.turbo_seed)
        kc, vc = alloc_cache(local, B, 0), alloc_cache(local, B, 1)
        kvq.kvq_append_quantize(local, kc, vc, k[:, lo:hi].contiguous(), v[:, lo:hi].contiguous(), B, 0, hi - lo)
        ws = torch.zeros(kvq.kvq_workspace_bytes(local, B, S), dtype=torch.uint8, device="cuda")
        assert kvq.kvq_partials_region(local, B, S) == (off, n)  # same layout on every rank
        if lens is None:
            kvq.kvq_decode_attention(local, kc, vc, q, B, hi - lo, scale, S, ws)
        else:
            here = torch.tensor([max(0, min(hi, L) - lo) for L in lens], dtype=torch.int32, device="cuda")
            kvq.kvq_decode_attention_varlen(local, kc, vc, q, B, here, hi - lo, scale, S, ws)
        regions.append(ws[off:off + n])
    return torch.cat(regions)


def _oracle(desc, q, k, v, b, g, n, scale):
    G = desc.n_q_heads // desc.n_kv_heads
    kt, vt = NAMES[desc.k_type], NAMES[desc.v_type]
    kh = oracle_dequant(kt, *oracle_rows(kt, k[b, :n, g].cpu().numpy(), desc.turbo_seed), desc.head_dim,
                        desc.turbo_seed)
    vh = oracle_dequant(vt, *oracle_rows(vt, v[b, :n, g].cpu().numpy(), desc.turbo_seed), desc.head_dim,
                        desc.turbo_seed)
    return oracle_attention_rows(q[b, g * G:(g + 1) * G].cpu().numpy(), kh, vh, scale)


@pytest.mark.parametrize("k_type,v_type", [("q8_0", "q4_0"), ("q8_0", "turbo3"), ("q4_0", "q4_0")])
@pytest.mark.parametrize("bounds", [[(0, 1000), (1000, 2000)], [(0, 33), (33, 900), (900, 1400), (1400, 2000)]])
def test_ranks_combine_to_the_whole_decode(k_type, v_type, bounds):
    B, n_q, n_kv, D, ctx, S = 2, 16, 4, 128, 2000, 6
    desc, q, k, v = _inputs(k_type, v_type, B, n_q, n_kv, D, ctx, seed=len(bounds))
    scale = 1 / math.sqrt(D)
    parts = _rank_partials(desc, q, k, v, B, bounds, S, scale)
    out = torch.empty((B, n_q, D), dtype=torch.float32, device="cuda")
    kvq.kvq_combine_ranks(desc, parts, len(bounds), B, S, out)
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k, v, B, 0, ctx)
    whole = decode(desc, kc, vc, q, B, ctx, scale)
    assert torch.allclose(out, whole, atol=2e-4, rtol=0)  # same rows, another merge order
    G = n_q // n_kv
    o = out.cpu().numpy()
    for b in range(B):
        for g in range(n_kv):
            assert_attention_close(o[b, g * G:(g + 1) * G], _oracle(desc, q, k, v, b, g, ctx, scale),
                                   f"{k_type}/{v_type} {len(bounds)} ranks b{b} g{g}")


def test_ranks_without_rows_of_a_sequence():
    """Per-sequence lengths: sequence 1 ends inside rank 0's rows, so the other
    ranks hold none of its rows (empty partials, weight 0)."""
    B, n_q, n_kv, D, ctx, S = 3, 8, 2, 128, 1500, 4
    desc, q, k, v = _inputs("q8_0", "q4_0", B, n_q, n_kv, D, ctx, seed=9)
    bounds = [(0, 500), (500, 1000), (1000, 1500)]
    lens = [1500, 321, 1001]
    scale = 1 / math.sqrt(D)
    parts = _rank_partials(desc, q, k, v, B, bounds, S, scale, lens=lens)
    out = torch.empty((B, n_q, D), dtype=torch.float32, device="cuda")
    kvq.kvq_combine_ranks(desc, parts, len(bounds), B, S, out)
    G = n_q // n_kv
    o = out.cpu().numpy()
    for b, n in enumerate(lens):
        for g in range(n_kv):
            assert_attention_close(o[b, g * G:(g + 1) * G], _oracle(desc, q, k, v, b, g, n, scale),
                                   f"b{b} len {n} g{g}")


def test_one_rank_equals_combine():
    """With one rank the rank combine is the plain combine, bit for bit."""
    B, n_q, n_kv, D, ctx, S = 2, 16, 4, 128, 700, 5
    desc, q, k, v = _inputs("q8_0", "turbo3", B, n_q, n_kv, D, ctx, seed=2)
    kc, vc = alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k, v, B, 0, ctx)
    ws = torch.zeros(kvq.kvq_workspace_bytes(desc, B, S), dtype=torch.uint8, device="cuda")
    kvq.kvq_decode_attention(desc, kc, vc, q, B, ctx, 0.1, S, ws)
    a = torch.empty((B, n_q, D), dtype=torch.float32, device="cuda")
    b_ = torch.empty_like(a)
    kvq.kvq_combine(desc, ws, B, ctx, S, a)
    off, n = kvq.kvq_partials_region(desc, B, S)
    kvq.kvq_combine_ranks(desc, ws[off:off + n].clone(), 1, B, S, b_)
    assert torch.equal(a, b_)
