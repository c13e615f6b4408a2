"""Paged pools (kvq_append_quantize_paged, kvq_decode_attention_paged,
kvq_decode_step_paged) on the GPU.  A pool holds each sequence's rows in pages
listed by a block table; the tests scatter the pages in a seeded random order.
Checked: the pool's pages hold, byte for byte, the rows a contiguous cache holds
at the same logical positions; the paged decode equals the contiguous
per-sequence-length decode bit for bit (same splits, same tiles); the fused
paged step matches the oracle; a block-table entry outside the pool yields NaN
and writes nothing."""

import math

import numpy as np
import pytest
import torch

import decode_attention_q8_b200 as kvq
import synth
from kvq_testlib import SENTINEL, alloc_cache, assert_attention_close, oracle_attention_rows, oracle_dequant, oracle_rows

pytestmark = pytest.mark.gpu

NAMES = {0: "f16", 1: "q8_0", 2: "q4_0", 3: "turbo3", 4: "turbo2", 5: "turbo4", 6: "q5_0", 7: "turbo3_qjl"}


def _inputs(k_type, v_type, B, n_q, n_kv, D, rows, max_ctx, seed):
    proj = synth.qjl_projection(seed + 17, D) if k_type == "turbo3_qjl" else None
    desc = kvq.make_desc(n_q, n_kv, D, k_type, v_type, max_ctx, turbo_seed=seed * 31 + 7,
                         qjl_proj=None if proj is None else proj.cuda())
    desc.qjl_host = None if proj is None else proj.numpy()
    w = synth.Workload("paged", B, 1, n_q, n_kv, D, rows, k_type, v_type, (3, 17), 10.0, seed)
    q, k, v = synth.layer_inputs(w, device="cuda")
    return desc, q, k, v


def _pool(desc, page_rows, n_pages):
    pools = []
    for which in (0, 1):
        n = kvq.kvq_paged_cache_bytes(desc, page_rows, n_pages, which)
        assert n > 0
        pools.append(torch.full((n,), SENTINEL, dtype=torch.uint8, device="cuda"))
    return pools


def _table(B, max_pages, n_pages, seed):
    """Block table with every sequence's pages at distinct, shuffled pool pages."""
    rng = np.random.default_rng(seed)
    ids = rng.permutation(n_pages)[:B * max_pages].astype(np.int32)
    return torch.from_numpy(ids.reshape(B, max_pages)).cuda()


def _pages_equal_contiguous(desc, pools, table, page_rows, n_pages, cont, B, lens):
    """Every page a sequence uses holds the contiguous cache's rows of that page."""
    tab = table.cpu().numpy()
    for which in (0, 1):
        lay_c = kvq.kvq_cache_layout(desc, B, which)
        lay_p = kvq.kvq_paged_layout(desc, page_rows, n_pages, which)
        host_c = cont[which].cpu().numpy()
        host_p = pools[which].cpu().numpy()
        cb, ns, T = lay_c.code_bytes, lay_c.n_scales, lay_c.rows_per_plane
        for b in range(B):
            for j in range((lens[b] + page_rows - 1) // page_rows):
                r0, r1 = j * page_rows, min(lens[b], (j + 1) * page_rows)
                pg = int(tab[b, j])
                for h in range(desc.n_kv_heads):
                    pc = b * desc.n_kv_heads + h
                    pp = pg * desc.n_kv_heads + h
                    o = pp * page_rows * cb
                    np.testing.assert_array_equal(host_p[o:o + (r1 - r0) * cb],
                                                  host_c[(pc * T + r0) * cb:(pc * T + r1) * cb],
                                                  err_msg=f"codes b{b} page {j}")
                    if ns:
                        sa = lay_c.scale_offset + (pc * T + r0) * ns * 2
                        sp = lay_p.scale_offset + pp * page_rows * ns * 2
                        np.testing.assert_array_equal(host_p[sp:sp + (r1 - r0) * ns * 2],
                                                      host_c[sa:sa + (r1 - r0) * ns * 2], err_msg=f"scales b{b}")


@pytest.mark.parametrize("k_type,v_type,page_rows", [("q8_0", "q4_0", 64), ("q8_0", "turbo3", 32),
                                                     ("q4_0", "q4_0", 256), ("f16", "q8_0", 128),
                                                     ("turbo3_qjl", "q4_0", 64)])
def test_paged_equals_contiguous(k_type, v_type, page_rows):
    B, n_q, n_kv, D, rows = 3, 16, 4, 128, 1500
    max_pages = (rows + page_rows - 1) // page_rows
    n_pages = B * max_pages + 5
    desc, q, k, v = _inputs(k_type, v_type, B, n_q, n_kv, D, rows, max_ctx=1536, seed=page_rows)
    table = _table(B, max_pages, n_pages, seed=page_rows)
    pages = kvq.make_paged(table, page_rows, n_pages)
    pools = _pool(desc, page_rows, n_pages)
    full = torch.full((B,), rows, dtype=torch.int32, device="cuda")
    kvq.kvq_append_quantize_paged(desc, pools[0], pools[1], k, v, B, pages, full, rows)
    cont = [alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)]
    kvq.kvq_append_quantize(desc, cont[0], cont[1], k, v, B, 0, rows)
    _pages_equal_contiguous(desc, pools, table, page_rows, n_pages, cont, B, [rows] * B)
    lens = [700, 64, 1500]
    lens_dev = torch.tensor(lens, dtype=torch.int32, device="cuda")
    scale = 1 / math.sqrt(D)
    for S in (0, 5):
        ws = torch.zeros(kvq.kvq_workspace_bytes(desc, B, S), dtype=torch.uint8, device="cuda")
        ref = torch.empty((B, n_q, D), dtype=torch.float32, device="cuda")
        kvq.kvq_decode_attention_varlen(desc, cont[0], cont[1], q, B, lens_dev, rows, scale, S, ws)
        kvq.kvq_combine(desc, ws, B, rows, S, ref)
        got = torch.empty_like(ref)
        ws.zero_()
        kvq.kvq_decode_attention_paged(desc, pools[0], pools[1], q, B, pages, lens_dev, rows, scale, S, ws)
        kvq.kvq_combine(desc, ws, B, rows, S, got)
        assert torch.equal(got, ref), f"S={S}"
    # and one group against the oracle directly
    G = n_q // n_kv
    b, g, n = 0, 1, lens[0]
    kh = oracle_dequant(k_type, *oracle_rows(k_type, k[b, :n, g].cpu().numpy(), desc.turbo_seed, desc.qjl_host), D,
                        desc.turbo_seed, desc.qjl_host)
    vh = oracle_dequant(v_type, *oracle_rows(v_type, v[b, :n, g].cpu().numpy(), desc.turbo_seed), D, desc.turbo_seed)
    assert_attention_close(got.cpu().numpy()[b, g * G:(g + 1) * G],
                           oracle_attention_rows(q[b, g * G:(g + 1) * G].cpu().numpy(), kh, vh, scale), "paged oracle")


def test_step_paged_matches_oracle():
    """The fused step writes each sequence's new row through the block table at
    ctx_lens[b] - 1 and attends rows 0 .. ctx_lens[b]-1 of its pages."""
    B, n_q, n_kv, D, rows, page_rows = 4, 64, 8, 128, 3000, 128
    max_pages = (rows + page_rows - 1) // page_rows
    n_pages = B * max_pages
    for k_type, v_type in (("q8_0", "q4_0"), ("q8_0", "turbo3")):
        desc, q, k, v = _inputs(k_type, v_type, B, n_q, n_kv, D, rows, max_ctx=rows, seed=41)
        table = _table(B, max_pages, n_pages, seed=41)
        pages = kvq.make_paged(table, page_rows, n_pages)
        pools = _pool(desc, page_rows, n_pages)
        kvq.kvq_append_quantize_paged(desc, pools[0], pools[1], k, v, B, pages,
                                      torch.full((B,), rows, dtype=torch.int32, device="cuda"), rows)
        lens = [1, 129, 3000, 2048]
        k2, v2 = k.clone(), v.clone()
        k_new = torch.empty((B, n_kv, D), dtype=torch.float16, device="cuda")
        v_new = torch.empty_like(k_new)
        for b, n in enumerate(lens):
            k_new[b] = -k[b, (n * 3) % rows]
            v_new[b] = v[b, (n * 5) % rows] * 0.25
            k2[b, n - 1], v2[b, n - 1] = k_new[b], v_new[b]
        ws = torch.zeros(kvq.kvq_workspace_bytes(desc, B, 0), dtype=torch.uint8, device="cuda")
        out = torch.empty((B, n_q, D), dtype=torch.float32, device="cuda")
        kvq.kvq_decode_step_paged(desc, pools[0], pools[1], q, k_new, v_new, B, pages,
                                  torch.tensor(lens, dtype=torch.int32, device="cuda"), rows, 1 / math.sqrt(D), 0,
                                  ws, out)
        G = n_q // n_kv
        o = out.cpu().numpy()
        for b, n in enumerate(lens):
            for g in (0, n_kv - 1):
                kh = oracle_dequant(k_type, *oracle_rows(k_type, k2[b, :n, g].cpu().numpy()), D)
                vh = oracle_dequant(v_type, *oracle_rows(v_type, v2[b, :n, g].cpu().numpy(), desc.turbo_seed), D,
                                    desc.turbo_seed)
                assert_attention_close(o[b, g * G:(g + 1) * G],
                                       oracle_attention_rows(q[b, g * G:(g + 1) * G].cpu().numpy(), kh, vh,
                                                             1 / math.sqrt(D)), f"{v_type} b{b} g{g}")
        # the pool now holds k2 / v2: the same bytes a paged append of them writes
        ref = _pool(desc, page_rows, n_pages)
        kvq.kvq_append_quantize_paged(desc, ref[0], ref[1], k2, v2, B, pages,
                                      torch.full((B,), rows, dtype=torch.int32, device="cuda"), rows)
        assert torch.equal(pools[0], ref[0]) and torch.equal(pools[1], ref[1])


def test_long_split_crosses_page_windows():
    """One split over 20000 rows of 32-row pages: each warp walks 78 tiles, so
    its 32-tile windows of page ids are refilled twice."""
    B, n_q, n_kv, D, rows, page_rows = 1, 8, 2, 128, 20000, 32
    max_pages = (rows + page_rows - 1) // page_rows
    n_pages = max_pages + 7
    desc, q, k, v = _inputs("q8_0", "q4_0", B, n_q, n_kv, D, rows, max_ctx=rows, seed=23)
    table = _table(B, max_pages, n_pages, seed=23)
    pages = kvq.make_paged(table, page_rows, n_pages)
    pools = _pool(desc, page_rows, n_pages)
    full = torch.full((B,), rows, dtype=torch.int32, device="cuda")
    kvq.kvq_append_quantize_paged(desc, pools[0], pools[1], k, v, B, pages, full, rows)
    cont = [alloc_cache(desc, B, 0), alloc_cache(desc, B, 1)]
    kvq.kvq_append_quantize(desc, cont[0], cont[1], k, v, B, 0, rows)
    scale = 1 / math.sqrt(D)
    ws = torch.zeros(kvq.kvq_workspace_bytes(desc, B, 1), dtype=torch.uint8, device="cuda")
    ref = torch.empty((B, n_q, D), dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attention_varlen(desc, cont[0], cont[1], q, B, full, rows, scale, 1, ws)
    kvq.kvq_combine(desc, ws, B, rows, 1, ref)
    got = torch.empty_like(ref)
    kvq.kvq_decode_attention_paged(desc, pools[0], pools[1], q, B, pages, full, rows, scale, 1, ws)
    kvq.kvq_combine(desc, ws, B, rows, 1, got)
    assert torch.equal(got, ref)


def test_page_ids_outside_the_pool():
    """A sequence whose block table names a page outside [0, n_pages) gets NaN
    (the other sequences are unaffected), and its appended rows are not
    written."""
    B, n_q, n_kv, D, rows, page_rows = 3, 8, 2, 128, 512, 64
    max_pages = rows // page_rows
    n_pages = B * max_pages
    desc, q, k, v = _inputs("q8_0", "q4_0", B, n_q, n_kv, D, rows, max_ctx=rows, seed=7)
    table = _table(B, max_pages, n_pages, seed=7)
    pages = kvq.make_paged(table, page_rows, n_pages)
    pools = _pool(desc, page_rows, n_pages)
    full = torch.full((B,), rows, dtype=torch.int32, device="cuda")
    kvq.kvq_append_quantize_paged(desc, pools[0], pools[1], k, v, B, pages, full, rows)
    before = [pools[0].clone(), pools[1].clone()]
    bad = table.clone()
    bad[1, 3] = n_pages          # one past the pool
    bad[2, 0] = -1
    bad_pages = kvq.make_paged(bad, page_rows, n_pages)
    lens = torch.tensor([rows, rows, 100], dtype=torch.int32, device="cuda")
    ws = torch.zeros(kvq.kvq_workspace_bytes(desc, B, 0), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, n_q, D), dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attention_paged(desc, pools[0], pools[1], q, B, bad_pages, lens, rows, 1 / math.sqrt(D), 0, ws)
    kvq.kvq_combine(desc, ws, B, rows, 0, out)
    o = out.cpu().numpy()
    assert np.isnan(o[1]).all() and np.isnan(o[2]).all()
    # the workspace's status word names the cause (it started at zero)
    off = kvq.kvq_workspace_status_offset(desc, B)
    assert int(ws[off:off + 4].view(torch.int32).item()) == kvq.STATUS_BAD_PAGE
    G = n_q // n_kv
    for g in range(n_kv):
        kh = oracle_dequant("q8_0", *oracle_rows("q8_0", k[0, :, g].cpu().numpy()), D)
        vh = oracle_dequant("q4_0", *oracle_rows("q4_0", v[0, :, g].cpu().numpy()), D)
        assert_attention_close(o[0, g * G:(g + 1) * G],
                               oracle_attention_rows(q[0, g * G:(g + 1) * G].cpu().numpy(), kh, vh, 1 / math.sqrt(D)),
                               f"good sequence g{g}")
    # appends through the bad entries write nothing: sequence 1's rows 192..255
    # (page 3) and sequence 2's rows 0..63 (page 0)
    kvq.kvq_append_quantize_paged(desc, pools[0], pools[1], k[:, :64].contiguous(), v[:, :64].contiguous(), B,
                                  bad_pages, torch.tensor([64, 256, 64], dtype=torch.int32, device="cuda"), 64)
    # sequence 0 rewrote its own rows 0..63 with the same bytes; nothing else changed
    assert torch.equal(pools[0], before[0]) and torch.equal(pools[1], before[1])
