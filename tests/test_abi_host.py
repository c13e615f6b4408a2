"""Host-side tests of the C ABI: the library loads, exports what include/kvq.h
declares, and its size / layout / turbo3 constants / argument checks behave.
No GPU: nothing here launches a kernel (every call below is rejected or answered
on the host)."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import decode_attention_q8_b200 as kvq
from oracle import cache_model, turbo, turbo3
from conftest import ROOT, read_golden

HEADER = os.path.join(ROOT, "include", "kvq.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", src)))


def test_exports_every_declared_symbol():
    names = _declared()
    assert len(names) == len(kvq.EXPORTED) and set(names) == set(kvq.EXPORTED)
    dyn = subprocess.run(["nm", "-D", "--defined-only", kvq.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (kvq_\w+)", dyn))
    for n in names:
        assert n in exported, n
        assert getattr(kvq._lib, n) is not None
    # nothing else leaks out under the kvq_ prefix
    assert exported == set(names)


def test_status_strings():
    for s in range(5):
        assert kvq.kvq_status_string(s)
    assert kvq.kvq_status_string(99) == "unknown status"


def test_row_bytes_match_oracle_model():
    for t in ("f16", "q8_0", "q4_0", "q5_0"):
        for d in (32, 64, 128, 256):
            assert kvq.kvq_row_bytes(t, d) == cache_model.row_bytes(t, d)
    for d in (32, 64, 128, 256):
        for t in ("turbo2", "turbo3", "turbo4", "turbo3_qjl"):
            assert kvq.kvq_row_bytes(t, d) == cache_model.row_bytes(t, d)
    assert kvq.kvq_row_bytes("q8_0", 48) == 0
    assert kvq.kvq_row_bytes("turbo3", 96) == 0
    assert kvq.kvq_row_bytes("turbo3_qjl", 96) == 0
    assert kvq.kvq_row_bytes(8, 128) == 0
    assert kvq.kvq_row_bytes("turbo2", 96) == 0


def test_cache_bytes_reproduce_pages():
    """Layer caches allocated by the library sum to the sizes the pages print."""
    mib = 1024.0 * 1024.0
    for row in read_golden("kv_cache_bytes.txt"):
        L, H, D, T, kt, vt, exp, which = row.split()
        L, H, D, T, exp = int(L), int(H), int(D), int(T), float(exp)
        desc = kvq.make_desc(H, H, D, kt, vt, T)
        k = L * kvq.kvq_cache_bytes(desc, 1, 0)
        v = L * kvq.kvq_cache_bytes(desc, 1, 1)
        got = {"K": k, "V": v, "KV": k + v}[which] / mib
        assert got == exp, row


def test_q5_0_layout():
    """q5_0: d/2 code bytes (q4_0's nibbles) and 3d/32 fp16 slots per row in the
    scale plane (block scales, then the qh words)."""
    desc = kvq.make_desc(32, 8, 128, "q5_0", "q5_0", 1000)
    L = kvq.kvq_cache_layout(desc, 2, 0)
    assert L.code_bytes == 64 and L.n_scales == 12
    assert L.total_bytes == L.scale_offset + 2 * 8 * 1008 * 12 * 2
    assert kvq.kvq_row_bytes("q5_0", 128) == 88 == cache_model.row_bytes("q5_0", 128)
    assert kvq.kvq_check_desc(desc) == kvq.KVQ_OK


def test_layout_formula():
    desc = kvq.make_desc(32, 8, 128, "q8_0", "turbo3", 1000, turbo_seed=5)
    L = kvq.kvq_cache_layout(desc, 3, 0)
    assert L.rows_per_plane == 1008 and L.code_bytes == 128 and L.n_scales == 4
    assert L.scale_offset == 3 * 8 * 1008 * 128
    assert L.total_bytes == L.scale_offset + 3 * 8 * 1008 * 4 * 2
    V = kvq.kvq_cache_layout(desc, 3, 1)
    assert V.code_bytes == 48 and V.n_scales == 1
    assert V.scale_offset % 256 == 0 and V.scale_offset >= 3 * 8 * 1008 * 48
    assert V.total_bytes == V.scale_offset + 3 * 8 * 1008 * 2


def test_turbo3_codebook_equals_oracle():
    lv, th = kvq.kvq_turbo3_codebook()
    olv, oth = turbo3.codebook_f32()
    np.testing.assert_array_equal(np.array(lv, np.float32), olv)
    np.testing.assert_array_equal(np.array(th, np.float32), oth)


@pytest.mark.parametrize("kind", ["turbo2", "turbo3", "turbo4"])
def test_turbo_codebooks_equal_oracle(kind):
    lv, th = kvq.kvq_turbo_codebook(kind)
    olv, oth = turbo.codebook_f32(turbo.BITS[kind])
    np.testing.assert_array_equal(np.array(lv, np.float32), olv)
    np.testing.assert_array_equal(np.array(th, np.float32), oth)


@pytest.mark.parametrize("seed", [0, 1, 1234567, 0x7475726233, 2**64 - 1])
def test_turbo3_signs_equal_oracle(seed):
    for d in (32, 128, 256):
        np.testing.assert_array_equal(np.array(kvq.kvq_turbo3_signs(seed, d), np.float32),
                                      turbo3.signs(seed, d))


def test_check_desc():
    ok = kvq.make_desc(64, 8, 128, "q8_0", "q4_0", 32768)
    assert kvq.kvq_check_desc(ok) == kvq.KVQ_OK
    bad = [
        (kvq.make_desc(63, 8, 128, "q8_0", "q4_0", 32768), kvq.KVQ_ERR_INVALID),   # n_q % n_kv
        (kvq.make_desc(64, 0, 128, "q8_0", "q4_0", 32768), kvq.KVQ_ERR_INVALID),
        (kvq.make_desc(64, 8, 128, "q8_0", "q4_0", 0), kvq.KVQ_ERR_INVALID),
        (kvq.make_desc(64, 8, 128, 9, "q4_0", 16), kvq.KVQ_ERR_INVALID),           # unknown type
        (kvq.make_desc(64, 8, 80, "q8_0", "q4_0", 16), kvq.KVQ_ERR_UNSUPPORTED),   # head_dim % 32
        (kvq.make_desc(64, 8, 512, "q8_0", "q4_0", 16), kvq.KVQ_ERR_UNSUPPORTED),  # head_dim > 256
        (kvq.make_desc(64, 8, 96, "turbo3", "q4_0", 16), kvq.KVQ_ERR_UNSUPPORTED),   # turbo K needs 2^k too
        (kvq.make_desc(64, 8, 96, "q8_0", "turbo3", 16), kvq.KVQ_ERR_UNSUPPORTED),   # WHT needs 2^k
        (kvq.make_desc(64, 8, 96, "turbo2", "q4_0", 16), kvq.KVQ_ERR_UNSUPPORTED),
        (kvq.make_desc(64, 8, 96, "q8_0", "turbo4", 16), kvq.KVQ_ERR_UNSUPPORTED),
        (kvq.make_desc(64, 8, 128, 8, "q4_0", 16), kvq.KVQ_ERR_INVALID),           # past the last type
        (kvq.make_desc(64, 8, 128, "q8_0", "turbo3_qjl", 16), kvq.KVQ_ERR_UNSUPPORTED),  # a key format
        (kvq.make_desc(64, 8, 96, "turbo3_qjl", "q8_0", 16), kvq.KVQ_ERR_UNSUPPORTED),
    ]
    for desc, st in bad:
        assert kvq.kvq_check_desc(desc) == st
    # turbo keys are a valid description (the decode pairs them with q8_0, q4_0 or the same type)
    for kt in ("turbo2", "turbo3", "turbo4", "turbo3_qjl"):
        assert kvq.kvq_check_desc(kvq.make_desc(64, 8, 128, kt, "q4_0", 16)) == kvq.KVQ_OK
    d = kvq.make_desc(64, 8, 128, "q8_0", "q4_0", 16)
    d.flags = 2                                        # an undefined flag bit
    assert kvq.kvq_check_desc(d) == kvq.KVQ_ERR_INVALID
    d.flags = kvq.KVQ_FLAG_OVERLAP_PREVIOUS
    assert kvq.kvq_check_desc(d) == kvq.KVQ_OK
    assert kvq.raw_status("kvq_check_desc", None) == kvq.KVQ_ERR_INVALID


FAKE = 0x7f0000000000  # 256-byte aligned address that is never dereferenced


def _append(desc, k_cache=FAKE, v_cache=FAKE, k_new=FAKE, v_new=FAKE, batch=1, pos=0, n_tok=1):
    return kvq.raw_status("kvq_append_quantize", ctypes.byref(desc), k_cache, v_cache, k_new, v_new,
                          batch, pos, n_tok, None)


def _decode(desc, k=FAKE, v=FAKE, q=FAKE, batch=1, ctx=16, scale=0.1, S=0, ws=FAKE, ws_bytes=1 << 40):
    return kvq.raw_status("kvq_decode_attention", ctypes.byref(desc), k, v, q, batch, ctx, scale, S, ws,
                          ws_bytes, None)


def _combine(desc, ws=FAKE, ws_bytes=1 << 40, batch=1, ctx=16, S=0, out=FAKE):
    return kvq.raw_status("kvq_combine", ctypes.byref(desc), ws, ws_bytes, batch, ctx, S, out, None)


def _step(desc, k=FAKE, v=FAKE, q=FAKE, k_new=FAKE, v_new=FAKE, batch=1, ctx=16, scale=0.1, S=0, ws=FAKE,
          ws_bytes=1 << 40, out=FAKE):
    return kvq.raw_status("kvq_decode_step", ctypes.byref(desc), k, v, q, k_new, v_new, batch, ctx, scale, S, ws,
                          ws_bytes, out, None)


def test_append_rejects_before_launch():
    d = kvq.make_desc(8, 2, 64, "q8_0", "q4_0", 256)
    assert _append(d, pos=250, n_tok=7) == kvq.KVQ_ERR_INVALID     # past max_ctx
    assert _append(d, pos=-1) == kvq.KVQ_ERR_INVALID
    assert _append(d, n_tok=0) == kvq.KVQ_ERR_INVALID
    assert _append(d, batch=0) == kvq.KVQ_ERR_INVALID
    assert _append(d, k_new=None) == kvq.KVQ_ERR_INVALID            # cache without rows
    assert _append(d, k_cache=None, k_new=None, v_cache=None, v_new=None) == kvq.KVQ_ERR_INVALID
    assert _append(d, k_cache=FAKE + 16) == kvq.KVQ_ERR_INVALID     # cache not 256-aligned
    assert _append(d, v_new=FAKE + 2) == kvq.KVQ_ERR_INVALID        # rows not 16-aligned
    assert _append(kvq.make_desc(8, 2, 96, "turbo3", "q4_0", 256)) == kvq.KVQ_ERR_UNSUPPORTED


def test_decode_and_combine_reject_before_launch():
    d = kvq.make_desc(32, 8, 128, "q8_0", "q4_0", 8192)
    assert _decode(d, ctx=0) == kvq.KVQ_ERR_INVALID
    assert _decode(d, ctx=8193) == kvq.KVQ_ERR_INVALID
    assert _decode(d, q=None) == kvq.KVQ_ERR_INVALID
    assert _decode(d, S=-1) == kvq.KVQ_ERR_INVALID
    assert _decode(d, S=5000) == kvq.KVQ_ERR_INVALID
    assert _decode(d, scale=float("nan")) == kvq.KVQ_ERR_INVALID
    assert _decode(d, ws=FAKE + 8) == kvq.KVQ_ERR_INVALID
    need = kvq.kvq_workspace_bytes(d, 1, 4)
    assert need > 0
    assert _decode(d, S=4, ws_bytes=need - 1) == kvq.KVQ_ERR_WORKSPACE
    assert _combine(d, S=4, ws_bytes=need - 1) == kvq.KVQ_ERR_WORKSPACE
    assert _combine(d, out=None) == kvq.KVQ_ERR_INVALID
    assert _combine(d, ctx=0) == kvq.KVQ_ERR_INVALID
    assert _decode(kvq.make_desc(32, 8, 128, "turbo3", "f16", 64)) == kvq.KVQ_ERR_UNSUPPORTED   # pairing
    assert _decode(kvq.make_desc(32, 8, 128, "turbo3", "turbo2", 64)) == kvq.KVQ_ERR_UNSUPPORTED


def test_decode_step_rejects_before_launch():
    d = kvq.make_desc(32, 8, 128, "q8_0", "q4_0", 8192)
    assert _step(d, k_new=None) == kvq.KVQ_ERR_INVALID
    assert _step(d, v_new=None) == kvq.KVQ_ERR_INVALID
    assert _step(d, out=None) == kvq.KVQ_ERR_INVALID
    assert _step(d, k_new=FAKE + 2) == kvq.KVQ_ERR_INVALID         # new rows not 16-aligned
    assert _step(d, out=FAKE + 4) == kvq.KVQ_ERR_INVALID
    assert _step(d, ctx=0) == kvq.KVQ_ERR_INVALID                  # the new row needs ctx_len >= 1
    assert _step(d, ctx=8193) == kvq.KVQ_ERR_INVALID
    assert _step(d, k=FAKE + 16) == kvq.KVQ_ERR_INVALID
    need = kvq.kvq_workspace_bytes(d, 1, 4)
    assert _step(d, S=4, ws_bytes=need - 1) == kvq.KVQ_ERR_WORKSPACE  # the counters are part of it
    assert _step(kvq.make_desc(32, 8, 128, "turbo3", "f16", 64)) == kvq.KVQ_ERR_UNSUPPORTED


def _decode_varlen(desc, lens=FAKE, max_ctx=16, q=FAKE, S=0, ws=FAKE, ws_bytes=1 << 40):
    return kvq.raw_status("kvq_decode_attention_varlen", ctypes.byref(desc), FAKE, FAKE, q, 1, lens, max_ctx,
                          0.1, S, ws, ws_bytes, None)


def _step_varlen(desc, lens=FAKE, max_ctx=16, k_new=FAKE, S=0, ws_bytes=1 << 40, out=FAKE):
    return kvq.raw_status("kvq_decode_step_varlen", ctypes.byref(desc), FAKE, FAKE, FAKE, k_new, FAKE, 1, lens,
                          max_ctx, 0.1, S, FAKE, ws_bytes, out, None)


def _append_varlen(desc, lens=FAKE, n_tok=1, batch=1, k_new=FAKE):
    return kvq.raw_status("kvq_append_quantize_varlen", ctypes.byref(desc), FAKE, FAKE, k_new, FAKE, batch, lens,
                          n_tok, None)


def test_varlen_entry_points_reject_before_launch():
    d = kvq.make_desc(32, 8, 128, "q8_0", "q4_0", 8192)
    # the lengths pointer: required, 4-byte aligned
    assert _decode_varlen(d, lens=None) == kvq.KVQ_ERR_INVALID
    assert _decode_varlen(d, lens=FAKE + 2) == kvq.KVQ_ERR_INVALID
    assert _step_varlen(d, lens=None) == kvq.KVQ_ERR_INVALID
    assert _step_varlen(d, lens=FAKE + 1) == kvq.KVQ_ERR_INVALID
    assert _append_varlen(d, lens=None) == kvq.KVQ_ERR_INVALID
    assert _append_varlen(d, lens=FAKE + 3) == kvq.KVQ_ERR_INVALID
    # the host bound on the lengths takes ctx_len's checks
    assert _decode_varlen(d, max_ctx=0) == kvq.KVQ_ERR_INVALID
    assert _decode_varlen(d, max_ctx=8193) == kvq.KVQ_ERR_INVALID
    assert _step_varlen(d, max_ctx=0) == kvq.KVQ_ERR_INVALID
    assert _step_varlen(d, max_ctx=8193) == kvq.KVQ_ERR_INVALID
    # everything else as in the uniform-length forms
    assert _decode_varlen(d, q=None) == kvq.KVQ_ERR_INVALID
    need = kvq.kvq_workspace_bytes(d, 1, 4)
    assert _decode_varlen(d, S=4, ws_bytes=need - 1) == kvq.KVQ_ERR_WORKSPACE
    assert _step_varlen(d, S=4, ws_bytes=need - 1) == kvq.KVQ_ERR_WORKSPACE
    assert _step_varlen(d, k_new=None) == kvq.KVQ_ERR_INVALID
    assert _step_varlen(d, out=FAKE + 4) == kvq.KVQ_ERR_INVALID
    assert _append_varlen(d, n_tok=0) == kvq.KVQ_ERR_INVALID
    assert _append_varlen(d, n_tok=8193) == kvq.KVQ_ERR_INVALID     # no sequence can hold them
    assert _append_varlen(d, batch=0) == kvq.KVQ_ERR_INVALID
    assert _append_varlen(d, k_new=FAKE + 8) == kvq.KVQ_ERR_INVALID
    t3k = kvq.make_desc(32, 8, 128, "turbo3", "q5_0", 64)     # a pairing the decode does not take
    assert _decode_varlen(t3k) == kvq.KVQ_ERR_UNSUPPORTED
    assert _append_varlen(kvq.make_desc(32, 8, 96, "turbo3", "q4_0", 64)) == kvq.KVQ_ERR_UNSUPPORTED


def test_paged_layout_is_the_contiguous_layout_of_pages():
    """A pool is laid out as a contiguous cache with the pages as batch rows
    and page_rows rows per plane."""
    for kt, vt, D in (("q8_0", "q4_0", 128), ("f16", "turbo3", 64), ("q4_0", "q8_0", 256)):
        for P, n in ((32, 1), (64, 700), (256, 33)):
            d = kvq.make_desc(32, 8, D, kt, vt, 100000)
            for which in (0, 1):
                got = kvq.kvq_paged_layout(d, P, n, which)
                ref = kvq.kvq_cache_layout(kvq.make_desc(32, 8, D, kt, vt, P), n, which)
                for f in ("rows_per_plane", "code_bytes", "n_scales", "scale_offset", "total_bytes"):
                    assert getattr(got, f) == getattr(ref, f), (kt, vt, D, P, n, which, f)
                assert kvq.kvq_paged_cache_bytes(d, P, n, which) == ref.total_bytes


def _pg(table=FAKE, max_pages=4, page_rows=64, n_pages=100):
    return kvq.kvq_paged(table, max_pages, page_rows, n_pages)


def test_paged_entry_points_reject_before_launch():
    d = kvq.make_desc(32, 8, 128, "q8_0", "q4_0", 8192)
    dec = lambda pg, lens=FAKE, mx=256: kvq.raw_status("kvq_decode_attention_paged", ctypes.byref(d), FAKE, FAKE,
                                                        FAKE, 1, ctypes.byref(pg) if pg else None, lens, mx, 0.1,
                                                        0, FAKE, 1 << 40, None)
    step = lambda pg, lens=FAKE, mx=256: kvq.raw_status("kvq_decode_step_paged", ctypes.byref(d), FAKE, FAKE, FAKE,
                                                         FAKE, FAKE, 1, ctypes.byref(pg) if pg else None, lens, mx,
                                                         0.1, 0, FAKE, 1 << 40, FAKE, None)
    app = lambda pg, lens=FAKE, n=1: kvq.raw_status("kvq_append_quantize_paged", ctypes.byref(d), FAKE, FAKE, FAKE,
                                                     FAKE, 1, ctypes.byref(pg) if pg else None, lens, n, None)
    for call in (dec, step, app):
        assert call(None) == kvq.KVQ_ERR_INVALID                          # no pool description
        assert call(_pg(), lens=None) == kvq.KVQ_ERR_INVALID              # no lengths
        assert call(_pg(table=None)) == kvq.KVQ_ERR_INVALID
        assert call(_pg(table=FAKE + 2)) == kvq.KVQ_ERR_INVALID           # table not 4-byte aligned
        assert call(_pg(max_pages=0)) == kvq.KVQ_ERR_INVALID
        assert call(_pg(n_pages=0)) == kvq.KVQ_ERR_INVALID
        assert call(_pg(page_rows=16)) == kvq.KVQ_ERR_UNSUPPORTED        # below one 32-row tile
        assert call(_pg(page_rows=96)) == kvq.KVQ_ERR_UNSUPPORTED        # not a power of two
        assert call(_pg(n_pages=1 << 28)) == kvq.KVQ_ERR_UNSUPPORTED     # n_pages * n_kv >= 2^31
    # the host bound on the lengths: within max_ctx and what the block table can address
    assert dec(_pg(max_pages=4, page_rows=64), mx=257) == kvq.KVQ_ERR_INVALID
    assert step(_pg(max_pages=4, page_rows=64), mx=257) == kvq.KVQ_ERR_INVALID
    assert dec(_pg(max_pages=1000, page_rows=64), mx=8193) == kvq.KVQ_ERR_INVALID
    assert kvq.kvq_paged_cache_bytes(d, 16, 10, 0) == 0


def test_partials_region_is_the_workspace_tail():
    """The partials (m, l, acc) follow the counters, the epoch words and the
    status word, and run to the end of the workspace."""
    d = kvq.make_desc(64, 8, 128, "q8_0", "q4_0", 32768)
    r256 = lambda v: (v + 255) // 256 * 256
    for B, S in ((1, 37), (4, 9), (16, 3), (32, 5)):
        off, n = kvq.kvq_partials_region(d, B, S)
        assert off == r256(B * 8 * 8 + 4)
        assert off + n == kvq.kvq_workspace_bytes(d, B, S)
    for bad in ((0, 4), (1, 0), (1, 5000)):
        with pytest.raises(kvq.KvqError):
            kvq.kvq_partials_region(d, *bad)
    rank = lambda **kw: kvq.raw_status("kvq_combine_ranks", ctypes.byref(d), kw.get("parts", FAKE), kw.get("r", 2),
                                        1, kw.get("s", 4), kw.get("out", FAKE), None)
    assert rank(parts=None) == kvq.KVQ_ERR_INVALID
    assert rank(r=0) == kvq.KVQ_ERR_INVALID
    assert rank(s=0) == kvq.KVQ_ERR_INVALID
    assert rank(parts=FAKE + 4) == kvq.KVQ_ERR_INVALID
    assert rank(r=4096, s=4) == kvq.KVQ_ERR_UNSUPPORTED  # more weights than the combine holds


def test_workspace_bytes_formula():
    d = kvq.make_desc(64, 8, 128, "q8_0", "q4_0", 32768)
    B, S = 4, 9
    rows = B * 64 * S
    r256 = lambda v: (v + 255) // 256 * 256
    # the fused step's arrival counters and epoch words, [B][n_kv] uint32 each, the status
    # word, then m, l, acc, each part 256-aligned
    assert kvq.kvq_workspace_bytes(d, B, S) == r256(B * 8 * 8 + 4) + 2 * r256(rows * 4) + rows * 128 * 4
    assert kvq.kvq_workspace_bytes(d, 0, S) == 0
    # the automatic split count never needs more workspace than n_splits = 0 reserves
    auto_ws = kvq.kvq_workspace_bytes(d, B, 0)
    for ctx in (1, 100, 4096, 32768):
        s = kvq.kvq_auto_splits(d, B, ctx)
        assert 1 <= s and kvq.kvq_workspace_bytes(d, B, s) <= auto_ws


def test_auto_splits_bounded_and_nonempty():
    for batch in (1, 4, 16):
        d = kvq.make_desc(32, 8, 128, "q4_0", "q4_0", 131072)
        bound = kvq.kvq_workspace_bytes(d, batch, 0)
        for ctx in (1, 15, 16, 17, 255, 256, 257, 1000, 4096, 8192, 65536, 100003, 131072):
            s = kvq.kvq_auto_splits(d, batch, ctx)
            assert 1 <= s <= 4096
            assert kvq.kvq_workspace_bytes(d, batch, s) <= bound
            # chunks are whole 32-row tiles and no automatic split is empty
            chunk = -(-(-(-ctx // s)) // 32) * 32
            assert (s - 1) * chunk < ctx
    assert kvq.kvq_auto_splits(d, 1, 0) == 0


def test_qjl_keys_need_their_projection():
    """turbo3_qjl keys: append, decode and the fused step read the projection,
    so a missing or misaligned one is INVALID before any launch; the decode
    pairs them with q8_0, q4_0 or turbo3 values only."""
    for proj in (None, FAKE + 4):
        d = kvq.make_desc(32, 8, 128, "turbo3_qjl", "q8_0", 64, qjl_proj=proj)
        assert _append(d) == kvq.KVQ_ERR_INVALID
        assert _decode(d) == kvq.KVQ_ERR_INVALID
        assert _step(d) == kvq.KVQ_ERR_INVALID
    for vt in ("f16", "q5_0", "turbo2", "turbo4"):
        d = kvq.make_desc(32, 8, 128, "turbo3_qjl", vt, 64, qjl_proj=FAKE)
        assert _decode(d) == kvq.KVQ_ERR_UNSUPPORTED
        assert _step(d) == kvq.KVQ_ERR_UNSUPPORTED
    lv, th = kvq.kvq_turbo_codebook("turbo3_qjl")
    lv2, th2 = kvq.kvq_turbo_codebook("turbo2")
    assert list(lv) == list(lv2) and list(th) == list(th2)


def test_binding_structs_and_enums_match_the_header(tmp_path):
    """The ctypes mirrors have the C structs' sizes and field offsets, and the
    binding's type and status codes are the header's enum values (the header is
    compiled by gcc as plain C)."""
    structs = {"kvq_cache_desc": kvq.kvq_cache_desc, "kvq_plane_layout": kvq.kvq_plane_layout,
               "kvq_paged": kvq.kvq_paged}
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "kvq.h"', 'int main(void) {']
    for name, cls in structs.items():
        lines.append(f'  printf("{name} size %zu\\n", sizeof({name}));')
        for field, _ in cls._fields_:
            lines.append(f'  printf("{name} {field} %zu\\n", offsetof({name}, {field}));')
    names = ["KVQ_F16", "KVQ_Q8_0", "KVQ_Q4_0", "KVQ_TURBO3", "KVQ_TURBO2", "KVQ_TURBO4", "KVQ_Q5_0",
             "KVQ_TURBO3_QJL", "KVQ_OK", "KVQ_ERR_INVALID", "KVQ_ERR_UNSUPPORTED", "KVQ_ERR_WORKSPACE",
             "KVQ_ERR_CUDA"]
    for n in names:
        lines.append(f'  printf("enum {n} %d\\n", (int){n});')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    seen = 0
    for line in filter(None, out):
        a, b, c = line.split()
        if a == "enum":
            assert getattr(kvq, b) == int(c), b
        elif b == "size":
            assert ctypes.sizeof(structs[a]) == int(c), a
        else:
            assert getattr(structs[a], b).offset == int(c), (a, b)
        seen += 1
    assert seen == len(names) + sum(1 + len(c._fields_) for c in structs.values())
    assert set(kvq.TYPES.values()) == set(range(8))


def test_qjl_layout():
    """turbo3_qjl keys: 3d/8 code bytes (2-bit levels, then 1-bit signs) and two
    fp16 slots per row (norm, gamma) in the scale plane."""
    desc = kvq.make_desc(32, 8, 128, "turbo3_qjl", "q8_0", 1000, qjl_proj=FAKE)
    L = kvq.kvq_cache_layout(desc, 2, 0)
    assert L.code_bytes == 48 and L.n_scales == 2
    assert L.scale_offset % 256 == 0 and L.scale_offset >= 2 * 8 * 1008 * 48
    assert L.total_bytes == L.scale_offset + 2 * 8 * 1008 * 2 * 2
    P = kvq.kvq_paged_layout(desc, 64, 10, 0)
    assert P.code_bytes == 48 and P.n_scales == 2 and P.rows_per_plane == 64


def test_workspace_status_word_place():
    """The status word follows the arrival counters and epoch words
    (8 bytes per (batch row, KV head)), does not move with the split count, and
    the split partials start after it."""
    desc = kvq.make_desc(64, 8, 128, "q8_0", "q4_0", 32768)
    for batch in (1, 4, 4096):
        off = kvq.kvq_workspace_status_offset(desc, batch)
        assert off == batch * 8 * 8
        for S in (1, 9, 300):
            p_off, p_bytes = kvq.kvq_partials_region(desc, batch, S)
            assert p_off >= off + 4 and p_off % 256 == 0
            assert kvq.kvq_workspace_bytes(desc, batch, S) == p_off + p_bytes
    with pytest.raises(kvq.KvqError):
        kvq.kvq_workspace_status_offset(desc, 0)
