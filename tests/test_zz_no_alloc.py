"""kvq_decode_attention_noalloc, the entry point for callers that cannot
allocate device memory when they decode (a fixed arena handed out up front, a
process that must not touch the allocator while another stream is being
captured, a foreign-language host that only passes pointers it was given).

It keeps the split partials in the library's own per-GPU scratch array instead
of a caller workspace.  It runs the same kernels with the same split count as
the workspace entry points (kvq_decode_attention + kvq_combine), so its output
must equal theirs bit for bit, call after call: the second call has other
inputs, and a later call with empty trailing splits follows a larger one, so
stale scratch contents would show.  One call is also checked against the
oracle directly.  Collected last so that a failure here cannot stop the rest of
the suite early."""

import numpy as np
import pytest
import torch

import decode_attention_q8_b200 as kvq
import synth
from kvq_testlib import alloc_cache, assert_attention_close, decode, oracle_attention_rows, oracle_dequant, oracle_rows

pytestmark = pytest.mark.gpu

SCRATCH = 8 << 20


def _caches(w, k_type, v_type, turbo_seed=0):
    desc = kvq.make_desc(w.n_q, w.n_kv, w.head_dim, k_type, v_type, w.ctx, turbo_seed=turbo_seed)
    q, k, v = synth.layer_inputs(w, device="cuda")
    kc, vc = alloc_cache(desc, w.batch, 0), alloc_cache(desc, w.batch, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k, v, w.batch, 0, w.ctx)
    return desc, q, k, v, kc, vc


def _noalloc(desc, w, q, kc, vc, n_splits, ctx=None):
    out = torch.full((w.batch, w.n_q, w.head_dim), float("nan"), dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attention_noalloc(desc, kc, vc, q, w.batch, ctx or w.ctx, w.scale, n_splits, out)
    torch.cuda.synchronize()
    return out


def test_noalloc_equals_workspace_entry_points_call_after_call():
    w1 = synth.WORKLOADS["llama8b_ctx8k"]
    w2 = synth.Workload("second", 2, 1, 16, 4, 128, 1500, "q8_0", "turbo3", (3, 17), 8.0, 777, turbo_seed=99)
    c1 = _caches(w1, "q8_0", "q4_0")
    c2 = _caches(w2, "q8_0", "turbo3", 99)
    for w, (desc, q, _, _, kc, vc) in ((w1, c1), (w2, c2)):     # two calls in a row, different problems
        out = _noalloc(desc, w, q, kc, vc, 0)
        ref = decode(desc, kc, vc, q, w.batch, w.ctx, w.scale)
        assert torch.equal(out, ref)
    # the first problem again with 3 splits, after the scratch held the second one
    w, (desc, q, _, _, kc, vc) = w1, c1
    assert torch.equal(_noalloc(desc, w, q, kc, vc, 3), decode(desc, kc, vc, q, w.batch, w.ctx, w.scale, 3))
    # a short context with more splits than 32-row tiles, right after the larger
    # calls filled the scratch: splits 4..7 are empty and must be written as such
    short = 100
    assert kvq.kvq_workspace_bytes(desc, w.batch, 8) <= SCRATCH
    out = _noalloc(desc, w, q, kc, vc, 8, ctx=short)
    assert torch.equal(out, decode(desc, kc, vc, q, w.batch, short, w.scale, 8))


def test_noalloc_against_the_oracle():
    w = synth.Workload("oracle_case", 2, 1, 16, 4, 128, 777, "q8_0", "q4_0", (3, 17), 8.0, 4321)
    desc, q, k, v, kc, vc = _caches(w, "q8_0", "q4_0")
    out = _noalloc(desc, w, q, kc, vc, 0).cpu().numpy()
    G = w.n_q // w.n_kv
    for b in range(w.batch):
        for g in range(w.n_kv):
            kh = oracle_dequant("q8_0", *oracle_rows("q8_0", k[b, :, g].cpu().numpy()), w.head_dim)
            vh = oracle_dequant("q4_0", *oracle_rows("q4_0", v[b, :, g].cpu().numpy()), w.head_dim)
            exp = oracle_attention_rows(q[b, g * G:(g + 1) * G].cpu().numpy(), kh, vh, w.scale)
            assert_attention_close(out[b, g * G:(g + 1) * G], exp, f"noalloc b{b} g{g}")


def test_noalloc_automatic_splits_fit_the_scratch():
    """With n_splits = 0 the automatic count is lowered until the partials fit
    the 8 MiB scratch; the result equals the workspace path at that count."""
    w = synth.Workload("wide", 16, 1, 64, 4, 256, 4096, "q8_0", "q4_0", (3, 17), 8.0, 99)
    desc, q, _, _, kc, vc = _caches(w, "q8_0", "q4_0")
    auto = kvq.kvq_auto_splits(desc, w.batch, w.ctx)
    S = auto
    while S > 1 and kvq.kvq_workspace_bytes(desc, w.batch, S) > SCRATCH:
        S -= 1
    out = _noalloc(desc, w, q, kc, vc, 0)
    assert torch.equal(out, decode(desc, kc, vc, q, w.batch, w.ctx, w.scale, S)), (auto, S)
    if S < auto:   # the automatic count itself would not have fitted
        with pytest.raises(kvq.KvqError) as e:
            _noalloc(desc, w, q, kc, vc, auto)
        assert e.value.status == kvq.KVQ_ERR_WORKSPACE


def test_noalloc_rejects_problems_beyond_its_scratch():
    w = synth.WORKLOADS["llama8b_ctx8k"]
    desc, q, _, _, kc, vc = _caches(w, "q8_0", "q4_0")
    out = torch.zeros((1, w.n_q, w.head_dim), dtype=torch.float32, device="cuda")
    # 4096 splits need 32 * 4096 * 130 * 4 bytes of partials, more than the 8 MiB scratch
    assert kvq.kvq_workspace_bytes(desc, 1, 4096) > SCRATCH
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attention_noalloc(desc, kc, vc, q, 1, w.ctx, w.scale, 4096, out)
    assert e.value.status == kvq.KVQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out == 0).all())
