"""kvq_decode_attention_noalloc, the entry point for callers that cannot
allocate device memory when they decode (a fixed arena handed out up front, a
process that must not touch the allocator while another stream is being
captured, a foreign-language host that only passes pointers it was given).

It keeps the split partials in the library's own per-GPU scratch array instead
of a caller workspace.  Checked through the C ABI against the workspace entry
points (kvq_decode_attention + kvq_combine) on two calls in a row -- the second
with other inputs, so stale scratch contents from the first call would show --
within the attention tolerance the other GPU tests use.  Collected last so that
a failure here cannot stop the rest of the suite early."""

import numpy as np
import pytest
import torch

import decode_attention_q8_b200 as kvq
import synth
from kvq_testlib import ATOL, REL_L2, alloc_cache, decode

pytestmark = pytest.mark.gpu


def _caches(w, k_type, v_type, turbo_seed=0):
    desc = kvq.make_desc(w.n_q, w.n_kv, w.head_dim, k_type, v_type, w.ctx, turbo_seed=turbo_seed)
    q, k, v = synth.layer_inputs(w, device="cuda")
    kc, vc = alloc_cache(desc, w.batch, 0), alloc_cache(desc, w.batch, 1)
    kvq.kvq_append_quantize(desc, kc, vc, k, v, w.batch, 0, w.ctx)
    return desc, q, kc, vc


def _close(got, ref):
    got, ref = got.double().cpu().numpy(), ref.double().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= ATOL
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= REL_L2


def test_noalloc_matches_workspace_entry_points_twice():
    w1 = synth.WORKLOADS["llama8b_ctx8k"]
    w2 = synth.Workload("second", 2, 1, 16, 4, 128, 1500, "q8_0", "turbo3", (3, 17), 8.0, 777, turbo_seed=99)
    cases = [(w1, *_caches(w1, "q8_0", "q4_0")), (w2, *_caches(w2, "q8_0", "turbo3", 99))]
    for w, desc, q, kc, vc in cases:     # two calls in a row, different problems
        ref = decode(desc, kc, vc, q, w.batch, w.ctx, w.scale)
        out = torch.full((w.batch, w.n_q, w.head_dim), float("nan"), dtype=torch.float32, device="cuda")
        kvq.kvq_decode_attention_noalloc(desc, kc, vc, q, w.batch, w.ctx, w.scale, 0, out)
        torch.cuda.synchronize()
        _close(out, ref)
    # and the first problem once more, after the scratch held the second one
    w, desc, q, kc, vc = cases[0]
    out = torch.empty((w.batch, w.n_q, w.head_dim), dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attention_noalloc(desc, kc, vc, q, w.batch, w.ctx, w.scale, 3, out)
    torch.cuda.synchronize()
    _close(out, decode(desc, kc, vc, q, w.batch, w.ctx, w.scale, 3))


def test_noalloc_rejects_problems_beyond_its_scratch():
    w = synth.WORKLOADS["llama8b_ctx8k"]
    desc, q, kc, vc = _caches(w, "q8_0", "q4_0")
    out = torch.zeros((1, w.n_q, w.head_dim), dtype=torch.float32, device="cuda")
    # 4096 splits need 32 * 4096 * 130 * 4 bytes of partials, more than the 8 MiB scratch
    assert kvq.kvq_workspace_bytes(desc, 1, 4096) > 8 << 20
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attention_noalloc(desc, kc, vc, q, 1, w.ctx, w.scale, 4096, out)
    assert e.value.status == kvq.KVQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out == 0).all())
