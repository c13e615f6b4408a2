"""kvq_decode_step launched to overlap the kernel before it on the stream
(KVQ_FLAG_OVERLAP_PREVIOUS: programmatic dependent launch).  The step may start
while that kernel finishes, but reads nothing it could have written before it
completes; so a chain of layer steps gives exactly the bytes and outputs of the
same chain launched one after the other -- eagerly and in a CUDA graph -- and a
step whose queries are written by the kernel right before it sees the new
queries."""

import math

import pytest
import torch

import decode_attention_q8_b200 as kvq
import synth
from kvq_testlib import alloc_cache, assert_attention_close, oracle_attention_rows, oracle_dequant, oracle_rows

pytestmark = pytest.mark.gpu

CASES = [  # (k_type, v_type, batch, n_q, n_kv, head_dim, ctx)
    ("q8_0", "q4_0", 4, 64, 8, 128, 4096),
    ("q8_0", "turbo3", 1, 64, 8, 128, 8192),
    ("q4_0", "q4_0", 1, 32, 8, 128, 16384),
]


class Chain:
    """L layers, each its own cache prefilled with rows 0 .. ctx-2 and its own
    inputs; steps append row ctx-1 and attend over ctx rows."""

    def __init__(self, case, L, seed):
        kt, vt, B, n_q, n_kv, D, ctx = case
        self.case, self.L, self.B, self.ctx = case, L, B, ctx
        self.scale = 1 / math.sqrt(D)
        self.descs = {f: kvq.make_desc(n_q, n_kv, D, kt, vt, ctx, turbo_seed=seed, flags=f)
                      for f in (0, kvq.KVQ_FLAG_OVERLAP_PREVIOUS)}
        w = synth.Workload("chain", B, L, n_q, n_kv, D, ctx, kt, vt, (3, 17), 8.0, seed)
        self.q, self.k, self.v, self.caches = [], [], [], []
        for layer in range(L):
            q, k, v = synth.layer_inputs(w, layer=layer, device="cuda")
            kc, vc = alloc_cache(self.descs[0], B, 0), alloc_cache(self.descs[0], B, 1)
            kvq.kvq_append_quantize(self.descs[0], kc, vc, k[:, :ctx - 1].contiguous(), v[:, :ctx - 1].contiguous(),
                                    B, 0, ctx - 1)
            self.q.append(q)
            self.k.append(k)
            self.v.append(v)
            self.caches.append((kc, vc))
        self.k_new = [k[:, ctx - 1].contiguous() for k in self.k]
        self.v_new = [v[:, ctx - 1].contiguous() for v in self.v]
        torch.cuda.synchronize()

    def copies(self):
        return [(kc.clone(), vc.clone()) for kc, vc in self.caches]

    def run(self, caches, flags, ws, outs, qs=None, q_from_prev=None):
        """The L steps on the current stream; q_from_prev(layer, prev_out, q_dst)
        runs between steps (a kernel of its own) when given."""
        desc = self.descs[flags]
        for layer in range(self.L):
            if q_from_prev is not None and layer > 0:
                q_from_prev(layer, outs[layer - 1], qs[layer])
            kc, vc = caches[layer]
            kvq.kvq_decode_step(desc, kc, vc, (qs or self.q)[layer], self.k_new[layer], self.v_new[layer], self.B,
                                self.ctx, self.scale, 0, ws, outs[layer])


def _outs(ch):
    kt, vt, B, n_q, n_kv, D, ctx = ch.case
    return [torch.full((B, n_q, D), float("nan"), dtype=torch.float32, device="cuda") for _ in range(ch.L)]


def _ws(ch):
    return torch.zeros(kvq.kvq_workspace_bytes(ch.descs[0], ch.B, 0), dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{c[1]}-b{c[2]}")
def test_overlapped_chain_equals_serial_chain(case):
    ch = Chain(case, 6, seed=31)
    serial_caches, serial_outs = ch.copies(), _outs(ch)
    ch.run(serial_caches, 0, _ws(ch), serial_outs)
    # eager, overlapped
    caches, outs = ch.copies(), _outs(ch)
    ch.run(caches, kvq.KVQ_FLAG_OVERLAP_PREVIOUS, _ws(ch), outs)
    torch.cuda.synchronize()
    for layer in range(ch.L):
        assert torch.equal(outs[layer], serial_outs[layer]), f"layer {layer} output"
        assert torch.equal(caches[layer][0], serial_caches[layer][0]) and \
            torch.equal(caches[layer][1], serial_caches[layer][1]), f"layer {layer} cache"
    # the same chain captured in a CUDA graph and replayed
    caches, outs, ws = ch.copies(), _outs(ch), _ws(ch)
    warm_caches = ch.copies()
    ch.run(warm_caches, kvq.KVQ_FLAG_OVERLAP_PREVIOUS, _ws(ch), _outs(ch))   # first calls outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        ch.run(caches, kvq.KVQ_FLAG_OVERLAP_PREVIOUS, ws, outs)
    graph.replay()
    torch.cuda.synchronize()
    for layer in range(ch.L):
        assert torch.equal(outs[layer], serial_outs[layer]), f"graph layer {layer} output"
        assert torch.equal(caches[layer][0], serial_caches[layer][0]), f"graph layer {layer} K cache"
    # replayed again: every row is rewritten with the same bytes, the output repeats
    graph.replay()
    torch.cuda.synchronize()
    for layer in range(ch.L):
        assert torch.equal(outs[layer], serial_outs[layer]), f"second replay layer {layer}"
    del graph


@pytest.mark.parametrize("graph", [False, True])
def test_overlapped_step_sees_queries_written_just_before_it(graph):
    """Layer l+1's queries are computed from layer l's output by a kernel that
    runs right before layer l+1's step (q = fp16(out + q_base)); the query
    buffers start as NaN, so a step that read its queries before that kernel
    completed would give NaN or stale outputs.  Overlapped and serial chains
    agree bit for bit, and the last layer matches the oracle on the queries
    actually produced."""
    case = CASES[0]
    ch = Chain(case, 5, seed=57)

    def q_from_prev(layer, prev_out, q_dst):
        # the last kernel before the step writes the step's queries
        q_dst.copy_((prev_out + ch.q[layer].float()).half())

    def chain(flags):
        qs = [ch.q[0].clone()] + [torch.full_like(ch.q[0], float("nan")) for _ in range(1, ch.L)]
        caches, outs, ws = ch.copies(), _outs(ch), _ws(ch)
        if graph:
            warm = [ch.q[0].clone()] + [torch.full_like(ch.q[0], float("nan")) for _ in range(1, ch.L)]
            ch.run(ch.copies(), flags, _ws(ch), _outs(ch), qs=warm, q_from_prev=q_from_prev)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                ch.run(caches, flags, ws, outs, qs=qs, q_from_prev=q_from_prev)
            g.replay()
            torch.cuda.synchronize()
            del g
        else:
            ch.run(caches, flags, ws, outs, qs=qs, q_from_prev=q_from_prev)
            torch.cuda.synchronize()
        return outs, qs

    serial, _ = chain(0)
    overlapped, qs = chain(kvq.KVQ_FLAG_OVERLAP_PREVIOUS)
    for layer in range(ch.L):
        assert torch.isfinite(overlapped[layer]).all(), f"layer {layer}"
        assert torch.equal(overlapped[layer], serial[layer]), f"layer {layer}"
    kt, vt, B, n_q, n_kv, D, ctx = case
    G = n_q // n_kv
    last = ch.L - 1
    o = overlapped[last].cpu().numpy()
    for b, g in ((0, 0), (B - 1, n_kv - 1)):
        kh = oracle_dequant(kt, *oracle_rows(kt, ch.k[last][b, :, g].cpu().numpy()), D)
        vh = oracle_dequant(vt, *oracle_rows(vt, ch.v[last][b, :, g].cpu().numpy()), D)
        exp = oracle_attention_rows(qs[last][b, g * G:(g + 1) * G].cpu().numpy(), kh, vh, ch.scale)
        assert_attention_close(o[b, g * G:(g + 1) * G], exp, f"last layer b{b} g{g}")
