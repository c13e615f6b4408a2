"""Benchmark of the quantized-KV decode hot path on B200.

One step = one decode token through every layer of the workload: for each
layer, quantize-on-append of the new token's K/V rows (kvq_append_quantize),
split-KV decode over the whole cache (kvq_decode_attention) and the split
combine (kvq_combine).  Default workload: Llama-3.1-70B-shaped cache, 80
layers, 64 query / 8 KV heads, head_dim 128, context 32768, batch 4,
K q8_0 / V q4_0 (~17.4 GB of quantized cache, every layer a distinct 218 MB
buffer, so nothing stays in the 126 MB L2 between layers).

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle
instead, on a bounded sample of the same workload.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-KV decode attention: achieved HBM GB/s (% of peak), µs/layer-step"
UNIT = "GB/s"
DEFAULT_WORKLOAD = "llama70b_ctx32k_b4"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (0 = workload's)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    return ap.parse_args()


def row_bytes(kind, d):
    from decode_attention_q8_b200 import kvq_row_bytes
    return kvq_row_bytes(kind, d)


def algorithmic_bytes(w, n_layers):
    """Bytes the step must move at minimum, per the format definitions:
    decode reads every cached row once (codes + scales) and the queries and
    writes the fp32 outputs; append reads the new fp16 rows and writes their
    cache rows."""
    rk, rv = row_bytes(w.k_type, w.head_dim), row_bytes(w.v_type, w.head_dim)
    decode = w.batch * w.n_kv * w.ctx * (rk + rv) + w.batch * w.n_q * w.head_dim * (2 + 4)
    append = w.batch * w.n_kv * (2 * w.head_dim * 2 + rk + rv)
    return decode, append, n_layers * (decode + append)


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event (throttle) reasons of one GPU, sampled every few
    ms by a thread through NVML (read-only queries), keeping the samples taken
    between begin() and end(), i.e. during the timed region.  Falls back to an
    `nvidia-smi -lms` process when the NVML binding is missing."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device_index, enabled=True, period_s=0.004, query=None):
        import threading
        self.samples = []            # (host time, sm MHz, set of reason names)
        self.window = [None, None]
        self.max_mhz = None
        self.proc = None
        self._stop = threading.Event()
        self._thread = None
        if not enabled:
            return
        if query is None:
            query = self._nvml_query(device_index)
        if query is None:
            self._start_smi(device_index)
            return
        self._query = query
        self._period = period_s
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()

    def _nvml_query(self, device_index):
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            masks = [(name, getattr(pynvml, sym)) for name, sym in self.REASONS if hasattr(pynvml, sym)]
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

            def query():
                sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                bits = get_reasons(h)
                return sm, {name for name, m in masks if bits & m}
            query()
            return query
        except Exception:
            return None

    def _run(self):
        while not self._stop.is_set():
            try:
                sm, reasons = self._query()
            except Exception:
                break
            self.samples.append((time.perf_counter(), sm, reasons))
            self._stop.wait(self._period)

    def _start_smi(self, device_index):
        q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={device_index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def _sample_now(self):
        if self._thread is not None:
            try:
                sm, reasons = self._query()
                self.samples.append((time.perf_counter(), sm, reasons))
            except Exception:
                pass

    def begin(self):
        self.window[0] = time.perf_counter()
        self._sample_now()  # a short timed region still gets samples at its ends

    def end(self):
        self._sample_now()
        self.window[1] = time.perf_counter()

    def stop(self):
        """Summary of the samples inside the window: median SM MHz, max MHz and
        every reason seen active, or None without samples."""
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for line in out.strip().splitlines():
                f = [x.strip() for x in line.split(",")]
                try:
                    sm, mx = float(f[0]), float(f[1])
                except (ValueError, IndexError):
                    continue
                self.max_mhz = max(self.max_mhz or 0.0, mx)
                self.samples.append((None, sm, {n for n, v in zip(names, f[2:6]) if v.lower() == "active"}))
        t0, t1 = self.window
        inside = [s for s in self.samples
                  if s[0] is None or ((t0 is None or s[0] >= t0) and (t1 is None or s[0] <= t1))]
        if not inside:
            return None
        reasons = set()
        for s in inside:
            reasons |= s[2]
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(inside)}


# ----------------------------------------------------------------- CPU oracle

def oracle_sample(w, seconds=10.0, max_units=None):
    """Times the oracle's decode step (append the new row, dequantize the cached
    rows, fp64 attention) on whole (batch row, KV head) units of one layer, as
    many as fit in about `seconds`; returns (GB/s, units, seconds, threads)."""
    import numpy as np
    from threadpoolctl import threadpool_limits
    import synth
    from oracle import attention, blocks, turbo3

    def quant(kind, x, seed):
        if kind == "q8_0":
            return blocks.quantize_q8_0(x)
        if kind == "q4_0":
            return blocks.quantize_q4_0(x)
        if kind == "turbo3":
            return turbo3.quantize_turbo3(x, seed)
        return None, x

    def deq(kind, s, c, seed):
        if kind == "q8_0":
            return blocks.dequantize_q8_0(s, c)
        if kind == "q4_0":
            return blocks.dequantize_q4_0(s, c)
        if kind == "turbo3":
            return turbo3.dequantize_turbo3(s, c, seed, w.head_dim)
        return blocks.dequantize_f16(c)

    G = w.n_q // w.n_kv
    q, k, v = synth.layer_inputs(w, layer=0, device="cpu", batch=1)
    q, k, v = q.numpy(), k.numpy(), v.numpy()
    units = []
    for g in range(w.n_kv):
        ks, kc = quant(w.k_type, k[0, :, g, :], w.turbo_seed)
        vs, vc = quant(w.v_type, v[0, :, g, :], w.turbo_seed)
        units.append((q[0, g * G:(g + 1) * G], k[0, -1:, g, :], v[0, -1:, g, :], ks, kc, vs, vc))
    limit = max_units or 4 * len(units)
    done, t_total = 0, 0.0
    with threadpool_limits(limits=1):
        while done < limit and t_total < seconds:
            qg, kn, vn, ks, kc, vs, vc = units[done % len(units)]
            t0 = time.perf_counter()
            quant(w.k_type, kn, w.turbo_seed)
            quant(w.v_type, vn, w.turbo_seed)
            kh = deq(w.k_type, ks, kc, w.turbo_seed)
            vh = deq(w.v_type, vs, vc, w.turbo_seed)
            attention.decode_attention(qg[None].astype(np.float64), kh[None, None], vh[None, None], w.scale)
            t_total += time.perf_counter() - t0
            done += 1
    rk, rv = row_bytes(w.k_type, w.head_dim), row_bytes(w.v_type, w.head_dim)
    unit_bytes = w.ctx * (rk + rv) + G * w.head_dim * 6 + 2 * w.head_dim * 2 + rk + rv
    return done * unit_bytes / t_total / 1e9, done, t_total, 1


def run_reference(args):
    import synth
    if rank_env()[1] != 0:
        return   # the oracle baseline runs on rank 0 only
    w = synth.WORKLOADS[args.workload]
    gbs, units, secs, cores = oracle_sample(w, seconds=max(3.0, 2.0 * (args.steps + args.warmup)))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 6), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _config(w, args, None),
        "cpu_baseline": {"value": round(gbs, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{units} (batch row, KV head) units of layer 0, ctx {w.ctx}, "
                                   f"{secs:.1f} s, 1 BLAS thread"},
        "e2e": {"value": round(gbs, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _config(w, args, n_layers):
    return {"workload": w.name, "layers": n_layers or w.layers, "batch": w.batch, "n_q_heads": w.n_q,
            "n_kv_heads": w.n_kv, "head_dim": w.head_dim, "ctx": w.ctx, "k_type": w.k_type,
            "v_type": w.v_type, "step": "per layer: one fused launch (append 1 row + split decode + combine)",
            "l2": "inputs larger than L2: every layer a distinct cache buffer larger than the 126 MB L2"}


# ----------------------------------------------------------------- ranks

def rank_env():
    """(world size, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, world, device):
    """Element-wise maximum over all ranks of this rank's timings; every rank
    takes part and gets the result."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_gbs(world, bytes_per_rank_step, steps, ms):
    """Weak scaling: each rank runs its own replica of the workload, so the job
    moves world x the per-rank bytes in the slowest rank's time (ms)."""
    return world * bytes_per_rank_step * steps / (ms * 1e-3) / 1e9


# ----------------------------------------------------------------- GPU arm

def run_kvq(args):
    import torch
    import torch.distributed as dist

    import decode_attention_q8_b200 as kvq
    import synth

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = synth.WORKLOADS[args.workload]
    L = args.layers or w.layers
    desc = kvq.make_desc(w.n_q, w.n_kv, w.head_dim, w.k_type, w.v_type, w.ctx, turbo_seed=w.turbo_seed)
    B, ctx = w.batch, w.ctx
    stream = torch.cuda.current_stream(dev)  # prefill and the timed steps run on it

    # ---- caches: prefill every layer with its own seeded rows (timed: bulk append)
    kcs, vcs, qs, kn, vn = [], [], [], [], []
    pre_ev = []
    for layer in range(L):
        q, k, v = synth.layer_inputs(w, layer=layer + 1000 * rank, device=dev)
        kc = torch.empty(kvq.kvq_cache_bytes(desc, B, 0), dtype=torch.uint8, device=dev)
        vc = torch.empty(kvq.kvq_cache_bytes(desc, B, 1), dtype=torch.uint8, device=dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        kvq.kvq_append_quantize(desc, kc, vc, k, v, B, 0, ctx, stream)
        e1.record(stream)
        pre_ev.append((e0, e1))
        kcs.append(kc)
        vcs.append(vc)
        qs.append(q)
        kn.append(k[:, ctx - 1:ctx].contiguous())
        vn.append(v[:, ctx - 1:ctx].contiguous())
        del k, v
    if L < 3:
        # the first call of a process includes loading the kernel: with few
        # layers, time warm repeats of layer 0's append too (same rows, same bytes)
        _, k, v = synth.layer_inputs(w, layer=1000 * rank, device=dev)
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            kvq.kvq_append_quantize(desc, kcs[0], vcs[0], k, v, B, 0, ctx, stream)
            e1.record(stream)
            pre_ev.append((e0, e1))
        del k, v
    torch.cuda.synchronize()
    prefill_ms = [a.elapsed_time(b) for a, b in pre_ev[1:]]
    torch.cuda.empty_cache()

    S = kvq.kvq_auto_splits(desc, B, ctx)
    ws = torch.zeros(kvq.kvq_workspace_bytes(desc, B, 0), dtype=torch.uint8, device=dev)  # counters start at 0
    outs = [torch.empty((B, w.n_q, w.head_dim), dtype=torch.float32, device=dev) for _ in range(L)]
    scale = w.scale

    def step(events=None):
        """One decode token through every layer, launched on the current stream:
        per layer one fused launch (append the token's K/V row, split decode,
        combine)."""
        for layer in range(L):
            if events is not None:
                events[layer][0].record()
            kvq.kvq_decode_step(desc, kcs[layer], vcs[layer], qs[layer], kn[layer], vn[layer], B, ctx, scale, 0,
                                ws, outs[layer])
            if events is not None:
                events[layer][1].record()

    def step_unfused():
        """The same step as three launches per layer (append, decode, combine)."""
        for layer in range(L):
            kvq.kvq_append_quantize(desc, kcs[layer], vcs[layer], kn[layer], vn[layer], B, ctx - 1, 1)
            kvq.kvq_decode_attention(desc, kcs[layer], vcs[layer], qs[layer], B, ctx, scale, 0, ws)
            kvq.kvq_combine(desc, ws, B, ctx, 0, outs[layer])

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize()

    # warm-up eagerly (first calls set kernel attributes), then capture one step
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(args.warmup):
        graph.replay()
    barrier()
    clocks = ClockSampler(local, enabled=not args.no_clocks)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    clocks.begin()
    t_start.record()
    for _ in range(args.steps):
        graph.replay()
    t_end.record()
    barrier()
    clocks.end()
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end)
    del graph

    # ---- each launch bracketed by event nodes (a separate replay: the nodes
    #      themselves add time, so the headline graph above has none)
    try:
        dec_ev = [(torch.cuda.Event(enable_timing=True, external=True),
                   torch.cuda.Event(enable_timing=True, external=True)) for _ in range(L)]
        egraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(egraph):
            step(dec_ev)
        for _ in range(2):
            egraph.replay()
        torch.cuda.synchronize()
        ev_ms = statistics.mean(a.elapsed_time(b) for a, b in dec_ev)
        del egraph
    except TypeError:
        ev_ms = float("nan")

    # ---- the same step as three launches per layer, for comparison (not the headline)
    step_unfused()
    torch.cuda.synchronize()
    ugraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ugraph):
        step_unfused()
    for _ in range(args.warmup):
        ugraph.replay()
    barrier()
    u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    u0.record()
    for _ in range(args.steps):
        ugraph.replay()
    u1.record()
    barrier()
    unfused_ms = u0.elapsed_time(u1)
    del ugraph

    # ---- end to end through the public API with host buffers: the step's
    #      inputs (every layer's query and new K/V rows) copied in from pinned
    #      host memory in one transfer, every layer's output copied back in
    #      one, all inside the timed region
    n_q_el, n_k_el = qs[0].numel(), kn[0].numel()
    per_layer = n_q_el + 2 * n_k_el
    in_h = torch.empty(L * per_layer, dtype=torch.float16).pin_memory()
    for layer in range(L):
        base = layer * per_layer
        in_h[base:base + n_q_el] = qs[layer].reshape(-1).cpu()
        in_h[base + n_q_el:base + n_q_el + n_k_el] = kn[layer].reshape(-1).cpu()
        in_h[base + n_q_el + n_k_el:base + per_layer] = vn[layer].reshape(-1).cpu()
    in_d = torch.empty_like(in_h, device=dev)
    out_d = torch.empty((L,) + tuple(outs[0].shape), dtype=torch.float32, device=dev)
    out_h = torch.empty_like(out_d, device="cpu").pin_memory()
    qd = [in_d[l * per_layer:l * per_layer + n_q_el].view(qs[0].shape) for l in range(L)]
    knd = [in_d[l * per_layer + n_q_el:l * per_layer + n_q_el + n_k_el].view(kn[0].shape) for l in range(L)]
    vnd = [in_d[l * per_layer + n_q_el + n_k_el:(l + 1) * per_layer].view(vn[0].shape) for l in range(L)]

    def e2e_step():
        in_d.copy_(in_h, non_blocking=True)
        for layer in range(L):
            kvq.kvq_decode_step(desc, kcs[layer], vcs[layer], qd[layer], knd[layer], vnd[layer], B, ctx, scale, 0,
                                ws, out_d[layer])
        out_h.copy_(out_d, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e2e_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(e2e_graph):
        e2e_step()
    for _ in range(args.warmup):
        e2e_graph.replay()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        e2e_graph.replay()
    e1.record()
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    del e2e_graph

    # ---- max over ranks
    ms, e2e_ms, ev_ms, unfused_ms = max_over_ranks([ms, e2e_ms, ev_ms, unfused_ms], world, dev)
    dec_avg = ms / (args.steps * L)   # one launch per layer step: the average launch period

    dec_bytes, app_bytes, step_bytes = algorithmic_bytes(w, L)
    value = whole_job_gbs(world, step_bytes, args.steps, ms)
    e2e_value = whole_job_gbs(world, step_bytes, args.steps, e2e_ms)
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except OSError:
        pass
    peak = peaks.get("hbm_gbs")
    peak_src = "measured" if peak else "fallback"
    peak = peak or 6650.0
    launch_bytes = dec_bytes + app_bytes          # what one fused step launch must move
    achieved = launch_bytes / (dec_avg * 1e-3) / 1e9
    ms_step = ms / args.steps
    traffic = _profiled_traffic(w.name)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": _config(w, args, L),
            "us_per_layer_step": round(1e3 * ms_step / L, 3),
            "tokens_per_s": round(world * B * 1e3 / ms_step, 2),
            "frac_of_8tbs": round(value / 8000.0, 4),
            "splits": S,
            "roofline": {"bound": "hbm", "kernel": "fused decode step (append + split decode + combine)",
                         "achieved": round(achieved, 2),
                         "peak": peak, "peak_source": f"{peak_src} copy bandwidth", "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "algorithmic_bytes_per_launch": launch_bytes,
                         "avg_launch_us": round(dec_avg * 1e3, 3),
                         "launch_us_between_event_nodes": None if ev_ms != ev_ms else round(ev_ms * 1e3, 3)},
            "e2e": {"value": round(e2e_value, 3), "unit": UNIT,
                    "h2d_bytes_per_step": in_h.numel() * in_h.element_size(),
                    "d2h_bytes_per_step": out_h.numel() * out_h.element_size()},
            "gpu_launches": args.steps * L,
            "step_unfused_us_per_layer": round(1e3 * unfused_ms / args.steps / L, 3),
            "timing": "CUDA-graph replays of whole steps (no event nodes); avg launch = timed region / launches",
            "append_bulk": {"rows_per_layer": B * ctx * w.n_kv, "us_per_layer": round(1e3 * statistics.median(prefill_ms), 2),
                            "GB_per_s": round((B * w.n_kv * ctx * (2 * w.head_dim * 2 + row_bytes(w.k_type, w.head_dim)
                                                                     + row_bytes(w.v_type, w.head_dim)))
                                              / (statistics.median(prefill_ms) * 1e-3) / 1e9, 2)},
        }
        if clk:
            line["clocks"] = clk
        if not args.no_cpu_baseline and world == 1:
            gbs, units, secs, cores = oracle_sample(w, seconds=10.0)
            line["cpu_baseline"] = {"value": round(gbs, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
                                    "sample": f"{units} (batch row, KV head) units of one layer (ctx {w.ctx}), "
                                              f"{secs:.1f} s, 1 BLAS thread"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()


def _decode_source_sha():
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "decode_attention_q8_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.startswith("decode"):
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def _profiled_traffic(name):
    """DRAM bytes per decode launch (dram__bytes_read.sum + dram__bytes_write.sum)
    from the committed ncu summary, scaled to this workload, or None when no
    summary was taken of the decode kernel as it is now (source hash differs)."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.txt")
    try:
        lines = open(p).read().splitlines()
    except OSError:
        return None
    sha = _decode_source_sha()
    for line in lines:
        f = line.split()
        if len(f) == 3 and f[0] == name and f[2] == sha:
            return int(f[1])
    return None


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_kvq(args)


if __name__ == "__main__":
    main()
