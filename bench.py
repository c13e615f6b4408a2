"""Benchmark of the quantized-KV decode hot path on B200.

One step = one decode token through every layer of the workload: for each
layer, quantize-on-append of the new token's K/V rows (kvq_append_quantize),
split-KV decode over the whole cache (kvq_decode_attention) and the split
combine (kvq_combine).  Default workload: Llama-3.1-70B-shaped cache, 80
layers, 64 query / 8 KV heads, head_dim 128, context 32768, batch 4,
K q8_0 / V q4_0 (~17.4 GB of quantized cache, every layer a distinct 218 MB
buffer, so nothing stays in the 126 MB L2 between layers).

Prints one JSON line (rank 0).  After the headline workload the same step is
timed on the other workloads (``workloads`` in the line): the Llama-3.1-8B
layer with its f16/f16 and q8_0/q8_0 controls, long-context K4V4 at batch 1, 4
and 16, and q8_0 keys with turbo3 values.  ``--impl reference`` times the CPU
oracle instead, on a bounded sample of the same workload.
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
    ap.add_argument("--no-workloads", action="store_true", help="time the headline workload only")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch each layer's step after the previous one has finished (no programmatic "
                         "dependent launch)")
    return ap.parse_args()


def row_bytes(kind, d):
    from decode_attention_q8_b200 import kvq_row_bytes
    return kvq_row_bytes(kind, d)


def oracle_row_bytes(kind, d):
    """Row bytes by the oracle's byte model (the CPU legs load nothing of the
    library)."""
    from oracle import cache_model
    return cache_model.row_bytes(kind, d)


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

def cpu_model():
    """The host CPU's model name (/proc/cpuinfo), or the platform's description."""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


class OracleStep:
    """The oracle's decode step on one batch row of one layer of workload w: the
    new token's K/V rows quantized, then every cached row of the KV heads
    dequantized and attended in binary64 (oracle/attention.cc,
    orc_decode_cache).  The cache is quantized once, by the oracle, from the
    workload's seeded inputs."""

    def __init__(self, w):
        import numpy as np
        import synth
        from oracle import blocks, qjl, turbo
        self.w = w
        q, k, v = synth.layer_inputs(w, layer=0, device="cpu", batch=1)
        self.q = q.numpy()
        k, v = k.numpy().transpose(0, 2, 1, 3), v.numpy().transpose(0, 2, 1, 3)  # [1, n_kv, T, D]
        self.proj = synth.qjl_projection(w.seed, w.head_dim).numpy() if "qjl" in w.k_type else None

        def store(kind, x):
            if kind == "f16":
                return np.ascontiguousarray(x).view(np.uint8), np.zeros((*x.shape[:-1], 0), np.float16)
            if kind == "q8_0":
                d, qq = blocks.quantize_q8_0(x)
                return qq.view(np.uint8), d
            if kind == "q4_0":
                d, qs = blocks.quantize_q4_0(x)
                return qs, d
            if kind == "q5_0":
                d, qs, qh = blocks.quantize_q5_0(x)
                return qs, np.concatenate([d, np.ascontiguousarray(qh).view(np.float16)], axis=-1)
            if kind == "turbo3_qjl":
                sc, codes = qjl.quantize(x, w.turbo_seed, self.proj)
                return codes, sc
            n, codes = turbo.quantize(x, w.turbo_seed, turbo.BITS[kind])
            return codes, n[..., None]

        self.store = store
        self.k, self.v = store(w.k_type, k), store(w.v_type, v)
        self.k_new, self.v_new = k[:, :, -1:], v[:, :, -1:]
        rk, rv = oracle_row_bytes(w.k_type, w.head_dim), oracle_row_bytes(w.v_type, w.head_dim)
        # algorithmic bytes of one batch row's step (as the GPU step counts them)
        self.bytes = (w.n_kv * w.ctx * (rk + rv) + w.n_q * w.head_dim * (2 + 4)
                      + w.n_kv * (2 * w.head_dim * 2 + rk + rv))

    def run(self, threads):
        from oracle import attention
        w = self.w
        self.store(w.k_type, self.k_new)
        self.store(w.v_type, self.v_new)
        attention.decode_cache(w.k_type, w.v_type, self.k[0], self.k[1], self.v[0], self.v[1], self.q, w.scale,
                               seed=w.turbo_seed, proj=self.proj, threads=threads)


def oracle_sample(w, seconds=10.0, threads=1, step=None):
    """Times the oracle's decode step (OracleStep) on `threads` host threads
    (<= 0: all), repeated while the total stays under about `seconds` (at
    least once); returns (GB/s, batch rows done, seconds, threads used)."""
    from oracle import attention
    step = step or OracleStep(w)
    used = threads if threads > 0 else attention.hardware_threads()
    done, total = 0, 0.0
    while done == 0 or total + total / done <= seconds:
        t0 = time.perf_counter()
        step.run(used)
        total += time.perf_counter() - t0
        done += 1
    return done * step.bytes / total / 1e9, done, total, used


def cpu_baseline(w, seconds_one=10.0, seconds_all=5.0):
    """The oracle's step on one host core and on all of them (bounded samples)."""
    step = OracleStep(w)
    one, n1, s1, _ = oracle_sample(w, seconds_one, 1, step)
    alln, na, sa, cores = oracle_sample(w, seconds_all, 0, step)
    return {"value": round(one, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
            "value_all_cores": round(alln, 6), "cores_all": cores, "cpu_model": cpu_model(),
            "sample": f"one batch row ({w.n_kv} KV heads) of one layer, ctx {w.ctx}: append the new row, "
                      f"dequantize every cached row, binary64 attention (C++ oracle); {n1} run(s) in {s1:.1f} s "
                      f"on 1 core, {na} run(s) in {sa:.1f} s on {cores} threads"}


def run_reference(args):
    import synth
    if rank_env()[1] != 0:
        return   # the oracle baseline runs on rank 0 only
    w = synth.WORKLOADS[args.workload]
    # one step = the oracle's decode step on one batch row of one layer, all host threads
    step = OracleStep(w)
    from oracle import attention
    cores = attention.hardware_threads()
    for _ in range(args.warmup):
        step.run(cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step.run(cores)
    secs = time.perf_counter() - t0
    gbs = args.steps * step.bytes / secs / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 6), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / max(args.steps, 1), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _config(w, args, None),
        "cpu_baseline": {"value": round(gbs, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "cpu_model": cpu_model(),
                         "sample": f"each step: one batch row ({w.n_kv} KV heads) of layer 0, ctx {w.ctx}, "
                                   f"append + dequantize + binary64 attention (C++ oracle), {cores} threads"},
        "e2e": {"value": round(gbs, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _config(w, args, n_layers):
    return {"workload": w.name, "layers": n_layers or w.layers, "batch": w.batch, "n_q_heads": w.n_q,
            "n_kv_heads": w.n_kv, "head_dim": w.head_dim, "ctx": w.ctx, "k_type": w.k_type,
            "v_type": w.v_type, "step": "per layer: one fused launch (append 1 row + split decode + combine)",
            "launch": ("each layer's step launched after the previous one finished" if args.no_overlap else
                       "programmatic dependent launch: each layer's step may start (and request its first cache "
                       "tiles) while the previous layer's finishes"),
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

# Workloads timed after the headline one (the line's "workloads" map):
# (entry name, workload, (k_type, v_type) override or None, layers override or 0).
# The 8B layer is one layer; 40 distinct layer caches keep its footprint above
# 4x the 126 MB L2 (13.6 MB each).
EXTRA_WORKLOADS = (
    ("llama8b_ctx8k", "llama8b_ctx8k", None, 40),
    ("llama8b_ctx8k_f16", "llama8b_ctx8k", ("f16", "f16"), 40),
    ("llama8b_ctx8k_q8_0", "llama8b_ctx8k", ("q8_0", "q8_0"), 40),
    ("k4v4_ctx128k_b1", "k4v4_ctx128k_b1", None, 0),
    ("k4v4_ctx128k_b4", "k4v4_ctx128k_b4", None, 0),
    ("k4v4_ctx128k_b16", "k4v4_ctx128k_b16", None, 0),
    ("turbo3_ctx32k", "turbo3_ctx32k", None, 0),
    ("turbo3_ctx32k_b4", "turbo3_ctx32k_b4", None, 0),
    ("qjl_ctx32k_b4", "qjl_ctx32k_b4", None, 0),
)


class StepRun:
    """One workload on this GPU: every layer's cache prefilled by the bulk
    append (timed), then the decode step (one fused launch per layer: append the
    token's K/V row, split decode, combine) captured in a CUDA graph and timed
    by replays."""

    def __init__(self, w, L, dev, world, local, overlap=True):
        import torch
        import decode_attention_q8_b200 as kvq
        import synth
        self.w, self.L, self.dev, self.world, self.local = w, L, dev, world, local
        self.kvq = kvq
        _, rank, _ = rank_env()
        # each layer's step may start while the previous layer's finishes: the
        # kernel before it on the stream is another layer's step (or the bulk
        # append of another layer's cache), which writes nothing this one reads
        # before the dependency resolves
        flags = kvq.KVQ_FLAG_OVERLAP_PREVIOUS if overlap else 0
        # turbo3_qjl keys: the seeded projection, on the device for the library
        self.proj = synth.qjl_projection(w.seed, w.head_dim).to(dev) if w.k_type == "turbo3_qjl" else None
        self.desc = kvq.make_desc(w.n_q, w.n_kv, w.head_dim, w.k_type, w.v_type, w.ctx, turbo_seed=w.turbo_seed,
                                  qjl_proj=self.proj, flags=flags)
        B, ctx = w.batch, w.ctx
        stream = torch.cuda.current_stream(dev)  # prefill and the timed steps run on it
        self.kcs, self.vcs, self.qs, self.kn, self.vn = [], [], [], [], []
        pre_ev = []
        for layer in range(L):
            q, k, v = synth.layer_inputs(w, layer=layer + 1000 * rank, device=dev)
            kc = torch.empty(kvq.kvq_cache_bytes(self.desc, B, 0), dtype=torch.uint8, device=dev)
            vc = torch.empty(kvq.kvq_cache_bytes(self.desc, B, 1), dtype=torch.uint8, device=dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            kvq.kvq_append_quantize(self.desc, kc, vc, k, v, B, 0, ctx, stream)
            e1.record(stream)
            pre_ev.append((e0, e1))
            self.kcs.append(kc)
            self.vcs.append(vc)
            self.qs.append(q)
            self.kn.append(k[:, ctx - 1:ctx].contiguous())
            self.vn.append(v[:, ctx - 1:ctx].contiguous())
            del k, v
        if L < 3:
            # the first call of a process includes loading the kernel: with few
            # layers, time warm repeats of layer 0's append too (same rows, same bytes)
            _, k, v = synth.layer_inputs(w, layer=1000 * rank, device=dev)
            for _ in range(3):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                kvq.kvq_append_quantize(self.desc, self.kcs[0], self.vcs[0], k, v, B, 0, ctx, stream)
                e1.record(stream)
                pre_ev.append((e0, e1))
            del k, v
        torch.cuda.synchronize()
        self.prefill_ms = [a.elapsed_time(b) for a, b in pre_ev[1:]]
        torch.cuda.empty_cache()
        self.S = kvq.kvq_auto_splits(self.desc, B, ctx)
        # arrival counters start at 0
        self.ws = torch.zeros(kvq.kvq_workspace_bytes(self.desc, B, 0), dtype=torch.uint8, device=dev)
        self.outs = [torch.empty((B, w.n_q, w.head_dim), dtype=torch.float32, device=dev) for _ in range(L)]

    def step(self, events=None, qs=None, kn=None, vn=None, outs=None):
        """One decode token through every layer, launched on the current stream."""
        w, kvq = self.w, self.kvq
        qs, kn, vn, outs = qs or self.qs, kn or self.kn, vn or self.vn, outs or self.outs
        for layer in range(self.L):
            if events is not None:
                events[layer][0].record()
            kvq.kvq_decode_step(self.desc, self.kcs[layer], self.vcs[layer], qs[layer], kn[layer], vn[layer], w.batch,
                                w.ctx, w.scale, 0, self.ws, outs[layer])
            if events is not None:
                events[layer][1].record()

    def step_unfused(self):
        """The same step as three launches per layer (append, decode, combine)."""
        w, kvq = self.w, self.kvq
        for layer in range(self.L):
            kvq.kvq_append_quantize(self.desc, self.kcs[layer], self.vcs[layer], self.kn[layer], self.vn[layer],
                                    w.batch, w.ctx - 1, 1)
            kvq.kvq_decode_attention(self.desc, self.kcs[layer], self.vcs[layer], self.qs[layer], w.batch, w.ctx,
                                     w.scale, 0, self.ws)
            kvq.kvq_combine(self.desc, self.ws, w.batch, w.ctx, 0, self.outs[layer])

    def barrier(self):
        import torch
        import torch.distributed as dist
        if self.world > 1:
            dist.barrier(device_ids=[self.local])
        torch.cuda.synchronize()

    def time_graph(self, fn, steps, warmup, clocks=None):
        """Captures fn() in a CUDA graph, replays it `warmup` times, then times
        `steps` replays between barriers with CUDA events; returns ms."""
        import torch
        fn()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            fn()
        for _ in range(warmup):
            graph.replay()
        self.barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if clocks is not None:
            clocks.begin()
        t0.record()
        for _ in range(steps):
            graph.replay()
        t1.record()
        self.barrier()
        if clocks is not None:
            clocks.end()
        del graph
        return t0.elapsed_time(t1)

    def event_launch_ms(self):
        """Mean launch time with each launch bracketed by event nodes (a separate
        replay: the nodes themselves add time, so the headline graph has none)."""
        import torch
        try:
            ev = [(torch.cuda.Event(enable_timing=True, external=True),
                   torch.cuda.Event(enable_timing=True, external=True)) for _ in range(self.L)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.step(ev)
            for _ in range(2):
                g.replay()
            torch.cuda.synchronize()
            ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
            del g
            return ms
        except TypeError:
            return float("nan")

    def e2e(self, steps, warmup):
        """The step through the public API with host buffers: every layer's query
        and new K/V rows copied in from pinned host memory in one transfer, every
        layer's output copied back in one, all inside the timed region.
        Returns (ms, h2d bytes, d2h bytes) per the `steps` replays."""
        import torch
        L, dev = self.L, self.dev
        n_q_el, n_k_el = self.qs[0].numel(), self.kn[0].numel()
        per_layer = n_q_el + 2 * n_k_el
        in_h = torch.empty(L * per_layer, dtype=torch.float16).pin_memory()
        for layer in range(L):
            base = layer * per_layer
            in_h[base:base + n_q_el] = self.qs[layer].reshape(-1).cpu()
            in_h[base + n_q_el:base + n_q_el + n_k_el] = self.kn[layer].reshape(-1).cpu()
            in_h[base + n_q_el + n_k_el:base + per_layer] = self.vn[layer].reshape(-1).cpu()
        in_d = torch.empty_like(in_h, device=dev)
        out_d = torch.empty((L,) + tuple(self.outs[0].shape), dtype=torch.float32, device=dev)
        out_h = torch.empty_like(out_d, device="cpu").pin_memory()
        qd = [in_d[l * per_layer:l * per_layer + n_q_el].view(self.qs[0].shape) for l in range(L)]
        knd = [in_d[l * per_layer + n_q_el:l * per_layer + n_q_el + n_k_el].view(self.kn[0].shape) for l in range(L)]
        vnd = [in_d[l * per_layer + n_q_el + n_k_el:(l + 1) * per_layer].view(self.vn[0].shape) for l in range(L)]
        outs = [out_d[l] for l in range(L)]

        def e2e_step():
            in_d.copy_(in_h, non_blocking=True)
            self.step(qs=qd, kn=knd, vn=vnd, outs=outs)
            out_h.copy_(out_d, non_blocking=True)

        ms = self.time_graph(e2e_step, steps, warmup)
        return ms, in_h.numel() * in_h.element_size(), out_h.numel() * out_h.element_size()

    def prefill_summary(self):
        w = self.w
        med = statistics.median(self.prefill_ms)
        moved = w.batch * w.n_kv * w.ctx * (2 * w.head_dim * 2 + row_bytes(w.k_type, w.head_dim)
                                            + row_bytes(w.v_type, w.head_dim))
        return {"rows_per_layer": w.batch * w.ctx * w.n_kv, "us_per_layer": round(1e3 * med, 2),
                "GB_per_s": round(moved / (med * 1e-3) / 1e9, 2)}

    def release(self):
        import torch
        self.kcs = self.vcs = self.qs = self.kn = self.vn = self.outs = self.ws = None
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def measured_peak():
    """(HBM GB/s, source): the measured copy bandwidth from MEASURED_PEAKS.json,
    else the profiling recipe's fallback."""
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        peaks = {}
    if peaks.get("hbm_gbs"):
        return float(peaks["hbm_gbs"]), "measured copy bandwidth"
    return 6650.0, "fallback copy bandwidth"


def run_extra(name, w, L, args, dev, world, local):
    """One entry of the line's "workloads" map: the fused step timed as the
    headline is (graph replays, max over ranks), its roofline fraction and its
    end-to-end rate through host buffers."""
    run = StepRun(w, L, dev, world, local, overlap=not args.no_overlap)
    clocks = ClockSampler(local, enabled=not args.no_clocks)
    ms = run.time_graph(run.step, args.steps, args.warmup, clocks)
    clk = clocks.stop()
    e2e_ms, h2d, d2h = run.e2e(args.steps, args.warmup)
    ms, e2e_ms = max_over_ranks([ms, e2e_ms], world, dev)
    dec_bytes, app_bytes, step_bytes = algorithmic_bytes(w, L)
    peak, _ = measured_peak()
    launch_us = 1e3 * ms / (args.steps * L)
    achieved = (dec_bytes + app_bytes) / (launch_us * 1e-6) / 1e9
    entry = {"workload": w.name, "layers": L, "batch": w.batch, "ctx": w.ctx, "k_type": w.k_type,
             "v_type": w.v_type, "splits": run.S, "us_per_layer_step": round(launch_us, 3),
             "GB_per_s": round(whole_job_gbs(world, step_bytes, args.steps, ms), 2),
             "frac": round(achieved / peak, 4), "frac_of_8tbs": round(achieved / 8000.0, 4),
             "algorithmic_bytes_per_launch": dec_bytes + app_bytes,
             "tokens_per_s": round(world * w.batch * 1e3 / (ms / args.steps), 2),
             "e2e": {"value": round(whole_job_gbs(world, step_bytes, args.steps, e2e_ms), 2), "unit": UNIT,
                     "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
             "traffic": _profiled_traffic(name), "append_bulk": run.prefill_summary()}
    if clk:
        entry["clocks"] = clk
    run.release()
    return entry


def run_kvq(args):
    import dataclasses
    import torch
    import torch.distributed as dist

    import synth

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = synth.WORKLOADS[args.workload]
    L = args.layers or w.layers
    B = w.batch
    run = StepRun(w, L, dev, world, local, overlap=not args.no_overlap)

    # warm-up eagerly (first calls set kernel attributes), then the timed replays
    for _ in range(args.warmup):
        run.step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local, enabled=not args.no_clocks)
    ms = run.time_graph(run.step, args.steps, args.warmup, clocks)
    clk = clocks.stop()
    ev_ms = run.event_launch_ms()
    unfused_ms = run.time_graph(run.step_unfused, args.steps, args.warmup)
    e2e_ms, h2d, d2h = run.e2e(args.steps, args.warmup)

    # ---- max over ranks
    ms, e2e_ms, ev_ms, unfused_ms = max_over_ranks([ms, e2e_ms, ev_ms, unfused_ms], world, dev)
    dec_avg = ms / (args.steps * L)   # one launch per layer step: the average launch period
    prefill = run.prefill_summary()
    S = run.S
    run.release()

    dec_bytes, app_bytes, step_bytes = algorithmic_bytes(w, L)
    value = whole_job_gbs(world, step_bytes, args.steps, ms)
    e2e_value = whole_job_gbs(world, step_bytes, args.steps, e2e_ms)
    peak, peak_src = measured_peak()
    launch_bytes = dec_bytes + app_bytes          # what one fused step launch must move
    achieved = launch_bytes / (dec_avg * 1e-3) / 1e9
    ms_step = ms / args.steps
    traffic = _profiled_traffic(w.name)

    # ---- the other workloads, each timed the same way (replicas on every rank)
    workloads = {}
    if not args.no_workloads and args.layers == 0:
        for name, wname, types, layers in EXTRA_WORKLOADS:
            wx = synth.WORKLOADS[wname]
            if types is not None:
                wx = dataclasses.replace(wx, k_type=types[0], v_type=types[1])
            if wname == w.name and types is None:
                continue
            workloads[name] = run_extra(name, wx, layers or wx.layers, args, dev, world, local)

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
                         "peak": peak, "peak_source": peak_src, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "algorithmic_bytes_per_launch": launch_bytes,
                         "avg_launch_us": round(dec_avg * 1e3, 3),
                         "launch_us_between_event_nodes": None if ev_ms != ev_ms else round(ev_ms * 1e3, 3)},
            "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps * L,
            "step_unfused_us_per_layer": round(1e3 * unfused_ms / args.steps / L, 3),
            "timing": "CUDA-graph replays of whole steps (no event nodes); avg launch = timed region / launches",
            "append_bulk": prefill,
        }
        if clk:
            line["clocks"] = clk
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(w)
            if "turbo3_ctx32k" in workloads:
                workloads["turbo3_ctx32k"]["cpu_baseline"] = cpu_baseline(synth.WORKLOADS["turbo3_ctx32k"],
                                                                          seconds_one=8.0, seconds_all=4.0)
        if workloads:
            line["workloads"] = workloads
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()


# Sources of the decode kernel: its own files and the headers it includes
# (the fused step's row append and the shared parameter structs).
DECODE_HEADERS = ("append_rows.cuh", "kvq_internal.h")


def _decode_source_sha():
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "decode_attention_q8_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.startswith("decode") or f in DECODE_HEADERS:
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
