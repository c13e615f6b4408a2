"""Host logic of bench.py without a GPU: the clock sampler's timed window, the
traffic record lookup, and the multi-rank path (max over ranks, whole-job
throughput, rank-0-only reference arm) on world-size-2 gloo process groups."""

import importlib.util
import json
import os
import socket
import subprocess
import sys
import time

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_clock_sampler_keeps_only_the_timed_window():
    bench = _bench()
    state = {"phase": "before"}

    def fake_query():
        if state["phase"] == "inside":
            return 1965.0, {"sw_power_cap"}
        return 1200.0, {"hw_slowdown"} if state["phase"] == "after" else set()

    s = bench.ClockSampler(0, enabled=True, period_s=0.002, query=fake_query)
    s.max_mhz = 1965.0
    time.sleep(0.03)
    state["phase"] = "inside"
    time.sleep(0.01)      # let the sampler see the new phase before the window opens
    s.begin()
    time.sleep(0.05)
    s.end()
    time.sleep(0.01)
    state["phase"] = "after"
    time.sleep(0.03)
    out = s.stop()
    assert out is not None and out["samples"] >= 5
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_sampler_disabled_returns_none():
    assert _bench().ClockSampler(0, enabled=False).stop() is None


def test_traffic_record_matches_source_hash(tmp_path, monkeypatch):
    bench = _bench()
    csrc = tmp_path / "decode_attention_q8_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "decode_x.cu").write_text("// kernel v1\n")
    (csrc / "other.cu").write_text("// not hashed\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench._decode_source_sha()
    (tmp_path / "profiles" / "decode_traffic.txt").write_text(
        f"# workload bytes sha\nwl_a 123456 {sha}\nwl_b 999 0000000000000000\n")
    assert bench._profiled_traffic("wl_a") == 123456
    assert bench._profiled_traffic("wl_b") is None          # taken of another kernel version
    (csrc / "other.cu").write_text("// edited\n")            # files not named decode* do not count
    assert bench._profiled_traffic("wl_a") == 123456
    (csrc / "decode_x.cu").write_text("// kernel v2\n")      # the kernel changed: counters are stale
    assert bench._profiled_traffic("wl_a") is None
    # the headers the decode kernel includes count too
    sha2 = bench._decode_source_sha()
    (tmp_path / "profiles" / "decode_traffic.txt").write_text(f"wl_a 123456 {sha2}\n")
    assert bench._profiled_traffic("wl_a") == 123456
    (csrc / "append_rows.cuh").write_text("// the fused step's row append\n")
    assert bench._profiled_traffic("wl_a") is None


def test_whole_job_throughput_is_weak_scaling():
    bench = _bench()
    one = bench.whole_job_gbs(1, 1e9, 10, 1000.0)
    assert one == pytest.approx(10.0)
    # two replicas, the slower rank's time: twice the bytes in that time
    assert bench.whole_job_gbs(2, 1e9, 10, 1250.0) == pytest.approx(16.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench = _bench()
        w, r, l = bench.rank_env()
        # rank-dependent timings: rank 1 is slower in the first, rank 0 in the second
        vals = bench.max_over_ranks([10.0 + r, 20.0 - r, 5.0], w, "cpu")
        dist.barrier()
        q.put((r, w, l, vals, bench.whole_job_gbs(w, 2e9, 4, vals[0])))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got.sort()
    assert [g[0] for g in got] == [0, 1] and all(g[1] == 2 for g in got)
    assert [g[2] for g in got] == [0, 1]
    for _, _, _, vals, gbs in got:
        assert vals == [11.0, 20.0, 5.0]            # every rank sees the max of each timing
        assert gbs == pytest.approx(2 * 2e9 * 4 / 11e-3 / 1e9)


def _gather_main(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import decode_attention_q8_b200 as kvq
        region = torch.arange(10, dtype=torch.uint8) + 100 * rank  # this rank's partials, as bytes
        q.put((rank, kvq.gather_partials(region).tolist()))
    finally:
        dist.destroy_process_group()


def test_partials_gather_is_rank_major_on_two_gloo_ranks():
    """The exchange step of a context split: every rank ends with all ranks'
    partial regions back to back, rank 0 first."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    expect = list(range(10)) + [100 + i for i in range(10)]
    assert sorted(got) == [(0, expect), (1, expect)]


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0", "--workload", "tiny"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_on_rank_zero():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--workload", "tiny"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_loads_nothing_of_the_library():
    """The oracle arm runs the C++ oracle only: after it, neither the library's
    binding nor libkvq.so is loaded in the process."""
    code = ("import runpy, sys\n"
            "sys.argv = ['bench.py', '--impl', 'reference', '--workload', 'tiny', '--steps', '1', '--warmup', '0']\n"
            f"runpy.run_path({os.path.join(ROOT, 'bench.py')!r}, run_name='__main__')\n"
            "maps = open('/proc/self/maps').read()\n"
            "print('LIB' if ('decode_attention_q8_b200' in sys.modules or 'libkvq' in maps) else 'CLEAN')\n"
            "print('ORACLE' if 'liboracle' in maps else 'NO-ORACLE')\n")
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    out = r.stdout.strip().splitlines()
    assert out[-2:] == ["CLEAN", "ORACLE"], out
