"""Host-side logic of bench.py on CPU: the N > 1 path's max-over-ranks timing
and whole-job aggregation with two gloo ranks, and the reference arm (the
oracle on the host cores), alone and under torch.distributed.run."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    import bench
    t = bench.max_over_ranks(100.0 + 7.0 * rank, world, torch.device("cpu"))
    v = bench.job_tflops(world, 10, bench.STEP_FLOPS, t)
    out.put((rank, t, v))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_job_value_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(2))
    sys.path.insert(0, ROOT)
    import bench
    for rank, t, v in res:
        assert t == 107.0                              # the slowest rank's time
        assert abs(v - 2 * 10 * bench.STEP_FLOPS / 0.107 / 1e12) < 1e-6


def _run(cmd, env=None):
    return subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600,
                          env={**os.environ, **(env or {})})


def test_reference_arm_prints_one_line():
    r = _run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["unit"] == "TFLOP/s" and j["higher_is_better"]
    assert j["value"] > 0 and j["cpu_baseline"]["kind"] == "oracle"
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["value"] == j["value"]


def test_reference_arm_under_two_ranks_only_rank0_prints():
    r = _run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
              "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
              "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1 and json.loads(lines[0])["n_gpus"] == 2


def test_clock_summary_counts_only_samples_inside_the_timed_region():
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler("GPU-none")
    c.h, c.max_mhz = object(), 1965
    c.samples = [(0.5, 1965, 200.0, 0), (1.5, 1500, 900.0, 0x4), (2.5, 1400, 1000.0, 0x4 | 0x8),
                 (3.5, 1965, 210.0, 0)]
    c.regions = [(1.0, 3.0)]
    s = c.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == 1450 and s["sm_min_mhz"] == 1400
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"] and s["power_w_max"] == 1000.0


def test_clock_region_follows_the_watched_events():
    """The region spans from when the first timed event is seen complete to
    when the last one is: samples before the first step ran on the device or
    after the last one finished do not count, whatever the host was doing."""
    sys.path.insert(0, ROOT)
    import bench

    class Ev:
        def __init__(self):
            self.done = False

        def query(self):
            return self.done

    c = bench.ClockSampler("GPU-none")
    c.h, c.max_mhz = object(), 1965
    start, end = Ev(), Ev()
    with c.region() as reg:
        c._poll_watch(0.1)                 # nothing armed yet
        reg.watch_start(start)
        c._poll_watch(0.2)                 # armed, not complete
        assert c._watch[2] is None
        start.done = True
        c._poll_watch(0.3)
        t_start = c._watch[2]              # host time just after that poll
        assert t_start is not None
        reg.watch_end(end)
        c._poll_watch(0.4)
        assert c._watch[3] is None
        end.done = True
        c._poll_watch(5.0)
    assert c._watch is None
    assert c.regions == [(t_start, 5.0)]
    # without the watched events the region is the host time of the block
    c2 = bench.ClockSampler("GPU-none")
    with c2.region():
        pass
    (a, b), = c2.regions
    assert a <= b


def test_config_roofline_arithmetic():
    """Roofline time of a GEMM set = FLOPs at the dense FP8 peak + cast bytes
    at HBM bandwidth; 4.5 TFLOP and 8 GB take 1 ms each at 4.5 PF and 8 TB/s."""
    sys.path.insert(0, ROOT)
    import bench
    peaks = dict(hbm=8000.0, bf16=2250.0, bf16_sus=2000.0)
    e = bench.config_entry("x", 4.5e12, 8e9, 4.0, 3.0, 1.0, peaks, 1)
    assert abs(e["roofline"]["ms_nominal"] - 2.0) < 1e-9
    assert abs(e["roofline"]["frac_nominal"] - 0.5) < 1e-9
    assert abs(e["roofline"]["frac_measured_peaks"] - 0.5) < 1e-9
    assert abs(e["tflops"] - 1125.0) < 1e-6 and abs(e["pct_of_dense_fp8_peak"] - 25.0) < 1e-9
