#!/usr/bin/env python
"""Throughput of the FP8 relu^2 MLP block, forward + dgrad + wgrad, on B200.

Workload: the 3.8B-shape relu^2 MLP block, M = 16384 tokens (8 x 2048),
d = 3072, f = 12288; X ~ N(0,1), W_up, W_down ~ N(0, 0.02), dY ~ N(0, 1e-3),
synthetic and seeded.  One step = lm_relu2_mlp_fwd + lm_relu2_mlp_bwd: six
FP8 GEMMs (2 * 16384 * 3072 * 12288 flops each) plus every amax/cast.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  N > 1 runs one independent replica per GPU
(launched by torch.distributed.run): the path has no exchange step, so there
is no data-path collective and scaling is weak.

Timing: CUDA events on the launching stream around each step, L2 flushed
(a 256 MiB write) before every timed step, W untimed warm-up steps, max over
ranks.  Each timed loop starts behind a short device-side sleep, so the host
is already ahead of the GPU when the first timed step starts and a host-side
stall while it issues later steps does not leave the GPU idle inside one.
SM clocks and clock-event reasons are sampled in-process through NVML every
few milliseconds; only samples taken while the timed steps ran on the device
count (the sampler watches the first start and the last end event).

Besides the headline (the fwd + bwd block at M = 16384), the same JSON line
carries the other GEMM sets of the little-lm model under "configs", each timed
the same way with its own oracle sample: the MLP forward alone (M = 16384),
the attention projections + LM head (M = 8192) and the 28-layer stack's
linear-layer set (M = 16384, t3 activations).
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP8 TFLOP/s (fwd+dgrad+wgrad) relu² MLP d=3072, % of dense FP8 peak"
M_TOK, D_MODEL, D_FF = 16384, 3072, 12288
GEMM_FLOPS = 2 * M_TOK * D_MODEL * D_FF        # each of the six GEMMs
STEP_FLOPS = 6 * GEMM_FLOPS
DENSE_FP8_PEAK_TFLOPS = 4500.0                 # public B200 dense FP8 figure
PAGES_FP8_PEAK_TFLOPS = 4190.0                 # the dense FP8 peak the pages' MFU figure implies
NOMINAL_FP8_OVER_BF16 = 2.0                    # 4.5 / 2.25 PFLOP/s dense
WORKLOAD = "relu2 MLP fwd+dgrad+wgrad M=16384 d=3072 f=12288"
LAUNCHES_PER_STEP = 10                         # kernels of ours per fwd+bwd: "acggacgggg"

# DRAM traffic of one GEMM launch from an ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum), valid only for the kernel source it was taken on;
# the summary and the command are in profiles/.  Taken on the source with
# sha256 a9aaa2d5389fdca3657e531b4b9b3ced39f8c2d80d4cd714ea66b6ab6f9cbb9e; the
# file recorded here differs from it in host code only (how the dispatcher
# treats an empty side-cast tensor), and its compiled device code without line
# information is byte-identical to that source's.
GEMM_TRAFFIC = {
    "source_sha256": "0e123c3b8a0053a031744441664db7012c4c4b211cd815114a45108732abcc4a",
    "bytes_per_launch": 493504981,  # mean over the step's six GEMM shapes, one capture each
}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-sample-tokens", type=int, default=256)
    p.add_argument("--no-configs", action="store_true",
                   help="skip the other GEMM sets (MLP forward, attention + head, stack)")
    p.add_argument("--config-steps", type=int, default=20)
    p.add_argument("--stack-steps", type=int, default=3)
    return p.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p["bf16_tflops_sustained"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ----------------------------------------------------------------- clocks
REASON_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}


class ClockSampler:
    """Samples the SM clock, power and clock-event reasons of one GPU through
    NVML from a host thread every ~2 ms.  region() marks the timed region; the
    summary uses only the samples taken inside it.  The thread also polls the
    region's watched CUDA events (Event.query is thread-safe)."""

    def __init__(self, uuid):
        self.uuid = uuid
        self.samples = []   # (t, sm_mhz, power_w, reasons)
        self.regions = []
        self._stop = threading.Event()
        self._watch = None  # [start event, end event, t seen done, t seen done]
        self.h = None
        self.max_mhz = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.h = None
        if self.h is not None:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def _run(self):
        nv, h = self.nv, self.h
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                t = time.perf_counter()
                self.samples.append((t, sm, pw, rs))
                self._poll_watch(t)
            except Exception:
                pass
            time.sleep(0.002)

    def _poll_watch(self, t):
        """After the sample taken at t: note when the watched start event is
        first seen complete (the samples after this one count) and then when
        the end event is (the sample at t is the last that counts)."""
        w = self._watch
        if w is None:
            return
        if w[2] is None and w[0] is not None and w[0].query():
            w[2] = time.perf_counter()
        if w[2] is not None and w[3] is None and w[1] is not None and w[1].query():
            w[3] = t

    def __exit__(self, *exc):
        self._stop.set()
        if self.h is not None:
            self.thread.join(timeout=5)
            try:
                self.nv.nvmlShutdown()
            except Exception:
                pass

    class _Region:
        def __init__(self, owner):
            self.owner = owner

        def __enter__(self):
            self.t0 = time.perf_counter()
            self.owner._watch = [None, None, None, None]
            return self

        def watch_start(self, ev):
            """ev: the first timed event, already recorded."""
            self.owner._watch[0] = ev

        def watch_end(self, ev):
            """ev: the last timed event, already recorded."""
            self.owner._watch[1] = ev

        def __exit__(self, *exc):
            o = self.owner
            w = o._watch
            if o.h is not None and w[1] is not None:
                deadline = time.perf_counter() + 0.5
                while w[3] is None and time.perf_counter() < deadline:
                    time.sleep(0.002)
            o._watch = None
            t1 = time.perf_counter()
            o.regions.append((w[2] if w[2] is not None else self.t0,
                              w[3] if w[3] is not None else t1))

    def region(self):
        """The timed region.  By default the host time inside the with-block;
        once watch_start() and watch_end() have handed it the recorded CUDA
        events that open and close the timed steps, the span from when the
        sampler thread first saw the first complete to when it first saw the
        second complete (2 ms resolution)."""
        return ClockSampler._Region(self)

    def summary(self, region=0):
        if self.h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"],
                    "samples": 0, "source": "nvml"}
        t0, t1 = self.regions[region]
        rows = [r for r in self.samples if t0 <= r[0] <= t1]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"],
                    "samples": 0, "source": "nvml"}
        sm = [r[1] for r in rows]
        reasons = sorted({n for r in rows for n, b in REASON_BITS.items() if r[3] & b})
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_p90_mhz":
                sorted(sm)[int(0.9 * (len(sm) - 1))], "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(rows),
                "region_s": round(t1 - t0, 4), "power_w_max": max(r[2] for r in rows),
                "source": "nvml, in-process, ~2 ms period, samples taken while the timed "
                          "steps ran on the device only"}


# ------------------------------------------------------------ GPU pieces
def make_inputs(torch, device):
    from fp8_gemms_b200 import synthetic
    t = synthetic.MLP_FWD_BWD.tensors()
    return t, {k: v.to(device) for k, v in t.items()}


def max_over_ranks(x, world, device):
    """Max of a per-rank float over all ranks (the job's time is its slowest
    rank's).  Every rank must call it, in the same order."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def host_ahead(torch, steps):
    """Queues a device-side sleep of about half a millisecond per step to come
    (at most 10 ms) ahead of a timed loop.  The host issues a step's launches
    in well under that (bench.py reports host_issue_ms_per_step), so it is
    several steps ahead when the first timed step starts and pulls further
    ahead with every step; a host-side stall while it issues later steps then
    cannot leave the GPU idle inside a timed step.  The sleep lies before the
    first timed event."""
    torch.cuda._sleep(int(min(10.0, 0.5 * steps) * 2.0e6))   # ~2e6 SM cycles per ms


def job_tflops(world, steps, flops_per_step, total_ms):
    """Whole-job throughput: the units all ranks processed over the job's time."""
    return world * steps * flops_per_step / (total_ms * 1e-3) / 1e12


# algorithmic bytes of the cast launches of one step: a full cast (amax pass +
# cast pass) moves 2 B (amax read) + 2 B (read) + 1 B (codes) per element; a
# cast whose amax came from a GEMM epilogue 2 + 1 B.  The launches: the amax
# of X, W_up and W_down; the casts of X and W_up; the amax and cast of dY.
# W_down's codes, h's and dH's (3 B/element each after their amax) are cast
# by side warps of the up, down and dW_down GEMMs, inside those launches.
# Only row-major codes are written: the backward's GEMMs read them MN-major.
def cast_bytes():
    Md, fd = M_TOK * D_MODEL, D_FF * D_MODEL
    return [5 * Md, 5 * fd, 2 * fd, 5 * Md]


def src_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def run_gpu(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from fp8_gemms_b200 import _lib as lib
    from fp8_gemms_b200 import api

    host, dev = make_inputs(torch, device)
    mlp = api.Relu2Mlp(M_TOK, D_MODEL, D_FF, device=device)
    for name, shape in [("Y", (M_TOK, D_MODEL)), ("dX", (M_TOK, D_MODEL)),
                        ("dW_up", (D_FF, D_MODEL)), ("dW_down", (D_MODEL, D_FF))]:
        dev[name] = torch.empty(*shape, dtype=torch.bfloat16, device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def step():
        mlp.forward(dev["X"], dev["W_up"], dev["W_down"], Y=dev["Y"])
        mlp.backward(dev["dY"], dX=dev["dX"], dW_up=dev["dW_up"], dW_down=dev["dW_down"])

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        step()
    st, where = lib.lm_get_error()
    if st != 0:
        raise RuntimeError(f"device error {st} at wait {where:#x}")

    # ---- timed region: K steps through the two C-ABI calls; the library
    # records an event before each of its kernel launches (lm_timing_attach).
    # A region whose clock record shows a hardware or thermal slowdown is
    # measured once more (every rank takes the same decision), and the line
    # names the reasons that the first one saw.
    K = args.steps
    props = torch.cuda.get_device_properties(device)
    uuid = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else ""
    slow_reasons = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")
    first_reasons = None
    for attempt in range(2):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        timers = [lib.KernelTimer(2 * LAUNCHES_PER_STEP) for _ in range(K)]
        barrier()
        with ClockSampler(uuid) as clk:
            host_ahead(torch, K)
            with clk.region() as reg:
                t_issue = time.perf_counter()
                for k in range(K):
                    flush.fill_(k & 0xFF)
                    starts[k].record()
                    if k == 0:
                        reg.watch_start(starts[0])
                    with timers[k]:
                        step()
                    ends[k].record()
                reg.watch_end(ends[-1])
                t_issue = time.perf_counter() - t_issue
                barrier()
        clocks = clk.summary()
        slow = sorted(set(clocks.get("reasons") or []) & set(slow_reasons))
        if attempt == 1 or max_over_ranks(1.0 if slow else 0.0, world, device) == 0.0:
            break
        first_reasons = slow or ["on another rank"]
        time.sleep(2.0)
    if first_reasons:
        clocks["remeasured_after"] = first_reasons
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), world, device)
    st, where = lib.lm_get_error()
    if st != 0:
        raise RuntimeError(f"device error {st} at wait {where:#x}")
    kinds = timers[0].kinds
    assert all(tm.kinds == kinds for tm in timers), "launch sequence changed between steps"
    assert len(kinds) == LAUNCHES_PER_STEP, kinds
    per_launch = [[] for _ in kinds]
    lead_ms = []
    for k in range(K):
        for j, d in enumerate(timers[k].durations_ms(ends[k])):
            per_launch[j].append(d)
        lead_ms.append(starts[k].elapsed_time(timers[k].events[0]))
    avg = [statistics.mean(v) for v in per_launch]
    gemm_ms = [a for a, kd in zip(avg, kinds) if kd == "g"]
    cast_ms = [a for a, kd in zip(avg, kinds) if kd != "g"]
    gemm_avg_ms = statistics.mean(gemm_ms)

    # ---- the same step with the weight casts cached: the forward reuses the
    # codes and scales of W_up and W_down (LM_MLP_REUSE_WEIGHT_CASTS), as every
    # micro-batch after the first of an optimizer step does.  Timed like the
    # headline region, from a similar power state: the GPU idles for a second
    # (the headline region starts after the process's set-up), then its own
    # warm-up steps, then the timed steps with their own clock record.
    Kc = min(K, 50)
    c_start = [torch.cuda.Event(enable_timing=True) for _ in range(Kc)]
    c_end = [torch.cuda.Event(enable_timing=True) for _ in range(Kc)]
    mlp.forward(dev["X"], dev["W_up"], dev["W_down"], Y=dev["Y"])  # casts of these weights

    def cached_step():
        mlp.forward(dev["X"], None, None, Y=dev["Y"], reuse_weight_casts=True)
        mlp.backward(dev["dY"], dX=dev["dX"], dW_up=dev["dW_up"], dW_down=dev["dW_down"])

    barrier()
    time.sleep(1.0)
    for _ in range(max(3, args.warmup)):
        cached_step()
    barrier()
    with ClockSampler(uuid) as cclk:
        host_ahead(torch, Kc)
        with cclk.region() as reg:
            for k in range(Kc):
                flush.fill_(k & 0xFF)
                c_start[k].record()
                if k == 0:
                    reg.watch_start(c_start[0])
                cached_step()
                c_end[k].record()
            reg.watch_end(c_end[-1])
            barrier()
    cached_clocks = cclk.summary()
    cached_steps = [a.elapsed_time(b) for a, b in zip(c_start, c_end)]
    cached_ms = max_over_ranks(sum(cached_steps), world, device)
    cached_median = statistics.median(cached_steps)
    st, where = lib.lm_get_error()
    if st != 0:
        raise RuntimeError(f"device error {st} at wait {where:#x}")

    # ---- end to end through the public API with host buffers: every step
    # uploads its inputs from pinned host memory and downloads its results.
    # Three streams (copy-in, compute, copy-out) and two device buffer sets
    # let step k's compute overlap step k+1's upload and step k-1's download.
    Ke = min(K, 100)  # long enough that the pipeline's fill and drain are a small share
    in_names, out_names = ("X", "W_up", "W_down", "dY"), ("Y", "dX", "dW_up", "dW_down")
    pinned_in = {k: host[k].pin_memory() for k in in_names}
    pinned_out = [{k: torch.empty(dev[k].shape, dtype=torch.bfloat16).pin_memory()
                   for k in out_names} for _ in range(2)]
    dbuf = [{k: torch.empty_like(dev[k]) for k in in_names + out_names} for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pinned_in.values())
    d2h = sum(v.numel() * v.element_size() for v in pinned_out[0].values())
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    s_comp = torch.cuda.current_stream(device)
    ev = lambda: torch.cuda.Event()
    in_ready, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    e_s = torch.cuda.Event(enable_timing=True)
    e_e = torch.cuda.Event(enable_timing=True)
    barrier()
    e_s.record(s_comp)
    s_in.wait_event(e_s)
    s_out.wait_event(e_s)
    for k in range(Ke):
        b = k % 2
        bufs = dbuf[b]
        if k >= 2:
            s_in.wait_event(comp_done[b])        # step k-2 no longer reads these inputs
        with torch.cuda.stream(s_in):
            for n in in_names:
                bufs[n].copy_(pinned_in[n], non_blocking=True)
            in_ready[b].record(s_in)
        s_comp.wait_event(in_ready[b])
        if k >= 2:
            s_comp.wait_event(out_done[b])       # step k-2's results are downloaded
        mlp.forward(bufs["X"], bufs["W_up"], bufs["W_down"], Y=bufs["Y"], stream=s_comp)
        mlp.backward(bufs["dY"], dX=bufs["dX"], dW_up=bufs["dW_up"], dW_down=bufs["dW_down"],
                     stream=s_comp)
        comp_done[b].record(s_comp)
        s_out.wait_event(comp_done[b])
        with torch.cuda.stream(s_out):
            for n in out_names:
                pinned_out[b][n].copy_(bufs[n], non_blocking=True)
            out_done[b].record(s_out)
    s_comp.wait_event(out_done[(Ke - 1) % 2])
    if Ke >= 2:
        s_comp.wait_event(out_done[(Ke - 2) % 2])
    e_e.record(s_comp)
    barrier()
    e2e_ms = max_over_ranks(e_s.elapsed_time(e_e), world, device)
    # the last step's results really arrived: spot-check against the device copy
    last = (Ke - 1) % 2
    assert torch.equal(pinned_out[last]["dX"][:4].float(), dbuf[last]["dX"][:4].cpu().float())

    peaks = read_peaks()
    value = job_tflops(world, K, STEP_FLOPS, total_ms)
    # the tensor pipe's dense FP8 peak at the SM clock sampled during the timed
    # region: SMs x 16384 FLOP per clock
    clock_peak = (world * props.multi_processor_count * 16384 * clocks["sm_mhz"] * 1e6 / 1e12
                  if clocks.get("sm_mhz") else None)
    e2e_value = job_tflops(world, Ke, STEP_FLOPS, e2e_ms)
    # The timed region is well under a second, so the kernel is compared with
    # the burst GEMM peak; the sustained (seconds-long, power-capped) one is
    # reported beside it.
    fp8_peak = peaks["bf16"] * NOMINAL_FP8_OVER_BF16
    fp8_peak_sus = peaks["bf16_sus"] * NOMINAL_FP8_OVER_BF16
    achieved = GEMM_FLOPS / (gemm_avg_ms * 1e-3) / 1e12
    traffic = None
    gemm_src = os.path.join(ROOT, "fp8_gemms_b200", "csrc", "lm_gemm.cu")
    if GEMM_TRAFFIC["source_sha256"] and GEMM_TRAFFIC["source_sha256"] == src_sha(gemm_src):
        traffic = GEMM_TRAFFIC["bytes_per_launch"]
    cb = cast_bytes()
    cast_gbs = sum(cb) / (sum(cast_ms) * 1e-3) / 1e9
    mhz = clocks.get("sm_mhz")
    configs = run_configs(args, device, world, flush, host, dev, mlp, peaks, rank)
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "pct_of_dense_fp8_peak": round(100.0 * value / (world * DENSE_FP8_PEAK_TFLOPS), 2),
        "pct_of_clock_scaled_peak": round(100.0 * value / clock_peak, 2) if clock_peak else None,
        "pct_of_pages_implied_peak": round(100.0 * value / (world * PAGES_FP8_PEAK_TFLOPS), 2),
        "n_gpus": world,
        "steps": K,
        "warmup": max(3, args.warmup),
        "ms_per_step": round(total_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8",
        "data": "synthetic (seeded N(0,1) X, N(0,0.02) weights, N(0,1e-3) dY)",
        "config": {"workload": WORKLOAD, "M": M_TOK, "d": D_MODEL, "f": D_FF,
                   "gemms_per_step": 6, "flops_per_step": STEP_FLOPS,
                   "l2": "flushed before every timed step (256 MiB write)",
                   "parallelism": f"{world} independent replica(s), no collective"},
        "roofline": {"bound": "tensor", "kernel": "gemm_fp8_pair_kernel (tcgen05, CTA pairs)",
                     "achieved": round(achieved, 2), "peak": round(fp8_peak, 1),
                     "unit": "TFLOP/s", "frac": round(achieved / fp8_peak, 4),
                     "peak_source": f"{peaks['src']} bf16 burst {peaks['bf16']} x nominal "
                                    f"fp8/bf16 ratio {NOMINAL_FP8_OVER_BF16} (timed region "
                                    f"under a second)",
                     "peak_sustained": round(fp8_peak_sus, 1),
                     "frac_of_sustained": round(achieved / fp8_peak_sus, 4),
                     "flops_per_launch": GEMM_FLOPS, "avg_launch_ms": round(gemm_avg_ms, 4),
                     "avg_launch_kcycles": round(gemm_avg_ms * mhz, 1) if mhz else None,
                     "traffic": traffic},
        "cast_kernels": {"achieved_gbs": round(cast_gbs, 1), "peak_gbs": peaks["hbm"],
                         "frac": round(cast_gbs / peaks["hbm"], 4),
                         "frac_of_8tbs": round(cast_gbs / 8000.0, 4),
                         "algorithmic_bytes_per_step": sum(cb),
                         "ms_per_step": round(sum(cast_ms), 4)},
        "gemm_ms_per_step": round(sum(gemm_ms), 4),
        "launch_sequence": kinds,
        "per_launch_ms": [round(a, 4) for a in avg],
        "per_gemm_kcycles": [round(a * mhz, 1) for a in gemm_ms] if mhz else None,
        "lead_in_ms_per_step": round(statistics.mean(lead_ms), 4),
        "host_issue_ms_per_step": round(1e3 * t_issue / K, 4),
        "step_ms_spread": {"min": round(min(step_ms), 4),
                           "median": round(statistics.median(step_ms), 4),
                           "max": round(max(step_ms), 4),
                           "first": round(step_ms[0], 4), "last": round(step_ms[-1], 4)},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "steps": Ke,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms / Ke, 4),
                "how": "pinned host inputs uploaded and results (Y, dX, dW_up, dW_down) "
                       "downloaded every step; copy-in / compute / copy-out streams overlap "
                       "across steps (double-buffered device copies)"},
        "weight_casts_cached": {
            "value": round(job_tflops(world, Kc, STEP_FLOPS, cached_ms), 2), "unit": "TFLOP/s",
            "steps": Kc, "ms_per_step": round(cached_ms / Kc, 4),
            "step_ms_median": round(cached_median, 4),
            "sm_mhz": cached_clocks.get("sm_mhz"), "reasons": cached_clocks.get("reasons"),
            "how": "forward reuses the W_up/W_down codes and scales, as after the first "
                   "micro-batch of an optimizer step"},
        "gpu_launches": K * LAUNCHES_PER_STEP,
        "clocks": clocks,
        "configs": configs,
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(host, args.cpu_sample_tokens)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# ------------------------------------------------- the other GEMM sets
def time_steps(step, K, W, flush, cap):
    """W warm-up steps, then K steps each preceded by an L2 flush and timed
    with CUDA events.  One more step runs with the library's launch events,
    for the split between GEMM launches and the rest; a host-side gap before
    a launch counts towards that launch, so where the host issues launches
    more slowly than the GPU runs them the split is of the instrumented
    eager step, not of device time alone.  Returns (ms per step, GEMM ms,
    other ms) of that step."""
    import torch
    from fp8_gemms_b200 import _lib as lib
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    host_ahead(torch, K)
    for k in range(K):
        flush.fill_(k & 0xFF)
        ev[k][0].record()
        step()
        ev[k][1].record()
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / K
    flush.fill_(0)
    t = lib.KernelTimer(cap)
    end = torch.cuda.Event(enable_timing=True)
    with t:
        step()
    end.record()
    torch.cuda.synchronize()
    d = t.durations_ms(end)
    assert len(t.kinds) == len(d) == t.n and t.n < cap, (len(t.kinds), len(d), t.n, cap)
    g = sum(x for x, kd in zip(d, t.kinds) if kd == "g")
    return ms, g, sum(d) - g


def time_graph(step, K, flush):
    """The same step captured once into a CUDA graph and replayed K times (L2
    flushed before each replay): device time without host launch gaps."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    host_ahead(torch, K)
    for k in range(K):
        flush.fill_(k & 0xFF)
        ev[k][0].record()
        g.replay()
        ev[k][1].record()
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / K
    del g
    return ms


def config_entry(name, flops, cast_bytes_total, ms, gemm_ms, other_ms, peaks, world):
    """Throughput and roofline of one GEMM set: the roofline time is the
    GEMMs' FLOPs at the dense FP8 peak plus the casts' algorithmic bytes at
    HBM bandwidth (each kernel bound by the slower of the two, which is FLOPs
    for every GEMM and bytes for every cast here)."""
    t_nom = flops / 4.5e15 + cast_bytes_total / 8e12
    t_meas = (flops / (peaks["bf16"] * NOMINAL_FP8_OVER_BF16 * 1e12) +
              cast_bytes_total / (peaks["hbm"] * 1e9))
    tflops = world * flops / (ms * 1e-3) / 1e12
    return {"workload": name, "ms_per_step": round(ms, 4), "tflops": round(tflops, 2),
            "flops_per_step": flops, "pct_of_dense_fp8_peak":
            round(100.0 * tflops / (world * DENSE_FP8_PEAK_TFLOPS), 2),
            "instrumented_step": {"gemm_ms": round(gemm_ms, 4), "other_ms": round(other_ms, 4)},
            "cast_bytes_per_step": cast_bytes_total,
            "roofline": {"ms_nominal": round(t_nom * 1e3, 4), "frac_nominal":
                         round(t_nom * 1e3 / ms, 4), "ms_measured_peaks":
                         round(t_meas * 1e3, 4), "frac_measured_peaks":
                         round(t_meas * 1e3 / ms, 4),
                         "how": "GEMM FLOPs at 4.5 PFLOP/s (nominal) or 2 x the measured "
                                "bf16 burst (measured) + cast bytes at 8 TB/s or the "
                                "measured copy bandwidth"}}


def add_graph(entry, flops, graph_ms, world):
    tf = world * flops / (graph_ms * 1e-3) / 1e12
    entry["graph_replay"] = {"ms_per_step": round(graph_ms, 4), "tflops": round(tf, 2),
                             "pct_of_dense_fp8_peak":
                             round(100.0 * tf / (world * DENSE_FP8_PEAK_TFLOPS), 2)}


def linear_cast_bytes(M, N, K):
    return 5 * (M * K + N * K + M * N)   # full casts of X, W and dY


def mlp_cast_bytes(M, d, f, backward=True):
    b = 5 * M * d + 10 * f * d + 3 * M * f           # X, W_up, W_down, h
    return b + (5 * M * d + 3 * M * f if backward else 0)   # dY, dH


def run_configs(args, device, world, flush, host, dev, mlp, peaks, rank):
    """Configs 2, 4 and 5 of the little-lm GEMM sets, each timed like the
    headline, with the oracle's sample time on rank 0."""
    import torch
    from fp8_gemms_b200 import api, synthetic
    if args.no_configs:
        return None
    out = {}
    K = args.config_steps
    # -- the MLP forward alone at M = 16384 (16 x 1024 tokens)
    fl = 2 * GEMM_FLOPS
    ms, g, o = time_steps(lambda: mlp.forward(dev["X"], dev["W_up"], dev["W_down"], Y=dev["Y"]),
                          K, 3, flush, 16)
    ms = max_over_ranks(ms, world, device)
    out["mlp_fwd_M16384"] = config_entry(synthetic.MLP_FWD.name, fl,
                                         mlp_cast_bytes(M_TOK, D_MODEL, D_FF, False), ms, g, o,
                                         peaks, world)
    # -- attention projections + LM head at M = 8192
    w = synthetic.ATTN_HEAD
    items = []
    for i, (name, n, k) in enumerate(w.linears):
        t = w.tensors(i, device=device)
        lin = api.Linear(w.M, k, n, device=device)
        bufs = (torch.empty(w.M, n, dtype=torch.bfloat16, device=device),
                torch.empty(w.M, k, dtype=torch.bfloat16, device=device),
                torch.empty(n, k, dtype=torch.bfloat16, device=device))
        items.append((lin, t, bufs))

    def step4():
        for lin, t, (Y, dX, dW) in items:
            lin.forward(t["X"], t["W"], Y=Y)
            lin.backward(t["dY"], dX=dX, dW=dW)

    ms, g, o = time_steps(step4, K, 3, flush, 64)
    ms = max_over_ranks(ms, world, device)
    cb = sum(linear_cast_bytes(w.M, n, k) for _, n, k in w.linears)
    out["attn_lmhead_M8192"] = config_entry(w.name, w.flops, cb, ms, g, o, peaks, world)
    add_graph(out["attn_lmhead_M8192"], w.flops,
              max_over_ranks(time_graph(step4, K, flush), world, device), world)
    del items
    torch.cuda.empty_cache()
    # -- the 28-layer stack: per layer Q, K, V, O and the relu^2 MLP, each layer
    # with its own seeded weights and t3 activations (drawn on the device)
    layers = []
    for layer in range(synthetic.N_LAYERS):
        lw, mw = synthetic.stack_layer(layer)
        layers.append(([lw.tensors(i, device=device) for i in range(len(lw.linears))],
                       mw.tensors(device=device)))
    lins = {(n, k): api.Linear(M_TOK, k, n, device=device) for _, n, k in synthetic.ATTN_LINEARS}
    lbuf = {(n, k): (torch.empty(M_TOK, n, dtype=torch.bfloat16, device=device),
                     torch.empty(M_TOK, k, dtype=torch.bfloat16, device=device),
                     torch.empty(n, k, dtype=torch.bfloat16, device=device))
            for _, n, k in synthetic.ATTN_LINEARS}
    shapes = [(n, k) for _, n, k in synthetic.ATTN_LINEARS]

    def step5():
        for lts, mt in layers:
            for (n, k), t in zip(shapes, lts):
                Y, dX, dW = lbuf[(n, k)]
                lins[(n, k)].forward(t["X"], t["W"], Y=Y)
                lins[(n, k)].backward(t["dY"], dX=dX, dW=dW)
            mlp.forward(mt["X"], mt["W_up"], mt["W_down"], Y=dev["Y"])
            mlp.backward(mt["dY"], dX=dev["dX"], dW_up=dev["dW_up"], dW_down=dev["dW_down"])

    K5 = max(1, min(K, args.stack_steps))
    ms, g, o = time_steps(step5, K5, 1, flush, 1400)
    ms = max_over_ranks(ms, world, device)
    per_layer_flops = (sum(6 * M_TOK * n * k for n, k in shapes) + 12 * M_TOK * D_MODEL * D_FF)
    cb = synthetic.N_LAYERS * (sum(linear_cast_bytes(M_TOK, n, k) for n, k in shapes) +
                               mlp_cast_bytes(M_TOK, D_MODEL, D_FF))
    out["stack28_M16384_t3"] = config_entry(
        "28-layer stack: Q, K, V, O + relu2 MLP per layer, fwd+dgrad+wgrad, M=16384, t3 "
        "activations", synthetic.N_LAYERS * per_layer_flops, cb, ms, g, o, peaks, world)
    out["stack28_M16384_t3"]["inputs"] = ("drawn on the device with the synthetic recipe "
                                          "(per-layer seeds, CUDA generators)")
    add_graph(out["stack28_M16384_t3"], synthetic.N_LAYERS * per_layer_flops,
              max_over_ranks(time_graph(step5, K5, flush), world, device), world)
    del layers, lins, lbuf
    torch.cuda.empty_cache()
    for v in out.values():
        v["steps"] = K if v is not out["stack28_M16384_t3"] else K5
    if rank == 0 and not args.no_cpu_baseline:
        for key, o in oracle_config_samples(host).items():
            out[key]["oracle"] = o
    return out


# --------------------------------------------------------------- oracle
def oracle_sample(host, tokens):
    """The oracle's relu^2 MLP fwd + bwd on the first `tokens` rows of the
    workload (full weights).  Returns (seconds, flops, threads)."""
    import oracle
    from fp8_gemms_b200 import synthetic
    b = {k: synthetic.bits_u16(v[:tokens] if k in ("X", "dY") else v) for k, v in host.items()}
    t0 = time.perf_counter()
    fwd = oracle.mlp_fwd(b["X"], b["W_up"], b["W_down"])
    oracle.mlp_bwd(b["dY"], fwd)
    dt = time.perf_counter() - t0
    return dt, 6 * 2 * tokens * D_MODEL * D_FF, oracle.num_threads()


def cpu_baseline(host, tokens):
    dt, flops, threads = oracle_sample(host, tokens)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": f"oracle relu2 MLP fwd+bwd on {tokens} of {M_TOK} tokens, full "
                      f"d={D_MODEL} f={D_FF} weights (casts of the full weights included); "
                      f"{dt:.1f} s"}


def oracle_config_samples(host):
    """The oracle, as it stands, on bounded samples of configs 2, 4 and 5 (host
    cores; a baseline, not a target).  Each sample keeps the full weights and
    takes the first T tokens of the activations; config 5 times one layer of
    the stack and multiplies by 28 (labelled extrapolated)."""
    import oracle
    from fp8_gemms_b200 import synthetic
    b = synthetic.bits_u16
    threads = oracle.num_threads()
    res = {}
    T = 128
    t0 = time.perf_counter()
    oracle.mlp_fwd(b(host["X"][:T]), b(host["W_up"]), b(host["W_down"]))
    dt = time.perf_counter() - t0
    res["mlp_fwd_M16384"] = {"tflops": round(4 * T * D_MODEL * D_FF / dt / 1e12, 6),
                             "seconds": round(dt, 3), "cores": threads, "kind": "oracle",
                             "sample": f"relu2 MLP forward on {T} of {M_TOK} tokens, full "
                                       "weights (their casts included)"}
    T = 64
    w = synthetic.ATTN_HEAD
    dt, fl = 0.0, 0
    for i, (name, n, k) in enumerate(w.linears):
        seed, base = w.seed, 4 * i
        X = synthetic.normal_bf16((T, k), 1.0, seed, base)
        W = synthetic.normal_bf16((n, k), 0.02, seed, base + 1)
        dY = synthetic.normal_bf16((T, n), 1e-3, seed, base + 2)
        t0 = time.perf_counter()
        oracle.linear_fwd_bwd(b(X), b(W), b(dY))
        dt += time.perf_counter() - t0
        fl += 6 * T * n * k
    res["attn_lmhead_M8192"] = {"tflops": round(fl / dt / 1e12, 6), "seconds": round(dt, 3),
                                "cores": threads, "kind": "oracle",
                                "sample": f"Q, K, V, O and LM head fwd+dgrad+wgrad on {T} of "
                                          f"{w.M} tokens, full weights"}
    T = 32
    lw, mw = synthetic.stack_layer(0)
    dt, fl = 0.0, 0
    for i, (name, n, k) in enumerate(lw.linears):
        X = synthetic.student_t3_bf16((T, k), lw.seed, 4 * i)
        W = synthetic.normal_bf16((n, k), 0.02, lw.seed, 4 * i + 1)
        dY = synthetic.normal_bf16((T, n), 1e-3, lw.seed, 4 * i + 2)
        t0 = time.perf_counter()
        oracle.linear_fwd_bwd(b(X), b(W), b(dY))
        dt += time.perf_counter() - t0
        fl += 6 * T * n * k
    X = synthetic.student_t3_bf16((T, D_MODEL), mw.seed, 0)
    Wu = synthetic.normal_bf16((D_FF, D_MODEL), 0.02, mw.seed, 1)
    Wd = synthetic.normal_bf16((D_MODEL, D_FF), 0.02, mw.seed, 2)
    dY = synthetic.normal_bf16((T, D_MODEL), 1e-3, mw.seed, 3)
    t0 = time.perf_counter()
    oracle.mlp_bwd(b(dY), oracle.mlp_fwd(b(X), b(Wu), b(Wd)))
    dt += time.perf_counter() - t0
    fl += 12 * T * D_MODEL * D_FF
    n = synthetic.N_LAYERS
    res["stack28_M16384_t3"] = {"tflops": round(fl / dt / 1e12, 6),
                                "seconds": round(dt * n, 3), "cores": threads,
                                "kind": "oracle", "extrapolated": True,
                                "sample": f"layer 0 (Q, K, V, O, relu2 MLP fwd+bwd) on {T} "
                                          f"of {M_TOK} tokens, full weights; seconds = that "
                                          f"layer's time x {n}"}
    return res


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from fp8_gemms_b200 import synthetic
    tokens = 16
    host = synthetic.MLP_FWD_BWD.tensors()
    for _ in range(max(0, args.warmup)):
        oracle_sample(host, tokens)
    secs, flops_total, threads = 0.0, 0, 1
    steps = max(1, args.steps)
    for _ in range(steps):
        dt, flops, threads = oracle_sample(host, tokens)
        secs += dt
        flops_total += flops
    value = flops_total / secs / 1e12
    sample = (f"oracle relu2 MLP fwd+bwd on {tokens} of {M_TOK} tokens per step, full "
              f"d={D_MODEL} f={D_FF} weights")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M_TOK, "d": D_MODEL, "f": D_FF},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
