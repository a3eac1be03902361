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
ranks.  SM clocks are sampled with nvidia-smi during the timed region.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
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
LAUNCHES_PER_STEP = 12                         # kernels of ours per fwd+bwd: "acgcgacggcgg"

# DRAM traffic of one GEMM launch from an ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum), valid only for the kernel source it was taken on;
# the summary and the command are in profiles/.
GEMM_TRAFFIC = {
    "source_sha256": "f46bdffe58b66ae3d9362e9e36f018cb84c2a6f5abe5393d9dd9a21f17fa71ae",
    "bytes_per_launch": 527555029,  # mean of the step's six GEMMs, profiles/gemm_fp8_pair_relu2_mlp_shapes.md
}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-sample-tokens", type=int, default=256)
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
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu = gpu_id  # nvidia-smi -i accepts an index or a GPU UUID
        self.proc = None
        self.out = None

    def __enter__(self):
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "50"], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.out.name) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) == 9:
                        rows.append(parts)
        finally:
            os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(pw) if pw else None}


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


def job_tflops(world, steps, flops_per_step, total_ms):
    """Whole-job throughput: the units all ranks processed over the job's time."""
    return world * steps * flops_per_step / (total_ms * 1e-3) / 1e12


# algorithmic bytes of the casts of one step (X, W_up, W_down, h, dY, dH):
# full cast (amax pass + cast pass) = 2 B amax read + 2 B read + 1 B codes per
# element; a cast whose amax came from a GEMM epilogue = 2 B read + 1 B codes.
# Only row-major codes are written: the backward's GEMMs read them MN-major.
def cast_bytes():
    Md, fd, Mf = M_TOK * D_MODEL, D_FF * D_MODEL, M_TOK * D_FF
    return [5 * Md, 5 * fd, 5 * fd, 3 * Mf, 5 * Md, 3 * Mf]


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
    # records an event before each of its kernel launches (lm_timing_attach)
    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    timers = [lib.KernelTimer(2 * LAUNCHES_PER_STEP) for _ in range(K)]
    barrier()
    props = torch.cuda.get_device_properties(device)
    smi_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    with ClockSampler(smi_id) as clk:
        for k in range(K):
            flush.fill_(k & 0xFF)
            starts[k].record()
            with timers[k]:
                step()
            ends[k].record()
        barrier()
    clocks = clk.summary()
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

    # ---- the same step with the weight casts cached: the forward reuses the
    # codes and scales of W_up and W_down (LM_MLP_REUSE_WEIGHT_CASTS), as every
    # micro-batch after the first of an optimizer step does
    Kc = min(K, 50)
    c_start = [torch.cuda.Event(enable_timing=True) for _ in range(Kc)]
    c_end = [torch.cuda.Event(enable_timing=True) for _ in range(Kc)]
    mlp.forward(dev["X"], dev["W_up"], dev["W_down"], Y=dev["Y"])  # casts of these weights
    barrier()
    for k in range(Kc):
        flush.fill_(k & 0xFF)
        c_start[k].record()
        mlp.forward(dev["X"], None, None, Y=dev["Y"], reuse_weight_casts=True)
        mlp.backward(dev["dY"], dX=dev["dX"], dW_up=dev["dW_up"], dW_down=dev["dW_down"])
        c_end[k].record()
    barrier()
    cached_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(c_start, c_end)), world,
                               device)
    st, where = lib.lm_get_error()
    if st != 0:
        raise RuntimeError(f"device error {st} at wait {where:#x}")

    peaks = read_peaks()
    value = job_tflops(world, K, STEP_FLOPS, total_ms)
    # the tensor pipe's dense FP8 peak at the SM clock sampled during the timed
    # region: SMs x 16384 FLOP per clock
    clock_peak = (world * props.multi_processor_count * 16384 * clocks["sm_mhz"] * 1e6 / 1e12
                  if clocks.get("sm_mhz") else None)
    e2e_value = job_tflops(world, Ke, STEP_FLOPS, e2e_ms)
    fp8_peak = peaks["bf16_sus"] * NOMINAL_FP8_OVER_BF16
    achieved = GEMM_FLOPS / (gemm_avg_ms * 1e-3) / 1e12
    traffic = None
    gemm_src = os.path.join(ROOT, "fp8_gemms_b200", "csrc", "lm_gemm.cu")
    if GEMM_TRAFFIC["source_sha256"] and GEMM_TRAFFIC["source_sha256"] == src_sha(gemm_src):
        traffic = GEMM_TRAFFIC["bytes_per_launch"]
    cb = cast_bytes()
    cast_gbs = sum(cb) / (sum(cast_ms) * 1e-3) / 1e9
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
                     "peak_source": f"{peaks['src']} bf16 sustained {peaks['bf16_sus']} x "
                                    f"nominal fp8/bf16 ratio {NOMINAL_FP8_OVER_BF16}",
                     "flops_per_launch": GEMM_FLOPS, "avg_launch_ms": round(gemm_avg_ms, 4),
                     "traffic": traffic},
        "cast_kernels": {"achieved_gbs": round(cast_gbs, 1), "peak_gbs": peaks["hbm"],
                         "frac": round(cast_gbs / peaks["hbm"], 4),
                         "algorithmic_bytes_per_step": sum(cb),
                         "ms_per_step": round(sum(cast_ms), 4)},
        "gemm_ms_per_step": round(sum(gemm_ms), 4),
        "launch_sequence": kinds,
        "per_launch_ms": [round(a, 4) for a in avg],
        "lead_in_ms_per_step": round(statistics.mean(lead_ms), 4),
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "steps": Ke,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms / Ke, 4),
                "how": "pinned host inputs uploaded and results (Y, dX, dW_up, dW_down) "
                       "downloaded every step; copy-in / compute / copy-out streams overlap "
                       "across steps (double-buffered device copies)"},
        "weight_casts_cached": {
            "value": round(job_tflops(world, Kc, STEP_FLOPS, cached_ms), 2), "unit": "TFLOP/s",
            "steps": Kc, "ms_per_step": round(cached_ms / Kc, 4),
            "how": "forward reuses the W_up/W_down codes and scales, as after the first "
                   "micro-batch of an optimizer step"},
        "gpu_launches": K * LAUNCHES_PER_STEP,
        "clocks": clocks,
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(host, args.cpu_sample_tokens)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


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
