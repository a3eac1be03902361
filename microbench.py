"""Time one C-ABI call on synthetic data (CUDA events, L2 flushed between
iterations).  Also the small, self-contained command to run under ncu.

    python microbench.py gemm --M 16384 --N 12288 --K 3072 --epi relu2_fwd
    python microbench.py cast --rows 16384 --cols 3072 --fmt e4m3
    python microbench.py cast --rows 16384 --cols 12288 --relu2 --amax-in
    python microbench.py mlp-compare --M 16384
        (the non-gated relu^2 block, f = 4d, against the gated SwiGLU block,
        f = 2.75d, both fwd + bwd in FP8: ms per step and tokens per second)
    python microbench.py scaled-mm
        (library calibration: torch._scaled_mm, i.e. cuBLASLt FP8, against this
        library's GEMM on the six GEMM shapes of the relu^2 MLP step, M = 16384)
    python microbench.py torch-composition --M 16384
        (the same relu^2 MLP step composed the way the pages' training code
        composes it -- per-tensor amax and cast in PyTorch, transposed copies,
        one torch._scaled_mm (cuBLASLt) per GEMM, unfused relu^2 / relu^2' --
        against this library's two calls, on the same GPU and inputs)
    python microbench.py linears --workload attn-head
        (the attention projections Q, K, V, O and the LM head at M = 8192, each
        fwd + dgrad + wgrad through lm_fp8_linear_fwd / _bwd: per linear, and
        the whole set eagerly and replayed from a CUDA graph)
    python microbench.py linears --workload stack
        (the per-step linear GEMM set of a 28-layer d = 3072 stack at M = 16384:
        per layer Q, K, V, O and the relu^2 MLP, fwd + dgrad + wgrad, each
        layer with its own weights and t3-distributed activations)
    python microbench.py mlp-fwd --M 16384
        (the relu^2 MLP forward alone: casts, the up GEMM, and the down GEMM
        whose side warps cast h; with --warmup 1 --iters 1 the 4th GEMM launch
        is the second forward's down GEMM, the one to capture under ncu)
    python microbench.py mlp-accum --M 16384 --micro 7
        (one optimizer step of gradient accumulation: the weights are cast by the
        first micro-batch's forward and reused by the others; every backward adds
        its weight gradients into fp32 accumulators)
"""
import argparse
import json
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from fp8_gemms_b200 import _lib  # noqa: E402
from fp8_gemms_b200._lib import E4M3, E5M2, EPI_NONE, EPI_RELU2_BWD, EPI_RELU2_FWD  # noqa: E402

FMT = {"e4m3": E4M3, "e5m2": E5M2}
EPI = {"none": EPI_NONE, "relu2_fwd": EPI_RELU2_FWD, "relu2_bwd": EPI_RELU2_BWD}
TDT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def random_codes(fmt, rows, cols, gen):
    v = torch.randn(rows, cols, device="cuda", generator=gen)
    return v.to(TDT[fmt]).view(torch.uint8)


def time_it(fn, iters, warmup, flush):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ms = []
    for i in range(iters):
        flush.fill_(i & 0xFF)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        e.synchronize()
        ms.append(s.elapsed_time(e))
    return ms


def _draw(shape, dist, gen):
    """Seeded device draw: N(0, sigma) or Student-t with 3 degrees of freedom
    (Z / sqrt(chi2_3 / 3)), rounded to bf16."""
    if dist == "t3":
        z = torch.randn(*shape, device="cuda", generator=gen)
        chi = torch.zeros_like(z)
        for _ in range(3):
            n = torch.randn(*shape, device="cuda", generator=gen)
            chi.addcmul_(n, n)
        return (z / torch.sqrt(chi / 3.0)).to(torch.bfloat16)
    return (torch.randn(*shape, device="cuda", generator=gen) * dist).to(torch.bfloat16)


def linears(a, gen, flush):
    from fp8_gemms_b200 import api, synthetic
    if a.workload == "attn-head":
        M, layers, x_dist = 8192, 1, 1.0
        shapes = synthetic.ATTN_LINEARS + [("lm_head", synthetic.VOCAB_PADDED,
                                            synthetic.D_MODEL)]
        mlp_dims = None
    else:
        M, layers, x_dist = 16384, a.layers, "t3"
        shapes = synthetic.ATTN_LINEARS
        mlp_dims = (synthetic.D_MODEL, synthetic.D_FF)
    lins = {(n, k): api.Linear(M, k, n) for _, n, k in shapes}
    outs = {(n, k): (torch.empty(M, n, dtype=torch.bfloat16, device="cuda"),
                     torch.empty(M, k, dtype=torch.bfloat16, device="cuda"),
                     torch.empty(n, k, dtype=torch.bfloat16, device="cuda"))
            for _, n, k in shapes}
    data = []   # per layer: [(name, n, k, X, W, dY)], and the MLP's tensors
    for _ in range(layers):
        lay = [(name, n, k, _draw((M, k), x_dist, gen), _draw((n, k), 0.02, gen),
                _draw((M, n), 1e-3, gen)) for name, n, k in shapes]
        mt = None
        if mlp_dims:
            d, f = mlp_dims
            mt = (_draw((M, d), x_dist, gen), _draw((f, d), 0.02, gen),
                  _draw((d, f), 0.02, gen), _draw((M, d), 1e-3, gen))
        data.append((lay, mt))
    mlp = api.Relu2Mlp(M, *mlp_dims) if mlp_dims else None
    if mlp:
        d, f = mlp_dims
        mY = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
        mdX = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
        mdWu = torch.empty(f, d, dtype=torch.bfloat16, device="cuda")
        mdWd = torch.empty(d, f, dtype=torch.bfloat16, device="cuda")

    def run_linear(name, n, k, X, W, dY):
        lin, (Y, dX, dW) = lins[(n, k)], outs[(n, k)]
        lin.forward(X, W, Y=Y)
        lin.backward(dY, dX=dX, dW=dW)

    def step():
        for lay, mt in data:
            for item in lay:
                run_linear(*item)
            if mt:
                mlp.forward(mt[0], mt[1], mt[2], Y=mY)
                mlp.backward(mt[3], dX=mdX, dW_up=mdWu, dW_down=mdWd)

    flops_lin = {name: 6 * M * n * k for name, n, k in shapes}
    flops = layers * (sum(flops_lin.values()) +
                      (12 * M * mlp_dims[0] * mlp_dims[1] if mlp_dims else 0))
    res = dict(op="linears", workload=a.workload, M=M, layers=layers,
               tflop_per_step=round(flops / 1e12, 4))
    per = []
    for item in data[0][0]:
        ms = time_it(lambda: run_linear(*item), a.iters, a.warmup, flush)
        t = sum(ms) / len(ms)
        per.append(dict(linear=item[0], N=item[1], K=item[2], ms=round(t, 4),
                        tflops=round(flops_lin[item[0]] / t / 1e9, 1)))
    res["per_linear_layer0"] = per
    iters = max(2, a.iters // (4 if layers > 1 else 1))
    ms = time_it(step, iters, a.warmup, flush)
    t = sum(ms) / len(ms)
    res.update(eager_ms=round(t, 4), eager_tflops=round(flops / t / 1e9, 1))
    if layers == 1:
        # replayed from a CUDA graph: no host launch overhead between the kernels
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                step()
        torch.cuda.current_stream().wait_stream(s)
        ms = time_it(g.replay, a.iters, a.warmup, flush)
        t = sum(ms) / len(ms)
        res.update(graph_ms=round(t, 4), graph_tflops=round(flops / t / 1e9, 1))
        del g
    res["pct_of_4500_tflops"] = round(100 * flops / (min(
        res.get("graph_ms", 1e30), res["eager_ms"]) * 1e9) / 4500.0, 1)
    return res


def main():
    p = argparse.ArgumentParser()
    p.add_argument("op", choices=["gemm", "cast", "mlp-accum", "mlp-fwd", "rmsnorm-cast",
                                  "mlp-compare", "lmhead-ce", "scaled-mm", "torch-composition",
                                  "linears"])
    p.add_argument("--workload", default="attn-head", choices=["attn-head", "stack"])
    p.add_argument("--layers", type=int, default=28)
    p.add_argument("--V", type=int, default=50304)
    p.add_argument("--chunk", type=int, default=4096)
    p.add_argument("--micro", type=int, default=7)
    p.add_argument("--d", type=int, default=3072)
    p.add_argument("--f", type=int, default=12288)
    p.add_argument("--M", type=int, default=16384)
    p.add_argument("--N", type=int, default=12288)
    p.add_argument("--K", type=int, default=3072)
    p.add_argument("--fa", default="e4m3")
    p.add_argument("--fb", default="e4m3")
    p.add_argument("--epi", default="none", choices=list(EPI))
    p.add_argument("--flags", type=int, default=0,
                   help="operand storage: 1 = A MN-major, 2 = B MN-major, 3 = both")
    p.add_argument("--no-ws", action="store_true",
                   help="gemm: no workspace, so no split-K tail")
    p.add_argument("--rows", type=int, default=16384)
    p.add_argument("--cols", type=int, default=3072)
    p.add_argument("--fmt", default="e4m3")
    p.add_argument("--relu2", action="store_true")
    p.add_argument("--amax-in", action="store_true")
    p.add_argument("--no-qT", action="store_true", help="cast: row-major codes only")
    p.add_argument("--iters", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    a = p.parse_args()
    gen = torch.Generator(device="cuda").manual_seed(0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    if a.op == "mlp-accum":
        pass
    elif a.op == "mlp-fwd":
        from fp8_gemms_b200 import api
        M, d, f = a.M, a.d, a.f
        mlp = api.Relu2Mlp(M, d, f)
        X = torch.randn(M, d, device="cuda", generator=gen).to(torch.bfloat16)
        Wu = (torch.randn(f, d, device="cuda", generator=gen) * 0.02).to(torch.bfloat16)
        Wd = (torch.randn(d, f, device="cuda", generator=gen) * 0.02).to(torch.bfloat16)
        Y = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
        ms = time_it(lambda: mlp.forward(X, Wu, Wd, Y=Y), a.iters, a.warmup, flush)
        avg = sum(ms) / len(ms)
        out = dict(op="mlp-fwd", M=M, d=d, f=f, avg_ms=round(avg, 4),
                   tflops=round(2 * 2 * M * d * f / avg / 1e9, 1))
    elif a.op == "linears":
        out = linears(a, gen, flush)
    elif a.op == "scaled-mm":
        # (name, M, N, K, A format, B format, operand storage in the step)
        shapes = [("up", 16384, 12288, 3072, E4M3, E4M3, 0),
                  ("down", 16384, 3072, 12288, E4M3, E4M3, 0),
                  ("dgrad-down", 16384, 12288, 3072, E5M2, E4M3, 2),
                  ("wgrad-down", 3072, 12288, 16384, E5M2, E4M3, 3),
                  ("dgrad-up", 16384, 3072, 12288, E5M2, E4M3, 2),
                  ("wgrad-up", 12288, 3072, 16384, E5M2, E4M3, 3)]
        ws = torch.empty(_lib.lm_fp8_gemm_workspace_size(), dtype=torch.uint8, device="cuda")
        one = torch.ones((), device="cuda")
        res = []
        for name, M, N, K, fa, fb, flags in shapes:
            A = random_codes(fa, M, K, gen)          # [M x K]
            B = random_codes(fb, N, K, gen)          # [N x K]
            At = A.t().contiguous() if flags & 1 else A
            Bt = B.t().contiguous() if flags & 2 else B
            ia = torch.full((1,), 1e-2, device="cuda")
            D = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            ours = lambda: _lib.lm_fp8_gemm_ex(At, fa, Bt, fb, ia, ia, D, flags=flags,
                                               workspace=ws)
            Af, Bf = A.view(TDT[fa]), B.view(TDT[fb])
            lib_mm = lambda: torch._scaled_mm(Af, Bf.t(), scale_a=one, scale_b=one,
                                              out_dtype=torch.bfloat16)
            t_ours = sum(time_it(ours, a.iters, a.warmup, flush)) / a.iters
            t_lib = sum(time_it(lib_mm, a.iters, a.warmup, flush)) / a.iters
            fl = 2 * M * N * K
            res.append(dict(gemm=name, M=M, N=N, K=K, ours_ms=round(t_ours, 4),
                            scaled_mm_ms=round(t_lib, 4),
                            ours_tflops=round(fl / t_ours / 1e9, 1),
                            scaled_mm_tflops=round(fl / t_lib / 1e9, 1)))
        tot_o = sum(r["ours_ms"] for r in res)
        tot_l = sum(r["scaled_mm_ms"] for r in res)
        out = dict(op="scaled-mm", gemms=res, ours_total_ms=round(tot_o, 4),
                   scaled_mm_total_ms=round(tot_l, 4),
                   ours_over_scaled_mm_speed=round(tot_l / tot_o, 4))
    elif a.op == "torch-composition":
        from fp8_gemms_b200 import api
        M, d, f = a.M, a.d, a.f
        bf = torch.bfloat16
        X = torch.randn(M, d, device="cuda", generator=gen).to(bf)
        Wu = (torch.randn(f, d, device="cuda", generator=gen) * 0.02).to(bf)
        Wd = (torch.randn(d, f, device="cuda", generator=gen) * 0.02).to(bf)
        dY = (torch.randn(M, d, device="cuda", generator=gen) * 1e-3).to(bf)
        fmax = {torch.float8_e4m3fn: 448.0, torch.float8_e5m2: 57344.0}

        def tcast(x, dt):
            # amax -> scale -> saturating RNE cast, and the inverse scale
            amax = x.abs().amax().float().clamp_min(1e-12)
            sc = fmax[dt] / amax
            q = (x.float() * sc).clamp(-fmax[dt], fmax[dt]).to(dt)
            return q, (1.0 / sc).reshape(())

        def mm(aq, ia, bq_nk, ib):
            # D [M x N] = A [M x K] B[N x K]^T; cuBLASLt wants B column-major
            return torch._scaled_mm(aq, bq_nk.t(), scale_a=ia, scale_b=ib, out_dtype=bf)

        e4, e5 = torch.float8_e4m3fn, torch.float8_e5m2

        def torch_step():
            Xq, iX = tcast(X, e4)
            Wuq, iWu = tcast(Wu, e4)
            Wdq, iWd = tcast(Wd, e4)
            H = mm(Xq, iX, Wuq, iWu)
            h = torch.relu(H).square()
            hq, ih = tcast(h, e4)
            Yt = mm(hq, ih, Wdq, iWd)                                # Y
            dYq, idY = tcast(dY, e5)
            g = mm(dYq, idY, Wdq.t().contiguous(), iWd)              # dY W_down
            dH = g * (2 * torch.relu(H))
            dHq, idH = tcast(dH, e5)
            dWd = mm(dYq.t().contiguous(), idY, hq.t().contiguous(), ih)   # dY^T h
            dX = mm(dHq, idH, Wuq.t().contiguous(), iWu)                   # dH W_up
            dWu = mm(dHq.t().contiguous(), idH, Xq.t().contiguous(), iX)   # dH^T X
            return Yt, dX, dWu, dWd  # returned, so a compiler cannot drop the work

        mlp = api.Relu2Mlp(M, d, f)
        Y = torch.empty(M, d, dtype=bf, device="cuda")
        ours_step = lambda: (mlp.forward(X, Wu, Wd, Y=Y), mlp.backward(dY))
        t_ref = sum(time_it(torch_step, a.iters, a.warmup, flush)) / a.iters
        # the same composition under torch.compile, as the pages ran it
        compiled = torch.compile(torch_step)
        t_cmp = sum(time_it(compiled, a.iters, a.warmup, flush)) / a.iters
        t_ours = sum(time_it(ours_step, a.iters, a.warmup, flush)) / a.iters
        flops = 6 * 2 * M * d * f
        out = dict(op="torch-composition", M=M, d=d, f=f,
                   eager_ms=round(t_ref, 4), eager_tflops=round(flops / t_ref / 1e9, 1),
                   compiled_ms=round(t_cmp, 4), compiled_tflops=round(flops / t_cmp / 1e9, 1),
                   ours_ms=round(t_ours, 4), ours_tflops=round(flops / t_ours / 1e9, 1),
                   speedup_vs_eager=round(t_ref / t_ours, 3),
                   speedup_vs_compiled=round(t_cmp / t_ours, 3))
    elif a.op == "mlp-compare":
        from fp8_gemms_b200 import api
        M, d = a.M, a.d
        res = {}
        for name, f in (("relu2", 4 * d), ("swiglu", (11 * d) // 4)):
            mk = lambda *sh, s=1.0: (torch.randn(*sh, device="cuda", generator=gen) * s).to(
                torch.bfloat16)
            X, dY = mk(M, d), mk(M, d, s=1e-3)
            Wd = mk(d, f, s=0.02)
            if name == "relu2":
                mlp, W1 = api.Relu2Mlp(M, d, f), mk(f, d, s=0.02)
                flops = 6 * 2 * M * d * f
            else:
                mlp, W1 = api.SwigluMlp(M, d, f), mk(2 * f, d, s=0.02)
                flops = 9 * 2 * M * d * f
            step = lambda: (mlp.forward(X, W1, Wd), mlp.backward(dY))
            ms = time_it(step, a.iters, a.warmup, flush)
            avg = sum(ms) / len(ms)
            res[name] = dict(f=f, ms_per_step=round(avg, 4),
                             tokens_per_s=round(M / avg * 1e3), tflops=round(flops / avg / 1e9, 1))
            del mlp
            torch.cuda.empty_cache()
        out = dict(op="mlp-compare", M=M, d=d, **res,
                   relu2_over_swiglu_tokens=round(res["relu2"]["tokens_per_s"] /
                                                  res["swiglu"]["tokens_per_s"], 4))
    elif a.op == "lmhead-ce":
        from fp8_gemms_b200 import api
        M, d, V = a.M, a.d, a.V
        head = api.LmHeadCE(M, d, V, a.chunk)
        X = torch.randn(M, d, device="cuda", generator=gen).to(torch.bfloat16)
        W = (torch.randn(V, d, device="cuda", generator=gen) * 0.02).to(torch.bfloat16)
        labels = torch.randint(0, 50257, (M,), device="cuda", generator=gen, dtype=torch.int32)
        dW = torch.zeros(V, d, dtype=torch.float32, device="cuda")
        dX = torch.empty_like(X)
        fn = lambda: head(X, W, labels, dW=dW, dX=dX)
        ms = time_it(fn, a.iters, a.warmup, flush)
        avg = sum(ms) / len(ms)
        flops = 3 * 2 * M * d * V
        # one more call with the library's per-launch events: time per launch kind
        timer = _lib.KernelTimer(16 * ((M + a.chunk - 1) // a.chunk) + 16)
        flush.fill_(1)
        end = torch.cuda.Event(enable_timing=True)
        with timer:
            fn()
        end.record()
        end.synchronize()
        by_kind = {}
        for kd, ms_k in zip(timer.kinds, timer.durations_ms(end)):
            by_kind[kd] = round(by_kind.get(kd, 0.0) + ms_k, 4)
        out = dict(op="lmhead-ce", M=M, d=d, V=V, chunk=a.chunk, avg_ms=round(avg, 4),
                   tokens_per_s=round(M / avg * 1e3), tflops=round(flops / avg / 1e9, 1),
                   workspace_bytes=head.workspace.numel(), full_logits_bytes=2 * M * V,
                   loss=round(float(head.loss.item()), 5),
                   ms_by_launch_kind=by_kind)
    elif a.op == "rmsnorm-cast":
        R = torch.randn(a.rows, a.cols, device="cuda", generator=gen).to(torch.bfloat16)
        w = torch.randn(a.cols, device="cuda", generator=gen).to(torch.bfloat16)
        X = torch.empty_like(R)
        q = torch.empty(a.rows, a.cols, dtype=torch.uint8, device="cuda")
        qT = torch.empty(a.cols, a.rows, dtype=torch.uint8, device="cuda")
        sc = torch.zeros(4, device="cuda")
        fn = lambda: _lib.lm_rmsnorm_fp8_cast(R, w, X, FMT[a.fmt], sc[0:1], sc[1:2], sc[2:3], q, qT)
        ms = time_it(fn, a.iters, a.warmup, flush)
        n = a.rows * a.cols
        avg = sum(ms) / len(ms)
        # R read, X write, X read, q, qT: 8 bytes per element
        out = dict(op="rmsnorm-cast", rows=a.rows, cols=a.cols, fmt=a.fmt, avg_ms=round(avg, 4),
                   gbs=round(8 * n / avg / 1e6, 1), algorithmic_bytes=8 * n)
    elif a.op == "gemm":
        fa, fb, epi = FMT[a.fa], FMT[a.fb], EPI[a.epi]
        A = random_codes(fa, *((a.K, a.M) if a.flags & 1 else (a.M, a.K)), gen)
        B = random_codes(fb, *((a.K, a.N) if a.flags & 2 else (a.N, a.K)), gen)
        ia = torch.full((1,), 1e-2, device="cuda")
        ib = torch.full((1,), 1e-2, device="cuda")
        D = torch.empty(a.M, a.N, dtype=torch.bfloat16, device="cuda")
        aux = torch.randn(a.M, a.N, device="cuda", generator=gen).to(torch.bfloat16) \
            if epi == EPI_RELU2_BWD else None
        am = torch.zeros(1, device="cuda")
        ws = None if a.no_ws else torch.empty(_lib.lm_fp8_gemm_workspace_size(),
                                              dtype=torch.uint8, device="cuda")
        fn = lambda: _lib.lm_fp8_gemm_ex(A, fa, B, fb, ia, ib, D, flags=a.flags, epi=epi, aux=aux,
                                         amax_out=am, workspace=ws)
        ms = time_it(fn, a.iters, a.warmup, flush)
        flops = 2 * a.M * a.N * a.K
        byts = a.M * a.K + a.N * a.K + 2 * a.M * a.N * (2 if epi == EPI_RELU2_BWD else 1)
        avg = sum(ms) / len(ms)
        out = dict(op="gemm", M=a.M, N=a.N, K=a.K, fa=a.fa, fb=a.fb, epi=a.epi, flags=a.flags,
                   workspace=not a.no_ws,
                   avg_ms=round(avg, 4), min_ms=round(min(ms), 4),
                   tflops=round(flops / avg / 1e9, 1), algorithmic_bytes=byts)
    else:
        fmt = FMT[a.fmt]
        x = (torch.randn(a.rows, a.cols, device="cuda", generator=gen)).to(torch.bfloat16)
        q = torch.empty(a.rows, a.cols, dtype=torch.uint8, device="cuda")
        qT = None if a.no_qT else torch.empty(a.cols, a.rows, dtype=torch.uint8, device="cuda")
        sc = torch.zeros(4, device="cuda")
        amax_in = torch.full((1,), 4.0, device="cuda") if a.amax_in else None
        fn = lambda: _lib.lm_fp8_amax_scale_cast(x, fmt, sc[0:1], sc[1:2], sc[2:3], q, qT,
                                                 relu2_input=a.relu2, amax_in=amax_in)
        ms = time_it(fn, a.iters, a.warmup, flush)
        n = a.rows * a.cols
        byts = n * ((2 if a.amax_in else 4) + (1 if a.no_qT else 2))
        avg = sum(ms) / len(ms)
        out = dict(op="cast", rows=a.rows, cols=a.cols, fmt=a.fmt, relu2=a.relu2,
                   amax_in=a.amax_in, qT=not a.no_qT, avg_ms=round(avg, 4),
                   min_ms=round(min(ms), 4),
                   gbs=round(byts / avg / 1e6, 1), algorithmic_bytes=byts)
    if a.op == "mlp-accum":
        from fp8_gemms_b200 import api  # noqa: F811
        M, d, f = a.M, a.d, a.f
        mlp = api.Relu2Mlp(M, d, f)
        Wu = (torch.randn(f, d, device="cuda", generator=gen) * 0.02).to(torch.bfloat16)
        Wd = (torch.randn(d, f, device="cuda", generator=gen) * 0.02).to(torch.bfloat16)
        Xs = [torch.randn(M, d, device="cuda", generator=gen).to(torch.bfloat16)
              for _ in range(a.micro)]
        dYs = [(torch.randn(M, d, device="cuda", generator=gen) * 1e-3).to(torch.bfloat16)
               for _ in range(a.micro)]
        dWu = torch.zeros(f, d, dtype=torch.float32, device="cuda")
        dWd = torch.zeros(d, f, dtype=torch.float32, device="cuda")
        Y = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
        dX = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")

        def opt_step():
            dWu.zero_()
            dWd.zero_()
            for i in range(a.micro):
                mlp.forward(Xs[i], Wu, Wd, Y=Y, reuse_weight_casts=i > 0)
                mlp.backward_accumulate(dYs[i], dWu, dWd, dX=dX)

        ms = time_it(opt_step, a.iters, a.warmup, flush)
        avg = sum(ms) / len(ms)
        flops = a.micro * 6 * 2 * M * d * f
        out = dict(op="mlp-accum", M=M, d=d, f=f, micro_batches=a.micro, avg_ms=round(avg, 4),
                   ms_per_micro_batch=round(avg / a.micro, 4),
                   tflops=round(flops / avg / 1e9, 1))
    st, where = _lib.lm_get_error()
    out["device_error"] = st
    print(json.dumps(out))


if __name__ == "__main__":
    main()
