"""Resources of the sm_100a kernels as ptxas reports them (-Xptxas -v), checked
on the host at build time (nvcc cross-compiles; no GPU is needed):

  - no kernel spills registers to local memory;
  - the persistent GEMMs (one 192-thread CTA per SM) stay within 255 registers
    per thread;
  - the TMA-fed cast keeps two CTAs per SM: its register use times its threads
    times two fits the SM's 65,536 registers.

A spill or a lost CTA per SM would slow the kernels without failing any parity
test, so the build is checked for it here."""
import os
import re
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "fp8_gemms_b200", "csrc")

pytestmark = pytest.mark.skipif(shutil.which(os.environ.get("NVCC", "nvcc")) is None,
                                reason="nvcc not found")


def ptxas_report(source):
    """{mangled kernel name: (registers, spill store bytes, spill load bytes)}"""
    from fp8_gemms_b200 import build
    nvcc = os.environ.get("NVCC", "nvcc")
    with tempfile.TemporaryDirectory() as d:
        cmd = [nvcc, "-Xptxas=-v", *build.NVCC_FLAGS, "-I", build.INCLUDE, "-I", CSRC, "-c",
               os.path.join(CSRC, source), "-o", os.path.join(d, "k.o")]
        out = subprocess.run(cmd, check=True, capture_output=True, text=True).stderr
    report, name = {}, None
    for line in out.splitlines():
        m = re.search(r"Compiling entry function '(\w+)'", line)
        if m:
            name = m.group(1)
            report[name] = [None, None, None]
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and name:
            report[name][1], report[name][2] = int(m.group(1)), int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m and name:
            report[name][0] = int(m.group(1))
    return {k: tuple(v) for k, v in report.items()}


@pytest.fixture(scope="module")
def reports():
    return {src: ptxas_report(src) for src in sorted(os.listdir(CSRC)) if src.endswith(".cu")}


def test_no_kernel_spills(reports):
    kernels = 0
    for src, rep in reports.items():
        for name, (regs, st, ld) in rep.items():
            kernels += 1
            assert regs is not None and st is not None, (src, name)
            assert st == 0 and ld == 0, f"{src}: {name} spills {st} B / loads {ld} B"
    assert kernels >= 20


def test_gemm_register_budget(reports):
    pair = {k: v for k, v in reports["lm_gemm.cu"].items() if "gemm_fp8_pair_kernel" in k}
    # four public epilogues x (lean, multi-part split) + the gated epilogue, and
    # the side-cast instantiations of the plain and relu^2-forward epilogues
    assert len(pair) == 11
    assert sum(re.search(r"ILi\d+ELb[01]ELb1EE", k) is not None for k in pair) == 2
    for name, (regs, _, _) in pair.items():
        # 192 threads: the 255-register cap; 320 threads (side warps): the
        # register file split evenly, 65536 / 320 rounded down to 8
        side = re.search(r"ILi\d+ELb[01]ELb1EE", name) is not None  # <EPI, MULTI, SIDE=true>
        assert regs <= (200 if side else 255), (name, regs)


def test_cast_keeps_two_ctas_per_sm(reports):
    src = open(os.path.join(CSRC, "lm_cast.cu")).read()
    consumers = int(re.search(r"constexpr int CONSUMERS = (\d+);", src).group(1))
    threads = consumers + 32  # eight converter warps and one TMA warp
    casts = {k: v for k, v in reports["lm_cast.cu"].items() if "cast_tma_kernel" in k}
    assert casts
    for name, (regs, _, _) in casts.items():
        # registers are granted per warp in units of 8 per thread
        per_thread = -(-regs // 8) * 8
        assert 2 * threads * per_thread <= 65536, (name, regs, threads)
