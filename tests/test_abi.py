"""The C-ABI library loads on a CPU-only host, exports every symbol that
include/*.h declares, and its host-side argument checks reject bad calls
before any launch (no GPU needed for any of this)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"^LM_API\s+[\w\s\*]+?\b(lm_\w+)\s*\(", text, flags=re.M)
    return names


@pytest.fixture(scope="module")
def L():
    from fp8_gemms_b200 import build
    build.build()
    from fp8_gemms_b200 import _lib
    return _lib


def test_header_declares_the_boundary():
    names = declared_functions()
    for fn in ["lm_fp8_amax_scale_cast", "lm_fp8_gemm", "lm_relu2_mlp_fwd", "lm_relu2_mlp_bwd"]:
        assert fn in names


def test_library_exports_every_declared_symbol(L):
    lib = ctypes.CDLL(L.LIB_PATH)
    for fn in declared_functions():
        assert hasattr(lib, fn), fn
    assert sorted(declared_functions()) == sorted(L.EXPORTED)


def test_status_strings_and_version(L):
    assert L.lm_version() >= 100
    for code, name in L.STATUS.items():
        assert L.lm_status_string(code).startswith(name)


def test_gemm_host_checks_reject_before_launch(L):
    g = L.lib.lm_fp8_gemm
    fake = 0x10000  # never dereferenced: every call below fails a host check first
    E4, E5 = L.E4M3, L.E5M2
    assert g(fake, E5, fake, E5, 16, 16, 16, fake, fake, 0, None, fake, None, None) == 4
    assert g(fake, 7, fake, E4, 16, 16, 16, fake, fake, 0, None, fake, None, None) == 4
    assert g(fake, E4, fake, E4, 16, 16, 16, fake, fake, 9, None, fake, None, None) == 4
    assert g(fake, E4, fake, E4, -1, 16, 16, fake, fake, 0, None, fake, None, None) == 1
    assert g(fake, E4, fake, E4, 16, 16, 16, None, fake, 0, None, fake, None, None) == 1
    assert g(fake, E4, fake, E4, 16, 16, 16, fake, fake, 2, None, fake, None, None) == 1
    assert g(fake, E4, fake, E4, 16, 16, 24, fake, fake, 0, None, fake, None, None) == 3
    assert g(fake, E4, fake, E4, 16, 12, 16, fake, fake, 0, None, fake, None, None) == 3
    assert g(fake + 8, E4, fake, E4, 16, 16, 16, fake, fake, 0, None, fake, None, None) == 2
    assert g(fake, E4, fake, E4, 16, 16, 16, fake, fake, 0, None, fake + 4, None, None) == 2
    # empty output: nothing to do, nothing launched
    assert g(fake, E4, fake, E4, 0, 16, 16, fake, fake, 0, None, fake, None, None) == 0


def test_cast_host_checks_reject_before_launch(L):
    c = L.lib.lm_fp8_amax_scale_cast
    fake = 0x10000
    assert c(fake, 32, 32, 32, 5, 0, None, fake, fake, fake, fake, fake, None) == 4
    assert c(fake, 32, 24, 24, 0, 0, None, fake, fake, fake, fake, None, None) == 3
    assert c(fake, 24, 32, 32, 0, 0, None, fake, fake, fake, None, fake, None) == 3
    assert c(fake, 32, 32, 16, 0, 0, None, fake, fake, fake, fake, fake, None) == 1
    assert c(fake, 32, 32, 32, 0, 0, None, None, fake, fake, fake, fake, None) == 1
    assert c(fake + 2, 32, 32, 32, 0, 0, None, fake, fake, fake, fake, fake, None) == 2


def test_mlp_sizes_and_carve(L):
    M, d, f = 256, 256, 1024
    r = lambda n: (n + 255) // 256 * 256
    # row-major codes only (the backward reads them MN-major): X, W_up, W_down,
    # H, h codes and the scales; scratch dY codes, dH, dH codes, scales
    assert L.lm_relu2_mlp_saved_bytes(M, d, f) == (r(M * d) + 2 * r(f * d) + r(2 * M * f)
                                                   + r(M * f) + r(64))
    # scratch: the GEMMs' split-K scratch (128 partial tiles x 256 KB of fp32 sums
    # plus a flag per CTA and warp), then dY codes, dH, dH codes, scales
    split = 128 * (256 * 1024 + 2 * 4 * 4)
    assert L.lib.lm_fp8_gemm_workspace_size() == split
    assert L.lm_relu2_mlp_workspace_size(M, d, f) == (r(split) + r(M * d) + r(2 * M * f)
                                                      + r(M * f) + r(32))
    assert L.lm_relu2_mlp_saved_bytes(M, d, 1000) == 0      # f not a multiple of 16
    s = L.MlpSaved()
    base = 0x100000
    n = L.lm_relu2_mlp_saved_bytes(M, d, f)
    assert L.lib.lm_relu2_mlp_saved_carve(base, n, M, d, f, ctypes.byref(s)) == 0
    assert s.Xq == base and s.Wuq == base + r(M * d) and s.scales == base + n - r(64)
    assert L.lib.lm_relu2_mlp_saved_carve(base, n - 1, M, d, f, ctypes.byref(s)) == 1
    assert L.lib.lm_relu2_mlp_saved_carve(base + 16, n, M, d, f, ctypes.byref(s)) == 2


def test_newer_entry_points_reject_before_launch(L):
    import ctypes as C
    fake = 0x10000
    lib = L.lib
    s = L.MlpSaved()
    # unknown flags
    assert lib.lm_relu2_mlp_fwd_ex(fake, fake, fake, 256, 256, 1024, fake, C.byref(s), None, 0, 4,
                                   None) == 1
    # a forward workspace must be 256-byte aligned
    assert lib.lm_relu2_mlp_fwd_ex(fake, fake, fake, 256, 256, 1024, fake, C.byref(s), fake + 16,
                                   1 << 30, 0, None) == 2
    assert lib.lm_relu2_mlp_bwd_ex(fake, C.byref(s), 256, 256, 1024, fake, fake, fake, fake,
                                   1 << 30, 1, None) == 1
    # rmsnorm: eps < 0, cols not a multiple of 16, misaligned weight
    f32 = C.c_float
    assert lib.lm_rmsnorm_fp8_cast(fake, None, 32, 64, f32(-1.0), 0, fake, fake, fake, fake,
                                   fake, fake, None) == 1
    assert lib.lm_rmsnorm_fp8_cast(fake, None, 32, 40, f32(1e-6), 0, fake, fake, fake, fake,
                                   fake, fake, None) == 3
    assert lib.lm_rmsnorm_fp8_cast(fake, fake + 2, 32, 64, f32(1e-6), 0, fake, fake, fake,
                                   fake, fake, fake, None) == 2
    # swiglu: f must be a multiple of 128
    assert L.lib.lm_swiglu_mlp_saved_bytes(256, 256, 200) == 0
    sw = L.SwigluSaved()
    assert lib.lm_swiglu_mlp_fwd(fake, fake, fake, 256, 256, 200, fake, C.byref(sw), None, 0,
                                 None) == 3
    # lm head: chunk not a multiple of 16, softcap <= 0, workspace too small
    assert lib.lm_fp8_lmhead_ce_workspace_size(64, 64, 128, 24) == 0
    n = lib.lm_fp8_lmhead_ce_workspace_size(64, 64, 128, 32)
    assert n > 0
    assert lib.lm_fp8_lmhead_ce(fake, fake, fake, 64, 64, 128, 32, f32(0.0), fake, fake, fake,
                                fake, n, None) == 1
    assert lib.lm_fp8_lmhead_ce(fake, fake, fake, 64, 64, 128, 32, f32(15.0), fake, fake, fake,
                                fake, n - 1, None) == 1
    # the internal gated epilogue is not reachable through the public GEMM
    assert lib.lm_fp8_gemm(fake, 0, fake, 0, 256, 256, 64, fake, fake, 4, None, fake, None,
                           None) == 4
    # operand-storage flags: unknown bits; MN-major rows not 16-byte aligned
    gx = lib.lm_fp8_gemm_ex
    assert gx(fake, 0, fake, 0, 256, 256, 64, 4, fake, fake, 0, None, fake, None, None, 0, None) == 1
    assert gx(fake, 0, fake, 0, 200, 256, 64, 1, fake, fake, 0, None, fake, None, None, 0, None) == 3
    assert gx(fake, 0, fake, 0, 256, 264, 64, 2, fake, fake, 0, None, fake, None, None, 0, None) == 3
    assert gx(fake, 0, fake, 0, 256, 264, 64, 1, fake, fake, 4, None, fake, None, None, 0, None) == 4
    # no-alloc backward: shape beyond its array
    assert lib.lm_relu2_mlp_bwd_noalloc(None, C.byref(s), 16384, 3072, 12288, None, None, None,
                                        None) == 3


def test_linear_sizes_carve_and_checks(L):
    import ctypes as C
    M, K, N = 256, 192, 320
    r = lambda n: (n + 255) // 256 * 256
    # saved: X codes, W codes, two scale blocks; scratch: split-K region, dY codes, one block
    assert L.lm_fp8_linear_saved_bytes(M, K, N) == r(M * K) + r(N * K) + r(32)
    split = L.lib.lm_fp8_gemm_workspace_size()
    assert L.lm_fp8_linear_workspace_size(M, K, N) == r(split) + r(M * N) + r(16)
    assert L.lm_fp8_linear_saved_bytes(M, K, 200) == 0      # N not a multiple of 16
    assert L.lm_fp8_linear_workspace_size(24, K, N) == 0    # M not a multiple of 16
    assert L.lm_fp8_linear_saved_bytes(0, K, N) == r(N * K) + r(32)
    s = L.LinearSaved()
    base, n = 0x100000, L.lm_fp8_linear_saved_bytes(M, K, N)
    assert L.lib.lm_fp8_linear_saved_carve(base, n, M, K, N, C.byref(s)) == 0
    assert s.Xq == base and s.Wq == base + r(M * K) and s.scales == base + n - r(32)
    assert L.lib.lm_fp8_linear_saved_carve(base, n - 1, M, K, N, C.byref(s)) == 1
    assert L.lib.lm_fp8_linear_saved_carve(base + 16, n, M, K, N, C.byref(s)) == 2
    fake = 0x10000
    fwd, bwd = L.lib.lm_fp8_linear_fwd, L.lib.lm_fp8_linear_bwd
    ws = L.lm_fp8_linear_workspace_size(M, K, N)
    assert fwd(fake, fake, M, K, 200, fake, C.byref(s), None, 0, 0, None) == 3
    assert fwd(fake, fake, M, K, N, fake, C.byref(s), None, 0, 4, None) == 1    # unknown flag
    assert fwd(fake, fake, M, K, N, fake, C.byref(s), fake + 16, ws, 0, None) == 2
    assert fwd(fake, None, M, K, N, fake, C.byref(s), None, 0, 0, None) == 1    # W needed
    assert fwd(None, fake, M, K, N, fake, C.byref(s), None, 0, 0, None) == 1
    assert bwd(fake, C.byref(s), M, K, N, fake, fake, fake, ws - 1, 0, None) == 1
    assert bwd(fake, C.byref(s), M, K, N, fake, fake, fake + 16, ws, 0, None) == 2
    assert bwd(fake, C.byref(s), M, K, N, fake, fake, fake, ws, 1, None) == 1   # fwd's flag
    assert bwd(fake, C.byref(s), M, K, N, fake, None, fake, ws, 0, None) == 1   # dW needed


def test_split_plan_on_a_148_sm_gpu(L):
    """The split-K tail plan (host arithmetic).  With 148 SMs there are C = 74
    CTA pairs; the last wave holds rem = tiles mod 74 tiles of 256 x 256."""
    plan = lambda M, N, K: L.lm_fp8_gemm_split_plan(M, N, K, 148)
    # relu^2 MLP, M = 16384: N = 3072 GEMMs have 768 tiles, rem 28 <= 37: halves
    assert plan(16384, 3072, 12288) == (2, 28)
    # N = 12288 GEMMs: 3072 tiles, rem 38 > 37, K = 3072 too short to gain: unsplit
    assert plan(16384, 12288, 3072) == (1, 0)
    # wgrads: 576 tiles, rem 58; more parts would need 2+ rounds each: unsplit
    assert plan(3072, 12288, 16384) == (1, 0) and plan(12288, 3072, 16384) == (1, 0)
    # K / V wgrad: 48 tiles, all in the last wave; three parts would take two
    # rounds and two partial reads each, measured slower: unsplit
    assert plan(1024, 3072, 8192) == (1, 0) and plan(1024, 3072, 16384) == (1, 0)
    # deep K pays for more parts: 44 tiles, K = 32768, three parts in two rounds
    assert plan(256 * 44, 256, 32768) == (3, 44)
    # LM head dgrad (K = 50304): 384 tiles, rem 14; five parts in one round
    assert plan(8192, 3072, 50304) == (5, 14)
    # a chunk's dgrad in the fused LM head: 192 tiles, rem 44: three parts
    assert plan(4096, 3072, 50304) == (3, 44)
    # short K with a small tail keeps halves (8 k-blocks: more parts do not pay)
    assert plan(8192, 3072, 1024) == (2, 14)
    # a single k-block is never split; M <= 128 takes the single-CTA kernel
    assert plan(512, 512, 128) == (1, 0) and plan(128, 4096, 4096) == (1, 0)
    # no last wave to fill
    assert plan(256 * 74, 256, 4096) == (1, 0)
    import ctypes as C
    p, t = C.c_int(), C.c_int()
    assert L.lib.lm_fp8_gemm_split_plan(256, 256, 256, 1, C.byref(p), C.byref(t)) == 1
    assert L.lib.lm_fp8_gemm_split_plan(-1, 256, 256, 148, C.byref(p), C.byref(t)) == 1
    assert L.lib.lm_fp8_gemm_split_plan(256, 256, 256, 148, None, C.byref(t)) == 1


def test_split_plan_invariants_over_shapes(L):
    """For every plan: parts in [1, 8]; a split tail has two k-blocks per part
    (one for halves) and its partials fit the workspace's 128 tiles."""
    for sms in (148, 132, 16):
        C = sms // 2
        for M in (256, 768, 4096, 16384, 40960):
            for N in (256, 1024, 3072, 12288, 50304):
                for K in (128, 256, 1024, 3072, 12288, 50304):
                    S, rem = L.lm_fp8_gemm_split_plan(M, N, K, sms)
                    tiles = -(-M // 256) * -(-N // 256)
                    kb = -(-K // 128)
                    assert 1 <= S <= 8
                    if S == 1:
                        assert rem == 0
                        continue
                    assert rem == tiles % C and rem > 0
                    assert kb >= (2 if S == 2 else 2 * S)
                    assert rem * (S - 1) <= 128
                    if 2 * rem <= C:
                        assert S >= 2   # a tail of at most half the pairs is always split


def test_plain_c_program_uses_the_boundary(L, tmp_path):
    """The header is plain C99, and a C program links against the library and
    calls its host-only entry points (no torch, no GPU)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    src = tmp_path / "use_abi.c"
    src.write_text(r"""
#include <stdio.h>
#include "lm_fp8.h"
int main(void) {
    int parts = 0, tail = 0;
    if (lm_fp8_gemm_split_plan(16384, 3072, 12288, 148, &parts, &tail) != LM_OK) return 1;
    lm_linear_saved s;
    if (lm_fp8_linear_saved_carve((void*)0x100000, lm_fp8_linear_saved_bytes(256, 192, 320),
                                  256, 192, 320, &s) != LM_OK) return 2;
    printf("%d|%d|%d|%zu|%s\n", parts, tail, (int)((char*)s.Wq - (char*)s.Xq),
           lm_fp8_gemm_workspace_size(), lm_status_string(LM_ERR_ALIGNMENT));
    return 0;
}
""")
    exe = tmp_path / "use_abi"
    libdir = os.path.dirname(L.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I",
                    os.path.join(ROOT, "include"), str(src), "-L", libdir, "-lfp8lm",
                    "-Wl,-rpath," + libdir, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True,
                         text=True).stdout.strip().split("|")
    assert out[:3] == ["2", "28", str(256 * 192)]
    assert int(out[3]) == L.lib.lm_fp8_gemm_workspace_size()
    assert out[4].startswith("LM_ERR_ALIGNMENT")


def test_composite_entry_points_refuse_misaligned_tensors_before_any_launch(L):
    """A misaligned output of a composite call is refused before its first
    launch: the status is LM_ERR_ALIGNMENT, not the LM_ERR_CUDA that reaching a
    CUDA call would give on a host without a GPU."""
    import ctypes as C
    fake, bad = 0x100000, 0x100008           # 16-byte aligned / 8 bytes off
    mlp = L.MlpSaved(*([fake] * 6))
    sw = L.SwigluSaved(*([fake] * 7))
    lin = L.LinearSaved(fake, fake, fake)
    ws = 1 << 31
    lib = L.lib
    M, d, f = 256, 256, 1024
    # relu^2 MLP: misaligned Y (forward), dX (backward), a saved tensor (both)
    assert lib.lm_relu2_mlp_fwd(fake, fake, fake, M, d, f, bad, C.byref(mlp), None, 0, None) == 2
    assert lib.lm_relu2_mlp_bwd(fake, C.byref(mlp), M, d, f, bad, fake, fake, fake, ws, None) == 2
    mlp_bad = L.MlpSaved(fake, fake, fake, bad, fake, fake)       # H
    assert lib.lm_relu2_mlp_fwd(fake, fake, fake, M, d, f, fake, C.byref(mlp_bad), None, 0,
                                None) == 2
    assert lib.lm_relu2_mlp_bwd(fake, C.byref(mlp_bad), M, d, f, fake, fake, fake, fake, ws,
                                None) == 2
    # gated MLP (f a multiple of 128)
    assert lib.lm_swiglu_mlp_fwd(fake, fake, fake, M, d, f, bad, C.byref(sw), None, 0, None) == 2
    assert lib.lm_swiglu_mlp_bwd(fake, C.byref(sw), M, d, f, fake, bad, fake, fake, ws, None) == 2
    # plain linear: misaligned Y, dW, saved codes
    K, N = 192, 320
    assert lib.lm_fp8_linear_fwd(fake, fake, M, K, N, bad, C.byref(lin), None, 0, 0, None) == 2
    assert lib.lm_fp8_linear_bwd(fake, C.byref(lin), M, K, N, fake, bad, fake, ws, 0, None) == 2
    lin_bad = L.LinearSaved(fake, bad, fake)
    assert lib.lm_fp8_linear_fwd(fake, fake, M, K, N, fake, C.byref(lin_bad), None, 0, 0,
                                 None) == 2
    # a missing saved buffer is an argument error, in the backward too
    sw_null = L.SwigluSaved(fake, fake, fake, None, fake, fake, fake)
    assert lib.lm_swiglu_mlp_bwd(fake, C.byref(sw_null), M, d, f, fake, fake, fake, fake, ws,
                                 None) == 1
