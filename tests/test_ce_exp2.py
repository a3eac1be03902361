"""The CE kernel's FMA-pipe base-2 exponential (ex2_fma in lm_lmhead_ce.cu),
evaluated step by step in IEEE fp32 on the host: the coefficients are read from
the source, the rounding trick (whose low bits, shifted into the exponent
field, must be the bits of 2^n for an integer n within 1/2 of x, with
f = x - n exact), the Horner steps (one rounding each, as
fused multiply-adds round once) and the final exact multiply are reproduced,
and the result is compared with 2^x in fp64 over the kernel's whole argument
range."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "fp8_gemms_b200", "csrc", "lm_lmhead_ce.cu")


def coefficients():
    text = open(SRC).read()
    c = {int(k): float(v) for k, v in re.findall(r"kExp2C(\d) = ([0-9.eE+-]+)f", text)}
    assert sorted(c) == list(range(6)), c
    return [np.float32(c[k]) for k in range(6)]


def fma32(a, b, c):
    # a*b + c rounded to fp32: the product of two fp32 is exact in fp64 and the
    # fp64 sum rounds far below fp32 precision, so this matches a fused
    # multiply-add's single rounding except in rare double-rounding ties
    return (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)


def ex2_fma(x):
    c = coefficients()
    magic = np.float32(12583039.0)   # 1.5 * 2^23 + 127
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = fma32(np.full_like(f, c[5]), f, c[4])
    for k in (3, 2, 1, 0):
        p = fma32(p, f, c[k])
    scale = (t.view(np.int32) << 23).view(np.float32)   # 2^n, n = x - f
    n = np.log2(scale.astype(np.float64))
    assert np.array_equal(n, np.round(n)) and np.all(np.abs(x.astype(np.float64) - n) <= 0.5)
    assert np.array_equal(f.astype(np.float64), x.astype(np.float64) - n)
    return (p * scale).astype(np.float32)


def test_ex2_fma_relative_error_over_the_kernels_range():
    # softcap 40 (the fast kernel's limit): arguments down to -2 log2(e) 40
    x = np.concatenate([np.linspace(-115.5, 0.0, 2_000_001, dtype=np.float64),
                        -np.random.default_rng(0).random(200_000) * 115.5]).astype(np.float32)
    got = ex2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 4e-7, rel.max()


def test_ex2_fma_exact_at_integers_and_halves():
    # 2^n for integer n needs p(0) = 1 up to the C0 coefficient's rounding
    n = np.arange(-115, 1, dtype=np.float32)
    assert np.all(np.abs(ex2_fma(n) / np.exp2(n.astype(np.float64)) - 1) < 2e-7)
    h = (n - 0.5).astype(np.float32)
    assert np.all(np.abs(ex2_fma(h) / np.exp2(h.astype(np.float64)) - 1) < 4e-7)
