"""Pins of the oracle's FP8 and bf16 codecs against the format definitions.

The oracle is checked against things other than itself: the published OCP
encoding parameters (tests/golden/ocp_fp8_formats.json), an exhaustive
256-code round trip, hand-built ties and boundaries, and PyTorch's own CPU
float8 / bfloat16 conversions used purely as an independent cross-check.
"""
import json
import math
import os
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

E4M3, E5M2 = 0, 1
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ocp_fp8_formats.json")


def torch_decode(fmt):
    return torch.arange(256, dtype=torch.uint8).view(TORCH_DT[fmt]).to(torch.float64).numpy()


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_decode_matches_published_parameters(orc, fmt):
    g = json.load(open(GOLDEN))["e4m3" if fmt == E4M3 else "e5m2"]
    dec = lambda s: orc.fp8_decode(int(s, 16), fmt)
    assert dec(g["max_normal_code"]) == g["max_normal"]
    assert dec(g["min_normal_code"]) == g["min_normal"]
    assert dec(g["max_subnormal_code"]) == g["max_subnormal"]
    assert dec(g["min_subnormal_code"]) == g["min_subnormal"]
    assert dec(g["one_code"]) == 1.0
    for c in g["nan_codes"]:
        assert math.isnan(dec(c))
    for c in g["infinity_codes"]:
        assert math.isinf(dec(c))
    nan_or_inf = {int(c, 16) for c in g["nan_codes"] + g["infinity_codes"]}
    finite = [c for c in range(256) if c not in nan_or_inf]
    assert all(math.isfinite(orc.fp8_decode(c, fmt)) for c in finite)
    assert max(orc.fp8_decode(c, fmt) for c in finite) == g["max_normal"]
    # the exponent bias: 2^0 sits at exponent field == bias
    mbits = 3 if fmt == E4M3 else 2
    assert orc.fp8_decode(g["exponent_bias"] << mbits, fmt) == 1.0


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_decode_all_codes_matches_torch(orc, fmt):
    ours = np.array([orc.fp8_decode(c, fmt) for c in range(256)])
    ref = torch_decode(fmt)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))  # -0 is 0x80


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_roundtrip_every_finite_code(orc, fmt):
    for c in range(256):
        v = orc.fp8_decode(c, fmt)
        if math.isnan(v):
            assert orc.fp8_encode(v, fmt) == (0x7F if fmt == E4M3 else 0x7E)
        elif math.isinf(v):
            assert orc.fp8_encode(v, fmt) == (0x7B if v > 0 else 0xFB)  # saturate
        else:
            assert orc.fp8_encode(v, fmt) == c, hex(c)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_ties_round_to_even_and_neighbours(orc, fmt):
    pos = sorted((orc.fp8_decode(c, fmt), c) for c in range(0x00, 0x80)
                 if math.isfinite(orc.fp8_decode(c, fmt)))
    for (v0, c0), (v1, c1) in zip(pos, pos[1:]):
        mid = (v0 + v1) / 2  # one extra bit: exact in fp32
        assert np.float32(mid) == mid
        even = c0 if c0 % 2 == 0 else c1
        assert orc.fp8_encode(mid, fmt) == even
        assert orc.fp8_encode(-mid, fmt) == even | 0x80
        below = float(np.nextafter(np.float32(mid), np.float32(0)))
        above = float(np.nextafter(np.float32(mid), np.float32(np.inf)))
        assert orc.fp8_encode(below, fmt) == c0
        assert orc.fp8_encode(above, fmt) == c1


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_saturation_and_specials(orc, fmt):
    mx, mxc = (448.0, 0x7E) if fmt == E4M3 else (57344.0, 0x7B)
    for v in [mx, mx * 1.0001, mx * 1.06, mx * 2, 1e30, float("inf")]:
        assert orc.fp8_encode(v, fmt) == mxc
        assert orc.fp8_encode(-v, fmt) == mxc | 0x80
    assert orc.fp8_encode(float("nan"), fmt) == (0x7F if fmt == E4M3 else 0x7E)
    assert orc.fp8_encode(0.0, fmt) == 0x00
    assert orc.fp8_encode(-0.0, fmt) == 0x80
    tiny = 2.0 ** (-9 if fmt == E4M3 else -16)  # min subnormal
    assert orc.fp8_encode(tiny, fmt) == 0x01
    assert orc.fp8_encode(tiny / 2, fmt) == 0x00            # tie -> even (zero)
    assert orc.fp8_encode(tiny / 2 * 1.0001, fmt) == 0x01
    assert orc.fp8_encode(-tiny / 4, fmt) == 0x80           # sign kept on underflow
    assert orc.fp8_encode(1e-30, fmt) == 0x00


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encode_matches_torch_on_random_fp32(orc, fmt):
    rng = np.random.default_rng(1234 + fmt)
    mx = 448.0 if fmt == E4M3 else 57344.0
    mags = np.exp2(rng.uniform(-20 if fmt == E4M3 else -26, math.log2(mx) + 0.5, 20000))
    vals = (mags * rng.choice([-1.0, 1.0], mags.size)).astype(np.float32)
    # torch's conversion does not saturate: clamp first (a test-side step only)
    clamped = np.clip(vals, -mx, mx)
    ref = torch.from_numpy(clamped).to(TORCH_DT[fmt]).view(torch.uint8).numpy()
    ours = np.array([orc.fp8_encode(float(v), fmt) for v in vals], dtype=np.uint8)
    assert np.array_equal(ours, ref)


def test_bf16_decode_and_round_once(orc):
    # decode: the bits are the upper half of a binary32
    for b, v in [(0x3F80, 1.0), (0xBF80, -1.0), (0x7F7F, (2 - 2 ** -7) * 2.0 ** 127),
                 (0x0001, 2.0 ** -133), (0x7F80, math.inf)]:
        assert orc.bf16_to_double(b) == v
    # exact fp32 inputs: identical to torch's RNE float32 -> bfloat16
    rng = np.random.default_rng(7)
    f = (rng.standard_normal(20000) * np.exp2(rng.uniform(-40, 40, 20000))).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = np.array([orc.bf16_from_double(float(x)) for x in f], dtype=np.uint16)
    assert np.array_equal(ours, ref)
    # a double just above a tie must round up (one rounding, not via fp32)
    assert orc.bf16_from_double(1 + 2 ** -8) == 0x3F80                # tie -> even
    assert orc.bf16_from_double(1 + 2 ** -8 + 2 ** -40) == 0x3F81     # not a tie
    assert orc.bf16_from_double(1 + 3 * 2 ** -8) == 0x3F82            # tie -> even (up)
    assert orc.bf16_from_double(-(1 + 2 ** -8 + 2 ** -40)) == 0xBF81
    top = (2 - 2 ** -7) * 2.0 ** 127
    assert orc.bf16_from_double(top) == 0x7F7F
    assert orc.bf16_from_double(top + 2.0 ** 119 * 1.0001) == 0x7F80  # overflow -> inf
    assert orc.bf16_from_double(2.0 ** -134) == 0x0000                 # tie -> even zero
    assert orc.bf16_from_double(2.0 ** -134 * 1.5) == 0x0001


def _exact_bf16(fr: Fraction) -> int:
    """Round an exact rational to bf16, ties to even, by integer arithmetic
    (an independent restatement used only to check the oracle)."""
    if fr == 0:
        return 0
    sign = 0x8000 if fr < 0 else 0
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)
    q = Fraction(2) ** (e - 7)
    n = a / q
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    val = fl * q
    f32 = np.float32(float(val))
    return sign | int(np.array([f32]).view(np.uint32)[0] >> 16)


def test_bf16_rounding_vs_exact_rationals(orc):
    rnd = random.Random(3)
    for _ in range(3000):
        num = rnd.randint(1, 2 ** 60)
        den = 2 ** rnd.randint(0, 100)
        fr = Fraction(num, den) * rnd.choice([-1, 1])
        v = float(fr)
        if Fraction(v) != fr:
            continue
        assert orc.bf16_from_double(v) == _exact_bf16(fr)
