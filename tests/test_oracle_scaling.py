"""Pins of the oracle's amax, scale and cast (dynamic tensorwise scaling).

Checked against: the closed form (the scaled amax encodes to exactly the
format's max code), a brute-force numpy max, and PyTorch's CPU float8 cast of
the same fp32 products (pre-clamped) as an independent implementation.
"""
import numpy as np
import pytest
import torch

from fp8_gemms_b200 import synthetic

E4M3, E5M2 = 0, 1
MAXC = {E4M3: 0x7E, E5M2: 0x7B}
FMAX = {E4M3: 448.0, E5M2: 57344.0}
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_scaled_amax_encodes_to_max_code(orc, fmt):
    rng = np.random.default_rng(11 + fmt)
    for a in np.exp2(rng.uniform(-30, 30, 4000)).astype(np.float32):
        s, inv = orc.scale(a, fmt)
        assert s == np.float32(np.float32(FMAX[fmt]) / a)          # one fp32 division
        assert inv == np.float32(np.float32(1.0) / s)
        assert orc.fp8_encode(float(np.float32(a) * s), fmt) == MAXC[fmt]
        assert orc.fp8_encode(float(-np.float32(a) * s), fmt) == MAXC[fmt] | 0x80


def test_scale_zero_and_nonfinite_amax(orc):
    s, inv = orc.scale(0.0, E4M3)
    assert s == np.float32(448.0) / np.float32(1e-12)
    s, _ = orc.scale(float("nan"), E4M3)
    assert np.isnan(s)
    s, _ = orc.scale(float("inf"), E5M2)
    assert s == 0.0


def _bits(t):
    return synthetic.bits_u16(t)


def test_amax_brute_force(orc):
    x = synthetic.normal_bf16((77, 130), 3.0, 5, 0)
    ref = np.float32(x.float().abs().max().item())
    assert orc.amax(_bits(x)) == ref
    h = (torch.relu(x.float()) ** 2).to(torch.bfloat16)  # exact square, one rounding
    assert orc.amax(_bits(x), relu2_input=True) == np.float32(h.float().max().item())
    xn = x.clone()
    xn[3, 4] = float("nan")
    assert np.isnan(orc.amax(_bits(xn)))


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
@pytest.mark.parametrize("relu2", [False, True])
def test_cast_matches_torch_reference(orc, fmt, relu2):
    x = synthetic.student_t3_bf16((96, 160), 9, fmt)
    r = orc.amax_scale_cast(_bits(x), fmt, relu2_input=relu2)
    src = (torch.relu(x.float()) ** 2).to(torch.bfloat16).float() if relu2 else x.float()
    assert r["amax"] == np.float32(src.abs().max().item())
    prod = src * torch.tensor(float(r["scale"]), dtype=torch.float32)  # fp32 multiply
    ref = prod.clamp(-FMAX[fmt], FMAX[fmt]).to(TORCH_DT[fmt]).view(torch.uint8).numpy()
    assert np.array_equal(r["q"], ref)
    assert np.array_equal(r["qT"], ref.T)
    # the largest magnitude lands exactly on the max code
    assert (r["q"] & 0x7F).max() == MAXC[fmt]


def test_cast_zero_tensor(orc):
    x = torch.zeros(16, 32, dtype=torch.bfloat16)
    r = orc.amax_scale_cast(_bits(x), E4M3)
    assert r["amax"] == 0.0
    assert not r["q"].any() and not r["qT"].any()
