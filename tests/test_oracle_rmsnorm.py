"""Pins of the oracle's RMSNorm (the producer of the FP8 GEMM input) against
closed forms and invariants of RMS normalisation."""
import numpy as np
import torch

from fp8_gemms_b200 import synthetic


def vals(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bits(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_constant_rows_normalise_to_the_sign(orc):
    R = np.zeros((4, 64), np.float32)
    R[0], R[1], R[2], R[3] = 3.0, -0.25, 1e-3, 50.0
    X = vals(orc.rmsnorm(bits(R), eps=0.0))
    assert np.array_equal(X, np.sign(R))                     # c / |c| exactly
    # with eps, a tiny row is damped: c / sqrt(c^2 + eps), rounded once
    X = vals(orc.rmsnorm(bits(R), eps=1e-6))
    c = vals(bits(R))[2, 0]
    assert X[2, 0] == vals(bits(np.float32(c / np.sqrt(c * c + 1e-6))))


def test_one_hot_row_and_weight(orc):
    d = 256
    R = np.zeros((1, d), np.float32)
    R[0, 7] = -2.0
    w = np.full(d, 0.5, np.float32)
    X = vals(orc.rmsnorm(bits(R), bits(w), eps=0.0))
    # mean square = 4/d, so the one nonzero becomes -2 / (2/sqrt(d)) * 0.5 = -sqrt(d)/2
    assert X[0, 7] == -8.0 and np.count_nonzero(X) == 1


def test_unit_rms_and_scale_invariance(orc):
    R = synthetic.normal_bf16((32, 512), 3.0, 61, 0)
    Rb = synthetic.bits_u16(R)
    X = vals(orc.rmsnorm(Rb, eps=0.0))
    rms = np.sqrt(np.mean(X * X, axis=1))
    assert np.all(np.abs(rms - 1.0) < 2.0 ** -7)              # within bf16 rounding
    R4 = synthetic.bits_u16((R.float() * 4.0).to(torch.bfloat16))   # exact power-of-two scale
    assert np.array_equal(orc.rmsnorm(R4, eps=0.0), orc.rmsnorm(Rb, eps=0.0))


def test_fused_producer_closed_forms(orc):
    """RMSNorm then the e4m3 cast, on rows whose outcome is known in closed
    form: constant rows normalise to +-1, so amax = 1, scale = 448 and every
    code is +-448 (0x7E / 0xFE); a one-hot row with weight 0.5 (d = 256)
    becomes -8 at its one entry, so amax = 8, scale = 56 and the codes are
    0xFE there and 0 elsewhere."""
    R = np.zeros((3, 256), np.float32)
    R[0], R[1], R[2] = 3.0, -0.25, 50.0
    out = orc.rmsnorm_fp8_cast(bits(R), eps=0.0)
    assert out["amax"] == 1.0 and out["scale"] == 448.0 and out["inv_scale"] == np.float32(1 / 448)
    assert np.all(out["q"][0] == 0x7E) and np.all(out["q"][1] == 0xFE) and np.all(out["q"][2] == 0x7E)
    R1 = np.zeros((1, 256), np.float32)
    R1[0, 7] = -2.0
    out = orc.rmsnorm_fp8_cast(bits(R1), bits(np.full(256, 0.5, np.float32)), eps=0.0)
    assert out["amax"] == 8.0 and out["scale"] == 56.0
    assert out["q"][0, 7] == 0xFE and np.count_nonzero(out["q"]) == 1
    assert out["qT"][7, 0] == 0xFE
