"""GPU parity of the fused RMSNorm -> amax -> FP8 cast producer.

X itself is a floating-point output (fp32 accumulation on the GPU, fp64 in
the oracle): each element within one bf16 rounding step of the oracle's
(|d| <= 2^-7 |ref|, the spacing of bf16 at the bottom of a binade).  The amax,
scales and codes are checked bit-exact against the oracle's cast of the GPU's
own X (stagewise)."""
import numpy as np
import pytest
import torch

from fp8_gemms_b200 import synthetic
from gpu_util import bf16_to_f64, f32, u8, u16

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1


def run(orc, R, w, fmt=E4M3, want_qT=True):
    from fp8_gemms_b200 import _lib
    rows, cols = R.shape
    Rd = R.cuda()
    wd = None if w is None else w.cuda()
    X = torch.empty(rows, cols, dtype=torch.bfloat16, device="cuda")
    sc = torch.zeros(4, device="cuda")
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    qT = torch.empty(cols, rows, dtype=torch.uint8, device="cuda") if want_qT else None
    _lib.lm_rmsnorm_fp8_cast(Rd, wd, X, fmt, sc[0:1], sc[1:2], sc[2:3], q, qT)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    Xg = u16(X)
    ref = orc.rmsnorm(synthetic.bits_u16(R), None if w is None else synthetic.bits_u16(w))
    g, r = bf16_to_f64(Xg), bf16_to_f64(ref)
    assert np.all(np.abs(g - r) <= 2.0 ** -7 * np.abs(r)), "X beyond one bf16 step"
    own = orc.amax_scale_cast(Xg, fmt)
    assert f32(sc[0]) == own["amax"] and f32(sc[1]) == own["scale"] and f32(sc[2]) == own["inv_scale"]
    assert np.array_equal(u8(q), own["q"])
    if want_qT:
        assert np.array_equal(u8(qT), own["qT"])


@pytest.mark.parametrize("rows,cols", [(256, 3072), (272, 144), (16, 16), (1040, 528)])
def test_rmsnorm_cast_with_weight(orc, rows, cols):
    R = synthetic.student_t3_bf16((rows, cols), 70, rows)
    w = synthetic.normal_bf16((cols,), 1.0, 70, cols)
    run(orc, R, w)


def test_rmsnorm_cast_without_weight_e5m2_and_q_only(orc):
    R = synthetic.normal_bf16((200, 256), 5.0, 71, 0)
    run(orc, R, None, fmt=E5M2, want_qT=False)


def test_rmsnorm_cast_full_size(orc):
    """The model's residual stream at M = 16384 tokens, d = 3072."""
    R = synthetic.student_t3_bf16((16384, 3072), 72, 0)
    w = synthetic.normal_bf16((3072,), 1.0, 72, 1)
    run(orc, R, w)
