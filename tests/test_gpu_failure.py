"""Device-side failure detection without a GPU fault: a bounded wait that
nothing satisfies runs out, records its code in the device error word and
returns; the host reads it with lm_get_error, the word is cleared, and the
context keeps working."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_expiry_is_reported_and_recoverable():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import _lib
    assert _lib.lm_get_error() == (0, 0)
    _lib.lm_selftest_bounded_wait(50)
    st, where = _lib.lm_get_error()
    assert _lib.STATUS[st] == "LM_ERR_TIMEOUT" and where == 0x301
    assert _lib.lm_get_error() == (0, 0)          # read and cleared
    # the context is still usable: a GEMM runs and is right
    A = torch.full((256, 64), 0x38, dtype=torch.uint8, device="cuda")   # e4m3 1.0
    B = torch.full((256, 64), 0x40, dtype=torch.uint8, device="cuda")   # e4m3 2.0
    one = torch.ones(1, device="cuda")
    D = torch.empty(256, 256, dtype=torch.bfloat16, device="cuda")
    _lib.lm_fp8_gemm(A, _lib.E4M3, B, _lib.E4M3, one, one, D)
    torch.cuda.synchronize()
    assert torch.all(D.float() == 128.0)
    assert _lib.lm_get_error() == (0, 0)


def test_selftest_rejects_bad_limits():
    from fp8_gemms_b200 import _lib
    assert _lib.STATUS[_lib.lib.lm_selftest_bounded_wait(0, None)] == "LM_ERR_INVALID_ARG"
    assert _lib.STATUS[_lib.lib.lm_selftest_bounded_wait(6000, None)] == "LM_ERR_INVALID_ARG"
