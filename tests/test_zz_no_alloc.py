"""The allocation-free relu^2 MLP backward (lm_relu2_mlp_bwd_noalloc).

It exists for callers that cannot allocate device memory -- during CUDA graph
capture, inside a host framework that owns the memory pool, or where the
synchronisation of cudaMalloc is unaffordable -- and keeps its workspace in a
fixed array owned by the library.  It must produce what the allocating
backward (lm_relu2_mlp_bwd) produces, on consecutive calls that reuse that
array, and must reject shapes whose workspace does not fit.

This file is collected last on purpose and sets up everything it needs, so it
passes alone in a fresh process as well as after the other tests.
"""
import pytest
import torch

from fp8_gemms_b200 import synthetic
from gpu_util import assert_close, u16

pytestmark = pytest.mark.gpu


def test_noalloc_backward_matches_allocating_backward_on_two_calls():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import _lib, api

    w = synthetic.TINY_MLP
    t = w.tensors()
    dev = {k: v.cuda() for k, v in t.items()}
    mlp = api.Relu2Mlp(w.M, w.d, w.f)
    mlp.forward(dev["X"], dev["W_up"], dev["W_down"])
    ref_dX, ref_dWu, ref_dWd = mlp.backward(dev["dY"])      # caller-provided workspace
    torch.cuda.synchronize()

    for call in range(2):                                    # the array is reused as-is
        dX = torch.full_like(ref_dX, float("nan"))
        dWu = torch.full_like(ref_dWu, float("nan"))
        dWd = torch.full_like(ref_dWd, float("nan"))
        _lib.lm_relu2_mlp_bwd_noalloc(dev["dY"], mlp.saved, dX, dWu, dWd)
        torch.cuda.synchronize()
        assert _lib.lm_get_error()[0] == 0
        assert_close(u16(dX), u16(ref_dX), f"dX, call {call}")
        assert_close(u16(dWu), u16(ref_dWu), f"dW_up, call {call}")
        assert_close(u16(dWd), u16(ref_dWd), f"dW_down, call {call}")


def test_noalloc_backward_rejects_shapes_beyond_its_array():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import _lib

    cap = _lib.lib.lm_relu2_mlp_bwd_noalloc_max_bytes()
    assert cap == 64 << 20
    M, d, f = 16384, 3072, 12288                              # needs ~0.9 GB of workspace
    assert _lib.lm_relu2_mlp_workspace_size(M, d, f) > cap
    s = _lib.MlpSaved()
    status = _lib.lib.lm_relu2_mlp_bwd_noalloc(None, s, M, d, f, None, None, None, None)
    assert _lib.STATUS[status] == "LM_ERR_UNSUPPORTED_SHAPE"
