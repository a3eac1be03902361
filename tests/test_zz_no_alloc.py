"""The allocation-free relu^2 MLP backward (lm_relu2_mlp_bwd_noalloc).

It exists for callers that cannot allocate device memory -- plugins inside a
host framework that owns the memory pool, or loops that cannot afford the
synchronisation of cudaMalloc -- and keeps its workspace in a fixed array
owned by the library.  It runs the same kernels with the same split plan as
the allocating backward (lm_relu2_mlp_bwd), so its outputs must be
bit-identical to that backward's on the same inputs, on consecutive calls that
reuse the array; and it must reject shapes whose workspace does not fit.

This file is collected last on purpose and sets up everything it needs, so it
passes alone in a fresh process as well as after the other tests.
"""
import numpy as np
import pytest
import torch

from fp8_gemms_b200 import synthetic
from gpu_util import assert_close, u16

pytestmark = pytest.mark.gpu


def test_noalloc_backward_matches_allocating_backward_on_two_calls(orc):
    """Two calls in a row through the C ABI.  The second uses dY / 4, so its
    amax, scales and every code differ from the first's: state the first call
    left in the shared array (amax accumulators, split-K flags, dH codes) would
    show as a mismatch."""
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import _lib, api

    w = synthetic.TINY_MLP
    t = w.tensors()
    dev = {k: v.cuda() for k, v in t.items()}
    mlp = api.Relu2Mlp(w.M, w.d, w.f)
    mlp.forward(dev["X"], dev["W_up"], dev["W_down"])
    torch.cuda.synchronize()

    for call, dY in enumerate([dev["dY"], dev["dY"] * 0.25]):
        ref_dX, ref_dWu, ref_dWd = mlp.backward(dY)          # caller-provided workspace
        dX = torch.full_like(ref_dX, float("nan"))
        dWu = torch.full_like(ref_dWu, float("nan"))
        dWd = torch.full_like(ref_dWd, float("nan"))
        _lib.lm_relu2_mlp_bwd_noalloc(dY, mlp.saved, dX, dWu, dWd)
        torch.cuda.synchronize()
        assert _lib.lm_get_error()[0] == 0
        assert torch.equal(dX, ref_dX), f"dX, call {call}"
        assert torch.equal(dWu, ref_dWu), f"dW_up, call {call}"
        assert torch.equal(dWd, ref_dWd), f"dW_down, call {call}"
        if call == 0:
            b = {k: synthetic.bits_u16(v) for k, v in t.items()}
            bwd = orc.mlp_bwd(b["dY"], orc.mlp_fwd(b["X"], b["W_up"], b["W_down"]))
            assert_close(u16(dX), bwd["dX"], "dX vs oracle")
            assert_close(u16(dWu), bwd["dW_up"], "dW_up vs oracle")
            assert_close(u16(dWd), bwd["dW_down"], "dW_down vs oracle")


def test_noalloc_backward_in_a_cuda_graph():
    """The entry point is meant for graph capture: after one eager call (which
    resolves the library array's address), the backward is captured once and
    replayed; every replay must reproduce the eager outputs bit for bit, and a
    replay after the inputs change must follow them."""
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import _lib, api

    w = synthetic.TINY_MLP
    dev = {k: v.cuda() for k, v in w.tensors().items()}
    mlp = api.Relu2Mlp(w.M, w.d, w.f)
    mlp.forward(dev["X"], dev["W_up"], dev["W_down"])
    dY = dev["dY"].clone()
    dX = torch.empty(w.M, w.d, dtype=torch.bfloat16, device="cuda")
    dWu = torch.empty(w.f, w.d, dtype=torch.bfloat16, device="cuda")
    dWd = torch.empty(w.d, w.f, dtype=torch.bfloat16, device="cuda")

    def bwd():
        _lib.lm_relu2_mlp_bwd_noalloc(dY, mlp.saved, dX, dWu, dWd)

    bwd()                                        # eager warm-up before capture
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    eager = [x.clone() for x in (dX, dWu, dWd)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            bwd()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        for x in (dX, dWu, dWd):
            x.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert _lib.lm_get_error()[0] == 0
        for name, a, b in zip(("dX", "dW_up", "dW_down"), eager, (dX, dWu, dWd)):
            assert torch.equal(a, b), name
    # new upstream gradient, same buffers: the replay follows it
    dY.mul_(0.25)
    g.replay()
    ref_dX, ref_dWu, ref_dWd = mlp.backward(dY)
    torch.cuda.synchronize()
    del g
    assert torch.equal(dX, ref_dX)
    assert torch.equal(dWu, ref_dWu)
    assert torch.equal(dWd, ref_dWd)


def test_noalloc_backward_rejects_shapes_beyond_its_array():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import _lib

    cap = _lib.lib.lm_relu2_mlp_bwd_noalloc_max_bytes()
    assert cap == 64 << 20
    assert _lib.lm_relu2_mlp_workspace_size(832, 3072, 12288) <= cap
    M, d, f = 848, 3072, 12288                                # the first M that does not fit
    assert _lib.lm_relu2_mlp_workspace_size(M, d, f) > cap
    s = _lib.MlpSaved()
    status = _lib.lib.lm_relu2_mlp_bwd_noalloc(None, s, M, d, f, None, None, None, None)
    assert _lib.STATUS[status] == "LM_ERR_UNSUPPORTED_SHAPE"
