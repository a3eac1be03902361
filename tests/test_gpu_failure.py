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


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), float("-inf")])
@pytest.mark.parametrize("path", ["tma", "ragged_rows", "scales_only"])
def test_nonfinite_amax_is_reported(bad, path):
    """A tensor holding a NaN or an infinity has a non-finite amax.  Each cast
    path then records code 0x501, and lm_get_error returns LM_ERR_NONFINITE
    once (the word is cleared).  The same tensor made finite reports LM_OK."""
    import math
    from fp8_gemms_b200 import _lib
    rows = 200 if path == "ragged_rows" else 64   # rows % 16 != 0: the per-tile kernel
    x = torch.randn(rows, 128, device="cuda").to(torch.bfloat16)
    x[3, 17] = bad
    sc = torch.zeros(4, device="cuda")
    q = None if path == "scales_only" else torch.empty(rows, 128, dtype=torch.uint8,
                                                        device="cuda")
    _lib.lm_fp8_amax_scale_cast(x, _lib.E4M3, sc[0:1], sc[1:2], sc[2:3], q, None)
    st, where = _lib.lm_get_error()
    assert _lib.STATUS[st] == "LM_ERR_NONFINITE" and where == 0x501
    assert _lib.lm_get_error() == (0, 0)
    amax = float(sc[0])
    assert math.isnan(amax) if math.isnan(bad) else amax == math.inf
    x[3, 17] = 0.0
    _lib.lm_fp8_amax_scale_cast(x, _lib.E4M3, sc[0:1], sc[1:2], sc[2:3], q, None)
    assert _lib.lm_get_error() == (0, 0)
    assert math.isfinite(float(sc[0])) and float(sc[1]) > 0


def test_nonfinite_input_to_the_mlp_is_reported():
    """A NaN in X reaches the forward's cast of X: the block reports
    LM_ERR_NONFINITE rather than returning codes silently derived from it."""
    from fp8_gemms_b200 import _lib, api, synthetic
    w = synthetic.TINY_MLP
    t = {k: v.cuda() for k, v in w.tensors().items()}
    t["X"][5, 9] = float("nan")
    mlp = api.Relu2Mlp(w.M, w.d, w.f)
    mlp.forward(t["X"], t["W_up"], t["W_down"])
    st, where = _lib.lm_get_error()
    assert _lib.STATUS[st] == "LM_ERR_NONFINITE" and where == 0x501
    assert _lib.lm_get_error() == (0, 0)


@pytest.mark.parametrize("where_bad", ["W_down", "saved H"])
def test_nonfinite_tensor_cast_beside_a_gemm_is_reported(where_bad):
    """W_down's codes are written by side warps of the up GEMM's launch, and
    dH's by side warps of the dW_down GEMM's launch.  A NaN in W_down (its
    amax is NaN), or an infinity in the saved H (dH = g 2 relu(H) is then
    infinite while dY is finite), is reported from there, and the scales
    follow the formula."""
    from fp8_gemms_b200 import _lib, api, synthetic
    w = synthetic.TINY_MLP
    t = {k: v.cuda() for k, v in w.tensors().items()}
    if where_bad == "W_down":
        t["W_down"][3, 7] = float("nan")
    mlp = api.Relu2Mlp(w.M, w.d, w.f)
    mlp.forward(t["X"], t["W_up"], t["W_down"])
    if where_bad == "saved H":
        assert _lib.lm_get_error() == (0, 0)
        mlp.view("H")[:, 5] = float("inf")       # one whole column: some g there is nonzero
        mlp.backward(t["dY"])
    st, where = _lib.lm_get_error()
    assert _lib.STATUS[st] == "LM_ERR_NONFINITE" and where == 0x501
    assert _lib.lm_get_error() == (0, 0)
    if where_bad == "W_down":
        sc = mlp.view("scales").cpu()
        assert torch.isnan(sc[2, 0]) and torch.isnan(sc[2, 1])
    else:
        # dH is +-inf (or NaN where g is exactly 0): a non-finite amax, and the
        # scale the formula gives (57344 / inf = 0, or NaN)
        g = mlp.workspace_view("scales").cpu()
        assert not torch.isfinite(g[1, 0]) and (g[1, 1] == 0.0 or torch.isnan(g[1, 1]))
