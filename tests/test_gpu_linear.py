"""GPU parity of the plain FP8 linear (forward, dgrad, wgrad) at the
attention-projection and LM-head shapes: X [M x K] and W [N x K] cast to e4m3,
dY [M x N] to e5m2 (each with its K-major transposed copy), then
Y = Xq Wq^T, dX = dYq (Wq^T)^T, dW = (dYq^T)(Xq^T)^T, all through the C ABI.

Casts are checked bit-exact over whole tensors; GEMM outputs elementwise
within the stated tolerance, on all rows for small M and on sampled rows at
full size."""
import numpy as np
import pytest
import torch

from fp8_gemms_b200 import synthetic
from gpu_util import assert_close, f32, u8, u16

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1


@pytest.fixture(scope="module")
def api():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import api as a
    return a


def check_linear(orc, api, X, W, dY, rows=None, wrows=None):
    Y, dX, dW, q = api.linear_fwd_bwd(X.cuda(), W.cuda(), dY.cuda())
    torch.cuda.synchronize()
    from fp8_gemms_b200 import _lib
    assert _lib.lm_get_error()[0] == 0
    sc = q["scales"].cpu().numpy()
    for i, (t, fmt, key) in enumerate([(X, E4M3, "Xq"), (W, E4M3, "Wq"), (dY, E5M2, "dYq")]):
        ref = orc.amax_scale_cast(synthetic.bits_u16(t), fmt)
        assert sc[i, 0] == ref["amax"] and sc[i, 1] == ref["scale"] and sc[i, 2] == ref["inv_scale"]
        assert np.array_equal(u8(q[key]), ref["q"]), key
    Xq, Wq, dYq = u8(q["Xq"]), u8(q["Wq"]), u8(q["dYq"])
    # dgrad and wgrad read the row-major codes MN-major; the oracle takes the
    # K-major operands (host transposes)
    XqT, WqT, dYqT = (np.ascontiguousarray(a.T) for a in (Xq, Wq, dYq))
    sel = lambda a, r: a if r is None else a[r]
    ref_Y, _ = orc.gemm(Xq, E4M3, Wq, E4M3, sc[0, 2], sc[1, 2], rows=rows)
    assert_close(sel(u16(Y), rows), ref_Y, "Y")
    ref_dX, _ = orc.gemm(dYq, E5M2, WqT, E4M3, sc[2, 2], sc[1, 2], rows=rows)
    assert_close(sel(u16(dX), rows), ref_dX, "dX")
    ref_dW, _ = orc.gemm(dYqT, E5M2, XqT, E4M3, sc[2, 2], sc[0, 2], rows=wrows)
    assert_close(sel(u16(dW), wrows), ref_dW, "dW")


@pytest.mark.parametrize("name,n_out,n_in", synthetic.ATTN_LINEARS +
                         [("lm_head", synthetic.VOCAB_PADDED, synthetic.D_MODEL)])
def test_linear_shapes_small_batch(orc, api, name, n_out, n_in):
    """All five projection shapes at M = 512 tokens; the LM head's N = 50,304
    is not a multiple of the 256-column tile."""
    w = synthetic.LinearWorkload("small", 512, [(name, n_out, n_in)])
    t = w.tensors(0)
    check_linear(orc, api, t["X"], t["W"], t["dY"])


def test_linear_student_t_activations(orc, api):
    w = synthetic.LinearWorkload("t3", 768, [("q", 3072, 3072)], ("t3", None), 3)
    t = w.tensors(0)
    check_linear(orc, api, t["X"], t["W"], t["dY"])


def _sample(n, k=24, seed=0):
    r = np.random.default_rng(seed)
    return np.sort(np.concatenate([np.arange(4), np.arange(n - 4, n),
                                   r.choice(np.arange(4, n - 4), k - 8, replace=False)]))


@pytest.mark.slow
@pytest.mark.parametrize("i", range(5))
def test_attention_and_head_full_size_sampled(orc, api, i):
    """Q, K, V, O and the LM head at M = 8192 tokens, X ~ N(0,1)."""
    w = synthetic.ATTN_HEAD
    t = w.tensors(i)
    check_linear(orc, api, t["X"], t["W"], t["dY"], rows=_sample(w.M),
                 wrows=_sample(t["W"].shape[0], seed=1))


@pytest.mark.slow
@pytest.mark.parametrize("layer", [0, 27])
def test_stack_layer_linears_full_size_sampled(orc, api, layer):
    """Layers of the 28-layer stack at M = 16384 with t3 activations: the
    four attention linears."""
    lin, _ = synthetic.stack_layer(layer)
    for i in range(len(lin.linears)):
        t = lin.tensors(i)
        check_linear(orc, api, t["X"], t["W"], t["dY"], rows=_sample(lin.M),
                     wrows=_sample(t["W"].shape[0], seed=1))
