"""GPU parity of the plain FP8 linear (lm_fp8_linear_fwd / lm_fp8_linear_bwd:
forward, dgrad, wgrad) at the attention-projection and LM-head shapes: X [M x K]
and W [N x K] cast to e4m3, dY [M x N] to e5m2 (row-major codes only), then
Y = Xq Wq^T, dX = dYq Wq, dW = dYq^T Xq, the last two reading the codes
MN-major.

Casts are checked bit-exact over whole tensors; GEMM outputs elementwise
within the stated tolerance, on all rows for small M and on sampled rows at
full size."""
import numpy as np
import pytest
import torch

from fp8_gemms_b200 import synthetic
from gpu_util import assert_close, assert_close_f32, f32, u8, u16

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
    sc = q["scales"]
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


def test_linear_ragged_shape(orc, api):
    """Every dimension off the 256-wide tile: M = 272, K = 208, N = 336."""
    w = synthetic.LinearWorkload("ragged", 272, [("r", 336, 208)])
    t = w.tensors(0)
    check_linear(orc, api, t["X"], t["W"], t["dY"])


def _lin_inputs(M, K, N, seed=0):
    t = synthetic.LinearWorkload("lin", M, [("l", N, K)], seed=seed).tensors(0)
    return t["X"].cuda(), t["W"].cuda(), t["dY"].cuda()


def test_linear_reused_weight_cast_and_skipped_dgrad(api):
    """The forward with LM_LINEAR_REUSE_WEIGHT_CAST uses W's codes and scale
    from the previous forward (they equal a fresh cast's); the backward with
    dX = NULL computes the same dW and leaves the dgrad out."""
    from fp8_gemms_b200 import _lib
    M, K, N = 512, 256, 384
    X, W, dY = _lin_inputs(M, K, N, seed=5)
    lin = api.Linear(M, K, N)
    lin.forward(X, W)
    w_scale, w_codes = lin.view("scales")[1].clone(), lin.view("Wq").clone()
    X2 = torch.roll(X, 7, dims=0).contiguous()
    Y2 = lin.forward(X2, None, reuse_weight_cast=True)
    fresh = api.Linear(M, K, N)
    Y3 = fresh.forward(X2, W)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    assert torch.equal(Y2.view(torch.int16), Y3.view(torch.int16))
    assert torch.equal(lin.view("scales")[1], w_scale) and torch.equal(lin.view("Wq"), w_codes)
    assert torch.equal(lin.view("scales"), fresh.view("scales"))
    dX, dW = lin.backward(dY)
    dX_none, dW2 = lin.backward(dY, need_dX=False)
    torch.cuda.synchronize()
    assert dX_none is None and dX is not None
    assert torch.equal(dW.view(torch.int16), dW2.view(torch.int16))


def test_linear_accumulating_wgrad(orc, api):
    """LM_LINEAR_ACCUMULATE_WGRAD over two calls: dW (fp32) += dYq^T Xq s each
    time, against the oracle's fp32-accumulating GEMM on the saved codes."""
    M, K, N = 384, 256, 320
    D0 = np.random.default_rng(6).standard_normal((N, K)).astype(np.float32) * 1e-3
    dW = torch.from_numpy(D0.copy()).cuda()
    ref = D0.copy()
    lin = api.Linear(M, K, N)
    for seed in (7, 8):
        X, W, dY = _lin_inputs(M, K, N, seed=seed)
        lin.forward(X, W)
        dX = lin.backward_accumulate(dY, dW)
        torch.cuda.synchronize()
        sx = lin.view("scales").cpu().numpy()
        sg = lin.workspace_view("scales").cpu().numpy()
        Xq, dYq = u8(lin.view("Xq")), u8(lin.workspace_view("dYq"))
        orc.gemm_accum_f32(np.ascontiguousarray(dYq.T), E5M2, np.ascontiguousarray(Xq.T), E4M3,
                           sg[2], sx[0, 2], ref)
        ref_dX, _ = orc.gemm(dYq, E5M2, np.ascontiguousarray(u8(lin.view("Wq")).T), E4M3,
                             sg[2], sx[1, 2])
        assert_close(u16(dX), ref_dX, "dX")
    from fp8_gemms_b200 import _lib
    assert _lib.lm_get_error()[0] == 0
    assert_close_f32(dW.cpu().numpy(), ref, "accumulated dW")


def test_linear_empty_batch(orc, api):
    """M = 0: nothing to multiply; W is still cast (its scale block is exact),
    Y and dX are empty and dW is zero."""
    K, N = 256, 128
    _, W, _ = _lin_inputs(16, K, N, seed=9)
    lin = api.Linear(0, K, N)
    X = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    Y = lin.forward(X, W)
    dX, dW = lin.backward(torch.empty(0, N, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    from fp8_gemms_b200 import _lib
    assert _lib.lm_get_error()[0] == 0
    assert Y.shape == (0, N) and dX.shape == (0, K)
    assert not bool(dW.view(torch.int16).any())
    ref = orc.amax_scale_cast(synthetic.bits_u16(W.cpu()), E4M3)
    sc = lin.view("scales").cpu().numpy()
    assert sc[1, 0] == ref["amax"] and sc[1, 1] == ref["scale"] and sc[1, 2] == ref["inv_scale"]
    assert np.array_equal(u8(lin.view("Wq")), ref["q"])


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


@pytest.mark.slow
@pytest.mark.parametrize("i", [0, 1, 4], ids=["q", "k", "lm_head"])
def test_attention_and_head_linears_are_deterministic_over_repeats(api, i):
    """Five fwd+dgrad+wgrad passes of the Q, K and LM-head linears at M = 8192
    (split tails, MN-major operands), L2 flushed between them: Y, dX and dW
    are bit-identical to the first pass's."""
    from fp8_gemms_b200 import _lib
    t = synthetic.ATTN_HEAD.tensors(i)
    X, W, dY = t["X"].cuda(), t["W"].cuda(), t["dY"].cuda()
    M, K = X.shape
    lin = api.Linear(M, K, W.shape[0])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    first = None
    for it in range(5):
        flush.fill_(it)
        Y = lin.forward(X, W)
        dX, dW = lin.backward(dY)
        torch.cuda.synchronize()
        assert _lib.lm_get_error()[0] == 0
        if first is None:
            first = [Y.clone(), dX.clone(), dW.clone()]
            continue
        for name, a, b in zip(("Y", "dX", "dW"), first, (Y, dX, dW)):
            assert torch.equal(a, b), f"{name} differs at repeat {it}"
