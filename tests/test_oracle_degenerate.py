"""The oracle on the method's degenerate inputs, pinned by what the
mathematics fixes for them: an empty reduction is zero, so a GEMM with K = 0
gives D = epi(0) = 0 and no tokens give zero weight gradients; zero inputs
quantise to zero codes whatever the scale; the epilogues' amax of an all-zero
output is zero.  These are the cases the GPU tests exercise as empty and
zero inputs."""
import numpy as np

from fp8_gemms_b200 import synthetic

E4M3, E5M2 = 0, 1


def test_empty_reduction_gives_zero_for_every_epilogue(orc):
    """Sum over an empty K: 0.  relu(0)^2 = 0, 2 relu(H) * 0 = 0 for any H."""
    A = np.zeros((5, 0), np.uint8)
    B = np.zeros((7, 0), np.uint8)
    one = np.float32(1.0)
    D, am = orc.gemm(A, E4M3, B, E4M3, one, one)
    assert D.shape == (5, 7) and not D.any()
    D, am = orc.gemm(A, E4M3, B, E4M3, one, one, epi=orc.EPI_RELU2_FWD)
    assert not D.any() and am == 0.0
    H = synthetic.bits_u16(synthetic.normal_bf16((5, 7), 3.0, 1, 0))
    D, am = orc.gemm(A, E5M2, B, E4M3, one, one, epi=orc.EPI_RELU2_BWD, aux=H)
    assert not (D & 0x7FFF).any() and am == 0.0   # +0 or -0 (a negative H's 0 * -x)


def test_zero_tensor_casts_to_zero_codes(orc):
    """amax 0; 0 times any finite scale is 0, which both formats code as 0x00."""
    z = np.zeros((16, 32), np.uint16)
    for fmt in (E4M3, E5M2):
        r = orc.amax_scale_cast(z, fmt)
        assert r["amax"] == 0.0 and np.isfinite(r["scale"]) and r["scale"] > 0
        assert not r["q"].any() and not r["qT"].any()


def test_no_tokens_give_empty_outputs_and_zero_weight_gradients(orc):
    """M = 0: Y and dX have no rows; dW_up = dH^T X and dW_down = dY^T h are
    sums over no tokens, so zero; the weights are still cast exactly as on
    their own."""
    t = synthetic.MlpWorkload("no tokens", 16, 32, 64, True, seed=3).tensors()
    b = {k: synthetic.bits_u16(v) for k, v in t.items()}
    fw = orc.mlp_fwd(b["X"][:0], b["W_up"], b["W_down"])
    assert fw["Y"].shape == (0, 32) and fw["h"]["amax"] == 0.0
    for name in ("W_up", "W_down"):
        ref = orc.amax_scale_cast(b[name], E4M3)
        assert np.array_equal(fw[name]["q"], ref["q"]) and fw[name]["scale"] == ref["scale"]
    bw = orc.mlp_bwd(b["dY"][:0], fw)
    assert bw["dX"].shape == (0, 32)
    assert bw["dW_up"].shape == (64, 32) and not (bw["dW_up"] & 0x7FFF).any()
    assert bw["dW_down"].shape == (32, 64) and not (bw["dW_down"] & 0x7FFF).any()


def test_lm_head_with_no_tokens(orc):
    """M = 0: dW is a sum over no tokens, so zero; dX has no rows; the mean
    loss over no tokens is taken as 0 (the library's reading)."""
    W = synthetic.bits_u16(synthetic.normal_bf16((48, 32), 0.02, 4, 1))
    X = np.zeros((0, 32), np.uint16)
    loss, dX, dW, rows = orc.lmhead_ce(X, W, np.zeros(0, np.int32), chunk=16)
    assert loss == 0.0 and dX.shape == (0, 32) and rows.shape == (0,)
    assert dW.shape == (48, 32) and not dW.any()
