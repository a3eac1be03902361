"""Gradient accumulation over micro-batches (the run's 7 grad-accum steps):
the fp32-accumulating wgrad epilogue (LM_EPI_ACCUM_F32, a TMA reduce-add in
the CTA-pair kernel) and the forward's reuse of the weight casts, against the
oracle."""
import numpy as np
import pytest
import torch

from fp8_gemms_b200 import synthetic
from gpu_util import assert_close, assert_close_f32, from_u8, u16

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import _lib
    return _lib


def codes(fmt, shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(TORCH_DT[fmt]).view(torch.uint8).numpy()


@pytest.mark.parametrize("M,N,K", [(384, 768, 512), (200, 328, 208), (128, 256, 128),
                                   (16, 8, 16), (3072, 1024, 2048)])
def test_accumulating_gemm_twice(lib, orc, M, N, K):
    A1, A2 = codes(E5M2, (M, K), 1), codes(E5M2, (M, K), 2)
    B1, B2 = codes(E4M3, (N, K), 3), codes(E4M3, (N, K), 4)
    D0 = np.random.default_rng(5).standard_normal((M, N)).astype(np.float32) * 1e-3
    D = torch.from_numpy(D0.copy()).cuda()
    ia = torch.tensor([1e-4], device="cuda")
    ib = torch.tensor([0.05], device="cuda")
    for A, B in [(A1, B1), (A2, B2)]:
        lib.lm_fp8_gemm(from_u8(A), E5M2, from_u8(B), E4M3, ia, ib, D, epi=lib.EPI_ACCUM_F32)
    torch.cuda.synchronize()
    assert lib.lm_get_error()[0] == 0
    ref = D0.copy()
    for A, B in [(A1, B1), (A2, B2)]:
        orc.gemm_accum_f32(A, E5M2, B, E4M3, np.float32(1e-4), np.float32(0.05), ref)
    assert_close_f32(D.cpu().numpy(), ref, f"accum M={M} N={N} K={K}")


@pytest.mark.parametrize("M,N,K", [(512, 336, 400), (96, 272, 160)])
def test_accumulating_gemm_mn_major(lib, orc, M, N, K):
    """The wgrad shape of the blocks: both operands MN-major (the row-major
    codes of dY / X read as their transposes), accumulated in fp32."""
    A, B = codes(E5M2, (M, K), 9), codes(E4M3, (N, K), 10)
    D0 = np.random.default_rng(11).standard_normal((M, N)).astype(np.float32) * 1e-3
    D = torch.from_numpy(D0.copy()).cuda()
    ia = torch.tensor([1e-4], device="cuda")
    ib = torch.tensor([0.05], device="cuda")
    At = torch.from_numpy(np.ascontiguousarray(A.T)).cuda()
    Bt = torch.from_numpy(np.ascontiguousarray(B.T)).cuda()
    lib.lm_fp8_gemm_ex(At, E5M2, Bt, E4M3, ia, ib, D, flags=3, epi=lib.EPI_ACCUM_F32)
    torch.cuda.synchronize()
    assert lib.lm_get_error()[0] == 0
    ref = D0.copy()
    orc.gemm_accum_f32(A, E5M2, B, E4M3, np.float32(1e-4), np.float32(0.05), ref)
    assert_close_f32(D.cpu().numpy(), ref, f"accum mn-major M={M} N={N} K={K}")


def test_mlp_grad_accumulation_three_micro_batches(lib, orc):
    from fp8_gemms_b200 import api
    w = synthetic.TINY_MLP
    t = w.tensors()
    mbs = [(t["X"], t["dY"])] + [
        (synthetic.normal_bf16((w.M, w.d), 1.0, 90 + i, 0),
         synthetic.normal_bf16((w.M, w.d), 1e-3, 90 + i, 1)) for i in range(2)]
    Wu, Wd = t["W_up"].cuda(), t["W_down"].cuda()
    mlp = api.Relu2Mlp(w.M, w.d, w.f)
    dWu = torch.zeros(w.f, w.d, dtype=torch.float32, device="cuda")
    dWd = torch.zeros(w.d, w.f, dtype=torch.float32, device="cuda")
    got = []
    for i, (X, dY) in enumerate(mbs):
        Y = mlp.forward(X.cuda(), Wu, Wd, reuse_weight_casts=i > 0)
        dX = mlp.backward_accumulate(dY.cuda(), dWu, dWd)
        got.append((u16(Y), u16(dX)))
    torch.cuda.synchronize()
    assert lib.lm_get_error()[0] == 0
    outs, rWu, rWd = orc.mlp_grad_accum(
        [(synthetic.bits_u16(X), synthetic.bits_u16(dY)) for X, dY in mbs],
        synthetic.bits_u16(t["W_up"]), synthetic.bits_u16(t["W_down"]))
    for i, ((gY, gdX), (rY, rdX)) in enumerate(zip(got, outs)):
        assert_close(gY, rY, f"Y[{i}]")
        assert_close(gdX, rdX, f"dX[{i}]")
    assert_close_f32(dWu.cpu().numpy(), rWu, "dW_up accumulated")
    assert_close_f32(dWd.cpu().numpy(), rWd, "dW_down accumulated")


def test_reused_weight_casts_give_the_same_forward(lib):
    from fp8_gemms_b200 import api
    w = synthetic.MlpWorkload("reuse", 512, 256, 1024, False)
    t = w.tensors()
    X2 = synthetic.normal_bf16((w.M, w.d), 1.0, 55, 0).cuda()
    mlp = api.Relu2Mlp(w.M, w.d, w.f)
    Wu, Wd = t["W_up"].cuda(), t["W_down"].cuda()
    mlp.forward(t["X"].cuda(), Wu, Wd)
    Y_reuse = mlp.forward(X2, None, None, reuse_weight_casts=True).clone()
    Y_full = mlp.forward(X2, Wu, Wd)
    torch.cuda.synchronize()
    assert torch.equal(Y_reuse, Y_full)
