"""Out-of-bounds writes would corrupt neighbouring memory without faulting,
so every output here lives inside a larger buffer whose guard bands (256
bytes before, 4 KB after) hold a pattern that must survive the call.  Ragged
shapes exercise every tile edge (TMA store clipping, partial transposes)."""
import pytest
import torch

pytestmark = pytest.mark.gpu

PAT = 0xA5
PRE, POST = 256, 4096


def guarded(nbytes, dtype, shape):
    buf = torch.full((PRE + nbytes + POST,), PAT, dtype=torch.uint8, device="cuda")
    view = buf[PRE:PRE + nbytes].view(dtype).view(*shape)
    return buf, view


def intact(buf, nbytes):
    return bool((buf[:PRE] == PAT).all()) and bool((buf[PRE + nbytes:] == PAT).all())


def codes(shape, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn(*shape, device="cuda", generator=g).to(torch.float8_e4m3fn).view(torch.uint8)


@pytest.mark.parametrize("M,N,K,epi", [(200, 328, 208, 0), (130, 264, 48, 1), (16, 8, 16, 0),
                                       (300, 1032, 1040, 2), (272, 520, 96, 3)])
def test_gemm_writes_stay_inside_D(M, N, K, epi):
    from fp8_gemms_b200 import _lib
    A, B = codes((M, K), 1), codes((N, K), 2)
    one = torch.full((1,), 0.01, device="cuda")
    dt = torch.float32 if epi == 3 else torch.bfloat16
    nbytes = M * N * (4 if epi == 3 else 2)
    buf, D = guarded(nbytes, dt, (M, N))
    if epi == 3:
        D.zero_()
    aux = torch.randn(M, N, device="cuda").to(torch.bfloat16) if epi == 2 else None
    _lib.lm_fp8_gemm(A, 0, B, 0, one, one, D, epi=epi, aux=aux)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    assert intact(buf, nbytes)


@pytest.mark.parametrize("M,N,K,epi", [(208, 336, 208, 0), (112, 528, 272, 3), (304, 1040, 96, 2)])
def test_gemm_mn_major_writes_stay_inside_D(M, N, K, epi):
    """Both operands stored MN-major (the transposes); ragged tiles in N and K."""
    from fp8_gemms_b200 import _lib
    At, Bt = codes((K, M), 3), codes((K, N), 4)
    one = torch.full((1,), 0.01, device="cuda")
    dt = torch.float32 if epi == 3 else torch.bfloat16
    nbytes = M * N * (4 if epi == 3 else 2)
    buf, D = guarded(nbytes, dt, (M, N))
    if epi == 3:
        D.zero_()
    aux = torch.randn(M, N, device="cuda").to(torch.bfloat16) if epi == 2 else None
    _lib.lm_fp8_gemm_ex(At, 0, Bt, 0, one, one, D, flags=3, epi=epi, aux=aux)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    assert intact(buf, nbytes)


@pytest.mark.parametrize("transposed", [True, False])
@pytest.mark.parametrize("rows,cols", [(272, 144), (16, 16), (1040, 48), (200, 96)])
def test_cast_writes_stay_inside_q_and_qT(rows, cols, transposed):
    from fp8_gemms_b200 import _lib
    x = torch.randn(rows, cols, device="cuda").to(torch.bfloat16)
    bq, q = guarded(rows * cols, torch.uint8, (rows, cols))
    want_qT = transposed and rows % 16 == 0
    bt, qT = guarded(rows * cols, torch.uint8, (cols, rows)) if want_qT else (None, None)
    sc = torch.zeros(4, device="cuda")
    _lib.lm_fp8_amax_scale_cast(x, 0, sc[0:1], sc[1:2], sc[2:3], q, qT)
    torch.cuda.synchronize()
    assert intact(bq, rows * cols)
    if want_qT:
        assert intact(bt, rows * cols)


def test_mlp_and_lmhead_outputs_stay_inside():
    from fp8_gemms_b200 import _lib, api
    M, d, f = 272, 208, 848
    X = torch.randn(M, d, device="cuda").to(torch.bfloat16)
    Wu = (torch.randn(f, d, device="cuda") * 0.02).to(torch.bfloat16)
    Wd = (torch.randn(d, f, device="cuda") * 0.02).to(torch.bfloat16)
    dY = (torch.randn(M, d, device="cuda") * 1e-3).to(torch.bfloat16)
    mlp = api.Relu2Mlp(M, d, f)
    by, Y = guarded(M * d * 2, torch.bfloat16, (M, d))
    bx, dX = guarded(M * d * 2, torch.bfloat16, (M, d))
    bu, dWu = guarded(f * d * 2, torch.bfloat16, (f, d))
    bd, dWd = guarded(d * f * 2, torch.bfloat16, (d, f))
    mlp.forward(X, Wu, Wd, Y=Y)
    mlp.backward(dY, dX=dX, dW_up=dWu, dW_down=dWd)
    Mh, dh, V = 96, 64, 400
    head = api.LmHeadCE(Mh, dh, V, 32)
    Xh = torch.randn(Mh, dh, device="cuda").to(torch.bfloat16)
    Wh = (torch.randn(V, dh, device="cuda") * 0.02).to(torch.bfloat16)
    labels = torch.randint(0, V, (Mh,), device="cuda", dtype=torch.int32)
    bhx, dXh = guarded(Mh * dh * 2, torch.bfloat16, (Mh, dh))
    bhw, dWh = guarded(V * dh * 4, torch.float32, (V, dh))
    dWh.zero_()
    head(Xh, Wh, labels, dW=dWh, dX=dXh)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    for b, n in [(by, M * d * 2), (bx, M * d * 2), (bu, f * d * 2), (bd, d * f * 2),
                 (bhx, Mh * dh * 2), (bhw, V * dh * 4)]:
        assert intact(b, n)
