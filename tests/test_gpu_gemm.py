"""GPU parity of the tcgen05 FP8 GEMM and its epilogues against the oracle.

Same FP8 codes and scales go to both sides.  Outputs must meet the stated
tolerance (elementwise 1e-2 |ref| + 1e-3 rms(ref), normwise 5e-3); the amax
the epilogue reports must equal, bit for bit, the amax of the GPU's own
output (stagewise: the next cast consumes exactly that)."""
import numpy as np
import pytest
import torch

from gpu_util import (ELEM_REL, ELEM_REL_RELU2_BWD, assert_close, bf16_neighbours, bf16_to_f64,
                      f32, from_u8, from_u16, u16)

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1
EPI_NONE, EPI_RELU2_FWD, EPI_RELU2_BWD = 0, 1, 2
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import _lib
    return _lib


def codes(fmt, shape, seed, spread=1.0):
    """Random finite FP8 codes: an N(0, spread) draw quantised at scale 1."""
    g = torch.Generator().manual_seed(seed)
    v = torch.randn(*shape, generator=g) * spread
    mx = 448.0 if fmt == E4M3 else 57344.0
    return v.clamp(-mx, mx).to(TORCH_DT[fmt]).view(torch.uint8).numpy()


def run(lib, orc, M, N, K, fa=E4M3, fb=E4M3, epi=EPI_NONE, inv_a=0.02, inv_b=0.5, seed=0):
    A = codes(fa, (M, K), seed)
    B = codes(fb, (N, K), seed + 1)
    aux = None
    if epi == EPI_RELU2_BWD:
        g = torch.Generator().manual_seed(seed + 2)
        aux = u16(torch.randn(M, N, generator=g).to(torch.bfloat16))
    ia = torch.tensor([inv_a], dtype=torch.float32, device="cuda")
    ib = torch.tensor([inv_b], dtype=torch.float32, device="cuda")
    D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    am = torch.zeros(1, dtype=torch.float32, device="cuda")
    lib.lm_fp8_gemm(from_u8(A), fa, from_u8(B), fb, ia, ib, D, epi=epi,
                    aux=None if aux is None else from_u16(aux), amax_out=am)
    torch.cuda.synchronize()
    assert lib.lm_get_error()[0] == 0
    ref, ref_amax = orc.gemm(A, fa, B, fb, np.float32(inv_a), np.float32(inv_b), epi=epi, aux=aux)
    got = u16(D)
    assert_close(got, ref, f"gemm M={M} N={N} K={K} fa={fa} fb={fb} epi={epi}",
                 ELEM_REL_RELU2_BWD if epi == EPI_RELU2_BWD else ELEM_REL)
    if epi == EPI_RELU2_BWD:
        # exact epilogue arithmetic: dH = bf16(g' * 2 relu(H)) for a g' equal to,
        # or one bf16 ulp from, the oracle's g = bf16(acc s)
        g, _ = orc.gemm(A, fa, B, fb, np.float32(inv_a), np.float32(inv_b))
        h = torch.from_numpy(aux.view(np.int16)).view(torch.bfloat16).float()
        ok = np.zeros(got.shape, bool)
        for cand in (g, *bf16_neighbours(g)):
            gc = torch.from_numpy(cand.view(np.int16)).view(torch.bfloat16).float()
            dh = u16((gc * 2.0 * torch.relu(h)).to(torch.bfloat16))  # exact product, one rounding
            ok |= dh == got
        assert ok.all(), f"{int((~ok).sum())} dH elements not explained by g within 1 ulp"
    # the amax written by the epilogue is exactly the amax of the GPU's own D
    own = orc.amax(got, relu2_input=(epi == EPI_RELU2_FWD))
    assert f32(am) == own
    # and close to the oracle's
    assert abs(float(f32(am)) - float(ref_amax)) <= 1e-2 * float(ref_amax) + 1e-30
    return got, ref


# several tiles plus ragged tails in M, N and K
SHAPES = [
    (128, 256, 128),    # exactly one tile, one k-block
    (384, 768, 512),    # 3 x 3 tiles, 4 k-blocks
    (200, 328, 208),    # ragged M, N (N % 256 != 0) and K (K % 128 != 0)
    (16, 8, 16),        # smaller than one tile in every dimension
    (1, 264, 48),       # a single row
    (2304, 256, 256),   # 9 row-blocks of 256: one raster group spans M
    (4608, 512, 128),   # 18 row-blocks: groups of 8 plus a ragged last group
    (300, 1032, 1040),  # ragged everywhere, many tiles
    (260, 296, 144),    # last column tile: 40 columns, two 32-column chunks in one 64-column box
]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_e4m3_plain(lib, orc, M, N, K):
    run(lib, orc, M, N, K)


@pytest.mark.parametrize("M,N,K", SHAPES[:4])
def test_gemm_e5m2_e4m3_plain(lib, orc, M, N, K):
    run(lib, orc, M, N, K, fa=E5M2, inv_a=1e-4)


def test_gemm_e4m3_e5m2(lib, orc):
    run(lib, orc, 256, 512, 256, fa=E4M3, fb=E5M2, inv_b=1e-4)


# (2048, 4096, 256): 128 tiles, so some CTA pairs take two and the epilogue's
# box slots carry over from one tile to the next
RELU2_SHAPES = [(384, 768, 512), (200, 328, 208), (260, 296, 144), (2048, 4096, 256)]


@pytest.mark.parametrize("M,N,K", RELU2_SHAPES)
def test_gemm_relu2_fwd_epilogue(lib, orc, M, N, K):
    run(lib, orc, M, N, K, epi=EPI_RELU2_FWD)


@pytest.mark.parametrize("M,N,K", RELU2_SHAPES)
def test_gemm_relu2_bwd_epilogue(lib, orc, M, N, K):
    run(lib, orc, M, N, K, fa=E5M2, epi=EPI_RELU2_BWD, inv_a=1e-4)


def test_gemm_long_k_like_wgrad(lib, orc):
    """K = 8192, the reduction length of a wgrad over a batch of tokens."""
    run(lib, orc, 256, 512, 8192, fa=E5M2, inv_a=1e-5, inv_b=0.01)


def test_gemm_persistent_many_tiles(lib, orc):
    """More tiles than SMs: each CTA walks several tiles and both TMEM
    accumulators, and the smem ring wraps many times."""
    run(lib, orc, 2048, 4096, 256)


MN_CASES = [
    # (M, N, K, flags): pair kernel (M > 128) and thin kernel (M <= 128), ragged
    # tails in M, N and K where the 16-row rule of MN-major storage allows
    (208, 336, 208, 1), (208, 336, 208, 2), (208, 336, 208, 3),
    (128, 256, 128, 3),      # one tile, one k-block
    (384, 768, 512, 1),
    (2048, 4096, 256, 2),    # many tiles per cluster
    (16, 16, 16, 3),         # thin kernel, smaller than a tile everywhere
    (112, 528, 272, 2),      # thin kernel: B in two 128-wide MN blocks plus a ragged third tile
    (96, 256, 8192, 1),      # thin kernel, long K (a wgrad's reduction length)
]


def mn_store(X, mn):
    """The codes as the GPU reads them: X itself, or its transpose, contiguous."""
    return from_u8(np.ascontiguousarray(X.T) if mn else X)


@pytest.mark.parametrize("M,N,K,flags", MN_CASES)
def test_gemm_mn_major_operands(lib, orc, M, N, K, flags):
    """Operands stored MN-major (the transposes of A [M x K] / B [N x K]): the
    oracle's result on the K-major codes, and bit-identical to the K-major run."""
    A, B = codes(E5M2, (M, K), 21), codes(E4M3, (N, K), 22)
    ia = torch.tensor([1e-4], device="cuda")
    ib = torch.tensor([0.5], device="cuda")
    D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    Dk = torch.empty_like(D)
    am = torch.zeros(1, device="cuda")
    amk = torch.zeros(1, device="cuda")
    lib.lm_fp8_gemm_ex(mn_store(A, flags & 1), E5M2, mn_store(B, flags & 2), E4M3, ia, ib, D,
                       flags=flags, amax_out=am)
    lib.lm_fp8_gemm(from_u8(A), E5M2, from_u8(B), E4M3, ia, ib, Dk, amax_out=amk)
    torch.cuda.synchronize()
    assert lib.lm_get_error()[0] == 0
    ref, _ = orc.gemm(A, E5M2, B, E4M3, np.float32(1e-4), np.float32(0.5))
    assert_close(u16(D), ref, f"mn-major flags={flags} M={M} N={N} K={K}", ELEM_REL)
    assert torch.equal(D.view(torch.int16), Dk.view(torch.int16))
    assert torch.equal(am, amk)


@pytest.mark.parametrize("epi", [EPI_RELU2_FWD, EPI_RELU2_BWD])
@pytest.mark.parametrize("M,N,K", [(208, 336, 208), (64, 272, 96)])
def test_gemm_mn_major_epilogues(lib, orc, epi, M, N, K):
    A, B = codes(E4M3, (M, K), 23), codes(E4M3, (N, K), 24)
    g = torch.Generator().manual_seed(25)
    aux = u16(torch.randn(M, N, generator=g).to(torch.bfloat16)) if epi == EPI_RELU2_BWD else None
    ia = torch.tensor([0.02], device="cuda")
    ib = torch.tensor([0.5], device="cuda")
    out = []
    for flags in (0, 3):
        D = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        am = torch.zeros(1, device="cuda")
        lib.lm_fp8_gemm_ex(mn_store(A, flags & 1), E4M3, mn_store(B, flags & 2), E4M3, ia, ib, D,
                           flags=flags, epi=epi, aux=None if aux is None else from_u16(aux),
                           amax_out=am)
        out.append((D, am))
    torch.cuda.synchronize()
    assert lib.lm_get_error()[0] == 0
    assert torch.equal(out[0][0].view(torch.int16), out[1][0].view(torch.int16))
    assert torch.equal(out[0][1], out[1][1])
    ref, _ = orc.gemm(A, E4M3, B, E4M3, np.float32(0.02), np.float32(0.5), epi=epi, aux=aux)
    assert_close(u16(out[1][0]), ref, f"mn-major epi={epi} M={M} N={N} K={K}",
                 ELEM_REL_RELU2_BWD if epi == EPI_RELU2_BWD else ELEM_REL)


def test_gemm_k_zero_and_empty(lib, orc):
    D = torch.full((32, 64), 1.0, dtype=torch.bfloat16, device="cuda")
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    A = torch.empty(32, 0, dtype=torch.uint8, device="cuda")
    B = torch.empty(64, 0, dtype=torch.uint8, device="cuda")
    lib.lm_fp8_gemm(A, E4M3, B, E4M3, one, one, D)
    torch.cuda.synchronize()
    assert float(D.float().abs().max()) == 0.0
    E = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    lib.lm_fp8_gemm(torch.empty(0, 16, dtype=torch.uint8, device="cuda"), E4M3,
                    torch.empty(64, 16, dtype=torch.uint8, device="cuda"), E4M3, one, one, E)


def test_gemm_identity_weights_reproduce_dequantised_input(lib, orc):
    """Identity B: D = bf16(dec(A) * inv_a), elementwise exact."""
    K = 256
    A = codes(E4M3, (300, K), 7)
    eye = np.where(np.eye(K, dtype=bool), 0x38, 0x00).astype(np.uint8)
    ia = torch.tensor([0.125], dtype=torch.float32, device="cuda")
    ib = torch.ones(1, dtype=torch.float32, device="cuda")
    D = torch.empty(300, K, dtype=torch.bfloat16, device="cuda")
    lib.lm_fp8_gemm(from_u8(A), E4M3, from_u8(eye), E4M3, ia, ib, D)
    torch.cuda.synchronize()
    want = torch.from_numpy(A).view(torch.float8_e4m3fn).float() * 0.125
    assert torch.equal(D.cpu(), want.to(torch.bfloat16))
