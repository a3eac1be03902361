"""GPU parity of the dynamic-scaling cast: amax, scale, inv_scale, the codes
and their transposed copy must equal the oracle's bit for bit."""
import numpy as np
import pytest
import torch

from fp8_gemms_b200 import synthetic
from gpu_util import f32, u8, u16

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1


@pytest.fixture(scope="module")
def api():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import api as a
    return a


def _check_cast(orc, api, x, fmt, relu2=False, want_qT=True):
    q, qT, sc = api.cast(x.cuda(), fmt, relu2_input=relu2, want_qT=want_qT)
    torch.cuda.synchronize()
    ref = orc.amax_scale_cast(u16(x), fmt, relu2_input=relu2)
    assert f32(sc[0]) == ref["amax"]
    assert f32(sc[1]) == ref["scale"]
    assert f32(sc[2]) == ref["inv_scale"]
    assert np.array_equal(u8(q), ref["q"])
    if want_qT:
        assert np.array_equal(u8(qT), ref["qT"])
    from fp8_gemms_b200 import _lib
    assert _lib.lm_get_error()[0] == 0


# shapes: full tiles, ragged rows (not a multiple of 256), ragged columns (not
# a multiple of 128), a single 16 x 16 block, and a tall/wide pair
SHAPES = [(256, 128), (512, 384), (272, 144), (16, 16), (48, 1040), (1040, 48)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_cast_bit_exact(orc, api, shape, fmt):
    x = synthetic.normal_bf16(shape, 1.0 if fmt == E4M3 else 1e-3, 40, shape[0] + fmt)
    _check_cast(orc, api, x, fmt)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_cast_relu2_input_bit_exact(orc, api, fmt):
    x = synthetic.student_t3_bf16((272, 400), 41, fmt)
    _check_cast(orc, api, x, fmt, relu2=True)


def test_cast_heavy_tails_and_ties(orc, api):
    """t3 outliers stress the tensorwise amax; values on FP8 rounding ties."""
    x = synthetic.student_t3_bf16((512, 256), 42, 0)
    _check_cast(orc, api, x, E4M3)
    # every bf16 value that is an exact e4m3 midpoint at scale 1 (amax 448)
    mids = []
    codes = torch.arange(0, 0x7E, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
    for a, b in zip(codes[:-1], codes[1:]):
        mids.append((a + b) / 2)
    v = torch.tensor(mids + [448.0], dtype=torch.float32)
    v = torch.cat([v, -v]).to(torch.bfloat16)
    x = torch.zeros(16, 256, dtype=torch.bfloat16)
    x.view(-1)[: v.numel()] = v
    _check_cast(orc, api, x, E4M3)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("relu2", [False, True])
def test_cast_row_major_only_bit_exact(orc, api, shape, relu2):
    """qT not requested: the TMA-fed kernel without its transpose stage (the
    blocks' casts, whose codes the GEMMs read MN-major where needed)."""
    x = synthetic.student_t3_bf16(shape, 44, int(relu2))
    _check_cast(orc, api, x, E5M2 if relu2 else E4M3, relu2=relu2, want_qT=False)


def _is_nan_code(c, fmt):
    c = np.asarray(c) & 0x7F
    return c == 0x7F if fmt == E4M3 else c > 0x7C


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
@pytest.mark.parametrize("amax", [1.0, 2.0 ** -20, 2.0 ** 40])
@pytest.mark.parametrize("want_qT", [False, True])
def test_cast_relu2_every_bf16_pattern(orc, api, fmt, amax, want_qT):
    """h = bf16(relu(x)^2) then the scaled cast, over all 65,536 bf16 bit
    patterns (zeros of both signs, subnormals, every rounding tie of a square,
    overflow to infinity, infinities, NaNs) with the amax supplied: codes equal
    the oracle's bit for bit; a NaN input gives a NaN code on both sides."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(4096, 16)
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    am = torch.tensor([amax], dtype=torch.float32, device="cuda")
    sc = torch.zeros(4, device="cuda")
    q = torch.empty(4096, 16, dtype=torch.uint8, device="cuda")
    qT = torch.empty(16, 4096, dtype=torch.uint8, device="cuda") if want_qT else None
    from fp8_gemms_b200 import _lib
    _lib.lm_fp8_amax_scale_cast(x.cuda(), fmt, sc[0:1], sc[1:2], sc[2:3], q, qT,
                                relu2_input=True, amax_in=am)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    s, inv = orc.scale(np.float32(amax), fmt)
    assert f32(sc[1:2]) == s and f32(sc[2:3]) == inv
    ref, refT = orc.cast(bits, fmt, s, relu2_input=True)
    for got, want in [(u8(q), ref)] + ([(u8(qT), refT)] if want_qT else []):
        nan = _is_nan_code(want, fmt)
        assert np.array_equal(_is_nan_code(got, fmt), nan)
        assert np.array_equal(got[~nan], want[~nan])


def test_cast_relu2_amax_pass_over_finite_patterns(orc, api):
    """The reduction pass of a relu^2 cast (no amax supplied) over every finite
    bf16 pattern whose square stays finite: amax, scale and codes bit-exact."""
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mag = b & 0x7FFF
    b = b[mag < 0x5F00]  # |x| < 2^63: finite squares, no NaN or infinity
    b = b[: (b.size // 16) * 16].reshape(-1, 16)
    x = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)
    _check_cast(orc, api, x, E4M3, relu2=True, want_qT=b.shape[0] % 16 == 0)


def test_cast_without_transpose_and_ragged_rows(orc, api):
    x = synthetic.normal_bf16((200, 96), 2.0, 43, 0)  # rows % 16 != 0: q only
    _check_cast(orc, api, x, E4M3, want_qT=False)


def test_cast_strided_input_and_amax_in(orc, api):
    from fp8_gemms_b200 import _lib
    big = synthetic.normal_bf16((64, 320), 1.0, 44, 0)
    x = big[:, :256]  # ld = 320
    ref = orc.amax_scale_cast(u16(x.contiguous()), E4M3)
    xd = big.cuda()[:, :256]
    sc = torch.zeros(4, dtype=torch.float32, device="cuda")
    q = torch.empty(64, 256, dtype=torch.uint8, device="cuda")
    qT = torch.empty(256, 64, dtype=torch.uint8, device="cuda")
    _lib.lm_fp8_amax_scale_cast(xd, E4M3, sc[0:1], sc[1:2], sc[2:3], q, qT)
    torch.cuda.synchronize()
    assert f32(sc[0]) == ref["amax"] and f32(sc[1]) == ref["scale"]
    assert np.array_equal(u8(q), ref["q"]) and np.array_equal(u8(qT), ref["qT"])
    # a supplied amax skips the reduction pass and is used as given
    amax_in = torch.tensor([3.5], dtype=torch.float32, device="cuda")
    _lib.lm_fp8_amax_scale_cast(xd, E4M3, sc[0:1], sc[1:2], sc[2:3], q, qT, amax_in=amax_in)
    torch.cuda.synchronize()
    s, inv = orc.scale(np.float32(3.5), E4M3)
    q_ref, qT_ref = orc.cast(u16(x.contiguous()), E4M3, s)
    assert f32(sc[0]) == np.float32(3.5) and f32(sc[1]) == s and f32(sc[2]) == inv
    assert np.array_equal(u8(q), q_ref) and np.array_equal(u8(qT), qT_ref)


def test_cast_empty_and_zero(orc, api):
    from fp8_gemms_b200 import _lib
    sc = torch.full((4,), 7.0, dtype=torch.float32, device="cuda")
    x = torch.empty(0, 32, dtype=torch.bfloat16, device="cuda")
    _lib.lm_fp8_amax_scale_cast(x, E4M3, sc[0:1], sc[1:2], sc[2:3], None, None)
    torch.cuda.synchronize()
    s, inv = orc.scale(np.float32(0.0), E4M3)
    assert f32(sc[0]) == 0.0 and f32(sc[1]) == s and f32(sc[2]) == inv
    _check_cast(orc, api, torch.zeros(32, 32, dtype=torch.bfloat16), E4M3)
