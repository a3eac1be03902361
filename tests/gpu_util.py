"""Helpers shared by the GPU parity tests: moving bits between the CUDA path
(torch tensors) and the oracle (numpy arrays), and the tolerance check."""
import numpy as np
import torch

# GEMM / MLP outputs (bf16): elementwise |d| <= 1e-2 |ref| + 1e-3 rms(ref),
# and normwise ||d||_F / ||ref||_F <= 5e-3.
ELEM_REL, ELEM_RMS, NORM_REL = 1e-2, 1e-3, 5e-3
# The relu^2-backward epilogue rounds twice: g = bf16(acc s), then
# dH = bf16(g * 2 relu(H)).  fp32 tensor-core accumulation and the oracle's
# fp64 sum can put g one bf16 ulp apart; the second rounding can then leave
# dH two ulps apart, i.e. up to 2 * 2^-7 = 2^-6 of |dH|.  Elementwise bound for
# that epilogue's output: 2^-6 |ref| + 1e-3 rms(ref) (normwise bound unchanged).
ELEM_REL_RELU2_BWD = 2.0 ** -6


def u16(t):
    """bf16 tensor (any device) -> numpy uint16 bits."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def u8(t):
    return t.detach().contiguous().cpu().numpy()


def bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def from_u8(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def from_u16(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def f32(t):
    """A one-element fp32 device tensor -> numpy float32 (bit-exact)."""
    return np.float32(t.detach().cpu().numpy().reshape(-1)[0])


def assert_close(got_bits, ref_bits, what="", elem_rel=ELEM_REL):
    g = bf16_to_f64(got_bits)
    r = bf16_to_f64(ref_bits)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    if r.size == 0:
        return
    rms = float(np.sqrt(np.mean(r * r)))
    d = np.abs(g - r)
    bound = elem_rel * np.abs(r) + ELEM_RMS * rms
    bad = d > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; "
                           f"worst |d|={d.max():.3e} at {np.unravel_index(d.argmax(), d.shape)}, "
                           f"rms(ref)={rms:.3e}")
    nr = np.linalg.norm(r)
    if nr > 0:
        assert np.linalg.norm(g - r) / nr <= NORM_REL, f"{what}: normwise {np.linalg.norm(g - r) / nr:.3e}"


def cast_ref(orc, bits, fmt, relu2_input=False, amax_in=None):
    """The oracle's dynamic cast of a whole tensor, row-major codes only:
    dict(amax, scale, inv_scale, q)."""
    a = orc.amax(bits, relu2_input) if amax_in is None else np.float32(amax_in)
    s, inv = orc.scale(a, fmt)
    q, _ = orc.cast(bits, fmt, s, relu2_input, want_qT=False)
    return dict(amax=a, scale=s, inv_scale=inv, q=q)


def bf16_neighbours(bits):
    """The bf16 values one ulp below and above each value (bits, same shape)."""
    b = np.asarray(bits, np.uint16).astype(np.int32)
    mag, neg = b & 0x7FFF, (b & 0x8000) != 0
    up_mag = np.minimum(mag + 1, 0x7F7F)
    dn_mag = np.where(mag == 0, 1, mag - 1)       # below +-0 is the smallest subnormal
    dn_neg = np.where(mag == 0, ~neg, neg)
    toward_big = np.where(neg, up_mag | 0x8000, up_mag)
    toward_small = np.where(dn_neg, dn_mag | 0x8000, dn_mag)
    return toward_small.astype(np.uint16), toward_big.astype(np.uint16)


def assert_close_f32(got, ref, what=""):
    """The same tolerance for fp32 results (numpy arrays)."""
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    rms = float(np.sqrt(np.mean(r * r)))
    d = np.abs(g - r)
    bad = d > ELEM_REL * np.abs(r) + ELEM_RMS * rms
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} out of tolerance, "
                           f"worst {d.max():.3e}, rms {rms:.3e}")
    nr = np.linalg.norm(r)
    if nr > 0:
        assert np.linalg.norm(g - r) / nr <= NORM_REL, what
