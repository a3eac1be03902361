"""Helpers shared by the GPU parity tests: moving bits between the CUDA path
(torch tensors) and the oracle (numpy arrays), and the tolerance check."""
import numpy as np
import torch

# GEMM / MLP outputs (bf16): elementwise |d| <= 1e-2 |ref| + 1e-3 rms(ref),
# and normwise ||d||_F / ||ref||_F <= 5e-3.
ELEM_REL, ELEM_RMS, NORM_REL = 1e-2, 1e-3, 5e-3


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


def assert_close(got_bits, ref_bits, what=""):
    g = bf16_to_f64(got_bits)
    r = bf16_to_f64(ref_bits)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    if r.size == 0:
        return
    rms = float(np.sqrt(np.mean(r * r)))
    d = np.abs(g - r)
    bound = ELEM_REL * np.abs(r) + ELEM_RMS * rms
    bad = d > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; "
                           f"worst |d|={d.max():.3e} at {np.unravel_index(d.argmax(), d.shape)}, "
                           f"rms(ref)={rms:.3e}")
    nr = np.linalg.norm(r)
    if nr > 0:
        assert np.linalg.norm(g - r) / nr <= NORM_REL, f"{what}: normwise {np.linalg.norm(g - r) / nr:.3e}"
