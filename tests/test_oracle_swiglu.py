"""Pins of the oracle's gated (SwiGLU) MLP variant: silu and its derivative
by closed forms and identities, the fp64 chain's backward by finite
differences, the gate/up interleaving, and the FP8 chain against fp64."""
import numpy as np
import torch

from fp8_gemms_b200 import synthetic


def vals(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bits(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def round_bf16(x):
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def gu_of(G, U):
    """Interleave G, U ([M x f] each) into the GU layout (blocks of 128)."""
    M, f = G.shape
    GU = np.empty((M, 2 * f), G.dtype)
    for b in range(f // 128):
        GU[:, 256 * b:256 * b + 128] = G[:, 128 * b:128 * b + 128]
        GU[:, 256 * b + 128:256 * b + 256] = U[:, 128 * b:128 * b + 128]
    return GU


def test_silu_closed_forms_and_odd_identity(orc):
    G = np.zeros((2, 128), np.float32)
    G[0, :] = np.linspace(-6, 6, 128)
    U = np.ones((2, 128), np.float32)
    h, _ = orc.swiglu_h(gu_of(bits(G), bits(U)))
    hv = vals(h)
    assert np.all(hv[1] == 0.0)                                   # silu(0) = 0
    g = vals(bits(G[0]))
    exact = g / (1.0 + np.exp(-g))
    assert np.array_equal(hv[0], round_bf16(exact))               # one rounding of x*sigma(x)
    hn, _ = orc.swiglu_h(gu_of(bits(-G), bits(U)))
    assert np.allclose(hv[0] - vals(hn)[0], g, atol=2 * 2.0 ** -8 * np.abs(g).max())


def test_silu_derivative_at_zero_and_far_out(orc):
    f = 128
    G = np.zeros((1, f), np.float32)
    G[0, 1], G[0, 2] = 30.0, -30.0
    U = np.full((1, f), 3.0, np.float32)
    g = np.ones((1, f), np.float32)
    dGU, _ = orc.swiglu_bwd(bits(g), gu_of(bits(G), bits(U)))
    d = vals(dGU)
    assert d[0, 0] == 1.5 and d[0, 128] == 0.0                    # silu'(0) = 1/2, silu(0) = 0
    assert d[0, 1] == 3.0 and d[0, 129] == 30.0                   # silu'(30) ~ 1, silu(30) ~ 30
    assert abs(d[0, 2]) < 1e-9 and abs(d[0, 130]) < 1e-9         # silu'(-30), silu(-30) ~ 0


def test_swiglu_f64_backward_by_finite_differences(orc):
    rng = np.random.default_rng(31)
    M, d, f = 3, 5, 7
    X = rng.standard_normal((M, d))
    Wg, Wu = rng.standard_normal((f, d)), rng.standard_normal((f, d))
    Wd = rng.standard_normal((d, f))
    dY = rng.standard_normal((M, d))
    out = orc.swiglu_f64(X, Wg, Wu, Wd, dY)
    loss = lambda a: float((orc.swiglu_f64(*a)["Y"] * dY).sum())
    base = [X, Wg, Wu, Wd]
    eps = 1e-6
    for i, key in enumerate(["dX", "dWg", "dWu", "dWd"]):
        for idx in np.ndindex(base[i].shape):
            p = [a.copy() for a in base]
            m = [a.copy() for a in base]
            p[i][idx] += eps
            m[i][idx] -= eps
            fd = (loss(p) - loss(m)) / (2 * eps)
            assert abs(fd - out[key][idx]) <= 1e-6 * max(1.0, abs(fd)), (key, idx)


def test_interleave_round_trip(orc):
    Wg = np.arange(256 * 3).reshape(256, 3)
    Wu = -np.arange(256 * 3).reshape(256, 3)
    Wgu = orc.interleave_gate_up(Wg, Wu)
    assert np.array_equal(Wgu[0:128], Wg[0:128]) and np.array_equal(Wgu[128:256], Wu[0:128])
    g2, u2 = orc.deinterleave_gate_up(Wgu)
    assert np.array_equal(g2, Wg) and np.array_equal(u2, Wu)


def test_fp8_swiglu_chain_within_fp8_error_of_f64(orc):
    M, d, f = 128, 128, 256
    X = synthetic.normal_bf16((M, d), 1.0, 33, 0)
    Wg = synthetic.normal_bf16((f, d), 0.05, 33, 1)
    Wu = synthetic.normal_bf16((f, d), 0.05, 33, 2)
    Wd = synthetic.normal_bf16((d, f), 0.05, 33, 3)
    dY = synthetic.normal_bf16((M, d), 1e-3, 33, 4)
    b = lambda t: synthetic.bits_u16(t)
    fwd = orc.swiglu_fwd(b(X), orc.interleave_gate_up(b(Wg), b(Wu)), b(Wd))
    bwd = orc.swiglu_bwd_chain(b(dY), fwd)
    ref = orc.swiglu_f64(*(t.double().numpy() for t in (X, Wg, Wu, Wd, dY)))
    dWg, dWu = orc.deinterleave_gate_up(bwd["dW_gu"])
    rel = lambda got, r: np.linalg.norm(vals(got) - r) / np.linalg.norm(r)
    assert rel(fwd["Y"], ref["Y"]) < 0.1
    assert rel(bwd["dX"], ref["dX"]) < 0.15
    assert rel(dWg, ref["dWg"]) < 0.15 and rel(dWu, ref["dWu"]) < 0.15
    assert rel(bwd["dW_down"], ref["dWd"]) < 0.15
