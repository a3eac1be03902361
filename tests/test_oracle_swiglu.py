"""Pins of the oracle's gated (SwiGLU) MLP variant: silu and its derivative
by closed forms and identities, dG and dU by finite differences of silu(G) U,
the fp64 chain's backward by finite differences of its forward, the shared
scale of the gate/up weight, and the FP8 chain against fp64."""
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


def test_silu_closed_forms_and_odd_identity(orc):
    G = np.zeros((2, 128), np.float32)
    G[0, :] = np.linspace(-6, 6, 128)
    U = np.ones((2, 128), np.float32)
    h, amax_h = orc.swiglu_h(bits(G), bits(U))
    hv = vals(h)
    assert np.all(hv[1] == 0.0)                                   # silu(0) = 0
    g = vals(bits(G[0]))
    exact = g / (1.0 + np.exp(-g))
    assert np.array_equal(hv[0], round_bf16(exact))               # one rounding of x*sigma(x)
    assert amax_h == np.float32(np.abs(hv).max())
    hn, _ = orc.swiglu_h(bits(-G), bits(U))
    assert np.allclose(hv[0] - vals(hn)[0], g, atol=2 * 2.0 ** -8 * np.abs(g).max())


def test_h_is_linear_in_u(orc):
    """h = silu(G) U: doubling U doubles h exactly (a power-of-two scale), and a
    negative U flips its sign; G and U are not interchangeable."""
    rng = np.random.default_rng(35)
    G = bits(rng.standard_normal((4, 64)) * 2)
    U = bits(rng.standard_normal((4, 64)))
    h, _ = orc.swiglu_h(G, U)
    h2, _ = orc.swiglu_h(G, bits(vals(U) * 2.0))
    hn, _ = orc.swiglu_h(G, bits(-vals(U)))
    assert np.array_equal(vals(h2), 2.0 * vals(h))
    assert np.array_equal(vals(hn), -vals(h))
    hs, _ = orc.swiglu_h(U, G)
    assert not np.array_equal(hs, h)


def test_silu_derivative_at_zero_and_far_out(orc):
    f = 128
    G = np.zeros((1, f), np.float32)
    G[0, 1], G[0, 2] = 30.0, -30.0
    U = np.full((1, f), 3.0, np.float32)
    g = np.ones((1, f), np.float32)
    dG, dU, amax_d = orc.swiglu_bwd(bits(g), bits(G), bits(U))
    dg, du = vals(dG), vals(dU)
    assert dg[0, 0] == 1.5 and du[0, 0] == 0.0                    # silu'(0) = 1/2, silu(0) = 0
    assert dg[0, 1] == 3.0 and du[0, 1] == 30.0                   # silu'(30) ~ 1, silu(30) ~ 30
    assert abs(dg[0, 2]) < 1e-9 and abs(du[0, 2]) < 1e-9         # silu'(-30), silu(-30) ~ 0
    assert amax_d == np.float32(30.0)                             # the amax spans dG and dU


def test_swiglu_bwd_by_finite_differences_of_h(orc):
    """dG and dU are the partial derivatives of silu(G) U times g: central
    differences of the fp64 silu(G) U at each point, within bf16 rounding."""
    rng = np.random.default_rng(36)
    G = vals(bits(rng.standard_normal((3, 40)) * 3))
    U = vals(bits(rng.standard_normal((3, 40))))
    g = vals(bits(rng.standard_normal((3, 40))))
    dG, dU, _ = orc.swiglu_bwd(bits(g), bits(G), bits(U))
    h = lambda a, b: a / (1.0 + np.exp(-a)) * b
    eps = 1e-6
    fdG = g * (h(G + eps, U) - h(G - eps, U)) / (2 * eps)
    fdU = g * (h(G, U + eps) - h(G, U - eps)) / (2 * eps)
    assert np.all(np.abs(vals(dG) - fdG) <= 2.0 ** -8 * np.abs(fdG) + 1e-8)
    assert np.all(np.abs(vals(dU) - fdU) <= 2.0 ** -8 * np.abs(fdU) + 1e-8)


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


def test_joint_cast_shares_one_scale(orc):
    """Gate and up weights are quantised as one tensor: the amax is the larger
    of the two, and each is cast at that one scale."""
    Wg = synthetic.normal_bf16((128, 64), 0.02, 34, 0)
    Wu = synthetic.normal_bf16((128, 64), 0.5, 34, 1)
    b = synthetic.bits_u16
    j = orc.amax_scale_cast_joint([b(Wg), b(Wu)], orc.E4M3)
    both = orc.amax_scale_cast(np.vstack([b(Wg), b(Wu)]), orc.E4M3)
    assert j["amax"] == both["amax"] == orc.amax(b(Wu))
    assert np.array_equal(np.vstack(j["q"]), both["q"])


def test_fp8_swiglu_chain_within_fp8_error_of_f64(orc):
    M, d, f = 128, 128, 256
    X = synthetic.normal_bf16((M, d), 1.0, 33, 0)
    Wg = synthetic.normal_bf16((f, d), 0.05, 33, 1)
    Wu = synthetic.normal_bf16((f, d), 0.05, 33, 2)
    Wd = synthetic.normal_bf16((d, f), 0.05, 33, 3)
    dY = synthetic.normal_bf16((M, d), 1e-3, 33, 4)
    b = lambda t: synthetic.bits_u16(t)
    fwd = orc.swiglu_fwd(b(X), b(Wg), b(Wu), b(Wd))
    bwd = orc.swiglu_bwd_chain(b(dY), fwd)
    ref = orc.swiglu_f64(*(t.double().numpy() for t in (X, Wg, Wu, Wd, dY)))
    rel = lambda got, r: np.linalg.norm(vals(got) - r) / np.linalg.norm(r)
    assert rel(fwd["Y"], ref["Y"]) < 0.1
    assert rel(bwd["dX"], ref["dX"]) < 0.15
    assert rel(bwd["dW_gate"], ref["dWg"]) < 0.15 and rel(bwd["dW_up"], ref["dWu"]) < 0.15
    assert rel(bwd["dW_down"], ref["dWd"]) < 0.15
    # a swapped gate/up pair is far outside that error
    assert rel(bwd["dW_up"], ref["dWg"]) > 0.5
