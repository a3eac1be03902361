"""Pins of the oracle's FP8 GEMM, its epilogues and the relu^2 MLP chain.

  * brute force: exact rational sums (Python Fractions over PyTorch-decoded
    FP8 values) against the oracle's fp64 accumulation;
  * identity and one-hot weights reproduce the dequantised input;
  * the relu^2 epilogues against their plain elementwise definitions;
  * the fp64 chain's backward against central finite differences of its
    forward (catches a transposed or swapped operand in the dgrad/wgrad
    wiring), and the FP8 chain against the fp64 chain within FP8 error.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from fp8_gemms_b200 import synthetic

E4M3, E5M2 = 0, 1
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def finite_codes(fmt, rng, shape, lo=None, hi=None):
    vals = torch.arange(256, dtype=torch.uint8).view(TORCH_DT[fmt]).float().numpy()
    ok = np.isfinite(vals)
    if lo is not None:
        ok &= (np.abs(vals) >= lo) & (np.abs(vals) <= hi)
    pool = np.nonzero(ok)[0].astype(np.uint8)
    return rng.choice(pool, size=shape)


def tdecode(codes, fmt):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(TORCH_DT[fmt]).double().numpy()


def round_bf16_np(x):
    """RNE to bf16 of float64 values (normal range), via frexp + rint."""
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def bf16_vals(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("fa", [E4M3, E5M2])
def test_gemm_acc_exact_vs_fractions(orc, fa):
    rng = np.random.default_rng(21 + fa)
    M, N, K = 5, 7, 48
    # restricted magnitudes: every partial sum is exact in fp64
    A = finite_codes(fa, rng, (M, K), 2.0 ** -4, 2.0 ** 4)
    B = finite_codes(E4M3, rng, (N, K), 2.0 ** -4, 2.0 ** 4)
    C = orc.gemm_acc(A, fa, B, E4M3)
    da, db = tdecode(A, fa), tdecode(B, E4M3)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(da[m, k])) * Fraction(float(db[n, k])) for k in range(K))
            assert Fraction(C[m, n]) == exact
    # full range: within the fp64 summation bound of the exact value
    A = finite_codes(fa, rng, (M, K))
    B = finite_codes(E4M3, rng, (N, K))
    C = orc.gemm_acc(A, fa, B, E4M3)
    da, db = tdecode(A, fa), tdecode(B, E4M3)
    for m in range(M):
        for n in range(N):
            terms = [Fraction(float(da[m, k])) * Fraction(float(db[n, k])) for k in range(K)]
            exact = sum(terms)
            bound = K * 2.0 ** -52 * float(sum(abs(t) for t in terms))
            assert abs(float(Fraction(C[m, n]) - exact)) <= bound
    # the row-subset form returns the same rows
    rows = [4, 0, 2]
    assert np.array_equal(orc.gemm_acc(A, fa, B, E4M3, rows=rows), C[rows])


def test_gemm_bf16_output_is_one_rounding(orc):
    rng = np.random.default_rng(5)
    M, N, K = 9, 11, 64
    A = finite_codes(E5M2, rng, (M, K))
    B = finite_codes(E4M3, rng, (N, K))
    inv_a, inv_b = np.float32(2.0 ** -7), np.float32(2.0 ** 3)  # powers of 2: exact
    D, amax = orc.gemm(A, E5M2, B, E4M3, inv_a, inv_b)
    exact = tdecode(A, E5M2) @ tdecode(B, E4M3).T * float(inv_a) * float(inv_b)
    assert np.array_equal(bf16_vals(D), round_bf16_np(exact))
    assert amax == np.float32(np.abs(bf16_vals(D)).max())


def test_identity_and_one_hot_weights_reproduce_quantised_input(orc):
    x = synthetic.normal_bf16((40, 64), 1.0, 3, 0)
    cx = orc.amax_scale_cast(synthetic.bits_u16(x), E4M3)
    deq = tdecode(cx["q"], E4M3) * float(cx["inv_scale"])
    eye = np.where(np.eye(64, dtype=bool), 0x38, 0x00).astype(np.uint8)  # e4m3 1.0
    D, _ = orc.gemm(cx["q"], E4M3, eye, E4M3, cx["inv_scale"], np.float32(1.0))
    assert np.array_equal(bf16_vals(D), round_bf16_np(deq))
    # and the dequantised input is within e4m3 precision of x itself
    xf = x.double().numpy()
    big = np.abs(xf) > 2.0 ** -6 * float(cx["amax"]) / 448 * 64
    assert np.all(np.abs(deq[big] - xf[big]) <= np.abs(xf[big]) * 2.0 ** -4)
    # one-hot rows pick one input column each, times a power-of-two weight
    rng = np.random.default_rng(8)
    pick = rng.integers(0, 64, 24)
    wcode = rng.choice(np.array([0x30, 0x38, 0x40, 0xB8], np.uint8), 24)  # .25 1 4 -1
    onehot = np.zeros((24, 64), np.uint8)
    onehot[np.arange(24), pick] = wcode
    D, _ = orc.gemm(cx["q"], E4M3, onehot, E4M3, cx["inv_scale"], np.float32(0.5))
    want = deq[:, pick] * tdecode(wcode, E4M3)[None, :] * 0.5
    assert np.array_equal(bf16_vals(D), round_bf16_np(want))


def test_relu2_epilogues_match_elementwise_definitions(orc):
    rng = np.random.default_rng(13)
    M, N, K = 12, 20, 32
    A = finite_codes(E4M3, rng, (M, K), 2.0 ** -3, 8.0)
    B = finite_codes(E4M3, rng, (N, K), 2.0 ** -3, 8.0)
    inv = np.float32(0.01)
    Hn, amax_n = orc.gemm(A, E4M3, B, E4M3, inv, inv)
    H, amax_h = orc.gemm(A, E4M3, B, E4M3, inv, inv, epi=orc.EPI_RELU2_FWD)
    assert np.array_equal(H, Hn)
    Ht = torch.from_numpy(H.view(np.int16)).view(torch.bfloat16).float()
    h = (torch.relu(Ht) ** 2).to(torch.bfloat16)   # exact square, one rounding
    assert amax_h == np.float32(h.float().max().item())
    assert amax_n == np.float32(Ht.abs().max().item())
    # backward: dH = bf16(g * 2 * relu(H)) with g = bf16 of the dgrad GEMM
    G = finite_codes(E5M2, rng, (M, K))
    Wt = finite_codes(E4M3, rng, (N, K))
    g, _ = orc.gemm(G, E5M2, Wt, E4M3, np.float32(1e-3), np.float32(0.05))
    dH, amax_dh = orc.gemm(G, E5M2, Wt, E4M3, np.float32(1e-3), np.float32(0.05),
                           epi=orc.EPI_RELU2_BWD, aux=H)
    gt = torch.from_numpy(g.view(np.int16)).view(torch.bfloat16).float()
    ref = (gt * 2.0 * torch.relu(Ht)).to(torch.bfloat16)  # exact product, one rounding
    assert np.array_equal(dH, synthetic.bits_u16(ref))
    assert amax_dh == np.float32(ref.float().abs().max().item())


def test_relu2_backward_epilogue_is_the_derivative_of_relu2(orc):
    """With the dgrad GEMM's value g = 1 exactly (one-hot codes of 1.0, unit
    scales), the oracle's relu^2 backward epilogue returns d/dH relu(H)^2 at
    every saved H: central differences of relu(x)^2 in fp64 at the same
    points (away from the kink), to 1e-6."""
    rng = np.random.default_rng(17)
    M, N, K = 4, 64, 16
    H = synthetic.bits_u16(torch.tensor(rng.uniform(-3, 3, (M, N)), dtype=torch.float32)
                           .to(torch.bfloat16))
    Hv = (H.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.min(np.abs(Hv)) > 1e-3
    A = np.zeros((M, K), np.uint8)
    B = np.zeros((N, K), np.uint8)
    A[:, 0] = orc.fp8_encode(1.0, E5M2)
    B[:, 0] = orc.fp8_encode(1.0, E4M3)
    dH, _ = orc.gemm(A, E5M2, B, E4M3, np.float32(1.0), np.float32(1.0),
                     epi=orc.EPI_RELU2_BWD, aux=H)
    got = (dH.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    eps = 1e-6
    f = lambda t: np.maximum(t, 0.0) ** 2
    fd = (f(Hv + eps) - f(Hv - eps)) / (2 * eps)
    assert np.all(np.abs(got - fd) <= 1e-6 * np.maximum(1.0, np.abs(fd)))


def test_f64_chain_backward_by_finite_differences(orc):
    rng = np.random.default_rng(19)
    M, d, f = 4, 6, 10
    X = rng.standard_normal((M, d))
    Wu = rng.standard_normal((f, d)) * 0.5
    Wd = rng.standard_normal((d, f)) * 0.5
    dY = rng.standard_normal((M, d))
    out = orc.mlp_f64(X, Wu, Wd, dY)
    loss = lambda X_, Wu_, Wd_: float((orc.mlp_f64(X_, Wu_, Wd_)["Y"] * dY).sum())
    H = X @ Wu.T
    assert np.min(np.abs(H)) > 1e-4  # no point within eps*|W| of the relu kink
    eps = 1e-6
    for name, arr, grad in [("X", X, out["dX"]), ("W_up", Wu, out["dW_up"]),
                            ("W_down", Wd, out["dW_down"])]:
        for idx in np.ndindex(arr.shape):
            p, m = arr.copy(), arr.copy()
            p[idx] += eps
            m[idx] -= eps
            args = {"X": (X, Wu, Wd), "W_up": (X, Wu, Wd), "W_down": (X, Wu, Wd)}[name]
            ap = [a if a is not arr else p for a in args]
            am = [a if a is not arr else m for a in args]
            fd = (loss(*ap) - loss(*am)) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx)
    # forward against a plain numpy composition
    Yref = (np.maximum(H, 0) ** 2) @ Wd.T
    assert np.allclose(out["Y"], Yref, rtol=1e-12, atol=1e-12)


def test_fp8_chain_within_fp8_error_of_f64_chain(orc):
    """Tiny relu^2 MLP block: the quantised chain approaches the unquantised
    one within FP8 error (a sanity bound, not parity)."""
    w = synthetic.TINY_MLP
    t = w.tensors()
    b = {k: synthetic.bits_u16(v) for k, v in t.items()}
    fwd = orc.mlp_fwd(b["X"], b["W_up"], b["W_down"])
    bwd = orc.mlp_bwd(b["dY"], fwd)
    ref = orc.mlp_f64(t["X"].double().numpy(), t["W_up"].double().numpy(),
                      t["W_down"].double().numpy(), t["dY"].double().numpy())

    def rel(bits, r):
        v = bf16_vals(bits)
        return np.linalg.norm(v - r) / np.linalg.norm(r)

    assert rel(fwd["Y"], ref["Y"]) < 0.08
    assert rel(bwd["dX"], ref["dX"]) < 0.15
    assert rel(bwd["dW_up"], ref["dW_up"]) < 0.15
    assert rel(bwd["dW_down"], ref["dW_down"]) < 0.15
    # and the backward reuses the forward's quantised operands and scales
    assert fwd["h"]["amax"] == np.float32(
        torch.relu(torch.from_numpy(fwd["H"].view(np.int16)).view(torch.bfloat16).float())
        .pow(2).to(torch.bfloat16).float().max().item())


def test_accumulating_gemm_adds_one_fp32_rounding_per_call(orc):
    """Gradient accumulation: D += fp32(C * inv_sa * inv_sb), one fp32 addition
    per call.  Pinned against exact products rounded by numpy's float32."""
    rng = np.random.default_rng(29)
    M, N, K = 7, 9, 48
    A = finite_codes(E5M2, rng, (M, K))
    B = finite_codes(E4M3, rng, (N, K))
    inv_a, inv_b = np.float32(2.0 ** -10), np.float32(0.25)   # powers of two: exact in fp64
    exact = tdecode(A, E5M2) @ tdecode(B, E4M3).T * float(inv_a) * float(inv_b)
    D = np.zeros((M, N), np.float32)
    orc.gemm_accum_f32(A, E5M2, B, E4M3, inv_a, inv_b, D)
    assert np.array_equal(D, exact.astype(np.float32))       # 0 + x = x: one rounding
    D0 = rng.standard_normal((M, N)).astype(np.float32)
    D = D0.copy()
    orc.gemm_accum_f32(A, E5M2, B, E4M3, inv_a, inv_b, D)
    assert np.array_equal(D, D0 + exact.astype(np.float32))   # numpy float32 add
    # a row subset touches only its own rows
    rows = [6, 1]
    Dr = D0[rows].copy()
    orc.gemm_accum_f32(A, E5M2, B, E4M3, inv_a, inv_b, Dr, rows=rows)
    assert np.array_equal(Dr, D0[rows] + exact[rows].astype(np.float32))


def test_grad_accum_chain_matches_sum_of_per_micro_batch_gradients(orc):
    """Accumulating two micro-batches equals the float32 sum of the two
    single-micro-batch wgrads computed with the same (reused) weight casts."""
    from fp8_gemms_b200 import synthetic
    w = synthetic.MlpWorkload("ga", 64, 64, 256, True)
    t = w.tensors()
    b = {k: synthetic.bits_u16(v) for k, v in t.items()}
    X2 = synthetic.bits_u16(synthetic.normal_bf16((64, 64), 1.0, 77, 0))
    dY2 = synthetic.bits_u16(synthetic.normal_bf16((64, 64), 1e-3, 77, 1))
    outs, dWu, dWd = orc.mlp_grad_accum([(b["X"], b["dY"]), (X2, dY2)], b["W_up"], b["W_down"])
    singles = [orc.mlp_grad_accum([mb], b["W_up"], b["W_down"]) for mb in
               [(b["X"], b["dY"]), (X2, dY2)]]
    assert np.array_equal(dWu, singles[0][1] + singles[1][1])
    assert np.array_equal(dWd, singles[0][2] + singles[1][2])
    # and each micro-batch's Y and dX equal the plain chain's
    fwd = orc.mlp_fwd(b["X"], b["W_up"], b["W_down"])
    bwd = orc.mlp_bwd(b["dY"], fwd)
    assert np.array_equal(outs[0][0], fwd["Y"]) and np.array_equal(outs[0][1], bwd["dX"])
    # the fp32 accumulator of one micro-batch equals the bf16 chain's wgrad to bf16 rounding
    dWu_bf = bf16_vals(bwd["dW_up"])
    assert np.all(np.abs(singles[0][1] - dWu_bf) <= 2.0 ** -8 * np.abs(dWu_bf) + 1e-30)


def test_fp8_linear_within_fp8_error_of_f64(orc):
    """The plain FP8 linear (forward, dgrad, wgrad) approaches the exact
    Y = X W^T, dX = dY W, dW = dY^T X within FP8 error; a transposed or
    swapped operand lands far outside it."""
    M, K, N = 96, 128, 80
    X = synthetic.normal_bf16((M, K), 1.0, 47, 0)
    W = synthetic.normal_bf16((N, K), 0.02, 47, 1)
    dY = synthetic.normal_bf16((M, N), 1e-3, 47, 2)
    out = orc.linear_fwd_bwd(*(synthetic.bits_u16(t) for t in (X, W, dY)))
    x, w, g = (t.double().numpy() for t in (X, W, dY))
    v = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    rel = lambda got, r: np.linalg.norm(v(got) - r) / np.linalg.norm(r)
    assert rel(out["Y"], x @ w.T) < 0.08
    assert rel(out["dX"], g @ w) < 0.15
    assert rel(out["dW"], g.T @ x) < 0.15
    assert rel(out["dW"], (g.T @ x)[::-1]) > 0.5
