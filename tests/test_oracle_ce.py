"""Pins of the oracle's softcapped cross-entropy (the LM head's loss)."""
import numpy as np
import torch


def bits(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def vals(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_uniform_logits_give_log_v(orc):
    V = 512
    loss, dl = orc.softcap_ce(bits(np.zeros((3, V))), [0, 7, 511], inv_count=1.0)
    assert np.allclose(loss, np.log(V), rtol=0, atol=1e-12)
    d = vals(dl)
    # softmax = 1/V everywhere, minus one at the label; tanh'(0) = 1
    assert d[1, 7] == vals(bits(1.0 / V - 1.0)) and d[1, 8] == vals(bits(1.0 / V))


def test_softcap_bounds_the_logits(orc):
    """z = c tanh(l/c) never exceeds c: a huge correct logit still costs
    log(1 + (V-1) e^{-c}) at c = 15, not ~0."""
    V, c = 64, 15.0
    l = np.zeros((1, V))
    l[0, 3] = 1e4
    loss, _ = orc.softcap_ce(bits(l), [3], softcap=c)
    assert abs(loss[0] - np.log1p((V - 1) * np.exp(-c))) < 1e-12


def test_ce_gradient_by_finite_differences(orc):
    """dloss/dl = (softmax(z) - onehot) * (1 - (z/c)^2): checked by central
    differences of the fp64 loss on logits exactly representable in bf16."""
    rng = np.random.default_rng(41)
    V, c = 96, 15.0
    lv = vals(bits(rng.standard_normal(V) * 8.0))
    label = 17

    def loss_f(x):
        z = c * np.tanh(x / c)
        m = z.max()
        return m + np.log(np.exp(z - m).sum()) - z[label]

    loss, dl = orc.softcap_ce(bits(lv[None]), [label], softcap=c, inv_count=1.0)
    assert abs(loss[0] - loss_f(lv)) < 1e-12
    eps = 1e-4   # truncation ~eps^2, cancellation ~1e-16 / eps: both far below 1e-8
    for v in range(V):
        p, m = lv.copy(), lv.copy()
        p[v] += eps
        m[v] -= eps
        fd = (loss_f(p) - loss_f(m)) / (2 * eps)
        assert abs(vals(dl)[0, v] - fd) <= 2.0 ** -8 * abs(fd) + 1e-8


def test_chunked_lm_head_is_chunk_independent_in_loss(orc):
    """Chunking changes no per-token loss (X and W carry whole-tensor scales)."""
    from fp8_gemms_b200 import synthetic
    M, d, V = 64, 64, 320
    X = synthetic.bits_u16(synthetic.normal_bf16((M, d), 1.0, 43, 0))
    W = synthetic.bits_u16(synthetic.normal_bf16((V, d), 0.02, 43, 1))
    labels = np.random.default_rng(43).integers(0, V, M).astype(np.int32)
    l1, dX1, dW1, r1 = orc.lmhead_ce(X, W, labels, chunk=M)
    l2, dX2, dW2, r2 = orc.lmhead_ce(X, W, labels, chunk=16)
    assert np.array_equal(r1, r2) and l1 == l2
    assert np.allclose(dW1, dW2, rtol=1e-5, atol=1e-9)


def test_lmhead_f64_gradient_by_finite_differences(orc):
    """The fp64 LM head + softcapped CE: dX and dW equal central differences
    of its mean loss in every entry.  Logits reach |l| ~ 20, so the softcap's
    derivative 1 - (z/c)^2 is far from 1 and a dropped factor would show; a
    transposed dW or a missing 1/M would too."""
    rng = np.random.default_rng(44)
    M, d, V, c = 5, 6, 9, 15.0
    X = rng.standard_normal((M, d)) * 3.0
    W = rng.standard_normal((V, d))
    labels = rng.integers(0, V, M).astype(np.int32)
    loss, dX, dW = orc.lmhead_ce_f64(X, W, labels, softcap=c)
    z = c * np.tanh((X @ W.T) / c)
    assert np.abs(z).max() > 0.5 * c
    eps = 1e-6
    f = lambda X_, W_: orc.lmhead_ce_f64(X_, W_, labels, softcap=c, want_grad=False)[0]
    for name, arr, grad in (("X", X, dX), ("W", W, dW)):
        for idx in np.ndindex(arr.shape):
            p, m = arr.copy(), arr.copy()
            p[idx] += eps
            m[idx] -= eps
            fd = (f(p, W) - f(m, W)) / (2 * eps) if name == "X" else (f(X, p) - f(X, m)) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-7 * max(1.0, abs(fd)), (name, idx)
    # the loss itself: the definition written out with numpy, row by row
    lse = np.log(np.exp(z).sum(axis=1))
    assert abs(loss - float(np.mean(lse - z[np.arange(M), labels]))) < 1e-12


def test_fp8_lmhead_within_fp8_error_of_f64(orc):
    """The FP8 chunked head (X, W e4m3 with whole-tensor scales; per-chunk
    e5m2 dlogits) approaches the unquantised fp64 head within FP8 error: a
    sanity bound, not parity.  A wrong chunk offset, a transposed dW, a scale
    applied twice or a dropped 1/M each land far outside it."""
    from fp8_gemms_b200 import synthetic
    M, d, V, chunk = 96, 64, 320, 32
    Xt = synthetic.normal_bf16((M, d), 2.0, 45, 0)
    Wt = synthetic.normal_bf16((V, d), 0.3, 45, 1)
    labels = np.random.default_rng(45).integers(0, V, M).astype(np.int32)
    loss8, dX8, dW8, _ = orc.lmhead_ce(synthetic.bits_u16(Xt), synthetic.bits_u16(Wt), labels,
                                       chunk=chunk)
    loss, dX, dW = orc.lmhead_ce_f64(Xt.double().numpy(), Wt.double().numpy(), labels)
    rel = lambda got, r: np.linalg.norm(got - r) / np.linalg.norm(r)
    assert abs(loss8 - loss) <= 0.01 * loss
    assert rel(vals(dX8), dX) < 0.1
    assert rel(dW8.astype(np.float64), dW) < 0.1
    assert rel(vals(dX8), 2 * dX) > 0.4 and rel(dW8.astype(np.float64).T, dW.T[::-1]) > 0.4
