"""GPU parity of the chunked FP8 LM head with softcapped cross-entropy
against the oracle: multi-chunk small cases end to end (loss, dX, fp32 dW),
the padded 50,304-entry vocabulary, and the run's micro-batch (M = 40,960,
d = 3072) on sampled tokens."""
import numpy as np
import pytest
import torch

from fp8_gemms_b200 import synthetic
from gpu_util import assert_close, assert_close_f32, u16

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1


def inputs(M, d, V, seed):
    X = synthetic.normal_bf16((M, d), 1.0, seed, 0)
    W = synthetic.normal_bf16((V, d), 0.02, seed, 1)
    labels = torch.randint(0, min(V, 50257), (M,), generator=torch.Generator().manual_seed(seed),
                           dtype=torch.int32)
    return X, W, labels


def run_gpu(X, W, labels, chunk):
    from fp8_gemms_b200 import _lib, api
    M, d = X.shape
    V = W.shape[0]
    head = api.LmHeadCE(M, d, V, chunk)
    dW = torch.zeros(V, d, dtype=torch.float32, device="cuda")
    loss, dX, dW = head(X.cuda(), W.cuda(), labels.cuda(), dW=dW)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    return head, float(loss.item()), dX, dW


@pytest.mark.parametrize("M,d,V,chunk", [(256, 256, 1024, 64), (512, 256, 50304, 256),
                                         (160, 128, 400, 160)])
def test_lmhead_ce_matches_oracle(orc, M, d, V, chunk):
    X, W, labels = inputs(M, d, V, M + V)
    head, loss, dX, dW = run_gpu(X, W, labels, chunk)
    ref_loss, ref_dX, ref_dW, ref_rows = orc.lmhead_ce(synthetic.bits_u16(X), synthetic.bits_u16(W),
                                                       labels.numpy(), chunk)
    assert abs(loss - ref_loss) <= 1e-3 * abs(ref_loss)
    rows = head.row_losses().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(rows - ref_rows) <= 1e-3 * np.abs(ref_rows) + 1e-4)
    assert_close(u16(dX), ref_dX, "dX")
    assert_close_f32(dW.cpu().numpy(), ref_dW, "dW")


@pytest.mark.parametrize("softcap", [5.0, 50.0])
def test_lmhead_ce_softcaps(orc, softcap):
    """Softcaps up to 40 take the sigmoid-form kernel (hardware exp2 and
    reciprocal, no running maximum); larger ones the tanhf / expf kernel."""
    M, d, V, chunk = 192, 256, 2048, 64
    X, W, labels = inputs(M, d, V, 12)
    X = X * 4  # larger logits: the softcap saturates for many of them
    from fp8_gemms_b200 import _lib, api
    head = api.LmHeadCE(M, d, V, chunk)
    dW = torch.zeros(V, d, dtype=torch.float32, device="cuda")
    loss, dX, dW = head(X.cuda(), W.cuda(), labels.cuda(), dW=dW, softcap=softcap)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    ref_loss, ref_dX, ref_dW, ref_rows = orc.lmhead_ce(synthetic.bits_u16(X), synthetic.bits_u16(W),
                                                       labels.numpy(), chunk, softcap=softcap)
    assert abs(float(loss.item()) - ref_loss) <= 1e-3 * abs(ref_loss)
    rows = head.row_losses().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(rows - ref_rows) <= 1e-3 * np.abs(ref_rows) + 1e-4)
    assert_close(u16(dX), ref_dX, f"dX softcap={softcap}")
    assert_close_f32(dW.cpu().numpy(), ref_dW, f"dW softcap={softcap}")


def test_lmhead_ce_accumulates_into_dW(orc):
    M, d, V = 128, 128, 256
    X, W, labels = inputs(M, d, V, 9)
    from fp8_gemms_b200 import api
    head = api.LmHeadCE(M, d, V, 64)
    dW = torch.zeros(V, d, dtype=torch.float32, device="cuda")
    head(X.cuda(), W.cuda(), labels.cuda(), dW=dW)
    once = dW.clone()
    head(X.cuda(), W.cuda(), labels.cuda(), dW=dW)
    torch.cuda.synchronize()
    assert torch.allclose(dW, 2 * once, rtol=1e-5, atol=1e-12)


def test_invalid_label_is_reported_not_read(orc):
    from fp8_gemms_b200 import _lib
    M, d, V = 32, 64, 128
    X, W, labels = inputs(M, d, V, 10)
    labels[5] = V + 7
    from fp8_gemms_b200 import api
    head = api.LmHeadCE(M, d, V, 32)
    head(X.cuda(), W.cuda(), labels.cuda())
    st, where = _lib.lm_get_error()
    assert _lib.STATUS[st] == "LM_ERR_INVALID_ARG" and where == 0x401
    assert _lib.lm_get_error() == (0, 0)


def test_lmhead_ce_run_shape_sampled(orc):
    """The run's micro-batch: M = 20 x 2048 = 40,960 tokens, d = 3072,
    V = 50,304, chunks of 4096.  Sampled tokens: row losses from the oracle's
    logits of bit-exact codes; the last chunk's dX rows from its own codes."""
    M, d, V, chunk = 40960, 3072, 50304, 4096
    X, W, labels = inputs(M, d, V, 11)
    head, loss, dX, dW = run_gpu(X, W, labels, chunk)
    rows_gpu = head.row_losses().cpu().numpy().astype(np.float64)
    assert abs(loss - rows_gpu.mean()) <= 1e-5 * abs(loss)
    Xb, Wb = synthetic.bits_u16(X), synthetic.bits_u16(W)
    cw = orc.amax_scale_cast(Wb, E4M3)
    sx, isx = orc.scale(orc.amax(Xb), E4M3)
    sample = np.sort(np.random.default_rng(1).choice(M, 24, replace=False))
    Xq_s, _ = orc.cast(Xb[sample], E4M3, sx, want_qT=False)
    logits, _ = orc.gemm(Xq_s, E4M3, cw["q"], E4M3, isx, cw["inv_scale"])
    ref_rows, _ = orc.softcap_ce(logits, labels.numpy()[sample], want_grad=False)
    assert np.all(np.abs(rows_gpu[sample] - ref_rows) <= 1e-3 * ref_rows + 1e-4)
