"""GPU parity of the chunked FP8 LM head with softcapped cross-entropy
against the oracle: multi-chunk small cases end to end (loss, dX, fp32 dW),
the padded 50,304-entry vocabulary, and the run's micro-batch (M = 40,960,
d = 3072) on sampled tokens."""
import numpy as np
import pytest
import torch

from fp8_gemms_b200 import synthetic
from gpu_util import assert_close, assert_close_f32, cast_ref, u8, u16

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1


def inputs(M, d, V, seed):
    X = synthetic.normal_bf16((M, d), 1.0, seed, 0)
    W = synthetic.normal_bf16((V, d), 0.02, seed, 1)
    labels = torch.randint(0, min(V, 50257), (M,), generator=torch.Generator().manual_seed(seed),
                           dtype=torch.int32)
    return X, W, labels


def run_gpu_with(head, X, W, labels):
    from fp8_gemms_b200 import _lib
    dW = torch.zeros(head.V, head.d, dtype=torch.float32, device="cuda")
    loss, dX, dW = head(X.cuda(), W.cuda(), labels.cuda(), dW=dW)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    return float(loss.item()), dX, dW


def run_gpu(X, W, labels, chunk):
    from fp8_gemms_b200 import api
    M, d = X.shape
    head = api.LmHeadCE(M, d, W.shape[0], chunk)
    return (head,) + run_gpu_with(head, X, W, labels)


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


def test_lmhead_ce_empty_batch(orc):
    """M = 0: no tokens.  W is still cast (bit-exact against the oracle), the
    loss is 0, dW keeps what it held, and X, labels and dX arrive as NULL."""
    from fp8_gemms_b200 import _lib, api
    d, V = 64, 128
    _, W, _ = inputs(16, d, V, 11)
    head = api.LmHeadCE(0, d, V, 32)
    head.loss.fill_(7.0)                     # the call must write the 0
    dW = torch.full((V, d), 0.5, dtype=torch.float32, device="cuda")
    loss, dX, _ = head(torch.empty(0, d, dtype=torch.bfloat16, device="cuda"), W.cuda(),
                       torch.empty(0, dtype=torch.int32, device="cuda"), dW=dW)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    assert float(loss) == 0.0 and dX.shape == (0, d)
    assert bool((dW == 0.5).all())
    ref = cast_ref(orc, synthetic.bits_u16(W), 0)
    assert np.array_equal(u8(head.view("Wq")), ref["q"])


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
    V = 50,304, chunks of 4096 (ten chunks).  Checked:
      * W's codes and the last chunk's X codes bit-exact (X at the whole
        tensor's scale);
      * row losses of sampled tokens of every chunk, from the oracle's logits
        of the bit-exact codes;
      * the last chunk (the state the workspace keeps): its dlogits on sampled
        rows against the oracle's CE of the same codes, the e5m2 cast of the
        GPU's dlogits bit-exact over the whole chunk, and dX of sampled rows
        against the oracle's dgrad of the GPU's own codes and scales;
      * dW on sampled vocabulary rows: a second call whose X is zero outside
        the last chunk, so that every other chunk adds exactly zero and dW is
        the last chunk's wgrad alone, against the oracle's fp32 wgrad of that
        call's own codes and scales."""
    from fp8_gemms_b200 import api
    M, d, V, chunk = 40960, 3072, 50304, 4096
    c0 = (M - 1) // chunk * chunk
    X, W, labels = inputs(M, d, V, 11)
    head, loss, dX, dW = run_gpu(X, W, labels, chunk)
    rows_gpu = head.row_losses().cpu().numpy().astype(np.float64)
    assert abs(loss - rows_gpu.mean()) <= 1e-5 * abs(loss)
    Xb, Wb = synthetic.bits_u16(X), synthetic.bits_u16(W)
    lab = labels.numpy()
    sc = head.view("scales").cpu().numpy()
    cw = cast_ref(orc, Wb, E4M3)
    assert sc[1, 0] == cw["amax"] and sc[1, 1] == cw["scale"]
    Wq = u8(head.view("Wq"))
    assert np.array_equal(Wq, cw["q"])
    ax = orc.amax(Xb)
    sx, isx = orc.scale(ax, E4M3)
    assert sc[0, 0] == ax and sc[0, 1] == sx and sc[0, 2] == isx
    Xq_last = u8(head.view("Xq"))
    assert np.array_equal(Xq_last, orc.cast(Xb[c0:], E4M3, sx, want_qT=False)[0])
    # row losses of sampled tokens, every chunk
    sample = np.sort(np.random.default_rng(1).choice(M, 24, replace=False))
    Xq_s, _ = orc.cast(Xb[sample], E4M3, sx, want_qT=False)
    logits, _ = orc.gemm(Xq_s, E4M3, Wq, E4M3, isx, cw["inv_scale"])
    ref_rows, _ = orc.softcap_ce(logits, lab[sample], want_grad=False)
    assert np.all(np.abs(rows_gpu[sample] - ref_rows) <= 1e-3 * ref_rows + 1e-4)
    # the last chunk: dlogits, their cast, dX
    ls = np.sort(np.random.default_rng(2).choice(M - c0, 16, replace=False))
    lg, _ = orc.gemm(Xq_last, E4M3, Wq, E4M3, isx, cw["inv_scale"], rows=ls)
    _, dl_ref = orc.softcap_ce(lg, lab[c0 + ls], inv_count=1.0 / M)
    dl = u16(head.view("dlogits"))
    assert_close(dl[ls], dl_ref, "dlogits of the last chunk")
    assert sc[2, 0] == orc.amax(dl)
    s_dl, inv_dl = orc.scale(sc[2, 0], E5M2)
    assert sc[2, 1] == s_dl and sc[2, 2] == inv_dl
    dLq = u8(head.view("dLq"))
    assert np.array_equal(dLq, orc.cast(dl, E5M2, s_dl, want_qT=False)[0])
    WqT = np.ascontiguousarray(Wq.T)
    ref_dX, _ = orc.gemm(dLq, E5M2, WqT, E4M3, inv_dl, cw["inv_scale"], rows=ls)
    assert_close(u16(dX)[c0 + ls], ref_dX, "dX of the last chunk")
    # dW: the last chunk's wgrad alone (X zero in every other chunk)
    X0 = X.clone()
    X0[:c0] = 0
    head0 = api.LmHeadCE(M, d, V, chunk)
    _, _, dW0 = run_gpu_with(head0, X0, W, labels)
    sc0 = head0.view("scales").cpu().numpy()
    dLq0, Xq0 = u8(head0.view("dLq")), u8(head0.view("Xq"))
    vrows = np.sort(np.concatenate([lab[c0:c0 + 8], [0, V - 1, 50257, 50300],
                                    np.random.default_rng(3).choice(V, 12, replace=False)]))
    vrows = np.unique(vrows)
    ref_dW = np.zeros((len(vrows), d), np.float32)
    orc.gemm_accum_f32(np.ascontiguousarray(dLq0.T), E5M2, np.ascontiguousarray(Xq0.T), E4M3,
                       sc0[2, 2], sc0[0, 2], ref_dW, rows=vrows)
    assert_close_f32(dW0.cpu().numpy()[vrows], ref_dW, "dW (last chunk's wgrad)")
