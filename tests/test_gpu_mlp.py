"""GPU parity of the relu^2 MLP forward and backward (single C-ABI calls)
against the oracle's chain.

Two kinds of check:
  * end to end: the same bf16 inputs go to lm_relu2_mlp_fwd/bwd and to the
    oracle chain; Y, dX, dW_up, dW_down within the stated tolerance;
  * stagewise: every cast the library runs is checked bit-exact against the
    oracle's cast of the GPU's own input to that cast (its H, its dH, its
    amax), and every GEMM within tolerance against the oracle's GEMM of the
    GPU's own codes and scales.
"""
import numpy as np
import pytest
import torch

from fp8_gemms_b200 import synthetic
from gpu_util import ELEM_REL_RELU2_BWD, assert_close, cast_ref, f32, u8, u16

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1


@pytest.fixture(scope="module")
def api():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import api as a
    return a


def run_chain(api, w):
    t = w.tensors()
    dev = {k: v.cuda() for k, v in t.items()}
    mlp = api.Relu2Mlp(w.M, w.d, w.f)
    Y = mlp.forward(dev["X"], dev["W_up"], dev["W_down"])
    dX, dWu, dWd = mlp.backward(dev["dY"]) if w.backward else (None, None, None)
    torch.cuda.synchronize()
    from fp8_gemms_b200 import _lib
    assert _lib.lm_get_error()[0] == 0
    return t, mlp, Y, dX, dWu, dWd


def T(codes):
    """Host transpose of a code matrix (the K-major operand the oracle takes)."""
    return np.ascontiguousarray(codes.T)


def Td(view):
    """The same transpose of a device code matrix, made on the device (a copy
    of bytes, no arithmetic) and brought to the host."""
    return u8(view.t().contiguous())


def check_stagewise(orc, mlp, t, Y, dX, dWu, dWd, rows=None, wd_rows=None, wu_rows=None):
    """rows: sample of output rows to check for the M x * GEMMs (None = all);
    wd_rows / wu_rows: rows of dW_down / dW_up to check (default: all when rows
    is None, else 24 evenly spaced rows)."""
    sc = mlp.view("scales").cpu().numpy()
    # casts of the inputs: bit-exact
    for name, key, si in [("X", "Xq", 0), ("W_up", "Wuq", 1), ("W_down", "Wdq", 2)]:
        ref = cast_ref(orc, synthetic.bits_u16(t[name]), E4M3)
        assert sc[si, 0] == ref["amax"] and sc[si, 1] == ref["scale"] and sc[si, 2] == ref["inv_scale"], name
        assert np.array_equal(u8(mlp.view(key)), ref["q"]), name
    Xq, Wuq, Wdq = u8(mlp.view("Xq")), u8(mlp.view("Wuq")), u8(mlp.view("Wdq"))
    H = u16(mlp.view("H"))
    # up GEMM (RELU2_FWD) from the GPU's codes and scales
    Href, _ = orc.gemm(Xq, E4M3, Wuq, E4M3, sc[0, 2], sc[1, 2], orc.EPI_RELU2_FWD, rows=rows)
    assert_close(H if rows is None else H[rows], Href, "H")
    # amax of h from the epilogue == amax of the GPU's own H, bit-exact
    assert sc[3, 0] == orc.amax(H, relu2_input=True)
    # cast of h from the GPU's H and amax: bit-exact
    s_h, inv_h = orc.scale(sc[3, 0], E4M3)
    assert sc[3, 1] == s_h and sc[3, 2] == inv_h
    hq_ref, _ = orc.cast(H, E4M3, s_h, relu2_input=True, want_qT=False)
    hq = u8(mlp.view("hq"))
    assert np.array_equal(hq, hq_ref)
    # down GEMM
    Yref, _ = orc.gemm(hq, E4M3, Wdq, E4M3, sc[3, 2], sc[2, 2], rows=rows)
    assert_close(u16(Y) if rows is None else u16(Y)[rows], Yref, "Y")
    if dX is None:
        return
    g = mlp.workspace_view("scales").cpu().numpy()
    ref = cast_ref(orc, synthetic.bits_u16(t["dY"]), E5M2)
    assert g[0, 0] == ref["amax"] and g[0, 1] == ref["scale"] and g[0, 2] == ref["inv_scale"]
    dYq = u8(mlp.workspace_view("dYq"))
    assert np.array_equal(dYq, ref["q"])
    # the backward's GEMMs read the row-major codes MN-major: the oracle gets
    # the K-major operands, i.e. the host transposes of those codes
    dH = u16(mlp.workspace_view("dH"))
    dHref, _ = orc.gemm(dYq, E5M2, Td(mlp.view("Wdq")), E4M3, g[0, 2], sc[2, 2],
                        orc.EPI_RELU2_BWD, aux=H, rows=rows)
    assert_close(dH if rows is None else dH[rows], dHref, "dH", ELEM_REL_RELU2_BWD)
    assert g[1, 0] == orc.amax(dH)
    s_dh, inv_dh = orc.scale(g[1, 0], E5M2)
    assert g[1, 1] == s_dh and g[1, 2] == inv_dh
    dHq_ref, _ = orc.cast(dH, E5M2, s_dh, want_qT=False)
    dHq = u8(mlp.workspace_view("dHq"))
    assert np.array_equal(dHq, dHq_ref)
    wrows = wd_rows
    if wrows is None and rows is not None:
        wrows = np.arange(0, dWd.shape[0], max(1, dWd.shape[0] // 24))
    ref_dWd, _ = orc.gemm(Td(mlp.workspace_view("dYq")), E5M2, Td(mlp.view("hq")), E4M3,
                          g[0, 2], sc[3, 2], rows=wrows)
    assert_close(u16(dWd) if wrows is None else u16(dWd)[wrows], ref_dWd, "dW_down")
    ref_dX, _ = orc.gemm(dHq, E5M2, Td(mlp.view("Wuq")), E4M3, g[1, 2], sc[1, 2], rows=rows)
    assert_close(u16(dX) if rows is None else u16(dX)[rows], ref_dX, "dX")
    urows = wu_rows
    if urows is None and rows is not None:
        urows = np.arange(0, dWu.shape[0], max(1, dWu.shape[0] // 24))
    ref_dWu, _ = orc.gemm(Td(mlp.workspace_view("dHq")), E5M2, Td(mlp.view("Xq")), E4M3,
                          g[1, 2], sc[0, 2], rows=urows)
    assert_close(u16(dWu) if urows is None else u16(dWu)[urows], ref_dWu, "dW_up")


def test_tiny_mlp_end_to_end(orc, api):
    """Tiny relu^2 MLP block fwd+bwd: X [256x256], W_up [1024x256],
    W_down [256x1024], dY [256x256]; GPU chain vs oracle chain."""
    w = synthetic.TINY_MLP
    t, mlp, Y, dX, dWu, dWd = run_chain(api, w)
    b = {k: synthetic.bits_u16(v) for k, v in t.items()}
    fwd = orc.mlp_fwd(b["X"], b["W_up"], b["W_down"])
    bwd = orc.mlp_bwd(b["dY"], fwd)
    assert_close(u16(Y), fwd["Y"], "Y")
    assert_close(u16(dX), bwd["dX"], "dX")
    assert_close(u16(dWu), bwd["dW_up"], "dW_up")
    assert_close(u16(dWd), bwd["dW_down"], "dW_down")


def test_tiny_mlp_stagewise(orc, api):
    w = synthetic.TINY_MLP
    t, mlp, Y, dX, dWu, dWd = run_chain(api, w)
    check_stagewise(orc, mlp, t, Y, dX, dWu, dWd)


def test_mlp_ragged_shapes(orc, api):
    """M, d, f multiples of 16 but not of any tile: every GEMM and cast has a
    ragged tail."""
    w = synthetic.MlpWorkload("ragged", 272, 208, 848, True)
    t, mlp, Y, dX, dWu, dWd = run_chain(api, w)
    check_stagewise(orc, mlp, t, Y, dX, dWu, dWd)


def test_mlp_small_model_dim(orc, api):
    """d = 128: the dW_down GEMM (M = d rows) runs on the single-CTA kernel,
    which carries no side warps, so the cast of dH runs as its own launch
    after it; the codes must be the same bits either way."""
    w = synthetic.MlpWorkload("d128", 512, 128, 512, True, seed=6)
    t, mlp, Y, dX, dWu, dWd = run_chain(api, w)
    check_stagewise(orc, mlp, t, Y, dX, dWu, dWd)


def test_mlp_student_t_inputs(orc, api):
    w = synthetic.MlpWorkload("t3", 512, 256, 1024, True, ("t3", None), 5)
    t, mlp, Y, dX, dWu, dWd = run_chain(api, w)
    check_stagewise(orc, mlp, t, Y, dX, dWu, dWd)


def test_mlp_repeated_calls_are_deterministic(orc, api):
    w = synthetic.TINY_MLP
    t, mlp, Y, dX, dWu, dWd = run_chain(api, w)
    dev = {k: v.cuda() for k, v in t.items()}
    Y2 = mlp.forward(dev["X"], dev["W_up"], dev["W_down"])
    dX2, dWu2, dWd2 = mlp.backward(dev["dY"])
    torch.cuda.synchronize()
    for a, b in [(Y, Y2), (dX, dX2), (dWu, dWu2), (dWd, dWd2)]:
        assert torch.equal(a, b)


@pytest.mark.slow
def test_full_size_mlp_sampled(orc, api):
    """The 3.8B-shape block (M=16384, d=3072, f=12288) fwd+bwd in the launch
    configuration bench.py times: casts bit-exact over whole tensors, GEMM
    outputs on sampled rows."""
    w = synthetic.MLP_FWD_BWD
    t, mlp, Y, dX, dWu, dWd = run_chain(api, w)
    rows = np.concatenate([np.arange(0, 16), np.arange(w.M - 16, w.M),
                           np.random.default_rng(0).choice(w.M, 16, replace=False)])
    check_stagewise(orc, mlp, t, Y, dX, dWu, dWd, rows=np.sort(rows))


@pytest.mark.slow
def test_full_size_mlp_forward_only_sampled(orc, api):
    """The 3.8B-shape forward alone (X [16384 x 3072] = 16 sequences x 1024
    tokens): up GEMM with the relu^2 epilogue and its amax, the cast of h,
    the down GEMM; casts bit-exact over whole tensors, GEMMs on sampled rows."""
    w = synthetic.MLP_FWD
    t, mlp, Y, *_ = run_chain(api, w)
    rows = np.sort(np.random.default_rng(2).choice(w.M, 32, replace=False))
    check_stagewise(orc, mlp, t, Y, None, None, None, rows=rows)


@pytest.mark.parametrize("workspace", [True, False])
@pytest.mark.parametrize("M,d,f", [(512, 256, 1024), (4096, 512, 2048), (1168, 256, 1040),
                                   (512, 768, 1024)])
def test_mlp_forward_h_cast_in_down_gemm_or_own_launch(orc, api, M, d, f, workspace):
    """With a workspace, h is cast by the down GEMM's side warps, unit by unit
    ahead of the tiles that read it (several units per CTA, ragged last row
    block and k-block at (1168, 1040); at (512, 768) the down GEMM's N exceeds
    its M, so its tiles sweep row blocks fastest and the units go k-block by
    k-block over all row blocks); without one, by its own launch before the
    GEMM.  Either way: casts bit-exact, the GEMMs within tolerance."""
    from fp8_gemms_b200 import _lib
    w = synthetic.MlpWorkload("h cast placement", M, d, f, False, ("t3", None), 11)
    t = w.tensors()
    dev = {k: v.cuda() for k, v in t.items()}
    mlp = api.Relu2Mlp(M, d, f)
    Y = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    _lib.lm_relu2_mlp_fwd(dev["X"], dev["W_up"], dev["W_down"], Y, mlp.saved,
                          workspace=mlp.workspace if workspace else None)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    check_stagewise(orc, mlp, t, Y, None, None, None)


def test_mlp_empty_batch(orc, api):
    """M = 0, an empty micro-batch: nothing to multiply.  Both weights are
    still cast (W_down's codes by the launch that stands in for the up GEMM's
    side warps), bit-exact against the oracle; Y and dX are empty; both weight
    gradients are zero; h's scale block is that of amax 0.  Tensors with M
    rows arrive as NULL pointers."""
    from fp8_gemms_b200 import _lib
    d, f = 256, 1024
    t = synthetic.MlpWorkload("empty", 16, d, f, False, seed=5).tensors()
    Wu, Wd = t["W_up"].cuda(), t["W_down"].cuda()
    mlp = api.Relu2Mlp(0, d, f)
    X = torch.empty(0, d, dtype=torch.bfloat16, device="cuda")
    Y = mlp.forward(X, Wu, Wd)
    dX, dWu, dWd = mlp.backward(torch.empty(0, d, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    assert Y.shape == (0, d) and dX.shape == (0, d)
    assert not bool(dWu.view(torch.int16).any()) and not bool(dWd.view(torch.int16).any())
    sc = mlp.view("scales").cpu().numpy()
    for row, name, W in ((1, "Wuq", t["W_up"]), (2, "Wdq", t["W_down"])):
        ref = orc.amax_scale_cast(synthetic.bits_u16(W), E4M3)
        assert sc[row, 0] == ref["amax"] and sc[row, 1] == ref["scale"], name
        assert sc[row, 2] == ref["inv_scale"], name
        assert np.array_equal(u8(mlp.view(name)), ref["q"]), name
    s0, inv0 = orc.scale(np.float32(0.0), E4M3)
    for row in (0, 3):                       # X and h: amax 0
        assert sc[row, 0] == 0.0 and sc[row, 1] == s0 and sc[row, 2] == inv0


@pytest.mark.slow
def test_full_size_step_is_deterministic_over_repeats(api):
    """Ten fwd+bwd steps of the 3.8B-shape block (M=16384, d=3072, f=12288) in
    the launch configuration bench.py times, L2 flushed between them: every
    output, the saved h codes and the dH codes are bit-identical to the first
    step's.  The side casts' ready bits, the split tails and the epilogues'
    amax must not make any result depend on timing."""
    from fp8_gemms_b200 import _lib
    w = synthetic.MLP_FWD_BWD
    dev = {k: v.cuda() for k, v in w.tensors().items()}
    mlp = api.Relu2Mlp(w.M, w.d, w.f)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    first = None
    for it in range(10):
        flush.fill_(it)
        Y = mlp.forward(dev["X"], dev["W_up"], dev["W_down"])
        dX, dWu, dWd = mlp.backward(dev["dY"])
        outs = [Y, dX, dWu, dWd, mlp.view("hq"), mlp.workspace_view("dHq"),
                mlp.view("scales"), mlp.workspace_view("scales")]
        torch.cuda.synchronize()
        assert _lib.lm_get_error()[0] == 0
        if first is None:
            first = [o.clone() for o in outs]
            continue
        names = ("Y", "dX", "dW_up", "dW_down", "hq", "dHq", "scales", "bwd scales")
        for name, a, b in zip(names, first, outs):
            assert torch.equal(a, b), f"{name} differs at repeat {it}"


@pytest.mark.slow
def test_mlp_forward_beyond_2_31_elements(orc, api):
    """M = 196,608 tokens, so H and h hold 2.4e9 elements, more than 2^31: the
    forward in bench.py's launch configuration (h cast by the down GEMM's side
    warps), checked on rows on both sides of element 2^31 and at the end.
    Whole-tensor amax of X and of h bit-exact; on the sampled rows X's and h's
    codes bit-exact, H and Y within the GEMM bar."""
    from fp8_gemms_b200 import _lib
    M, d, f = 196608, 3072, 12288
    assert M * f > 2 ** 31
    X = synthetic.normal_bf16((M, d), 1.0, 7, 0, device="cuda")
    Wu = synthetic.normal_bf16((f, d), 0.02, 7, 1).cuda()
    Wd = synthetic.normal_bf16((d, f), 0.02, 7, 2).cuda()
    mlp = api.Relu2Mlp(M, d, f)
    Y = mlp.forward(X, Wu, Wd)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    edge = 2 ** 31 // f                       # the row holding element 2^31 of H
    rows = np.array([0, 1, edge - 1, edge, edge + 1, M // 2, M - 2, M - 1])
    sc = mlp.view("scales").cpu().numpy()
    xb = synthetic.bits_u16(X.cpu())
    s_x, inv_x = orc.scale(orc.amax(xb), E4M3)
    assert sc[0, 0] == orc.amax(xb) and sc[0, 1] == s_x and sc[0, 2] == inv_x
    Xq_rows = u8(mlp.view("Xq")[torch.as_tensor(rows, device="cuda")])
    q_ref, _ = orc.cast(np.ascontiguousarray(xb[rows]), E4M3, s_x, want_qT=False)
    assert np.array_equal(Xq_rows, q_ref)
    del xb
    for name, key, si in [("W_up", "Wuq", 1), ("W_down", "Wdq", 2)]:
        ref = cast_ref(orc, synthetic.bits_u16((Wu if si == 1 else Wd).cpu()), E4M3)
        assert sc[si, 0] == ref["amax"] and np.array_equal(u8(mlp.view(key)), ref["q"]), name
    H = u16(mlp.view("H"))
    Href, _ = orc.gemm(u8(mlp.view("Xq")), E4M3, u8(mlp.view("Wuq")), E4M3, sc[0, 2], sc[1, 2],
                       orc.EPI_RELU2_FWD, rows=rows)
    assert_close(H[rows], Href, "H")
    assert sc[3, 0] == orc.amax(H, relu2_input=True)
    s_h, inv_h = orc.scale(sc[3, 0], E4M3)
    assert sc[3, 1] == s_h and sc[3, 2] == inv_h
    hq_ref, _ = orc.cast(np.ascontiguousarray(H[rows]), E4M3, s_h, relu2_input=True,
                         want_qT=False)
    del H
    hq = u8(mlp.view("hq"))
    assert np.array_equal(hq[rows], hq_ref)
    Yref, _ = orc.gemm(hq, E4M3, u8(mlp.view("Wdq")), E4M3, sc[3, 2], sc[2, 2], rows=rows)
    assert_close(u16(Y)[rows], Yref, "Y")
