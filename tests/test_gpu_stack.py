"""GPU parity of the 28-layer stack's linear-layer GEMM set against the oracle.

Each layer of the little-lm 3.8B model (decomputer.nl, "Het trainen van een
3.8B LLM tot 0.384 CORE voor $998", "Appendix: De configuratie": 28 layers,
d = 3072, 24 query / 8 KV heads of 128, a non-gated relu^2 MLP of 12288) runs
its Q, K, V and O projections and its MLP block forward, dgrad and wgrad in
FP8, here at M = 16384 tokens with Student-t(3) activations whose outliers
stress the tensorwise amax.  Every layer has its own seeded inputs.

  * layers 0 and 27: the MLP block checked stagewise on scattered rows (the
    attention linears of those layers: tests/test_gpu_linear.py);
  * every layer: each cast the layer runs (X, W and dY of the four linears;
    X, W_up, W_down, h, dY and dH of the MLP) bit-exact over the whole tensor
    against the oracle's cast of the same input, and one 128-row block of
    every GEMM output (all columns) within the stated tolerance against the
    oracle on the GPU's own codes and scales.

The inputs are drawn on the host (the synthetic recipe), several tensors at a
time in threads, the next layer's while the current one is checked.
"""
import concurrent.futures

import numpy as np
import pytest
import torch

from fp8_gemms_b200 import synthetic
from gpu_util import assert_close, cast_ref, u8, u16
from test_gpu_mlp import Td, check_stagewise

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

E4M3, E5M2 = 0, 1
BLOCK = 128


@pytest.fixture(scope="module")
def api():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import api as a
    return a


def draw_layer(pool, layer):
    """Futures of the layer's tensors: four linears' dicts and the MLP's dict."""
    lin, mlp = synthetic.stack_layer(layer)
    return ([pool.submit(lin.tensors, i) for i in range(len(lin.linears))],
            pool.submit(mlp.tensors), lin, mlp)


def block_rows(n, layer, salt):
    """A 128-row block (all columns) at a seeded position."""
    r0 = int(np.random.default_rng(layer * 7919 + salt).integers(0, n - BLOCK + 1))
    return np.arange(r0, r0 + BLOCK)


def check_casts_equal(orc, sc_row, codes, bits, fmt, what):
    ref = cast_ref(orc, bits, fmt)
    assert sc_row[0] == ref["amax"] and sc_row[1] == ref["scale"] and \
        sc_row[2] == ref["inv_scale"], what
    assert np.array_equal(codes, ref["q"]), what


def check_linear_layer(orc, api, t, layer, i):
    X, W, dY = t["X"], t["W"], t["dY"]
    Y, dX, dW, q = api.linear_fwd_bwd(X.cuda(), W.cuda(), dY.cuda())
    torch.cuda.synchronize()
    from fp8_gemms_b200 import _lib
    assert _lib.lm_get_error()[0] == 0
    sc = q["scales"]
    Xq, Wq, dYq = u8(q["Xq"]), u8(q["Wq"]), u8(q["dYq"])
    what = f"layer {layer} {t['name']}"
    check_casts_equal(orc, sc[0], Xq, synthetic.bits_u16(X), E4M3, what + " X")
    check_casts_equal(orc, sc[1], Wq, synthetic.bits_u16(W), E4M3, what + " W")
    check_casts_equal(orc, sc[2], dYq, synthetic.bits_u16(dY), E5M2, what + " dY")
    rows = block_rows(X.shape[0], layer, i)
    wrows = block_rows(W.shape[0], layer, 100 + i)
    ref_Y, _ = orc.gemm(Xq, E4M3, Wq, E4M3, sc[0, 2], sc[1, 2], rows=rows)
    assert_close(u16(Y)[rows], ref_Y, what + " Y")
    ref_dX, _ = orc.gemm(dYq, E5M2, Td(q["Wq"]), E4M3, sc[2, 2], sc[1, 2], rows=rows)
    assert_close(u16(dX)[rows], ref_dX, what + " dX")
    ref_dW, _ = orc.gemm(Td(q["dYq"]), E5M2, Td(q["Xq"]), E4M3, sc[2, 2], sc[0, 2], rows=wrows)
    assert_close(u16(dW)[wrows], ref_dW, what + " dW")


def run_mlp(api, t, M):
    dev = {k: v.cuda() for k, v in t.items()}
    mlp = api.Relu2Mlp(M, synthetic.D_MODEL, synthetic.D_FF)
    Y = mlp.forward(dev["X"], dev["W_up"], dev["W_down"])
    dX, dWu, dWd = mlp.backward(dev["dY"])
    torch.cuda.synchronize()
    from fp8_gemms_b200 import _lib
    assert _lib.lm_get_error()[0] == 0
    return mlp, Y, dX, dWu, dWd


@pytest.mark.parametrize("layer", [0, 27])
def test_stack_layer_mlp_full_size_sampled(orc, api, layer):
    """The relu^2 MLP block of layers 0 and 27 at M = 16384 with t3 inputs:
    every cast bit-exact over the whole tensor, every GEMM on scattered rows."""
    _, w = synthetic.stack_layer(layer)
    t = w.tensors()
    mlp, Y, dX, dWu, dWd = run_mlp(api, t, w.M)
    rows = np.sort(np.concatenate([np.arange(0, 8), np.arange(w.M - 8, w.M),
                                   np.random.default_rng(layer).choice(w.M, 16, replace=False)]))
    check_stagewise(orc, mlp, t, Y, dX, dWu, dWd, rows=rows)


def test_stack_all_layers_casts_and_gemm_blocks(orc, api):
    """All 28 layers: bit-exact casts and a 128-row block of every GEMM."""
    with concurrent.futures.ThreadPoolExecutor(max_workers=6) as pool:
        nxt = draw_layer(pool, 0)
        for layer in range(synthetic.N_LAYERS):
            lin_f, mlp_f, lin, w = nxt
            if layer + 1 < synthetic.N_LAYERS:
                nxt = draw_layer(pool, layer + 1)
            for i, fut in enumerate(lin_f):
                check_linear_layer(orc, api, fut.result(), layer, i)
            t = mlp_f.result()
            mlp, Y, dX, dWu, dWd = run_mlp(api, t, w.M)
            check_stagewise(orc, mlp, t, Y, dX, dWu, dWd,
                            rows=block_rows(w.M, layer, 10),
                            wd_rows=block_rows(synthetic.D_MODEL, layer, 11),
                            wu_rows=block_rows(synthetic.D_FF, layer, 12))
            del mlp, Y, dX, dWu, dWd, t
