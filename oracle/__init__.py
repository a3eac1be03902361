"""CPU oracle for the FP8 training-GEMM path (test infrastructure only).

Only tests/, ``__graft_entry__.smoke()`` and bench.py's ``cpu_baseline`` and
``--impl reference`` legs may import this package.  It shares no code with the
CUDA path: the arithmetic lives in ``fp8_oracle.c`` (plain C, fp64); this
module only marshals numpy arrays into it and composes the relu^2 MLP chain in
the order the method runs it.

Tensors cross this interface as numpy arrays of raw bits: bf16 as uint16,
FP8 codes as uint8, all row-major.

The chain (``mlp_fwd`` / ``mlp_bwd``) follows the method described on
decomputer.nl, "Het trainen van een 3.8B LLM tot 0.384 CORE voor $998":
section "Vroege experimenten" item 4 and section "Doorvoer (Throughput)
verhogen" (FP8 with dynamic tensorwise scaling on the forward GEMM and both
backward GEMMs), with the non-gated relu^2 MLP of the "Niet-gated MLPs" bullet
and of "Appendix: De configuratie".  Every tensor is quantised once per call
with one tensorwise scale; the backward reuses the forward's quantised X,
W_up, W_down and h and their scales.

Parity status: no page prints a numeric value for any cast or GEMM of this
path, so every value check rests on pins against the format definitions,
closed forms, brute force and finite differences (tests/test_oracle_*.py).
"""
import ctypes
import os

import numpy as np

from . import build as _build

E4M3, E5M2 = 0, 1
EPI_NONE, EPI_RELU2_FWD, EPI_RELU2_BWD = 0, 1, 2
FP8_MAX = {E4M3: 448.0, E5M2: 57344.0}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_fp8_decode.argtypes = [ctypes.c_uint8, ctypes.c_int]
        L.orc_fp8_decode.restype = ctypes.c_double
        L.orc_fp8_encode.argtypes = [ctypes.c_float, ctypes.c_int]
        L.orc_fp8_encode.restype = ctypes.c_uint8
        L.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_double.restype = ctypes.c_double
        L.orc_bf16_from_double.argtypes = [ctypes.c_double]
        L.orc_bf16_from_double.restype = ctypes.c_uint16
        L.orc_amax.argtypes = [P, i64, i64, i64, ctypes.c_int]
        L.orc_amax.restype = ctypes.c_float
        L.orc_scale.argtypes = [ctypes.c_float, ctypes.c_int, P, P]
        L.orc_scale.restype = None
        L.orc_cast.argtypes = [P, i64, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_float, P, P]
        L.orc_cast.restype = None
        L.orc_gemm_acc.argtypes = [P, ctypes.c_int, P, ctypes.c_int, i64, i64, i64, P, i64, P]
        L.orc_gemm_acc.restype = None
        L.orc_gemm.argtypes = [P, ctypes.c_int, P, ctypes.c_int, i64, i64, i64, ctypes.c_float,
                               ctypes.c_float, ctypes.c_int, P, P, i64, P, P]
        L.orc_gemm.restype = None
        L.orc_gemm_accum_f32.argtypes = [P, ctypes.c_int, P, ctypes.c_int, i64, i64, i64,
                                         ctypes.c_float, ctypes.c_float, P, i64, P]
        L.orc_gemm_accum_f32.restype = None
        L.orc_rmsnorm.argtypes = [P, P, i64, i64, ctypes.c_double, P]
        L.orc_rmsnorm.restype = None
        L.orc_swiglu_h.argtypes = [P, P, i64, i64, P]
        L.orc_swiglu_h.restype = ctypes.c_float
        L.orc_swiglu_bwd.argtypes = [P, P, P, i64, i64, P, P]
        L.orc_swiglu_bwd.restype = ctypes.c_float
        L.orc_swiglu_f64.argtypes = [P, P, P, P, P, i64, i64, i64, P, P, P, P, P]
        L.orc_swiglu_f64.restype = None
        L.orc_softcap_ce.argtypes = [P, P, i64, i64, ctypes.c_double, ctypes.c_double, P, P]
        L.orc_softcap_ce.restype = None
        L.orc_mlp_f64.argtypes = [P, P, P, P, i64, i64, i64, P, P, P, P]
        L.orc_mlp_f64.restype = None
        L.orc_lmhead_ce_f64.argtypes = [P, P, P, i64, i64, i64, ctypes.c_double, P, P, P]
        L.orc_lmhead_ce_f64.restype = None
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


def num_threads() -> int:
    return lib().orc_num_threads()


# ------------------------------------------------------------------ codecs
def fp8_decode(code: int, fmt: int) -> float:
    return lib().orc_fp8_decode(code, fmt)


def fp8_encode(x: float, fmt: int) -> int:
    return lib().orc_fp8_encode(x, fmt)


def fp8_decode_array(codes, fmt):
    table = np.array([fp8_decode(c, fmt) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def bf16_to_double(b: int) -> float:
    return lib().orc_bf16_to_double(b)


def bf16_from_double(v: float) -> int:
    return lib().orc_bf16_from_double(v)


def bf16_bits_to_f64(bits):
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ------------------------------------------------------ amax / scale / cast
def amax(x, relu2_input=False) -> np.float32:
    x = _c(x, np.uint16)
    rows, cols = x.shape
    return np.float32(lib().orc_amax(_ptr(x), rows, cols, cols, int(relu2_input)))


def scale(amax_value, fmt):
    s = np.zeros(1, np.float32)
    inv = np.zeros(1, np.float32)
    lib().orc_scale(float(np.float32(amax_value)), fmt, _ptr(s), _ptr(inv))
    return s[0], inv[0]


def cast(x, fmt, scale_value, relu2_input=False, want_q=True, want_qT=True):
    """Return (q, qT) codes of a rows x cols bf16 tensor at a given scale."""
    x = _c(x, np.uint16)
    rows, cols = x.shape
    q = np.zeros((rows, cols), np.uint8) if want_q else None
    qT = np.zeros((cols, rows), np.uint8) if want_qT else None
    lib().orc_cast(_ptr(x), rows, cols, cols, fmt, int(relu2_input),
                   float(np.float32(scale_value)), _ptr(q), _ptr(qT))
    return q, qT


def amax_scale_cast(x, fmt, relu2_input=False, amax_in=None):
    """The full dynamic-scaling cast: amax -> scale -> codes (+ transpose)."""
    a = amax(x, relu2_input) if amax_in is None else np.float32(amax_in)
    s, inv = scale(a, fmt)
    q, qT = cast(x, fmt, s, relu2_input)
    return dict(amax=a, scale=s, inv_scale=inv, q=q, qT=qT)


# ------------------------------------------------------------------- GEMM
def gemm_acc(A, fa, B, fb, rows=None):
    """fp64 C = dec(A) dec(B)^T over the listed rows of A (all if None)."""
    A = _c(A, np.uint8)
    B = _c(B, np.uint8)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2
    r = None if rows is None else _c(np.asarray(rows, dtype=np.int64), np.int64)
    nr = M if r is None else len(r)
    C = np.zeros((nr, N), np.float64)
    lib().orc_gemm_acc(_ptr(A), fa, _ptr(B), fb, M, N, K, _ptr(r), nr, _ptr(C))
    return C


def gemm(A, fa, B, fb, inv_sa, inv_sb, epi=EPI_NONE, aux=None, rows=None):
    """bf16 D = epi((dec(A) dec(B)^T) inv_sa inv_sb) and the amax of what the
    next cast consumes.  Returns (D bits, amax)."""
    A = _c(A, np.uint8)
    B = _c(B, np.uint8)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2
    if epi == EPI_RELU2_BWD:
        aux = _c(aux, np.uint16)
        assert aux.shape == (M, N)
    r = None if rows is None else _c(np.asarray(rows, dtype=np.int64), np.int64)
    nr = M if r is None else len(r)
    D = np.zeros((nr, N), np.uint16)
    am = np.zeros(1, np.float32)
    lib().orc_gemm(_ptr(A), fa, _ptr(B), fb, M, N, K, float(np.float32(inv_sa)),
                   float(np.float32(inv_sb)), epi, _ptr(aux), _ptr(r), nr, _ptr(D), _ptr(am))
    return D, am[0]


def gemm_accum_f32(A, fa, B, fb, inv_sa, inv_sb, D, rows=None):
    """In place: D (fp32, rows x N) += fp32(dec(A) dec(B)^T inv_sa inv_sb) for the
    listed rows of A (all if None); D holds those rows in order."""
    A = _c(A, np.uint8)
    B = _c(B, np.uint8)
    assert D.dtype == np.float32 and D.flags.c_contiguous
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2
    r = None if rows is None else _c(np.asarray(rows, dtype=np.int64), np.int64)
    nr = M if r is None else len(r)
    assert D.shape == (nr, N)
    lib().orc_gemm_accum_f32(_ptr(A), fa, _ptr(B), fb, M, N, K, float(np.float32(inv_sa)),
                             float(np.float32(inv_sb)), _ptr(r), nr, _ptr(D))
    return D


def rmsnorm(R, w=None, eps=1e-6):
    """bf16 X = RMSNorm(R) * w, fp64 then one rounding (bits in, bits out)."""
    R = _c(R, np.uint16)
    rows, cols = R.shape
    if w is not None:
        w = _c(w, np.uint16)
        assert w.shape == (cols,)
    X = np.zeros((rows, cols), np.uint16)
    lib().orc_rmsnorm(_ptr(R), _ptr(w), rows, cols, float(eps), _ptr(X))
    return X


def rmsnorm_fp8_cast(R, w=None, eps=1e-6, fmt=E4M3):
    """The fused producer: X = RMSNorm(R) * w, then X's dynamic cast."""
    X = rmsnorm(R, w, eps)
    out = amax_scale_cast(X, fmt)
    out["X"] = X
    return out


# ---------------------------------------------------------- plain linear
def linear_fwd_bwd(X, W, dY):
    """Plain FP8 linear Y = X W^T with its dgrad and wgrad (the attention
    projections and the LM head): X and W quantised to e4m3 and dY to e5m2,
    each once with its own tensorwise scale (decomputer.nl, "Het trainen van
    een 3.8B LLM tot 0.384 CORE voor $998", section "Vroege experimenten" item
    4: all three GEMMs of a linear in FP8).
      Y = Xq Wq^T,  dX = dYq Wq,  dW = dYq^T Xq   (bf16 bits out)."""
    cx = amax_scale_cast(X, E4M3)
    cw = amax_scale_cast(W, E4M3)
    cg = amax_scale_cast(dY, E5M2)
    Y, _ = gemm(cx["q"], E4M3, cw["q"], E4M3, cx["inv_scale"], cw["inv_scale"])
    dX, _ = gemm(cg["q"], E5M2, cw["qT"], E4M3, cg["inv_scale"], cw["inv_scale"])
    dW, _ = gemm(cg["qT"], E5M2, cx["qT"], E4M3, cg["inv_scale"], cx["inv_scale"])
    return dict(Y=Y, dX=dX, dW=dW, X=cx, W=cw, dY=cg)


# -------------------------------------------------------------- MLP chain
def mlp_fwd(X, W_up, W_down):
    """relu^2 MLP forward with dynamic tensorwise FP8 scaling.

    X: M x d, W_up: f x d, W_down: d x f (bf16 bits).  Returns a dict holding
    Y and every intermediate the backward reuses.
    """
    cx = amax_scale_cast(X, E4M3)
    cu = amax_scale_cast(W_up, E4M3)
    cd = amax_scale_cast(W_down, E4M3)
    H, amax_h = gemm(cx["q"], E4M3, cu["q"], E4M3, cx["inv_scale"], cu["inv_scale"],
                     EPI_RELU2_FWD)
    ch = amax_scale_cast(H, E4M3, relu2_input=True, amax_in=amax_h)
    Y, amax_y = gemm(ch["q"], E4M3, cd["q"], E4M3, ch["inv_scale"], cd["inv_scale"])
    return dict(Y=Y, X=cx, W_up=cu, W_down=cd, H=H, h=ch, amax_y=amax_y)


def mlp_bwd(dY, saved):
    """relu^2 MLP backward: dgrad and wgrad of both linears in FP8, e5m2
    gradients against e4m3 saved operands."""
    cg = amax_scale_cast(dY, E5M2)
    cx, cu, cd, ch = saved["X"], saved["W_up"], saved["W_down"], saved["h"]
    dH, amax_dh = gemm(cg["q"], E5M2, cd["qT"], E4M3, cg["inv_scale"], cd["inv_scale"],
                       EPI_RELU2_BWD, aux=saved["H"])
    dW_down, _ = gemm(cg["qT"], E5M2, ch["qT"], E4M3, cg["inv_scale"], ch["inv_scale"])
    cdh = amax_scale_cast(dH, E5M2, amax_in=amax_dh)
    dX, _ = gemm(cdh["q"], E5M2, cu["qT"], E4M3, cdh["inv_scale"], cu["inv_scale"])
    dW_up, _ = gemm(cdh["qT"], E5M2, cx["qT"], E4M3, cdh["inv_scale"], cx["inv_scale"])
    return dict(dX=dX, dW_up=dW_up, dW_down=dW_down, dY=cg, dH=dH, dh=cdh)


def mlp_grad_accum(micro_batches, W_up, W_down):
    """One optimizer step of gradient accumulation over micro-batches
    [(X, dY), ...]: the weights are cast once (first micro-batch) and their
    codes reused; each backward adds its weight gradients into fp32
    accumulators.  Returns per-micro-batch (Y, dX) and the fp32 dW_up, dW_down."""
    f, d = W_up.shape
    dWu = np.zeros((f, d), np.float32)
    dWd = np.zeros((d, f), np.float32)
    outs = []
    cu = amax_scale_cast(W_up, E4M3)
    cd = amax_scale_cast(W_down, E4M3)
    for X, dY in micro_batches:
        cx = amax_scale_cast(X, E4M3)
        H, amax_h = gemm(cx["q"], E4M3, cu["q"], E4M3, cx["inv_scale"], cu["inv_scale"],
                         EPI_RELU2_FWD)
        ch = amax_scale_cast(H, E4M3, relu2_input=True, amax_in=amax_h)
        Y, _ = gemm(ch["q"], E4M3, cd["q"], E4M3, ch["inv_scale"], cd["inv_scale"])
        cg = amax_scale_cast(dY, E5M2)
        dH, amax_dh = gemm(cg["q"], E5M2, cd["qT"], E4M3, cg["inv_scale"], cd["inv_scale"],
                           EPI_RELU2_BWD, aux=H)
        gemm_accum_f32(cg["qT"], E5M2, ch["qT"], E4M3, cg["inv_scale"], ch["inv_scale"], dWd)
        cdh = amax_scale_cast(dH, E5M2, amax_in=amax_dh)
        dX, _ = gemm(cdh["q"], E5M2, cu["qT"], E4M3, cdh["inv_scale"], cu["inv_scale"])
        gemm_accum_f32(cdh["qT"], E5M2, cx["qT"], E4M3, cdh["inv_scale"], cx["inv_scale"], dWu)
        outs.append((Y, dX))
    return outs, dWu, dWd


def mlp_f64(X, W_up, W_down, dY=None):
    """Unquantised fp64 relu^2 MLP forward and backward (float64 arrays)."""
    X = _c(X, np.float64)
    W_up = _c(W_up, np.float64)
    W_down = _c(W_down, np.float64)
    M, d = X.shape
    f = W_up.shape[0]
    Y = np.zeros((M, d))
    out = dict(Y=Y)
    if dY is not None:
        dY = _c(dY, np.float64)
        out.update(dX=np.zeros((M, d)), dW_up=np.zeros((f, d)), dW_down=np.zeros((d, f)))
    lib().orc_mlp_f64(_ptr(X), _ptr(W_up), _ptr(W_down), _ptr(dY), M, d, f, _ptr(Y),
                      _ptr(out.get("dX")), _ptr(out.get("dW_up")), _ptr(out.get("dW_down")))
    return out


# ------------------------------------------------ gated (SwiGLU) variant
def amax_scale_cast_joint(tensors, fmt, amax_in=None):
    """Several tensors quantised as ONE tensor: one amax over all of them, one
    scale, then each tensor's codes (+ transposes) at that scale.  The gated
    block's gate and up weights form one fused weight, and its dG and dU one
    gradient, so each pair shares a tensorwise scale."""
    a = max(amax(t) for t in tensors) if amax_in is None else np.float32(amax_in)
    s, inv = scale(a, fmt)
    out = dict(amax=np.float32(a), scale=s, inv_scale=inv, q=[], qT=[])
    for t in tensors:
        q, qT = cast(t, fmt, s)
        out["q"].append(q)
        out["qT"].append(qT)
    return out


def swiglu_h(G, U):
    """h = bf16(silu(G) U) from bf16 G, U [M x f]; returns (h, amax of h)."""
    G = _c(G, np.uint16)
    U = _c(U, np.uint16)
    assert G.shape == U.shape
    M, f = G.shape
    h = np.zeros((M, f), np.uint16)
    a = lib().orc_swiglu_h(_ptr(G), _ptr(U), M, f, _ptr(h))
    return h, np.float32(a)


def swiglu_bwd(g, G, U):
    """dG = bf16(g U silu'(G)), dU = bf16(g silu(G)); returns (dG, dU, amax over both)."""
    g = _c(g, np.uint16)
    G = _c(G, np.uint16)
    U = _c(U, np.uint16)
    assert g.shape == G.shape == U.shape
    M, f = g.shape
    dG = np.zeros((M, f), np.uint16)
    dU = np.zeros((M, f), np.uint16)
    a = lib().orc_swiglu_bwd(_ptr(g), _ptr(G), _ptr(U), M, f, _ptr(dG), _ptr(dU))
    return dG, dU, np.float32(a)


def swiglu_fwd(X, W_gate, W_up, W_down):
    """Gated MLP forward in FP8 (bf16 bits in): G = Xq Wgq^T, U = Xq Wuq^T,
    h = silu(G) U, Y = hq Wdq^T.  W_gate and W_up share one scale."""
    cx = amax_scale_cast(X, E4M3)
    cw = amax_scale_cast_joint([W_gate, W_up], E4M3)
    cd = amax_scale_cast(W_down, E4M3)
    G, _ = gemm(cx["q"], E4M3, cw["q"][0], E4M3, cx["inv_scale"], cw["inv_scale"])
    U, _ = gemm(cx["q"], E4M3, cw["q"][1], E4M3, cx["inv_scale"], cw["inv_scale"])
    h, amax_h = swiglu_h(G, U)
    ch = amax_scale_cast(h, E4M3, amax_in=amax_h)
    Y, _ = gemm(ch["q"], E4M3, cd["q"], E4M3, ch["inv_scale"], cd["inv_scale"])
    return dict(Y=Y, X=cx, W_gu=cw, W_down=cd, G=G, U=U, h_bf16=h, h=ch)


def swiglu_bwd_chain(dY, saved):
    """Gated MLP backward in FP8: g = dYq Wd (plain dgrad), dG and dU from g,
    cast to e5m2 with one shared scale; dX = dGq Wgq + dUq Wuq as one GEMM over
    the concatenated reduction [G | U]; dW_gate = dGq^T Xq, dW_up = dUq^T Xq,
    dW_down = dYq^T hq."""
    cg = amax_scale_cast(dY, E5M2)
    cx, cw, cd, ch = saved["X"], saved["W_gu"], saved["W_down"], saved["h"]
    g, _ = gemm(cg["q"], E5M2, cd["qT"], E4M3, cg["inv_scale"], cd["inv_scale"])
    dW_down, _ = gemm(cg["qT"], E5M2, ch["qT"], E4M3, cg["inv_scale"], ch["inv_scale"])
    dG, dU, amax_d = swiglu_bwd(g, saved["G"], saved["U"])
    cdg = amax_scale_cast_joint([dG, dU], E5M2, amax_in=amax_d)
    dX, _ = gemm(np.hstack(cdg["q"]), E5M2, np.hstack(cw["qT"]), E4M3, cdg["inv_scale"],
                 cw["inv_scale"])
    dW_gate, _ = gemm(cdg["qT"][0], E5M2, cx["qT"], E4M3, cdg["inv_scale"], cx["inv_scale"])
    dW_up, _ = gemm(cdg["qT"][1], E5M2, cx["qT"], E4M3, cdg["inv_scale"], cx["inv_scale"])
    return dict(dX=dX, dW_gate=dW_gate, dW_up=dW_up, dW_down=dW_down, dY=cg, g=g, dG=dG,
                dU=dU, dgu=cdg)


def swiglu_f64(X, Wg, Wu, Wd, dY=None):
    X, Wg, Wu, Wd = (_c(a, np.float64) for a in (X, Wg, Wu, Wd))
    M, d = X.shape
    f = Wg.shape[0]
    out = dict(Y=np.zeros((M, d)))
    if dY is not None:
        dY = _c(dY, np.float64)
        out.update(dX=np.zeros((M, d)), dWg=np.zeros((f, d)), dWu=np.zeros((f, d)),
                   dWd=np.zeros((d, f)))
    lib().orc_swiglu_f64(_ptr(X), _ptr(Wg), _ptr(Wu), _ptr(Wd), _ptr(dY), M, d, f,
                         _ptr(out["Y"]), _ptr(out.get("dX")), _ptr(out.get("dWg")),
                         _ptr(out.get("dWu")), _ptr(out.get("dWd")))
    return out


# ------------------------------------- LM head with softcapped cross-entropy
def softcap_ce(logits, labels, softcap=15.0, inv_count=None, want_grad=True):
    """Row losses (fp64) and bf16 dlogits of the softcapped CE over bf16 logits."""
    logits = _c(logits, np.uint16)
    labels = _c(np.asarray(labels, dtype=np.int32), np.int32)
    rows, V = logits.shape
    inv = 1.0 / rows if inv_count is None else inv_count
    dl = np.zeros((rows, V), np.uint16) if want_grad else None
    loss = np.zeros(rows, np.float64)
    lib().orc_softcap_ce(_ptr(logits), _ptr(labels), rows, V, float(softcap), float(inv),
                         _ptr(dl), _ptr(loss))
    return loss, dl


def lmhead_ce_f64(X, W, labels, softcap=15.0, want_grad=True):
    """Unquantised, unchunked fp64 LM head + softcapped CE (float64 arrays in):
    mean loss, dX [M x d], dW [V x d] of loss = mean(lse(z) - z[label]),
    z = c tanh(X W^T / c)."""
    X = _c(X, np.float64)
    W = _c(W, np.float64)
    labels = _c(np.asarray(labels, dtype=np.int32), np.int32)
    M, d = X.shape
    V = W.shape[0]
    loss = np.zeros(1, np.float64)
    dX = np.zeros((M, d)) if want_grad else None
    dW = np.zeros((V, d)) if want_grad else None
    lib().orc_lmhead_ce_f64(_ptr(X), _ptr(W), _ptr(labels), M, d, V, float(softcap), _ptr(loss),
                            _ptr(dX), _ptr(dW))
    return float(loss[0]), dX, dW


def lmhead_ce(X, W, labels, chunk, softcap=15.0):
    """FP8 LM head inside a chunked, softcapped fused linear cross-entropy:
    X and W are quantised once (X's per-chunk codes use the whole tensor's
    scale); per chunk of rows: bf16 logits = Xq_c Wq^T, CE -> dlogits,
    dlogits cast to e5m2 (its own tensorwise scale), dX_c = dL_c W,
    dW += fp32(dL_c^T X_c).  Returns mean loss, dX (bf16 bits), dW (fp32)."""
    M, d = X.shape
    V = W.shape[0]
    cw = amax_scale_cast(W, E4M3)
    ax = amax(X)
    sx, isx = scale(ax, E4M3)
    dX = np.zeros((M, d), np.uint16)
    dW = np.zeros((V, d), np.float32)
    losses = np.zeros(M, np.float64)
    for c0 in range(0, M, chunk):
        c1 = min(M, c0 + chunk)
        Xq, XqT = cast(X[c0:c1], E4M3, sx)
        logits, _ = gemm(Xq, E4M3, cw["q"], E4M3, isx, cw["inv_scale"])
        loss, dl = softcap_ce(logits, labels[c0:c1], softcap, inv_count=1.0 / M)
        losses[c0:c1] = loss
        cdl = amax_scale_cast(dl, E5M2)
        dX[c0:c1], _ = gemm(cdl["q"], E5M2, cw["qT"], E4M3, cdl["inv_scale"], cw["inv_scale"])
        gemm_accum_f32(cdl["qT"], E5M2, XqT, E4M3, cdl["inv_scale"], isx, dW)
    # no tokens: the mean over an empty batch is taken as 0 (a reading; the
    # pages only ever average over a full micro-batch)
    return (losses.mean() if M else 0.0), dX, dW, losses
