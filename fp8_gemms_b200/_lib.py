"""ctypes binding of libfp8lm.so (include/lm_fp8.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  If the
library is missing the import fails loudly -- there is no fallback.
"""
import ctypes
import os

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libfp8lm.so")

E4M3, E5M2 = 0, 1
EPI_NONE, EPI_RELU2_FWD, EPI_RELU2_BWD, EPI_ACCUM_F32 = 0, 1, 2, 3
GEMM_A_MN_MAJOR, GEMM_B_MN_MAJOR = 1, 2
MLP_REUSE_WEIGHT_CASTS, MLP_ACCUMULATE_WGRAD = 1, 2
LINEAR_REUSE_WEIGHT_CAST, LINEAR_ACCUMULATE_WGRAD = 1, 2

STATUS = {0: "LM_OK", 1: "LM_ERR_INVALID_ARG", 2: "LM_ERR_ALIGNMENT",
          3: "LM_ERR_UNSUPPORTED_SHAPE", 4: "LM_ERR_UNSUPPORTED_FORMAT", 5: "LM_ERR_CUDA",
          6: "LM_ERR_TIMEOUT", 7: "LM_ERR_NONFINITE"}

EXPORTED = ["lm_fp8_amax_scale_cast", "lm_fp8_gemm", "lm_relu2_mlp_saved_bytes",
            "lm_relu2_mlp_saved_carve", "lm_relu2_mlp_workspace_size", "lm_relu2_mlp_fwd",
            "lm_relu2_mlp_bwd", "lm_get_error", "lm_status_string", "lm_version",
            "lm_timing_attach", "lm_timing_detach", "lm_timing_kinds",
            "lm_relu2_mlp_bwd_noalloc", "lm_relu2_mlp_bwd_noalloc_max_bytes",
            "lm_selftest_bounded_wait", "lm_relu2_mlp_fwd_ex", "lm_relu2_mlp_bwd_ex",
            "lm_rmsnorm_fp8_cast", "lm_swiglu_mlp_saved_bytes", "lm_swiglu_mlp_saved_carve",
            "lm_swiglu_mlp_workspace_size", "lm_swiglu_mlp_fwd", "lm_swiglu_mlp_bwd",
            "lm_fp8_lmhead_ce_workspace_size", "lm_fp8_lmhead_ce", "lm_fp8_gemm_ex",
            "lm_fp8_gemm_workspace_size", "lm_fp8_linear_saved_bytes",
            "lm_fp8_linear_saved_carve", "lm_fp8_linear_workspace_size", "lm_fp8_linear_fwd",
            "lm_fp8_linear_bwd", "lm_fp8_gemm_split_plan"]


class LmError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class MlpSaved(ctypes.Structure):
    """Mirror of lm_mlp_saved."""
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("Xq", "Wuq", "Wdq", "H", "hq", "scales")]


class LinearSaved(ctypes.Structure):
    """Mirror of lm_linear_saved."""
    _fields_ = [(n, ctypes.c_void_p) for n in ("Xq", "Wq", "scales")]


class SwigluSaved(ctypes.Structure):
    """Mirror of lm_swiglu_saved."""
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("Xq", "Wguq", "Wdq", "GU", "h", "hq", "scales")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m fp8_gemms_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i64, i32, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int
    L.lm_fp8_amax_scale_cast.argtypes = [P, i64, i64, i64, i32, i32, P, P, P, P, P, P, P]
    L.lm_fp8_amax_scale_cast.restype = st
    L.lm_fp8_gemm.argtypes = [P, i32, P, i32, i64, i64, i64, P, P, i32, P, P, P, P]
    L.lm_fp8_gemm.restype = st
    L.lm_fp8_gemm_ex.argtypes = [P, i32, P, i32, i64, i64, i64, ctypes.c_uint32, P, P, i32, P, P,
                                 P, P, ctypes.c_size_t, P]
    L.lm_fp8_gemm_ex.restype = st
    L.lm_fp8_gemm_workspace_size.argtypes = []
    L.lm_fp8_gemm_workspace_size.restype = ctypes.c_size_t
    L.lm_relu2_mlp_saved_bytes.argtypes = [i64, i64, i64]
    L.lm_relu2_mlp_saved_bytes.restype = ctypes.c_size_t
    L.lm_relu2_mlp_saved_carve.argtypes = [P, ctypes.c_size_t, i64, i64, i64,
                                           ctypes.POINTER(MlpSaved)]
    L.lm_relu2_mlp_saved_carve.restype = st
    L.lm_relu2_mlp_workspace_size.argtypes = [i64, i64, i64]
    L.lm_relu2_mlp_workspace_size.restype = ctypes.c_size_t
    L.lm_relu2_mlp_fwd.argtypes = [P, P, P, i64, i64, i64, P, ctypes.POINTER(MlpSaved), P,
                                   ctypes.c_size_t, P]
    L.lm_relu2_mlp_fwd.restype = st
    L.lm_relu2_mlp_bwd.argtypes = [P, ctypes.POINTER(MlpSaved), i64, i64, i64, P, P, P, P,
                                   ctypes.c_size_t, P]
    L.lm_relu2_mlp_bwd.restype = st
    L.lm_get_error.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    L.lm_get_error.restype = st
    L.lm_status_string.argtypes = [st]
    L.lm_status_string.restype = ctypes.c_char_p
    L.lm_version.restype = ctypes.c_int
    L.lm_timing_attach.argtypes = [ctypes.POINTER(ctypes.c_void_p), i32]
    L.lm_timing_attach.restype = None
    L.lm_timing_detach.argtypes = []
    L.lm_timing_detach.restype = i32
    L.lm_timing_kinds.argtypes = [ctypes.c_char_p, i32]
    L.lm_timing_kinds.restype = i32
    L.lm_relu2_mlp_bwd_noalloc.argtypes = [P, ctypes.POINTER(MlpSaved), i64, i64, i64, P, P, P, P]
    L.lm_relu2_mlp_bwd_noalloc.restype = st
    L.lm_relu2_mlp_bwd_noalloc_max_bytes.argtypes = []
    L.lm_relu2_mlp_bwd_noalloc_max_bytes.restype = ctypes.c_size_t
    L.lm_relu2_mlp_fwd_ex.argtypes = [P, P, P, i64, i64, i64, P, ctypes.POINTER(MlpSaved),
                                      P, ctypes.c_size_t, ctypes.c_uint32, P]
    L.lm_relu2_mlp_fwd_ex.restype = st
    L.lm_relu2_mlp_bwd_ex.argtypes = [P, ctypes.POINTER(MlpSaved), i64, i64, i64, P, P, P, P,
                                      ctypes.c_size_t, ctypes.c_uint32, P]
    L.lm_relu2_mlp_bwd_ex.restype = st
    L.lm_rmsnorm_fp8_cast.argtypes = [P, P, i64, i64, ctypes.c_float, i32, P, P, P, P, P, P, P]
    L.lm_rmsnorm_fp8_cast.restype = st
    L.lm_swiglu_mlp_saved_bytes.argtypes = [i64, i64, i64]
    L.lm_swiglu_mlp_saved_bytes.restype = ctypes.c_size_t
    L.lm_swiglu_mlp_saved_carve.argtypes = [P, ctypes.c_size_t, i64, i64, i64,
                                            ctypes.POINTER(SwigluSaved)]
    L.lm_swiglu_mlp_saved_carve.restype = st
    L.lm_swiglu_mlp_workspace_size.argtypes = [i64, i64, i64]
    L.lm_swiglu_mlp_workspace_size.restype = ctypes.c_size_t
    L.lm_swiglu_mlp_fwd.argtypes = [P, P, P, i64, i64, i64, P, ctypes.POINTER(SwigluSaved), P,
                                    ctypes.c_size_t, P]
    L.lm_swiglu_mlp_fwd.restype = st
    L.lm_swiglu_mlp_bwd.argtypes = [P, ctypes.POINTER(SwigluSaved), i64, i64, i64, P, P, P, P,
                                    ctypes.c_size_t, P]
    L.lm_swiglu_mlp_bwd.restype = st
    L.lm_fp8_lmhead_ce_workspace_size.argtypes = [i64, i64, i64, i64]
    L.lm_fp8_lmhead_ce_workspace_size.restype = ctypes.c_size_t
    L.lm_fp8_lmhead_ce.argtypes = [P, P, P, i64, i64, i64, i64, ctypes.c_float, P, P, P, P,
                                   ctypes.c_size_t, P]
    L.lm_fp8_lmhead_ce.restype = st
    L.lm_selftest_bounded_wait.argtypes = [ctypes.c_uint32, P]
    L.lm_selftest_bounded_wait.restype = st
    L.lm_fp8_gemm_split_plan.argtypes = [i64, i64, i64, i32, ctypes.POINTER(ctypes.c_int),
                                         ctypes.POINTER(ctypes.c_int)]
    L.lm_fp8_gemm_split_plan.restype = st
    for fn in ("lm_fp8_linear_saved_bytes", "lm_fp8_linear_workspace_size"):
        getattr(L, fn).argtypes = [i64, i64, i64]
        getattr(L, fn).restype = ctypes.c_size_t
    L.lm_fp8_linear_saved_carve.argtypes = [P, ctypes.c_size_t, i64, i64, i64,
                                            ctypes.POINTER(LinearSaved)]
    L.lm_fp8_linear_saved_carve.restype = st
    L.lm_fp8_linear_fwd.argtypes = [P, P, i64, i64, i64, P, ctypes.POINTER(LinearSaved), P,
                                    ctypes.c_size_t, ctypes.c_uint32, P]
    L.lm_fp8_linear_fwd.restype = st
    L.lm_fp8_linear_bwd.argtypes = [P, ctypes.POINTER(LinearSaved), i64, i64, i64, P, P, P,
                                    ctypes.c_size_t, ctypes.c_uint32, P]
    L.lm_fp8_linear_bwd.restype = st
    return L


lib = _load()


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _check(status, what):
    if status != 0:
        raise LmError(status, what)


# ------------------------------------------------------- C-ABI mirrors
def lm_fp8_amax_scale_cast(x, fmt, amax_out, scale_out, inv_scale_out, q=None, qT=None,
                           relu2_input=False, amax_in=None, stream=None):
    """x: 2-D bf16 CUDA tensor (row stride = ld).  Scales are 1-element (or
    sliced) fp32 CUDA tensors.  Raises LmError on a non-zero status."""
    rows, cols = x.shape
    ld = x.stride(0) if rows > 1 else cols
    assert x.dtype == torch.bfloat16 and x.stride(-1) == 1
    _check(lib.lm_fp8_amax_scale_cast(_p(x), rows, cols, ld, fmt, int(relu2_input), _p(amax_in),
                                      _p(amax_out), _p(scale_out), _p(inv_scale_out), _p(q),
                                      _p(qT), _stream(stream)), "lm_fp8_amax_scale_cast")


def lm_fp8_gemm(A, fa, B, fb, inv_scale_a, inv_scale_b, D, epi=EPI_NONE, aux=None,
                amax_out=None, stream=None):
    """D[M x N] (bf16) = epi(A[M x K] B[N x K]^T * inv_a * inv_b); A, B uint8 codes."""
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2 and tuple(D.shape) == (M, N)
    _check(lib.lm_fp8_gemm(_p(A), fa, _p(B), fb, M, N, K, _p(inv_scale_a), _p(inv_scale_b), epi,
                           _p(aux), _p(D), _p(amax_out), _stream(stream)), "lm_fp8_gemm")


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def lm_fp8_gemm_workspace_size():
    return lib.lm_fp8_gemm_workspace_size()


def lm_fp8_gemm_split_plan(M, N, K, sm_count):
    """(parts, tail_tiles): the split-K tail lm_fp8_gemm_ex uses for this shape
    on a GPU of sm_count multiprocessors (host arithmetic only)."""
    parts, tail = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib.lm_fp8_gemm_split_plan(M, N, K, sm_count, ctypes.byref(parts), ctypes.byref(tail)),
           "lm_fp8_gemm_split_plan")
    return parts.value, tail.value


def lm_fp8_gemm_ex(A, fa, B, fb, inv_scale_a, inv_scale_b, D, flags=0, epi=EPI_NONE, aux=None,
                   amax_out=None, workspace=None, stream=None):
    """lm_fp8_gemm with per-operand storage: with GEMM_A_MN_MAJOR, A is given as
    its [K x M] transpose (row-major); with GEMM_B_MN_MAJOR, B as [K x N].
    workspace (a device buffer, or None) enables the split-K tail."""
    M, K = (A.shape[1], A.shape[0]) if flags & GEMM_A_MN_MAJOR else tuple(A.shape)
    N, K2 = (B.shape[1], B.shape[0]) if flags & GEMM_B_MN_MAJOR else tuple(B.shape)
    assert K == K2 and tuple(D.shape) == (M, N)
    _check(lib.lm_fp8_gemm_ex(_p(A), fa, _p(B), fb, M, N, K, flags, _p(inv_scale_a),
                              _p(inv_scale_b), epi, _p(aux), _p(D), _p(amax_out), _p(workspace),
                              _nbytes(workspace), _stream(stream)),
           "lm_fp8_gemm_ex")


def lm_rmsnorm_fp8_cast(R, weight, X, fmt, amax_out, scale_out, inv_scale_out, q=None, qT=None,
                        eps=1e-6, stream=None):
    rows, cols = R.shape
    assert R.is_contiguous() and X.is_contiguous()
    _check(lib.lm_rmsnorm_fp8_cast(_p(R), _p(weight), rows, cols, eps, fmt, _p(X), _p(amax_out),
                                   _p(scale_out), _p(inv_scale_out), _p(q), _p(qT),
                                   _stream(stream)), "lm_rmsnorm_fp8_cast")


def lm_relu2_mlp_saved_bytes(M, d, f):
    return lib.lm_relu2_mlp_saved_bytes(M, d, f)


def lm_relu2_mlp_workspace_size(M, d, f):
    return lib.lm_relu2_mlp_workspace_size(M, d, f)


def lm_relu2_mlp_saved_carve(buf, M, d, f):
    s = MlpSaved()
    _check(lib.lm_relu2_mlp_saved_carve(_p(buf), buf.numel() * buf.element_size(), M, d, f,
                                        ctypes.byref(s)), "lm_relu2_mlp_saved_carve")
    return s


def lm_relu2_mlp_fwd(X, W_up, W_down, Y, saved, workspace=None, stream=None):
    M, d = X.shape
    f = W_up.shape[0]
    _check(lib.lm_relu2_mlp_fwd(_p(X), _p(W_up), _p(W_down), M, d, f, _p(Y),
                                ctypes.byref(saved), _p(workspace), _nbytes(workspace),
                                _stream(stream)),
           "lm_relu2_mlp_fwd")


def lm_relu2_mlp_bwd(dY, saved, dX, dW_up, dW_down, workspace, stream=None):
    M, d = dY.shape
    f = dW_up.shape[0]
    _check(lib.lm_relu2_mlp_bwd(_p(dY), ctypes.byref(saved), M, d, f, _p(dX), _p(dW_up),
                                _p(dW_down), _p(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream)),
           "lm_relu2_mlp_bwd")


def lm_relu2_mlp_fwd_ex(X, W_up, W_down, Y, saved, f, flags=0, workspace=None, stream=None):
    """f: hidden size (W_up may be None when its cast is reused)."""
    M, d = X.shape
    _check(lib.lm_relu2_mlp_fwd_ex(_p(X), _p(W_up), _p(W_down), M, d, f, _p(Y),
                                   ctypes.byref(saved), _p(workspace), _nbytes(workspace), flags,
                                   _stream(stream)),
           "lm_relu2_mlp_fwd_ex")


def lm_relu2_mlp_bwd_ex(dY, saved, dX, dW_up, dW_down, workspace, flags=0, stream=None):
    M, d = dY.shape
    f = dW_up.shape[0]
    _check(lib.lm_relu2_mlp_bwd_ex(_p(dY), ctypes.byref(saved), M, d, f, _p(dX), _p(dW_up),
                                   _p(dW_down), _p(workspace),
                                   workspace.numel() * workspace.element_size(), flags,
                                   _stream(stream)), "lm_relu2_mlp_bwd_ex")


def lm_relu2_mlp_bwd_noalloc(dY, saved, dX, dW_up, dW_down, stream=None):
    """The relu^2 MLP backward with the library's own fixed scratch (no workspace
    argument); see include/lm_fp8.h for its size limit and sharing rules."""
    M, d = dY.shape
    f = dW_up.shape[0]
    _check(lib.lm_relu2_mlp_bwd_noalloc(_p(dY), ctypes.byref(saved), M, d, f, _p(dX), _p(dW_up),
                                        _p(dW_down), _stream(stream)),
           "lm_relu2_mlp_bwd_noalloc")


def lm_fp8_linear_saved_bytes(M, K, N):
    return lib.lm_fp8_linear_saved_bytes(M, K, N)


def lm_fp8_linear_workspace_size(M, K, N):
    return lib.lm_fp8_linear_workspace_size(M, K, N)


def lm_fp8_linear_saved_carve(buf, M, K, N):
    s = LinearSaved()
    _check(lib.lm_fp8_linear_saved_carve(_p(buf), _nbytes(buf), M, K, N, ctypes.byref(s)),
           "lm_fp8_linear_saved_carve")
    return s


def lm_fp8_linear_fwd(X, W, Y, saved, N, flags=0, workspace=None, stream=None):
    """X [M x K] -> Y [M x N]; N is given because W may be None when its cast
    is reused (LINEAR_REUSE_WEIGHT_CAST)."""
    M, K = X.shape
    _check(lib.lm_fp8_linear_fwd(_p(X), _p(W), M, K, N, _p(Y), ctypes.byref(saved),
                                 _p(workspace), _nbytes(workspace), flags, _stream(stream)),
           "lm_fp8_linear_fwd")


def lm_fp8_linear_bwd(dY, saved, K, dX, dW, workspace, flags=0, stream=None):
    """dY [M x N]; dX [M x K] (or None: no dgrad); dW [N x K] bf16, or fp32
    with LINEAR_ACCUMULATE_WGRAD."""
    M, N = dY.shape
    _check(lib.lm_fp8_linear_bwd(_p(dY), ctypes.byref(saved), M, K, N, _p(dX), _p(dW),
                                 _p(workspace), _nbytes(workspace), flags, _stream(stream)),
           "lm_fp8_linear_bwd")


def lm_swiglu_mlp_saved_carve(buf, M, d, f):
    s = SwigluSaved()
    _check(lib.lm_swiglu_mlp_saved_carve(_p(buf), buf.numel() * buf.element_size(), M, d, f,
                                         ctypes.byref(s)), "lm_swiglu_mlp_saved_carve")
    return s


def lm_swiglu_mlp_fwd(X, W_gu, W_down, Y, saved, workspace=None, stream=None):
    M, d = X.shape
    f = W_gu.shape[0] // 2
    _check(lib.lm_swiglu_mlp_fwd(_p(X), _p(W_gu), _p(W_down), M, d, f, _p(Y),
                                 ctypes.byref(saved), _p(workspace), _nbytes(workspace),
                                 _stream(stream)), "lm_swiglu_mlp_fwd")


def lm_swiglu_mlp_bwd(dY, saved, dX, dW_gu, dW_down, workspace, stream=None):
    M, d = dY.shape
    f = dW_gu.shape[0] // 2
    _check(lib.lm_swiglu_mlp_bwd(_p(dY), ctypes.byref(saved), M, d, f, _p(dX), _p(dW_gu),
                                 _p(dW_down), _p(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "lm_swiglu_mlp_bwd")


def lm_fp8_lmhead_ce(X, W, labels, loss_out, dX, dW, workspace, chunk, softcap=15.0,
                     stream=None):
    M, d = X.shape
    V = W.shape[0]
    assert labels.dtype == torch.int32 and dW.dtype == torch.float32
    _check(lib.lm_fp8_lmhead_ce(_p(X), _p(W), _p(labels), M, d, V, chunk, softcap, _p(loss_out),
                                _p(dX), _p(dW), _p(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream)),
           "lm_fp8_lmhead_ce")


def lm_get_error(stream=None):
    where = ctypes.c_uint32(0)
    st = lib.lm_get_error(_stream(stream), ctypes.byref(where))
    return st, where.value


def lm_selftest_bounded_wait(limit_ms, stream=None):
    _check(lib.lm_selftest_bounded_wait(limit_ms, _stream(stream)), "lm_selftest_bounded_wait")


def lm_status_string(status):
    return lib.lm_status_string(status).decode()


def lm_version():
    return lib.lm_version()


class KernelTimer:
    """Context manager over lm_timing_attach/detach: records a CUDA event before
    every library kernel launched on this host thread (at most `capacity`).
    After exit, `.kinds` labels each launch and `.durations_ms(end_event)`
    gives per-launch times, the last one ending at `end_event`."""

    def __init__(self, capacity=64):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(capacity)]
        for e in self.events:       # torch creates the CUDA event on first record
            e.record()
        self._arr = (ctypes.c_void_p * capacity)(*[e.cuda_event for e in self.events])
        self.n = 0
        self.kinds = ""

    def __enter__(self):
        lib.lm_timing_attach(self._arr, len(self.events))
        return self

    def __exit__(self, *exc):
        self.n = lib.lm_timing_detach()
        buf = ctypes.create_string_buffer(self.n + 1)
        k = lib.lm_timing_kinds(buf, self.n)
        self.kinds = buf.raw[:k].decode()

    def durations_ms(self, end_event):
        marks = self.events[:self.n] + [end_event]
        return [a.elapsed_time(b) for a, b in zip(marks[:-1], marks[1:])]
